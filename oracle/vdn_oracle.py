"""Float64 CPU oracle for the forward pass of the VDN-H3 bidirectional linear branch.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain definition that the CUDA
path is checked against.  Only the test-suite, the package smoke check and the
benchmark's CPU-baseline leg may import it; the library never does.  It shares no
code with the CUDA path (only the seeded input generator serves both).

Source: "VDN-Minimax-H3 bidirectional linear branch in five steps"
(icman.com.cn/news/81972), the sections "Step 1" to "Step 5" and "text state".
The page lost every '+' and '=' when it was turned into text; the restored forms
are used here:  A = sum_s beta_s k_s k_s^T,  B = sum_s beta_s v_s k_s^T,
S_out = (S_in D + B)(I + A)^-1, and so on (see each function).

Readings taken where the page is silent (each one is a keyword argument here):
  * short conv: depthwise, 1-D along each frame's token order, centred, zero
    padded at the frame edges, no bias; tap j reads token s + j - (K-1)//2;
  * SiLU on q, k and v (k and v after the conv); L2 norm x / sqrt(sum x^2 + 1e-12)
    on q and k;
  * D_f = diag(alpha_f) over key channels, right-multiplying the state; both scans
    absorb frame f with its own alpha_f;
  * window: chunk index c = t // chunk, lo = max(0, chunk (c - r)),
    hi = min(F - 1, chunk (c + r + 1) - 1);
  * bridge: the prefix state P[lo-1] is carried to frame t through D_lo..D_t and
    the suffix state Q[hi+1] through D_t..D_hi (column scaling, nothing absorbed);
  * seeds: both scans start from 0.5 * text_state (zero without a text state) and
    a window at a clip edge reads that decayed seed;
  * read-out o = W_t q', RMSNorm over d with eps 1e-6 and weight rms_w[d], then
    the (post-sigmoid) output gate.

The page also places the branch in its layer: the windowed softmax branch sees
the frames of the chunk-aligned window through the RoPE-rotated q/k, the linear
branch everything outside it, and the two outputs are added (section on why
video models stall on attention and what the far field is).  Readings: scaled
dot-product softmax with scale 1/sqrt(d), bidirectional over all keys of frames
lo..hi, no mask inside the window; the rotation is applied by the caller (its
parameters are not on the page), so the softmax branch takes q_rope, k_rope.

Parity status: every function here is pinned by tests/test_oracle_pins.py and
tests/test_oracle_softmax_pins.py against closed forms, textbook reductions,
library routines or brute force.
"""
from __future__ import annotations

import numpy as np

TEXT_STATE_SCALE = 0.5
L2_EPS = 1e-12
RMS_EPS = 1e-6
RULES = ("sana_scaled", "vdn_solve", "vdn_scaled", "additive")


# --------------------------------------------------------------------------- geometry
def window_bounds(t: int, F: int, chunk: int, radius: int) -> tuple[int, int]:
    """Chunk-aligned softmax window of query frame t ("what is the far field":
    chunks of `chunk` latent frames, the query's chunk widened by `radius` chunks
    on each side).  Frames outside [lo, hi] belong to the linear branch."""
    c = t // chunk
    lo = max(0, chunk * (c - radius))
    hi = min(F - 1, chunk * (c + radius + 1) - 1)
    return lo, hi


# --------------------------------------------------------------------------- step 1
def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def l2_normalize(x: np.ndarray, eps: float = L2_EPS) -> np.ndarray:
    """Row-wise x / sqrt(sum x^2 + eps) over the last axis."""
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def short_conv_frame(x: np.ndarray, w: np.ndarray | None, causal: bool = False) -> np.ndarray:
    """Depthwise 1-D conv over the tokens of ONE frame.

    x: [S, d] tokens of one frame and head, w: [d, K] taps (None: identity).
    out[s, c] = sum_j w[c, j] * x[s + j - p, c] for in-frame indices only,
    p = (K-1)//2 (centred) or K-1 (causal)."""
    if w is None:
        return x.copy()
    S, d = x.shape
    K = w.shape[1]
    p = (K - 1) if causal else (K - 1) // 2
    out = np.zeros_like(x)
    for j in range(K):
        off = j - p
        lo, hi = max(0, -off), min(S, S - off)
        if lo < hi:
            out[lo:hi] += w[:, j][None, :] * x[lo + off:hi + off]
    return out


def prepare_features(qh, kh, vh, F, S, wk=None, wv=None, silu_v=True, causal=False):
    """Step 1 (NoPE features) for one (batch, head).

    qh, kh, vh: [F*S, d] pre-RoPE features.  k and v go through the short conv
    (within each frame), then SiLU; q goes through SiLU only; q and k are then
    L2-normalised.  Returns q', k', v' as [F, S, d]."""
    d = qh.shape[-1]
    q = qh.reshape(F, S, d)
    k = kh.reshape(F, S, d)
    v = vh.reshape(F, S, d)
    kc = np.stack([short_conv_frame(k[f], wk, causal) for f in range(F)])
    vc = np.stack([short_conv_frame(v[f], wv, causal) for f in range(F)])
    qf = l2_normalize(silu(q))
    kf = l2_normalize(silu(kc))
    vf = silu(vc) if silu_v else vc
    return qf, kf, vf


# --------------------------------------------------------------------------- step 2
def frame_statistics(kf: np.ndarray, vf: np.ndarray, beta: np.ndarray):
    """Step 2: per frame, A = sum_s beta_s k_s k_s^T (d_k x d_k) and
    B = sum_s beta_s v_s k_s^T (d_v x d_k).  kf, vf: [F, S, d]; beta: [F, S]."""
    bk = beta[..., None] * kf
    A = np.einsum("fsi,fsj->fij", kf, bk)
    Bm = np.einsum("fsi,fsj->fij", vf, bk)
    return A, Bm


# --------------------------------------------------------------------------- step 3
def rule_step(S_in, A_f, B_f, alpha_f, rule: str, c: float = 1.0):
    """Step 3: one frame of the delta-rule recurrence (state is d_v x d_k).

    vdn_solve:   S_out = (S_in D + B)(I + A)^-1
    vdn_scaled:  S_out = (S_in D + cB)(I + c^2 A)^-1
    sana_scaled: S_out = (S_in D)(I - c^2 A) + cB
    additive:    S_out = S_in D + B            (test-only: A taken as 0)
    with D = diag(alpha_f).  The inverse is never formed: S_out solves
    S_out (I + c^2 A) = X, i.e. (I + c^2 A)^T S_out^T = X^T."""
    d = A_f.shape[0]
    I = np.eye(d)
    D = np.diag(alpha_f)
    if rule == "vdn_solve":
        X = S_in @ D + B_f
        return np.linalg.solve((I + A_f).T, X.T).T
    if rule == "vdn_scaled":
        X = S_in @ D + c * B_f
        return np.linalg.solve((I + c * c * A_f).T, X.T).T
    if rule == "sana_scaled":
        return (S_in @ D) @ (I - c * c * A_f) + c * B_f
    if rule == "additive":
        return S_in @ D + B_f
    raise ValueError(rule)


def seed_state(text_state_h, d):
    """Scan seed: TEXT_STATE_SCALE x the text state (zero without one)."""
    if text_state_h is None:
        return np.zeros((d, d))
    return TEXT_STATE_SCALE * np.asarray(text_state_h, dtype=np.float64)


# --------------------------------------------------------------------------- step 4
def bidirectional_scan(A, Bm, alpha_h, seed, rule, c=1.0):
    """Forward prefix scan P_f (frames 0..f absorbed) and backward suffix scan
    Q_f (frames f..F-1 absorbed), both starting from `seed`.  alpha_h: [F, d]."""
    F = A.shape[0]
    P = np.empty_like(A)
    Q = np.empty_like(A)
    s = seed
    for f in range(F):
        s = rule_step(s, A[f], Bm[f], alpha_h[f], rule, c)
        P[f] = s
    s = seed
    for f in reversed(range(F)):
        s = rule_step(s, A[f], Bm[f], alpha_h[f], rule, c)
        Q[f] = s
    return P, Q


def gather_state(P, Q, seed, alpha_h, t, chunk, radius, bridge="to_query"):
    """Step 4 (gather + bridge) for query frame t: the prefix state just before
    the window and the suffix state just after it, each decayed across the
    window frames up to the query frame, then summed.

    bridge="to_query":  P[lo-1] diag(prod_{f=lo..t} alpha_f) + Q[hi+1] diag(prod_{f=t..hi} alpha_f)
    bridge="window":    both sides decayed by prod_{f=lo..hi} alpha_f (alternative reading)."""
    F = P.shape[0]
    lo, hi = window_bounds(t, F, chunk, radius)
    pre = seed if lo == 0 else P[lo - 1]
    suf = seed if hi == F - 1 else Q[hi + 1]
    if bridge == "to_query":
        dpre = np.prod(alpha_h[lo:t + 1], axis=0)
        dsuf = np.prod(alpha_h[t:hi + 1], axis=0)
    elif bridge == "window":
        dpre = dsuf = np.prod(alpha_h[lo:hi + 1], axis=0)
    else:
        raise ValueError(bridge)
    return pre @ np.diag(dpre) + suf @ np.diag(dsuf)


# --------------------------------------------------------------------------- step 5
def readout(W_t, qf_tokens, gate_tokens, rms_w, prenorm=False):
    """Step 5: o = W_t q' per token, RMSNorm over d (eps 1e-6, weight rms_w),
    times the output gate.  qf_tokens, gate_tokens: [n, d]."""
    o = qf_tokens @ W_t.T
    if prenorm:
        return o
    y = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + RMS_EPS) * rms_w
    return y * gate_tokens


# --------------------------------------------------------------------------- whole branch
def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):          # torch tensor (CPU)
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def head_state(inp: dict, b: int, h: int, F: int, S: int, rule: str, c: float, chunk: int, radius: int,
               bridge="to_query", silu_v=True, causal=False):
    """Steps 1-4 for one (batch, head).  Returns a dict with q' [F,S,d], k', v',
    A, B [F,d,d], P, Q [F,d,d] and W [F,d,d] (the gathered state per query frame)."""
    q = _f64(inp["q"][b, :, h, :])
    k = _f64(inp["k"][b, :, h, :])
    v = _f64(inp["v"][b, :, h, :])
    beta = _f64(inp["beta"][b, :, h]).reshape(F, S)
    alpha_h = _f64(inp["alpha"][b, :, h, :])
    wk = None if inp.get("conv_k_w") is None else _f64(inp["conv_k_w"][h])
    wv = None if inp.get("conv_v_w") is None else _f64(inp["conv_v_w"][h])
    d = q.shape[-1]
    ts = inp.get("text_state")
    seed = seed_state(None if ts is None else _f64(ts[h]), d)
    qf, kf, vf = prepare_features(q, k, v, F, S, wk, wv, silu_v=silu_v, causal=causal)
    A, Bm = frame_statistics(kf, vf, beta)
    P, Q = bidirectional_scan(A, Bm, alpha_h, seed, rule, c)
    W = np.stack([gather_state(P, Q, seed, alpha_h, t, chunk, radius, bridge) for t in range(F)])
    return {"qf": qf, "kf": kf, "vf": vf, "A": A, "B": Bm, "P": P, "Q": Q, "W": W, "seed": seed}


def branch_forward(inp: dict, F: int, S: int, rule: str = "vdn_solve", c: float = 1.0, chunk: int = 5,
                   radius: int = 1, heads=None, batches=None, prenorm=False, **kw):
    """The whole branch for the selected (batch, head) pairs.

    Returns out [B, F*S, H, d] float64; entries of heads/batches not selected stay NaN."""
    q = inp["q"]
    B, N, H, d = q.shape
    out = np.full((B, N, H, d), np.nan)
    rms_w = _f64(inp["rms_w"])
    for b in (range(B) if batches is None else batches):
        for h in (range(H) if heads is None else heads):
            st = head_state(inp, b, h, F, S, rule, c, chunk, radius, **kw)
            g = _f64(inp["gate"][b, :, h, :]).reshape(F, S, d)
            for t in range(F):
                out[b, t * S:(t + 1) * S, h, :] = readout(st["W"][t], st["qf"][t], g[t], rms_w, prenorm)
    return out


def sampled_outputs(inp: dict, F: int, S: int, rule: str, c: float, chunk: int, radius: int,
                    b: int, h: int, tokens, prenorm=False):
    """Outputs of selected tokens (indices into F*S) of one (batch, head), for
    checks at full size where the whole output is too large to recompute."""
    st = head_state(inp, b, h, F, S, rule, c, chunk, radius)
    rms_w = _f64(inp["rms_w"])
    tokens = np.asarray(tokens)
    d = st["qf"].shape[-1]
    g = _f64(inp["gate"][b, :, h, :])
    res = np.empty((len(tokens), d))
    for i, n in enumerate(tokens):
        t, s = divmod(int(n), S)
        res[i] = readout(st["W"][t], st["qf"][t, s][None, :], g[n][None, :], rms_w, prenorm)[0]
    return res


# --------------------------------------------------------------------------- windowed softmax branch
def window_softmax_frame(qr_t, kr_win, v_win, scale):
    """softmax(q k^T * scale) v for the query rows qr_t [n, d] against the keys
    kr_win [m, d] and values v_win [m, d] of their window (one frame's queries
    share the window).  Max-subtracted, so large scores do not overflow."""
    sc = (qr_t @ kr_win.T) * scale
    sc -= sc.max(axis=1, keepdims=True)
    w = np.exp(sc)
    w /= w.sum(axis=1, keepdims=True)
    return w @ v_win


def window_softmax_head(qr_h, kr_h, v_h, F: int, S: int, chunk: int, radius: int, scale=None, frames=None):
    """Windowed softmax branch of one (batch, head): query frame t attends to
    every token of frames lo..hi = window_bounds(t).  Inputs [F*S, d]; returns
    [F*S, d] (rows of frames not in `frames` stay NaN)."""
    d = qr_h.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.full(qr_h.shape, np.nan)
    for t in (range(F) if frames is None else frames):
        lo, hi = window_bounds(t, F, chunk, radius)
        keys = slice(lo * S, (hi + 1) * S)
        out[t * S:(t + 1) * S] = window_softmax_frame(qr_h[t * S:(t + 1) * S], kr_h[keys], v_h[keys], scale)
    return out


def window_softmax_forward(inp: dict, F: int, S: int, chunk: int = 5, radius: int = 1, heads=None, batches=None,
                           scale=None):
    """The windowed softmax branch for the selected (batch, head) pairs:
    [B, F*S, H, d] float64 (unselected entries NaN).  Uses inp["q_rope"],
    inp["k_rope"] and inp["v"]."""
    qr = inp["q_rope"]
    B, N, H, d = qr.shape
    out = np.full((B, N, H, d), np.nan)
    for b in (range(B) if batches is None else batches):
        for h in (range(H) if heads is None else heads):
            out[b, :, h, :] = window_softmax_head(_f64(inp["q_rope"][b, :, h, :]), _f64(inp["k_rope"][b, :, h, :]),
                                                  _f64(inp["v"][b, :, h, :]), F, S, chunk, radius, scale)
    return out


def sampled_window_softmax(inp: dict, F: int, S: int, chunk: int, radius: int, b: int, h: int, tokens, scale=None):
    """Softmax-branch outputs of selected tokens (indices into F*S) of one (batch, head)."""
    qr = _f64(inp["q_rope"][b, :, h, :])
    kr = _f64(inp["k_rope"][b, :, h, :])
    v = _f64(inp["v"][b, :, h, :])
    d = qr.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    tokens = np.asarray(tokens)
    res = np.empty((len(tokens), d))
    for i, n in enumerate(tokens):
        t = int(n) // S
        lo, hi = window_bounds(t, F, chunk, radius)
        keys = slice(lo * S, (hi + 1) * S)
        res[i] = window_softmax_frame(qr[int(n)][None, :], kr[keys], v[keys], scale)[0]
    return res


def hybrid_forward(inp: dict, F: int, S: int, rule: str = "vdn_solve", c: float = 1.0, chunk: int = 5,
                   radius: int = 1, heads=None, batches=None, scale=None):
    """The hybrid attention layer's two branches summed: windowed softmax over
    the near field plus the bidirectional linear branch over the far field."""
    return (window_softmax_forward(inp, F, S, chunk, radius, heads, batches, scale)
            + branch_forward(inp, F, S, rule, c, chunk, radius, heads, batches))
