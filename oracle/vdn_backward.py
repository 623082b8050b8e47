"""Float64 oracle of the BACKWARD pass of the VDN-H3 bidirectional linear branch.

Test infrastructure, like vdn_oracle.py: only tests/, the package smoke check and
bench.py's CPU legs use it; nothing on the product path imports it.

The page ("VDN-Minimax-H3 bidirectional linear branch in five steps", section on
how the branch was trained: stages A1/A2 align the new branch layer by layer, then
end to end) trains the branch but gives no backward formulas.  Reading: the
backward pass is the exact gradient of the forward of vdn_oracle.py (the five
steps and the text-state seeds), taken step by step in reverse order by the
adjoint method.  For a loss L with dL/dout = dout it returns dL/d of every input:
q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w and text_state.

Each step below names the forward step it reverses.  Nothing here is blocked,
fused or reordered; the pins are central finite differences of the forward oracle
(tests/test_oracle_backward_pins.py).  The divergent sana_scaled settings whose
states leave any floating-point range are out of scope for gradients as they are
for fp32 forward values.
"""
from __future__ import annotations

import numpy as np

from oracle import vdn_oracle as O


# --------------------------------------------------------------------------- step 1 reversed
def silu_grad(x: np.ndarray, g: np.ndarray) -> np.ndarray:
    """d silu(x) = sigma(x) (1 + x (1 - sigma(x))) dx."""
    s = 1.0 / (1.0 + np.exp(-x))
    return g * s * (1.0 + x * (1.0 - s))


def l2_normalize_grad(x: np.ndarray, g: np.ndarray, eps: float = O.L2_EPS) -> np.ndarray:
    """x_hat = x / n with n = sqrt(sum x^2 + eps): dx = (g - x_hat (x_hat . g)) / n, row-wise."""
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)
    xh = x / n
    return (g - xh * np.sum(xh * g, axis=-1, keepdims=True)) / n


def short_conv_frame_grad(x: np.ndarray, w: np.ndarray | None, g: np.ndarray):
    """Reverse of vdn_oracle.short_conv_frame (centred taps, in-frame only):
    out[s, c] = sum_j w[c, j] x[s + j - p, c]  gives
    dx[s + j - p, c] += w[c, j] g[s, c]  and  dw[c, j] = sum_s g[s, c] x[s + j - p, c]."""
    if w is None:
        return g.copy(), None
    S, d = x.shape
    K = w.shape[1]
    p = (K - 1) // 2
    dx = np.zeros_like(x)
    dw = np.zeros_like(w)
    for j in range(K):
        off = j - p
        lo, hi = max(0, -off), min(S, S - off)
        if lo < hi:
            dx[lo + off:hi + off] += w[:, j][None, :] * g[lo:hi]
            dw[:, j] += np.sum(g[lo:hi] * x[lo + off:hi + off], axis=0)
    return dx, dw


# --------------------------------------------------------------------------- step 5 reversed
def readout_grad(W_t, qf, gate, rms_w, dout):
    """Reverse of vdn_oracle.readout for one frame's tokens.

    Forward: o = W_t q', r = (mean(o^2) + eps)^-1/2, y = o r rms_w, out = y gate.
    Returns dW_t, dq' [n, d], dgate [n, d], drms_w [d]."""
    o = qf @ W_t.T
    d = o.shape[-1]
    r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + O.RMS_EPS)
    oh = o * r
    y = oh * rms_w
    dgate = dout * y
    dy = dout * gate
    drms = np.sum(dy * oh, axis=0)
    doh = dy * rms_w
    # oh = o r: do_j = r doh_j - r^3 o_j / d * sum_i doh_i o_i
    do = r * doh - (r ** 3) * o * np.sum(doh * o, axis=-1, keepdims=True) / d
    dW = do.T @ qf
    dqf = do @ W_t
    return dW, dqf, dgate, drms


# --------------------------------------------------------------------------- step 4 (gather) reversed
def gather_grad(P, Q, seed, alpha_h, t, chunk, radius, dW, acc):
    """Reverse of vdn_oracle.gather_state (bridge "to_query") for query frame t.

    W_t = pre diag(a) + suf diag(b), a = prod_{lo..t} alpha, b = prod_{t..hi} alpha.
    Adds into acc["dP"][f] / acc["dQ"][f] (or acc["dseed"] at a clip edge) and
    acc["dalpha"]."""
    F = P.shape[0]
    lo, hi = O.window_bounds(t, F, chunk, radius)
    pre = seed if lo == 0 else P[lo - 1]
    suf = seed if hi == F - 1 else Q[hi + 1]
    a = np.prod(alpha_h[lo:t + 1], axis=0)
    b = np.prod(alpha_h[t:hi + 1], axis=0)
    if lo == 0:
        acc["dseed"] += dW * a[None, :]
    else:
        acc["dP"][lo - 1] += dW * a[None, :]
    if hi == F - 1:
        acc["dseed"] += dW * b[None, :]
    else:
        acc["dQ"][hi + 1] += dW * b[None, :]
    da = np.sum(pre * dW, axis=0)
    db = np.sum(suf * dW, axis=0)
    for f in range(lo, t + 1):
        others = [g for g in range(lo, t + 1) if g != f]
        acc["dalpha"][f] += da * (np.prod(alpha_h[others], axis=0) if others else 1.0)
    for f in range(t, hi + 1):
        others = [g for g in range(t, hi + 1) if g != f]
        acc["dalpha"][f] += db * (np.prod(alpha_h[others], axis=0) if others else 1.0)


# --------------------------------------------------------------------------- step 3 reversed
def rule_step_grad(S_in, A_f, B_f, alpha_f, rule, c, dS_out):
    """Reverse of vdn_oracle.rule_step.  Returns dS_in, dA_f, dB_f, dalpha_f.

    vdn_solve / vdn_scaled: S_out = X N^-1, X = S_in D + cB, N = I + c^2 A
        dX = dS_out N^-T (a solve), dN = -S_out^T dX, dA = c^2 dN, dB = c dX
    sana_scaled: S_out = Y (I - c^2 A) + cB, Y = S_in D
        dY = dS_out (I - c^2 A)^T, dA = -c^2 Y^T dS_out, dB = c dS_out
    additive: S_out = S_in D + B.
    In all cases dS_in = dX D (D = diag(alpha_f)) and dalpha_j = sum_i S_in[i, j] dX[i, j]."""
    d = A_f.shape[0]
    I = np.eye(d)
    D = np.diag(alpha_f)
    if rule in ("vdn_solve", "vdn_scaled"):
        cc = 1.0 if rule == "vdn_solve" else c
        N = I + cc * cc * A_f
        X = S_in @ D + cc * B_f
        S_out = np.linalg.solve(N.T, X.T).T
        dX = np.linalg.solve(N, dS_out.T).T          # dS_out N^-T
        dA = -cc * cc * (S_out.T @ dX)
        dB = cc * dX
    elif rule == "sana_scaled":
        Y = S_in @ D
        dX = dS_out @ (I - c * c * A_f).T
        dA = -c * c * (Y.T @ dS_out)
        dB = c * dS_out
    elif rule == "additive":
        dX = dS_out.copy()
        dA = np.zeros_like(A_f)
        dB = dS_out.copy()
    else:
        raise ValueError(rule)
    dS_in = dX @ D
    dalpha = np.sum(S_in * dX, axis=0)
    return dS_in, dA, dB, dalpha


# --------------------------------------------------------------------------- step 2 reversed
def frame_statistics_grad(kf, vf, beta, dA, dB):
    """Reverse of vdn_oracle.frame_statistics: A = sum beta k k^T, B = sum beta v k^T.
    dk_s = beta_s (dA + dA^T) k_s + beta_s dB^T v_s, dv_s = beta_s dB k_s,
    dbeta_s = k_s^T dA k_s + v_s^T dB k_s.  kf, vf: [F, S, d]; dA, dB: [F, d, d]."""
    dAs = dA + np.transpose(dA, (0, 2, 1))
    dkf = beta[..., None] * (np.einsum("fij,fsj->fsi", dAs, kf) + np.einsum("fji,fsj->fsi", dB, vf))
    dvf = beta[..., None] * np.einsum("fij,fsj->fsi", dB, kf)
    dbeta = np.einsum("fsi,fij,fsj->fs", kf, dA, kf) + np.einsum("fsi,fij,fsj->fs", vf, dB, kf)
    return dkf, dvf, dbeta


# --------------------------------------------------------------------------- whole branch reversed
def head_backward(inp: dict, b: int, h: int, F: int, S: int, rule: str, c: float, chunk: int, radius: int,
                  dout_bh: np.ndarray):
    """Gradients of one (batch, head): dout_bh [F*S, d] -> dict of per-(b, h) gradients
    (dq, dk, dv [F*S, d]; dbeta [F*S]; dalpha [F, d]; dgate [F*S, d]; drms_w [d];
    dconv_k_w, dconv_v_w [d, K] or None; dtext_state [d, d] or None)."""
    q = O._f64(inp["q"][b, :, h, :])
    k = O._f64(inp["k"][b, :, h, :])
    v = O._f64(inp["v"][b, :, h, :])
    beta = O._f64(inp["beta"][b, :, h]).reshape(F, S)
    alpha_h = O._f64(inp["alpha"][b, :, h, :])
    wk = None if inp.get("conv_k_w") is None else O._f64(inp["conv_k_w"][h])
    wv = None if inp.get("conv_v_w") is None else O._f64(inp["conv_v_w"][h])
    gate = O._f64(inp["gate"][b, :, h, :]).reshape(F, S, -1)
    rms_w = O._f64(inp["rms_w"])
    d = q.shape[-1]
    ts = inp.get("text_state")
    seed = O.seed_state(None if ts is None else O._f64(ts[h]), d)
    dout = O._f64(dout_bh).reshape(F, S, d)

    # forward, keeping what the reverse steps read
    q3, k3, v3 = q.reshape(F, S, d), k.reshape(F, S, d), v.reshape(F, S, d)
    kc = np.stack([O.short_conv_frame(k3[f], wk) for f in range(F)])
    vc = np.stack([O.short_conv_frame(v3[f], wv) for f in range(F)])
    qs, ks = O.silu(q3), O.silu(kc)
    qf, kf, vf = O.l2_normalize(qs), O.l2_normalize(ks), O.silu(vc)
    A, Bm = O.frame_statistics(kf, vf, beta)
    P, Q = O.bidirectional_scan(A, Bm, alpha_h, seed, rule, c)
    W = np.stack([O.gather_state(P, Q, seed, alpha_h, t, chunk, radius) for t in range(F)])

    # step 5 reversed
    dW = np.zeros_like(W)
    dqf = np.zeros_like(qf)
    dgate = np.zeros_like(gate)
    drms = np.zeros(d)
    for t in range(F):
        dW[t], dqf[t], dgate[t], dr = readout_grad(W[t], qf[t], gate[t], rms_w, dout[t])
        drms += dr

    # step 4 (gather + bridge) reversed
    acc = {"dP": np.zeros_like(P), "dQ": np.zeros_like(Q), "dseed": np.zeros((d, d)),
           "dalpha": np.zeros_like(alpha_h)}
    for t in range(F):
        gather_grad(P, Q, seed, alpha_h, t, chunk, radius, dW[t], acc)

    # steps 3-4 (both scans) reversed
    dA = np.zeros_like(A)
    dB = np.zeros_like(Bm)
    dalpha = acc["dalpha"]
    lam = np.zeros((d, d))                       # prefix scan: P_f = step(P_{f-1}, f)
    for f in reversed(range(F)):
        lam = lam + acc["dP"][f]
        S_in = seed if f == 0 else P[f - 1]
        lam, a_, b_, al_ = rule_step_grad(S_in, A[f], Bm[f], alpha_h[f], rule, c, lam)
        dA[f] += a_
        dB[f] += b_
        dalpha[f] += al_
    dseed = acc["dseed"] + lam
    mu = np.zeros((d, d))                        # suffix scan: Q_f = step(Q_{f+1}, f)
    for f in range(F):
        mu = mu + acc["dQ"][f]
        S_in = seed if f == F - 1 else Q[f + 1]
        mu, a_, b_, al_ = rule_step_grad(S_in, A[f], Bm[f], alpha_h[f], rule, c, mu)
        dA[f] += a_
        dB[f] += b_
        dalpha[f] += al_
    dseed += mu

    # step 2 reversed
    dkf, dvf, dbeta = frame_statistics_grad(kf, vf, beta, dA, dB)

    # step 1 reversed
    dq = silu_grad(q3, l2_normalize_grad(qs, dqf))
    dkc = silu_grad(kc, l2_normalize_grad(ks, dkf))
    dvc = silu_grad(vc, dvf)
    dk = np.empty_like(k3)
    dv = np.empty_like(v3)
    dwk = None if wk is None else np.zeros_like(wk)
    dwv = None if wv is None else np.zeros_like(wv)
    for f in range(F):
        dk[f], g1 = short_conv_frame_grad(k3[f], wk, dkc[f])
        dv[f], g2 = short_conv_frame_grad(v3[f], wv, dvc[f])
        if dwk is not None:
            dwk += g1
        if dwv is not None:
            dwv += g2
    return {"dq": dq.reshape(F * S, d), "dk": dk.reshape(F * S, d), "dv": dv.reshape(F * S, d),
            "dbeta": dbeta.reshape(F * S), "dalpha": dalpha, "dgate": dgate.reshape(F * S, d), "drms_w": drms,
            "dconv_k_w": dwk, "dconv_v_w": dwv,
            "dtext_state": None if ts is None else O.TEXT_STATE_SCALE * dseed}


def branch_backward(inp: dict, dout, F: int, S: int, rule: str = "vdn_solve", c: float = 1.0, chunk: int = 5,
                    radius: int = 1) -> dict:
    """Gradients of <dout, branch_forward(inp)> with respect to every input, float64:
    dq, dk, dv, dgate [B, F*S, H, d]; dbeta [B, F*S, H]; dalpha [B, F, H, d];
    drms_w [d] (summed over batch and heads); dconv_k_w, dconv_v_w [H, d, K] and
    dtext_state [H, d, d] (summed over the batch; None when the input is None)."""
    q = inp["q"]
    B, N, H, d = q.shape
    dout = O._f64(dout)
    g = {n: np.zeros((B, N, H, d)) for n in ("dq", "dk", "dv", "dgate")}
    g["dbeta"] = np.zeros((B, N, H))
    g["dalpha"] = np.zeros((B, F, H, d))
    g["drms_w"] = np.zeros(d)
    g["dconv_k_w"] = None if inp.get("conv_k_w") is None else np.zeros(np.shape(inp["conv_k_w"]))
    g["dconv_v_w"] = None if inp.get("conv_v_w") is None else np.zeros(np.shape(inp["conv_v_w"]))
    g["dtext_state"] = None if inp.get("text_state") is None else np.zeros(np.shape(inp["text_state"]))
    for b in range(B):
        for h in range(H):
            r = head_backward(inp, b, h, F, S, rule, c, chunk, radius, dout[b, :, h, :])
            for n in ("dq", "dk", "dv", "dgate"):
                g[n][b, :, h, :] = r[n]
            g["dbeta"][b, :, h] = r["dbeta"]
            g["dalpha"][b, :, h, :] = r["dalpha"]
            g["drms_w"] += r["drms_w"]
            for n in ("dconv_k_w", "dconv_v_w", "dtext_state"):
                if g[n] is not None:
                    g[n][h] += r[n]
    return g
