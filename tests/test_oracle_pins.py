"""Pins of the float64 oracle against things other than itself.

The source page ("VDN-Minimax-H3 bidirectional linear branch in five steps")
prints no worked example, so each step is pinned by a closed form, a textbook
reduction, a library routine or brute force on tiny inputs, chosen so that a
dropped term, a wrong sign, an off-by-one window or a transposed operand fails
at least one test.  CPU only.
"""
import numpy as np
import pytest
import scipy.special

from oracle import vdn_oracle as O
from video_diffusion_linear_b200 import synth

RULES = ["sana_scaled", "vdn_solve", "vdn_scaled", "additive"]


def _sig(x):
    return scipy.special.expit(x)


def _inputs(rng, B=1, H=1, d=6, F=12, S=3, K=3, text=False, alpha_one=False):
    N = F * S
    inp = {
        "q": rng.normal(size=(B, N, H, d)),
        "k": rng.normal(size=(B, N, H, d)),
        "v": rng.normal(size=(B, N, H, d)),
        "beta": _sig(rng.normal(size=(B, N, H))),
        "alpha": np.ones((B, F, H, d)) if alpha_one else _sig(rng.normal(2.0, 1.0, size=(B, F, H, d))),
        "gate": _sig(rng.normal(size=(B, N, H, d))),
        "rms_w": 1 + 0.1 * rng.normal(size=d),
        "conv_k_w": rng.normal(size=(H, d, K)) / np.sqrt(K) if K > 1 else None,
        "conv_v_w": rng.normal(size=(H, d, K)) / np.sqrt(K) if K > 1 else None,
        "text_state": 0.5 * 0.1 * rng.normal(size=(H, d, d)) if text else None,
    }
    return inp


# ----------------------------------------------------------------------------- window
@pytest.mark.parametrize("chunk", range(1, 7))
@pytest.mark.parametrize("radius", [0, 1, 2])
def test_window_partitions_frames(chunk, radius):
    """prefix frames [0, lo-1], window [lo, hi] and suffix frames [hi+1, F-1]
    cover [0, F) with no overlap, and the window is exactly the frames whose
    chunk is within `radius` chunks of the query's chunk."""
    for F in range(1, 41):
        for t in range(F):
            lo, hi = O.window_bounds(t, F, chunk, radius)
            assert 0 <= lo <= t <= hi <= F - 1
            pre = set(range(0, lo))
            win = set(range(lo, hi + 1))
            suf = set(range(hi + 1, F))
            assert not (pre & win) and not (win & suf) and not (pre & suf)
            assert pre | win | suf == set(range(F))
            by_chunk = {g for g in range(F) if abs(g // chunk - t // chunk) <= radius}
            assert win == by_chunk


def test_window_page_geometry():
    """chunk 5, radius 1: an interior frame sees about 15 frames (three chunks)."""
    for t in range(5, 95):
        lo, hi = O.window_bounds(t, 100, 5, 1)
        assert hi - lo + 1 == 15 and lo % 5 == 0


# ----------------------------------------------------------------------------- step 1
@pytest.mark.parametrize("K", [1, 3, 5])
def test_short_conv_is_numpy_convolve_same(K):
    rng = np.random.default_rng(1)
    S, d = 11, 4
    x = rng.normal(size=(S, d))
    w = rng.normal(size=(d, K))
    y = O.short_conv_frame(x, w)
    for c in range(d):
        ref = np.convolve(x[:, c], w[c, ::-1], mode="same")
        np.testing.assert_allclose(y[:, c], ref, rtol=1e-14, atol=1e-14)


def test_short_conv_causal_flag():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(9, 3))
    w = rng.normal(size=(3, 3))
    y = O.short_conv_frame(x, w, causal=True)
    for c in range(3):
        ref = np.convolve(x[:, c], w[c, ::-1], mode="full")[:9]
        np.testing.assert_allclose(y[:, c], ref, rtol=1e-14, atol=1e-14)


def test_identity_conv_when_no_weights():
    x = np.arange(12.0).reshape(4, 3)
    np.testing.assert_array_equal(O.short_conv_frame(x, None), x)


def test_silu_and_l2():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(50, 7)) * 3
    np.testing.assert_allclose(O.silu(x), x * scipy.special.expit(x), rtol=1e-14, atol=1e-15)
    y = O.l2_normalize(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=1e-12)
    np.testing.assert_array_equal(O.l2_normalize(np.zeros((2, 5))), 0.0)


def test_features_conv_stays_inside_frame():
    """The conv must not read across a frame edge: changing frame 1 leaves
    frame 0's and frame 2's features untouched."""
    rng = np.random.default_rng(4)
    F, S, d = 3, 5, 4
    q, k, v = (rng.normal(size=(F * S, d)) for _ in range(3))
    wk, wv = rng.normal(size=(d, 3)), rng.normal(size=(d, 3))
    a = O.prepare_features(q, k, v, F, S, wk, wv)
    k2, v2 = k.copy(), v.copy()
    k2[S:2 * S] += 10
    v2[S:2 * S] -= 10
    b = O.prepare_features(q, k2, v2, F, S, wk, wv)
    for i in (1, 2):
        np.testing.assert_array_equal(a[i][0], b[i][0])
        np.testing.assert_array_equal(a[i][2], b[i][2])
    np.testing.assert_array_equal(a[0], b[0])            # q has no conv


# ----------------------------------------------------------------------------- step 2 / 3
def test_frame_statistics_is_sum_of_outer_products():
    rng = np.random.default_rng(5)
    F, S, d = 3, 7, 5
    kf, vf = rng.normal(size=(F, S, d)), rng.normal(size=(F, S, d))
    beta = _sig(rng.normal(size=(F, S)))
    A, Bm = O.frame_statistics(kf, vf, beta)
    for f in range(F):
        Al = sum(beta[f, s] * np.outer(kf[f, s], kf[f, s]) for s in range(S))
        Bl = sum(beta[f, s] * np.outer(vf[f, s], kf[f, s]) for s in range(S))
        np.testing.assert_allclose(A[f], Al, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(Bm[f], Bl, rtol=1e-13, atol=1e-13)


def test_I_plus_A_is_spd_and_inverse_exact():
    """P-ii: I + A symmetric positive definite with spectrum in [1, 1 + sum beta |k|^2];
    (I + A) X = I to 1e-10 for its inverse."""
    rng = np.random.default_rng(6)
    inp = _inputs(rng, d=16, F=4, S=40)
    st = O.head_state(inp, 0, 0, 4, 40, "vdn_solve", 1.0, 5, 1)
    beta = inp["beta"][0, :, 0].reshape(4, 40)
    for f in range(4):
        M = np.eye(16) + st["A"][f]
        np.testing.assert_allclose(M, M.T, rtol=1e-13, atol=1e-13)
        np.linalg.cholesky(M)
        ev = np.linalg.eigvalsh(M)
        bound = 1 + np.sum(beta[f] * np.sum(st["kf"][f] ** 2, axis=-1))
        assert ev.min() >= 1 - 1e-12 and ev.max() <= bound + 1e-9
        X = np.linalg.inv(M)
        assert np.abs(M @ X - np.eye(16)).max() <= 1e-10


@pytest.mark.parametrize("c", [1.0, 0.5])
def test_solve_is_ridge_regression_least_squares(c):
    """P-ii': vdn_scaled's S_out is the minimiser of
    |S - S_in D|_F^2 + sum_s beta_s |S (c k_s) - v_s|^2, solved here by LAPACK
    least squares on the raw tokens (A and B never formed)."""
    rng = np.random.default_rng(7)
    d, S = 6, 9
    kf = O.l2_normalize(rng.normal(size=(S, d)))
    vf = rng.normal(size=(S, d))
    beta = _sig(rng.normal(size=S))
    alpha = _sig(rng.normal(2, 1, size=d))
    S_in = rng.normal(size=(d, d))
    A, Bm = O.frame_statistics(kf[None], vf[None], beta[None])
    S_out = O.rule_step(S_in, A[0], Bm[0], alpha, "vdn_scaled", c)
    sb = np.sqrt(beta)
    Z = np.concatenate([np.eye(d), (c * kf * sb[:, None]).T], axis=1)
    Y = np.concatenate([S_in * alpha[None, :], (vf * sb[:, None]).T], axis=1)
    St, *_ = np.linalg.lstsq(Z.T, Y.T, rcond=None)
    np.testing.assert_allclose(S_out, St.T, rtol=1e-10, atol=1e-12)


def test_sana_vs_vdn_scaled_small_c():
    """P-iii: (I + c^2 A)^-1 = I - c^2 A + c^4 A^2 - ..., so
    vdn_scaled - sana_scaled = -c^3 B A + c^4 S D A^2 + O(c^5)."""
    rng = np.random.default_rng(8)
    d = 5
    R = rng.normal(size=(d, d))
    A = R @ R.T / d
    Bm = rng.normal(size=(d, d))
    Sst = rng.normal(size=(d, d))
    alpha = _sig(rng.normal(2, 1, size=d))
    D = np.diag(alpha)
    errs = []
    for e in range(4, 11):
        c = 2.0 ** -e
        diff = O.rule_step(Sst, A, Bm, alpha, "vdn_scaled", c) - O.rule_step(Sst, A, Bm, alpha, "sana_scaled", c)
        errs.append(np.abs(diff / c ** 3 + Bm @ A).max())
    errs = np.array(errs)
    assert np.all(errs[1:] < errs[:-1] * 0.6)          # O(c) remainder
    assert errs[-1] < 1e-2
    errs0 = []
    for e in range(3, 9):
        c = 2.0 ** -e
        diff = O.rule_step(Sst, A, 0 * Bm, alpha, "vdn_scaled", c) - O.rule_step(Sst, A, 0 * Bm, alpha, "sana_scaled", c)
        errs0.append(np.abs(diff / c ** 4 - Sst @ D @ A @ A).max())
    errs0 = np.array(errs0)
    assert np.all(errs0[1:] < errs0[:-1] * 0.35)       # O(c^2) remainder
    assert errs0[-1] < 5e-4


def test_vdn_scaled_at_one_is_vdn_solve():
    """P-vi: bitwise."""
    rng = np.random.default_rng(9)
    inp = _inputs(rng, d=8, F=12, S=4, text=True)
    a = O.branch_forward(inp, 12, 4, "vdn_solve", 1.0, 3, 1)
    b = O.branch_forward(inp, 12, 4, "vdn_scaled", 1.0, 3, 1)
    np.testing.assert_array_equal(a, b)


# ----------------------------------------------------------------------------- step 3 (textbook)
@pytest.mark.parametrize("rule", ["vdn_solve", "sana_scaled"])
def test_one_token_per_frame_is_gated_delta_rule(rule):
    """P-v: with one token per frame and |k| = 1, vdn_solve is the gated delta rule
    S <- S D (I - b' k k^T) + b' v k^T with b' = beta / (1 + beta) (Sherman-Morrison),
    and sana_scaled at c = 1 is the same rule with rate beta."""
    rng = np.random.default_rng(10)
    F, d = 9, 6
    inp = _inputs(rng, d=d, F=F, S=1, K=1, text=True)
    st = O.head_state(inp, 0, 0, F, 1, rule, 1.0, 3, 1)
    kf, vf = st["kf"][:, 0], st["vf"][:, 0]
    beta = inp["beta"][0, :, 0]
    alpha = inp["alpha"][0, :, 0]
    Sst = 0.5 * inp["text_state"][0]
    for f in range(F):
        rate = beta[f] / (1 + beta[f]) if rule == "vdn_solve" else beta[f]
        Sst = (Sst * alpha[f][None, :]) @ (np.eye(d) - rate * np.outer(kf[f], kf[f])) + rate * np.outer(vf[f], kf[f])
        np.testing.assert_allclose(st["P"][f], Sst, rtol=1e-11, atol=1e-13)


# ----------------------------------------------------------------------------- step 4
@pytest.mark.parametrize("rule", RULES)
def test_text_state_only_decays_to_half_prompt(rule):
    """P-iv: with k = v = 0 (A = B = 0), P_f = 0.5 T prod_{g<=f} D_g and
    Q_f = 0.5 T prod_{g>=f} D_g; with alpha = 1 the pre-norm read-out is T q'."""
    rng = np.random.default_rng(11)
    F, S, d = 14, 3, 6
    for alpha_one in (False, True):
        inp = _inputs(rng, d=d, F=F, S=S, text=True, alpha_one=alpha_one)
        inp["k"][:] = 0
        inp["v"][:] = 0
        st = O.head_state(inp, 0, 0, F, S, rule, 0.7, 5, 1)
        T = inp["text_state"][0]
        alpha = inp["alpha"][0, :, 0]
        for f in range(F):
            decay_p = np.ones(d)
            for g in range(f + 1):
                decay_p = decay_p * alpha[g]
            decay_q = np.ones(d)
            for g in range(f, F):
                decay_q = decay_q * alpha[g]
            np.testing.assert_allclose(st["P"][f], 0.5 * T * decay_p[None, :], rtol=1e-12, atol=1e-15)
            np.testing.assert_allclose(st["Q"][f], 0.5 * T * decay_q[None, :], rtol=1e-12, atol=1e-15)
        if alpha_one:
            o = O.branch_forward(inp, F, S, rule, 0.7, 5, 1, prenorm=True)[0, :, 0, :]
            qf = st["qf"].reshape(F * S, d)
            np.testing.assert_allclose(o, qf @ T.T, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("chunk,radius", [(2, 1), (3, 0), (1, 2), (5, 1)])
def test_additive_unit_alpha_is_bruteforce_far_field_attention(chunk, radius):
    """P-i: with A := 0 (additive rule), alpha = 1 and no text, the pre-norm output
    is beta-weighted linear attention of q' against exactly the tokens of frames
    outside the query's window:  o_s = sum_{s' not in window} beta_s' v'_s' (k'_s' . q'_s)."""
    rng = np.random.default_rng(12)
    F, S, d = 13, 3, 5
    inp = _inputs(rng, d=d, F=F, S=S, alpha_one=True)
    o = O.branch_forward(inp, F, S, "additive", 1.0, chunk, radius, prenorm=True)[0, :, 0, :]
    st = O.head_state(inp, 0, 0, F, S, "additive", 1.0, chunk, radius)
    qf = st["qf"].reshape(-1, d)
    kf = st["kf"].reshape(-1, d)
    vf = st["vf"].reshape(-1, d)
    beta = inp["beta"][0, :, 0]
    for n in range(F * S):
        t = n // S
        acc = np.zeros(d)
        for m in range(F * S):
            g = m // S
            if abs(g // chunk - t // chunk) > radius:       # outside the softmax window
                acc += beta[m] * vf[m] * np.dot(kf[m], qf[n])
        np.testing.assert_allclose(o[n], acc, rtol=1e-11, atol=1e-13)


def test_bridge_decays_across_exactly_the_frames_between():
    """P-vii: additive rule, only frame g carries values: a query frame t outside
    g's window reads B_g diag(prod_{f in (g, t]} alpha_f) (g before the window) or
    B_g diag(prod_{f in [t, g)} alpha_f) (g after it), with B_g summed token by token."""
    rng = np.random.default_rng(13)
    F, S, d, chunk, radius = 17, 2, 5, 3, 1
    for g in (1, 8, 15):
        inp = _inputs(rng, d=d, F=F, S=S)
        vmask = np.zeros(F * S)
        vmask[g * S:(g + 1) * S] = 1
        inp["v"] = inp["v"] * vmask[None, :, None, None]
        inp["conv_v_w"] = None          # keep v zero outside frame g
        o = O.branch_forward(inp, F, S, "additive", 1.0, chunk, radius, prenorm=True)[0, :, 0, :]
        st = O.head_state(inp, 0, 0, F, S, "additive", 1.0, chunk, radius)
        beta = inp["beta"][0, :, 0]
        alpha = inp["alpha"][0, :, 0]
        Bg = sum(beta[g * S + s] * np.outer(st["vf"][g, s], st["kf"][g, s]) for s in range(S))
        for t in range(F):
            if abs(g // chunk - t // chunk) <= radius:
                continue
            frames = range(g + 1, t + 1) if g < t else range(t, g)
            decay = np.ones(d)
            for f in frames:
                decay = decay * alpha[f]
            expect = st["qf"][t] @ (Bg * decay[None, :]).T
            np.testing.assert_allclose(o[t * S:(t + 1) * S], expect, rtol=1e-11, atol=1e-14)


@pytest.mark.parametrize("rule", RULES)
def test_suffix_scan_is_prefix_scan_of_reversed_frames(rule):
    """P-viii (mirror)."""
    rng = np.random.default_rng(14)
    F, d = 10, 5
    R = rng.normal(size=(F, d, d))
    A = np.einsum("fij,fkj->fik", R, R) / d
    Bm = rng.normal(size=(F, d, d))
    alpha = _sig(rng.normal(2, 1, size=(F, d)))
    seed = rng.normal(size=(d, d))
    P, Q = O.bidirectional_scan(A, Bm, alpha, seed, rule, 0.8)
    Pr, _ = O.bidirectional_scan(A[::-1], Bm[::-1], alpha[::-1], seed, rule, 0.8)
    np.testing.assert_allclose(Q, Pr[::-1], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("rule", RULES)
def test_steps_are_affine_maps_that_compose(rule):
    """P-viii (associativity): each frame is S -> S G_f + B'_f, and composing the
    maps of a chunk, (G1,B1) o (G2,B2) = (G1 G2, B1 G2 + B2), equals stepping."""
    rng = np.random.default_rng(15)
    F, d = 5, 6
    R = rng.normal(size=(F, d, d))
    A = np.einsum("fij,fkj->fik", R, R) / d
    Bm = rng.normal(size=(F, d, d))
    alpha = _sig(rng.normal(2, 1, size=(F, d)))
    S0 = rng.normal(size=(d, d))
    G = np.eye(d)
    Bc = np.zeros((d, d))
    Sst = S0
    for f in range(F):
        Bp = O.rule_step(np.zeros((d, d)), A[f], Bm[f], alpha[f], rule, 0.9)
        Gf = O.rule_step(np.eye(d), A[f], Bm[f], alpha[f], rule, 0.9) - Bp
        X = rng.normal(size=(d, d))
        np.testing.assert_allclose(O.rule_step(X, A[f], Bm[f], alpha[f], rule, 0.9), X @ Gf + Bp,
                                   rtol=1e-11, atol=1e-12)
        G, Bc = G @ Gf, Bc @ Gf + Bp
        Sst = O.rule_step(Sst, A[f], Bm[f], alpha[f], rule, 0.9)
    np.testing.assert_allclose(S0 @ G + Bc, Sst, rtol=1e-11, atol=1e-12)


def test_vdn_solve_state_is_stable_over_85_frames():
    """P-ix: with vdn_solve, |(I + A)^-1|_2 <= 1 and alpha <= 1, so
    |P_f|_2 <= |P_{f-1}|_2 + |B'_f|_2 over a 14 s clip's 85 latent frames."""
    rng = np.random.default_rng(16)
    F, S, d = 85, 6, 8
    inp = _inputs(rng, d=d, F=F, S=S, text=True)
    st = O.head_state(inp, 0, 0, F, S, "vdn_solve", 1.0, 5, 1)
    prev = st["seed"]
    alpha = inp["alpha"][0, :, 0]
    for f in range(F):
        M = np.linalg.inv(np.eye(d) + st["A"][f])
        assert np.linalg.norm(M, 2) <= 1 + 1e-12
        Bp = O.rule_step(np.zeros((d, d)), st["A"][f], st["B"][f], alpha[f], "vdn_solve")
        n = np.linalg.norm(st["P"][f], 2)
        assert n <= np.linalg.norm(prev, 2) + np.linalg.norm(Bp, 2) + 1e-12
        prev = st["P"][f]


# ----------------------------------------------------------------------------- step 5
def test_rmsnorm_gate_readout():
    rng = np.random.default_rng(17)
    d, n = 8, 20
    W = rng.normal(size=(d, d))
    qf = O.l2_normalize(rng.normal(size=(n, d)))
    gate = _sig(rng.normal(size=(n, d)))
    w = 1 + 0.1 * rng.normal(size=d)
    y = O.readout(W, qf, np.ones((n, d)), w)
    o = qf @ W.T
    ms = np.mean(o * o, axis=-1)
    np.testing.assert_allclose(np.mean((y / w) ** 2, axis=-1), ms / (ms + 1e-6), rtol=1e-12)
    np.testing.assert_allclose(y / w / o, np.broadcast_to((ms + 1e-6) ** -0.5, (d, n)).T, rtol=1e-12)
    out = O.readout(W, qf, gate, w)
    np.testing.assert_allclose(out, y * gate, rtol=1e-14)
    # scale invariance of the norm (up to eps)
    np.testing.assert_allclose(O.readout(1e3 * W, qf, gate, w), out, rtol=1e-5)


# ----------------------------------------------------------------------------- workloads
def test_tiny_workload_output_is_exactly_zero():
    """P-x: F = 10 frames, chunk 5, radius 1: every window covers all frames and
    there is no text state, so the branch output is identically 0."""
    w = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs(w)
    out = O.branch_forward(inp, w.F, w.S, w.rule, w.c, w.chunk, w.radius)
    assert np.all(out == 0.0)


def test_tiny_f20_workloads_are_not_degenerate():
    for name in ("tiny_f20", "tiny_f20_text"):
        w = synth.WORKLOADS[name]
        inp = synth.make_inputs(w)
        out = O.branch_forward(inp, w.F, w.S, w.rule, w.c, w.chunk, w.radius)
        assert np.isfinite(out).all() and np.abs(out).max() > 0.1


def test_prepare_features_from_library_routines():
    """Step 1 composed from library routines: numpy's 'same' convolution per
    channel and frame, x * expit(x), and division by numpy's vector norm."""
    rng = np.random.default_rng(18)
    F, S, d = 3, 6, 5
    q, k, v = (rng.normal(size=(F * S, d)) for _ in range(3))
    wk, wv = rng.normal(size=(d, 3)), rng.normal(size=(d, 3))
    qf, kf, vf = O.prepare_features(q, k, v, F, S, wk, wv)
    for f in range(F):
        sl = slice(f * S, (f + 1) * S)
        kc = np.stack([np.convolve(k[sl, c], wk[c, ::-1], mode="same") for c in range(d)], axis=1)
        vc = np.stack([np.convolve(v[sl, c], wv[c, ::-1], mode="same") for c in range(d)], axis=1)
        ks = kc * scipy.special.expit(kc)
        qs = q[sl] * scipy.special.expit(q[sl])
        np.testing.assert_allclose(kf[f], ks / np.linalg.norm(ks, axis=1, keepdims=True), rtol=1e-10)
        np.testing.assert_allclose(qf[f], qs / np.linalg.norm(qs, axis=1, keepdims=True), rtol=1e-10)
        np.testing.assert_allclose(vf[f], vc * scipy.special.expit(vc), rtol=1e-12, atol=1e-15)


# ----------------------------------------------------------------------------- sampled outputs
def _frame_edge_tokens(F, S, rng, extra=2):
    """First and last token of every frame plus a few random ones (indices into F*S)."""
    toks = []
    for t in range(F):
        toks += [t * S, t * S + S - 1]
        toks += list(t * S + rng.integers(0, S, size=extra))
    return np.array(sorted(set(int(x) for x in toks)))


@pytest.mark.parametrize("rule", RULES)
@pytest.mark.parametrize("text", [False, True])
def test_sampled_outputs_are_rows_of_the_whole_branch(rule, text):
    """The full-size checker: sampled_outputs(b, h, tokens) must be exactly the
    rows (b, tokens, h) of branch_forward, for every batch and head, the first
    and last token of each frame, and a frame length (S = 7) that is not a
    multiple of anything in the window geometry."""
    rng = np.random.default_rng(40)
    B, H, d, F, S = 2, 3, 6, 13, 7
    inp = _inputs(rng, B=B, H=H, d=d, F=F, S=S, text=text)
    c = 0.5 if rule in ("sana_scaled", "vdn_scaled") else 1.0
    full = O.branch_forward(inp, F, S, rule, c, 5, 1)
    for b in range(B):
        for h in range(H):
            toks = _frame_edge_tokens(F, S, rng)
            got = O.sampled_outputs(inp, F, S, rule, c, 5, 1, b, h, toks)
            np.testing.assert_allclose(got, full[b, toks, h, :], rtol=1e-13, atol=1e-13)


def test_sampled_outputs_prenorm_is_bruteforce_far_field_attention():
    """sampled_outputs against a definition that shares none of its indexing:
    additive rule, alpha = 1, no text, batch 2 and 2 heads: the pre-norm output
    of token n of (b, h) is the beta-weighted linear attention of its q' against
    every token of the frames outside its window."""
    rng = np.random.default_rng(41)
    B, H, d, F, S, chunk, radius = 2, 2, 5, 11, 4, 2, 1
    inp = _inputs(rng, B=B, H=H, d=d, F=F, S=S, alpha_one=True)
    for b in range(B):
        for h in range(H):
            st = O.head_state(inp, b, h, F, S, "additive", 1.0, chunk, radius)
            qf, kf, vf = (st[n].reshape(-1, d) for n in ("qf", "kf", "vf"))
            beta = inp["beta"][b, :, h]
            toks = _frame_edge_tokens(F, S, rng, extra=1)
            got = O.sampled_outputs(inp, F, S, "additive", 1.0, chunk, radius, b, h, toks, prenorm=True)
            for i, n in enumerate(toks):
                t = n // S
                far = [m for m in range(F * S) if abs((m // S) // chunk - t // chunk) > radius]
                ref = sum(beta[m] * vf[m] * np.dot(kf[m], qf[n]) for m in far) if far else np.zeros(d)
                np.testing.assert_allclose(got[i], ref, rtol=1e-11, atol=1e-13)
