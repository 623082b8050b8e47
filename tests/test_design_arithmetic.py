"""The arithmetic the tensor-core path uses in place of the plain definition, checked against it.

The kernels do not evaluate the oracle's formulas literally in four places:
  * scans: each state is kept as 2^e x an fp32 matrix.  After a step whose result has an entry
    above 2^32 the matrix is multiplied by 2^-32 and e grows by 32; B_f enters the next steps
    scaled by 2^-e (through the rule's coefficients); a stored state is the matrix before that
    rescale, with its e;
  * gather: the two bridged sides are added after aligning them to the larger exponent;
  * read-out: the scaled row is normalised with the RMSNorm eps scaled by 2^-2e;
  * scan products: X N runs as Xh Nl + Xh Nh + Xl Nh on bf16 hi/lo splits, accumulated in fp32.
Each scheme is restated here in float64 and compared with the oracle ("Step 4" and "Step 5" of
"VDN-Minimax-H3 bidirectional linear branch in five steps"): exactly where the scheme only moves
powers of two, within the derived bound for the hi/lo products.  These check the schemes, not the
kernels; the GPU parity tests check the kernels."""
import numpy as np
import pytest
import torch

from oracle import vdn_oracle as O

RENORM_ABOVE = 2.0 ** 32
RENORM_EXP = 32


def _divergent_frames(F=31, S=1024, d=16, seed=7):
    """Per-frame A, B from SiLU / L2 features with a large common component (as the workloads'
    k' have), so sana_scaled at c = 1 grows the state by a factor of tens per frame."""
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((F * S, d))
    v = rng.standard_normal((F * S, d))
    _, kf, vf = O.prepare_features(k, k, v, F, S)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((F, S))))
    A, Bm = O.frame_statistics(kf, vf, beta)
    alpha = 1.0 / (1.0 + np.exp(-(2.0 + rng.standard_normal((F, d)))))
    seed_T = O.seed_state(0.5 * rng.normal(0.0, 0.1, (d, d)), d)
    return A, Bm, alpha, seed_T


def _aligned_frames(F=12, S=4096, d=16, seed=3):
    """The worst case of the growth bound: every token of a frame carries the same unit key
    with beta = 1, so A = S u u^T and |1 - c^2 lambda_max| = S - 1 at c = 1."""
    rng = np.random.default_rng(seed)
    A = np.empty((F, d, d))
    Bm = np.empty((F, d, d))
    for f in range(F):
        u = rng.standard_normal(d)
        u /= np.linalg.norm(u)
        A[f] = S * np.outer(u, u)
        w = rng.standard_normal(d)
        Bm[f] = S * np.outer(w / np.linalg.norm(w), u)
    alpha = np.ones((F, d))
    return A, Bm, alpha, np.eye(d)


def _scan_block_exponent(A, Bm, alpha, seed, rule, c, order):
    """One scan direction with the kernels' block exponent: returns the stored matrices and
    their exponents in frame order (state = 2^e x matrix)."""
    s, e = seed.copy(), 0
    mats, exps = np.empty_like(A), np.zeros(A.shape[0], dtype=np.int64)
    for f in order:
        s = O.rule_step(s, A[f], np.ldexp(Bm[f], -e), alpha[f], rule, c)
        mats[f], exps[f] = s, e
        if np.abs(s).max() > RENORM_ABOVE:
            s = np.ldexp(s, -RENORM_EXP)
            e += RENORM_EXP
    return mats, exps


@pytest.mark.parametrize("rule,c", [("sana_scaled", 1.0), ("sana_scaled", 0.5), ("vdn_scaled", 1.0),
                                    ("vdn_solve", 1.0)])
def test_block_exponent_scan_reproduces_the_states(rule, c):
    A, Bm, alpha, seed = _divergent_frames()
    F = A.shape[0]
    P, Q = O.bidirectional_scan(A, Bm, alpha, seed, rule, c)
    Pm, Pe = _scan_block_exponent(A, Bm, alpha, seed, rule, c, range(F))
    Qm, Qe = _scan_block_exponent(A, Bm, alpha, seed, rule, c, reversed(range(F)))
    for f in range(F):
        assert np.array_equal(np.ldexp(Pm[f], Pe[f]), P[f])
        assert np.array_equal(np.ldexp(Qm[f], Qe[f]), Q[f])
    if rule == "sana_scaled" and c == 1.0:
        assert np.abs(P[-1]).max() > 2.0 ** 128        # beyond fp32: the exponent is needed
        assert Pe[-1] >= 128
    if rule != "sana_scaled":
        assert Pe.max() == 0 and Qe.max() == 0         # the exact-solve rules contract


@pytest.mark.parametrize("make", [_divergent_frames, _aligned_frames])
@pytest.mark.parametrize("c", [1.0, 0.5])
def test_stored_states_stay_below_two_to_48(make, c):
    # one step grows a row norm by at most 1 + c^2 S (|k'| = 1, beta <= 1, alpha <= 1), and a
    # matrix whose entries are at most 2^32 has row norms at most 2^32 sqrt(d): the fp32 gather
    # can add two aligned sides without overflow
    A, Bm, alpha, seed = make()
    F = A.shape[0]
    for order in (range(F), reversed(range(F))):
        mats, _ = _scan_block_exponent(A, Bm, alpha, seed, "sana_scaled", c, order)
        assert np.abs(mats).max() < 2.0 ** 48
    # the same bound at the kernels' sizes: d = 128, S up to 4096 tokens per frame
    assert 2.0 ** 32 * np.sqrt(128) * (1 + c * c * 4096) < 2.0 ** 48


@pytest.mark.parametrize("chunk,radius", [(5, 1), (3, 0), (4, 2)])
def test_aligned_gather_and_scaled_eps_readout_reproduce_the_output(chunk, radius):
    A, Bm, alpha, seed = _divergent_frames()
    F, d = A.shape[0], A.shape[1]
    rule, c = "sana_scaled", 1.0
    P, Q = O.bidirectional_scan(A, Bm, alpha, seed, rule, c)
    Pm, Pe = _scan_block_exponent(A, Bm, alpha, seed, rule, c, range(F))
    Qm, Qe = _scan_block_exponent(A, Bm, alpha, seed, rule, c, reversed(range(F)))
    rng = np.random.default_rng(11)
    q = O.l2_normalize(O.silu(rng.standard_normal((8, d))))
    gate = 1.0 / (1.0 + np.exp(-rng.standard_normal((8, d))))
    rms_w = 1.0 + 0.1 * rng.standard_normal(d)
    for t in range(F):
        lo, hi = O.window_bounds(t, F, chunk, radius)
        pre, ep = (seed, 0) if lo == 0 else (Pm[lo - 1], Pe[lo - 1])
        suf, eq = (seed, 0) if hi == F - 1 else (Qm[hi + 1], Qe[hi + 1])
        dpre = np.prod(alpha[lo:t + 1], axis=0)
        dsuf = np.prod(alpha[t:hi + 1], axis=0)
        em = max(ep, eq)
        W_e = np.ldexp(pre * dpre[None, :], ep - em) + np.ldexp(suf * dsuf[None, :], eq - em)
        W = O.gather_state(P, Q, seed, alpha, t, chunk, radius)
        assert np.array_equal(np.ldexp(W_e, em), W)
        o = q @ W_e.T
        y = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + np.ldexp(O.RMS_EPS, -2 * em)) * rms_w
        assert np.array_equal(y * gate, O.readout(W, q, gate, rms_w))


def _bf16(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest even) and back, exactly."""
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def test_hi_lo_product_keeps_sixteen_bits():
    # X = Xh + Xl + dX, |Xl| <= 2^-8 |X|, |dX| <= 2^-16 |X| (same for N): the dropped terms
    # Xl Nl, Xh dN, dX N are each at most about 2^-16 |X| |N|
    rng = np.random.default_rng(5)
    d = 128
    X = (rng.standard_normal((d, d)) * np.exp2(rng.integers(-6, 7, (d, d)))).astype(np.float32).astype(np.float64)
    K = O.l2_normalize(O.silu(rng.standard_normal((512, d))))
    N = np.linalg.inv(np.eye(d) + (K.T * rng.uniform(0, 1, 512)) @ K).astype(np.float32).astype(np.float64)
    Xh = _bf16(X)
    Xl = _bf16((X.astype(np.float32) - Xh.astype(np.float32)).astype(np.float64))
    Nh = _bf16(N)
    Nl = _bf16((N.astype(np.float32) - Nh.astype(np.float32)).astype(np.float64))
    got = Xh @ Nl + Xh @ Nh + Xl @ Nh
    exact = X @ N
    scale = np.abs(X) @ np.abs(N)
    assert np.all(np.abs(got - exact) <= 3.1 * 2.0 ** -16 * scale)
    # a single bf16 product misses that bound by far: the split is what buys the bits
    plain = Xh @ Nh
    assert np.max(np.abs(plain - exact) / scale) > 2.0 ** -12


def _sweep_every_pivot(M: np.ndarray, dtype=np.float64):
    """The per-frame solve's elimination, without pivoting: for pivot k with d = M[k, k],
    M[i, j] -= (M[i, k] / d) M[k, j] for every (i, j), then row and column k divided by d and
    M[k, k] = -1 / d.  Sweeping every pivot of a symmetric positive definite M leaves -M^-1.
    Returns that matrix and the pivots in elimination order."""
    M = M.astype(dtype).copy()
    piv = np.empty(M.shape[0])
    for k in range(M.shape[0]):
        d = M[k, k]
        piv[k] = d
        r = dtype(1) / d
        col, row = M[:, k].copy(), M[k, :].copy()
        M -= np.outer(col * r, row)
        M[k, :] = row * r
        M[:, k] = col * r
        M[k, k] = -r
    return M, piv


def _frame_matrix(d, S, c, seed):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((S, d))
    _, kf, _ = O.prepare_features(k, k, k, 1, S)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((1, S))))
    A, _ = O.frame_statistics(kf, kf, beta)
    return np.eye(d) + c * c * A[0]


@pytest.mark.parametrize("d,S,c", [(16, 1024, 1.0), (128, 1024, 1.0), (128, 4096, 0.5)])
def test_sweep_without_pivoting_inverts_and_every_pivot_is_at_least_one(d, S, c):
    # every pivot is a Schur complement of M = I + c^2 A; its inverse is a diagonal block of
    # M^-1, which is at most I because M is at least I, so each pivot is at least 1: the
    # elimination never divides by a small number and needs no row exchanges
    M = _frame_matrix(d, S, c, seed=d + S)
    neg_inv, piv = _sweep_every_pivot(M)
    assert piv.min() >= 1.0 - 1e-12
    np.testing.assert_allclose(-neg_inv, np.linalg.inv(M), rtol=0, atol=1e-13)
    # the rule step with the swept inverse equals the oracle's solve
    rng = np.random.default_rng(1)
    S_in, Bf = rng.standard_normal((d, d)), rng.standard_normal((d, d))
    alpha = rng.uniform(0.5, 1.0, d)
    A = (M - np.eye(d)) / (c * c)
    X = S_in @ np.diag(alpha) + c * Bf
    np.testing.assert_allclose(X @ -neg_inv, O.rule_step(S_in, A, Bf, alpha, "vdn_scaled", c), rtol=0, atol=1e-12)


def test_fp32_sweep_error_within_the_conditioning_bound():
    # in fp32 the sweep's forward error stays within n u cond(M) of the inverse's largest
    # entry (u = 2^-24): the solve's fp32 arithmetic is as accurate as the problem allows
    d = 128
    M = _frame_matrix(d, 4096, 1.0, seed=2)
    neg_inv32, piv32 = _sweep_every_pivot(M.astype(np.float32), np.float32)
    inv = np.linalg.inv(M)
    cond = np.linalg.cond(M)
    assert cond > 10                                   # lambda_max(A) ~ 250: one dominant key direction
    err = np.abs(-neg_inv32.astype(np.float64) - inv).max()
    assert err <= d * 2.0 ** -24 * cond * np.abs(inv).max()
    assert piv32.min() >= 1.0 - 1e-4


def test_fp16_row_block_image_of_w_keeps_eleven_bits():
    # the gather scales W_t by the power of two that puts its largest entry in [0.5, 1), then
    # writes each block of 32 rows in fp16 scaled again so that the block's largest entry is in
    # [0.5, 1); the read-out undoes both exponents in its RMSNorm.  Each entry then carries fp16's
    # 11 significant bits (2^-25 absolute below the block's normal range).
    A, Bm, alpha, seed = _divergent_frames(d=128)
    F, d = A.shape[0], A.shape[1]
    P, Q = O.bidirectional_scan(A, Bm, alpha, seed, "sana_scaled", 1.0)
    rng = np.random.default_rng(4)
    q = O.l2_normalize(O.silu(rng.standard_normal((64, d))))
    gate = 1.0 / (1.0 + np.exp(-rng.standard_normal((64, d))))
    rms_w = 1.0 + 0.1 * rng.standard_normal(d)
    worst = {"fp16": 0.0, "bf16": 0.0}
    for t in range(F):
        W = O.gather_state(P, Q, seed, alpha, t, 5, 1)
        _, ew = np.frexp(np.abs(W).max())
        Wn = np.ldexp(W, -int(ew))                                    # largest entry in [0.5, 1)
        _, eb = np.frexp(np.abs(Wn).reshape(d // 32, -1).max(axis=1))
        eb = np.repeat(np.clip(eb, -125, 126), 32)[:, None]
        img = np.ldexp(Wn, -eb).astype(np.float16).astype(np.float64)
        back = np.ldexp(img, eb)
        bound = np.ldexp(np.maximum(2.0 ** -11 * np.abs(np.ldexp(Wn, -eb)), 2.0 ** -25), eb)
        assert np.all(np.abs(back - Wn) <= bound)
        ref = O.readout(W, q, gate, rms_w)
        for name, img_w in (("fp16", back), ("bf16", np.ldexp(_bf16(np.ldexp(Wn, -eb)), eb))):
            o = q @ img_w.T
            y = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + np.ldexp(O.RMS_EPS, -2 * int(ew))) * rms_w
            worst[name] = max(worst[name], np.abs(y * gate - ref).max() / np.abs(ref).max())
    assert np.abs(P[-1]).max() > 2.0 ** 128
    assert worst["fp16"] < 2e-3 and worst["bf16"] > 4 * worst["fp16"]   # the three extra bits show


def _lazy_two_group_softmax(qr, kr, v, scale, tile=128, move_above=8.0):
    """The windowed softmax kernel's schedule for one block of query rows: key tiles alternate
    between two groups; each group keeps, per row, a reference maximum m (log2 units), a running
    normaliser l and an accumulator O, and moves m to a tile's maximum only when that maximum
    exceeds m by more than `move_above` (O and l then scaled by 2^(m_old - m_new)); exponents
    are taken against m, so every weight is at most 2^move_above.  The groups are combined at
    the end against their larger reference.  Returns the output and the largest weight used."""
    n, L = qr.shape[0], kr.shape[0]
    s2 = (qr @ kr.T) * scale * np.log2(np.e)                     # scores in log2 units
    m = np.full((2, n), -np.inf)
    l = np.zeros((2, n))
    acc = np.zeros((2, n, v.shape[1]))
    pmax = 0.0
    for j, t0 in enumerate(range(0, L, tile)):
        g, t1 = j % 2, min(L, t0 + tile)
        tmax = s2[:, t0:t1].max(axis=1)
        move = tmax > m[g] + move_above
        corr = np.where(move, np.exp2(np.where(np.isinf(m[g]), -np.inf, m[g] - tmax)), 1.0)
        l[g] *= corr
        acc[g] *= corr[:, None]
        m[g] = np.where(move, tmax, m[g])
        p = np.exp2(s2[:, t0:t1] - m[g][:, None])
        pmax = max(pmax, p.max())
        l[g] += p.sum(axis=1)
        acc[g] += p @ v[t0:t1]
    top = m.max(axis=0)
    w = np.where(np.isinf(m), 0.0, np.exp2(m - top))
    return (acc[0] * w[0][:, None] + acc[1] * w[1][:, None]) / (l[0] * w[0] + l[1] * w[1])[:, None], pmax


@pytest.mark.parametrize("L,rising", [(128, False), (200, False), (1000, True), (4 * 1560 + 37, True)])
def test_lazy_reference_two_group_softmax_equals_softmax(L, rising):
    rng = np.random.default_rng(L)
    d = 32
    qr = 2.0 * rng.standard_normal((16, d))
    kr = rng.standard_normal((L, d))
    if rising:                                       # key norms rising along the window: the
        kr *= np.linspace(0.5, 6.0, L)[:, None]      # reference maximum moves again and again
    v = rng.standard_normal((L, d))
    scale = 1.0 / np.sqrt(d)
    got, pmax = _lazy_two_group_softmax(qr, kr, v, scale)
    np.testing.assert_allclose(got, O.window_softmax_frame(qr, kr, v, scale), rtol=0, atol=1e-12)
    assert pmax <= 2.0 ** 8 * (1 + 1e-12)            # stored as bf16 without overflow, l < L 2^8


# The kernels run every rule as one generic step with coefficients (cpre, cpost, c2, solve,
# identity):  S_out = (S_in D + cpre B) N + cpost B,  N = (I + c2 A)^-1 (solve), I - c2 A, or I.
_RULE_COEF = {
    "vdn_solve": lambda c: (1.0, 0.0, 1.0, True, False),
    "vdn_scaled": lambda c: (c, 0.0, c * c, True, False),
    "sana_scaled": lambda c: (0.0, c, c * c, False, False),
    "additive": lambda c: (1.0, 0.0, 0.0, False, True),
}


def _generic_step_and_adjoint(S_in, A, B, alpha, rule, c, lam):
    """The generic step and its adjoint as the backward kernels form them from the forward's
    explicit N: dX = lam N^T, dS_in = dX D, dB = cpre dX + cpost lam, dalpha_j = sum_i S_in[i, j]
    dX[i, j], and dA = -c2 S_out^T dX when N is an inverse (dN^-1 = -N^T dN N^T), -c2 X^T lam
    when N = I - c2 A, 0 for the identity."""
    cpre, cpost, c2, solve, identity = _RULE_COEF[rule](c)
    d = A.shape[0]
    N = np.eye(d) if identity else (np.linalg.inv(np.eye(d) + c2 * A) if solve else np.eye(d) - c2 * A)
    X = S_in * alpha[None, :] + cpre * B
    S_out = X @ N + cpost * B
    dX = lam @ N.T
    dA = np.zeros_like(A) if identity else (-c2 * S_out.T @ dX if solve else -c2 * X.T @ lam)
    return S_out, (dX * alpha[None, :], dA, cpre * dX + cpost * lam, np.sum(S_in * dX, axis=0))


@pytest.mark.parametrize("rule,c", [("vdn_solve", 1.0), ("vdn_scaled", 0.6), ("sana_scaled", 0.3),
                                    ("additive", 1.0)])
def test_generic_step_and_its_adjoint_match_the_oracles_rules(rule, c):
    from oracle import vdn_backward as OB
    A, Bm, alpha, _ = _divergent_frames(F=3, S=64, d=16)
    rng = np.random.default_rng(9)
    for f in range(A.shape[0]):
        S_in = rng.standard_normal((16, 16))
        lam = rng.standard_normal((16, 16))
        S_out, grads = _generic_step_and_adjoint(S_in, A[f], Bm[f], alpha[f], rule, c, lam)
        ref_out = O.rule_step(S_in, A[f], Bm[f], alpha[f], rule, c)
        np.testing.assert_allclose(S_out, ref_out, rtol=0, atol=1e-12 * np.abs(ref_out).max())
        for got, ref in zip(grads, OB.rule_step_grad(S_in, A[f], Bm[f], alpha[f], rule, c, lam)):
            np.testing.assert_allclose(got, ref, rtol=0, atol=1e-11 * max(1.0, np.abs(ref).max()))


def test_stream_k_owner_and_partial_slots():
    # CTA i of G owns units [floor(i T / G), floor((i + 1) T / G)) of the T (frame, block) units,
    # frames in unit order; the solve finds the CTAs covering a frame from the closed form
    # owner(x) = ceil((x + 1) G / T) - 1 and reads slot (CTA + frame).  The closed form must be the
    # CTA whose range holds x, and no two (CTA, frame) pairs may share a slot.
    rng = np.random.default_rng(0)
    cases = [(744, 42, 148), (31, 42, 148), (1, 1, 148), (3, 5, 148), (2976, 43, 148), (5, 1, 7)]
    cases += [(int(rng.integers(1, 400)), int(rng.integers(1, 50)), int(rng.integers(1, 300))) for _ in range(40)]
    for NF, nb, G0 in cases:
        T = NF * nb
        G = min(G0, T)
        begin = [(i * T) // G for i in range(G + 1)]
        owner_def = np.repeat(np.arange(G), np.diff(begin))           # the CTA holding each unit
        x = np.arange(T)
        owner = -((-(x + 1) * G) // T) - 1                           # ceil((x + 1) G / T) - 1
        assert np.array_equal(owner, owner_def)
        slots = {}
        for i in range(G):
            for pf in range(begin[i] // nb, (begin[i + 1] - 1) // nb + 1) if begin[i + 1] > begin[i] else ():
                assert (i + pf) not in slots
                slots[i + pf] = (i, pf)
        assert max(slots) < NF + G
        for pf in range(NF):                                          # the solve's CTA range per frame
            i0, i1 = owner[pf * nb], owner[pf * nb + nb - 1]
            assert {i for i, f in slots.values() if f == pf} == set(range(i0, i1 + 1))
