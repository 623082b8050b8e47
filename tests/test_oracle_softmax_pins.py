"""Pins of the oracle's windowed softmax branch and of the hybrid sum against
things other than the oracle itself: closed forms (uniform weights give the
window mean, one dominant key gives its value), invariances (a key outside the
window cannot matter; a common shift of one query's scores cannot matter) and a
library routine (torch's scaled_dot_product_attention with a boolean window mask).
A wrong scale, an off-by-one window, a missing max subtraction or a transposed
operand fails at least one test.  Mutations planted in the oracle are checked in
test_oracle_mutations.py.  CPU only.
"""
import numpy as np
import pytest
import torch

from oracle import vdn_oracle as O


def _rope_inputs(rng, B=1, H=2, d=8, F=12, S=4, qsd=2.0):
    N = F * S
    return {
        "q_rope": qsd * rng.normal(size=(B, N, H, d)),
        "k_rope": rng.normal(size=(B, N, H, d)),
        "v": rng.normal(size=(B, N, H, d)),
    }


def _window_of(t, F, chunk, radius):
    # chunk-aligned window written out from the page's description: the query's
    # chunk and `radius` chunks on each side, clipped to the clip
    first_chunk = max(0, t // chunk - radius)
    last_frame = min(F - 1, (t // chunk + radius + 1) * chunk - 1)
    return first_chunk * chunk, last_frame


@pytest.mark.parametrize("chunk,radius", [(5, 1), (3, 0), (2, 2)])
def test_uniform_scores_give_the_window_mean(chunk, radius):
    rng = np.random.default_rng(1)
    F, S = 12, 4
    inp = _rope_inputs(rng, F=F, S=S)
    inp["q_rope"][:] = 0.0                      # every score 0: uniform weights
    out = O.window_softmax_forward(inp, F, S, chunk, radius)
    v = inp["v"]
    for t in range(F):
        lo, hi = _window_of(t, F, chunk, radius)
        mean = v[:, lo * S:(hi + 1) * S].mean(axis=1)     # [B, H, d]
        for s in range(S):
            np.testing.assert_allclose(out[:, t * S + s], mean, rtol=1e-12, atol=1e-12)


def test_one_dominant_key_inside_the_window_selects_its_value():
    rng = np.random.default_rng(2)
    F, S, d = 12, 4, 8
    inp = _rope_inputs(rng, F=F, S=S, d=d, qsd=0.01)
    n_q, n_k = 7 * S + 1, 5 * S + 2             # frame 7 (chunk 1, window 0..14 -> 0..11), key in frame 5
    inp["k_rope"][0, n_k, 0] = 1e3 * inp["q_rope"][0, n_q, 0] / np.linalg.norm(inp["q_rope"][0, n_q, 0]) ** 2
    out = O.window_softmax_forward(inp, F, S, 5, 1, heads=[0])
    np.testing.assert_allclose(out[0, n_q, 0], inp["v"][0, n_k, 0], rtol=1e-9, atol=1e-9)


def test_a_key_outside_the_window_has_no_influence():
    rng = np.random.default_rng(3)
    F, S, d = 20, 3, 8
    inp = _rope_inputs(rng, F=F, S=S, d=d)
    ref = O.window_softmax_forward(inp, F, S, 5, 1, heads=[1])
    # query frame 2 (chunk 0): window 0..9; frame 10 is outside
    t, n_out = 2, 10 * S + 1
    inp2 = {k: v.copy() for k, v in inp.items()}
    q = inp2["q_rope"][0, t * S, 1]
    inp2["k_rope"][0, n_out, 1] = 1e6 * q
    inp2["v"][0, n_out, 1] = 1e6
    out = O.window_softmax_forward(inp2, F, S, 5, 1, heads=[1])
    np.testing.assert_array_equal(out[0, t * S:(t + 1) * S, 1], ref[0, t * S:(t + 1) * S, 1])
    # and a frame-10 query does see it (frame 10 is in its own window)
    assert not np.allclose(out[0, 10 * S:11 * S, 1], ref[0, 10 * S:11 * S, 1])


def test_common_shift_of_one_querys_scores_is_invisible():
    rng = np.random.default_rng(4)
    F, S, d = 10, 4, 8
    inp = _rope_inputs(rng, F=F, S=S, d=d)
    n = 3 * S + 2
    ref = O.sampled_window_softmax(inp, F, S, 5, 1, 0, 0, [n])
    # k_j -> k_j + u with q_n . u = 700 for every key j: every score of query n moves by the same amount
    q = inp["q_rope"][0, n, 0]
    inp2 = {k: v.copy() for k, v in inp.items()}
    inp2["k_rope"][0, :, 0] += 700.0 * q / np.dot(q, q)
    out = O.sampled_window_softmax(inp2, F, S, 5, 1, 0, 0, [n])
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("chunk,radius,scale", [(5, 1, None), (4, 0, None), (3, 1, 0.37)])
def test_matches_masked_scaled_dot_product_attention(chunk, radius, scale):
    rng = np.random.default_rng(5)
    B, H, d, F, S = 2, 3, 16, 11, 5
    inp = _rope_inputs(rng, B=B, H=H, d=d, F=F, S=S)
    out = O.window_softmax_forward(inp, F, S, chunk, radius, scale=scale)
    N = F * S
    mask = torch.zeros(N, N, dtype=torch.bool)
    for t in range(F):
        lo, hi = _window_of(t, F, chunk, radius)
        mask[t * S:(t + 1) * S, lo * S:(hi + 1) * S] = True
    q = torch.from_numpy(inp["q_rope"]).permute(0, 2, 1, 3)
    k = torch.from_numpy(inp["k_rope"]).permute(0, 2, 1, 3)
    v = torch.from_numpy(inp["v"]).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
    np.testing.assert_allclose(out, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-10, atol=1e-12)


def test_sampled_outputs_agree_with_the_full_branch():
    rng = np.random.default_rng(6)
    F, S = 12, 4
    inp = _rope_inputs(rng, F=F, S=S)
    full = O.window_softmax_forward(inp, F, S, 5, 1)
    toks = [0, 5, 17, 33, 47]
    np.testing.assert_allclose(O.sampled_window_softmax(inp, F, S, 5, 1, 0, 1, toks), full[0, toks, 1],
                               rtol=1e-13, atol=1e-13)


def test_large_scores_do_not_overflow():
    rng = np.random.default_rng(7)
    F, S = 10, 4
    inp = _rope_inputs(rng, F=F, S=S, qsd=400.0)      # scores of order 1e3: exp would overflow unshifted
    out = O.window_softmax_forward(inp, F, S, 5, 1)
    assert np.isfinite(out).all()
    assert np.abs(out).max() <= np.abs(inp["v"]).max() + 1e-12   # a convex combination of values


def test_hybrid_is_the_sum_of_the_two_branches():
    rng = np.random.default_rng(8)
    B, H, d, F, S = 1, 2, 6, 12, 3
    N = F * S
    sig = lambda x: 1 / (1 + np.exp(-x))
    inp = _rope_inputs(rng, B=B, H=H, d=d, F=F, S=S)
    inp.update({
        "q": rng.normal(size=(B, N, H, d)), "k": rng.normal(size=(B, N, H, d)),
        "beta": sig(rng.normal(size=(B, N, H))), "alpha": sig(rng.normal(2.0, 1.0, size=(B, F, H, d))),
        "gate": sig(rng.normal(size=(B, N, H, d))), "rms_w": 1 + 0.1 * rng.normal(size=d),
        "conv_k_w": None, "conv_v_w": None, "text_state": None,
    })
    hyb = O.hybrid_forward(inp, F, S)
    lin = O.branch_forward(inp, F, S)
    soft = O.window_softmax_forward(inp, F, S)
    np.testing.assert_allclose(hyb, lin + soft, rtol=0, atol=0)
