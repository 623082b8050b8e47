"""Pins of the float64 backward oracle (oracle/vdn_backward.py) against something
other than itself: central finite differences of the forward oracle, which is
pinned on its own (test_oracle_pins.py).  For L = <dout, out>, every input X and a
random direction U, (L(X + eU) - L(X - eU)) / 2e must equal <dL/dX, U>; the
central difference is exact up to O(e^2) and rounding, far below the 1e-6
relative bound used here.  Every rule, with and without the conv taps and the
text state, and windows clipped at both clip ends are covered; planted mistakes
in the backward (a dropped term, a transposed operand, a wrong sign, an index
off by one) must each fail a check.  CPU only.
"""
import numpy as np
import pytest

from oracle import vdn_backward as BW
from oracle import vdn_oracle as O

F, S, D, H = 7, 3, 4, 2
INPUTS = ["q", "k", "v", "beta", "alpha", "gate", "rms_w", "conv_k_w", "conv_v_w", "text_state"]


def _inputs(seed, conv=True, text=True):
    rng = np.random.default_rng(seed)
    N = F * S
    sig = lambda x: 1 / (1 + np.exp(-x))
    return {
        "q": rng.normal(size=(1, N, H, D)), "k": rng.normal(size=(1, N, H, D)), "v": rng.normal(size=(1, N, H, D)),
        "beta": sig(rng.normal(size=(1, N, H))), "alpha": sig(rng.normal(2.0, 1.0, size=(1, F, H, D))),
        "gate": sig(rng.normal(size=(1, N, H, D))), "rms_w": 1 + 0.1 * rng.normal(size=D),
        "conv_k_w": rng.normal(0, 0.6, size=(H, D, 3)) if conv else None,
        "conv_v_w": rng.normal(0, 0.6, size=(H, D, 3)) if conv else None,
        "text_state": rng.normal(0, 0.5, size=(H, D, D)) if text else None,
    }


def _loss(inp, dout, rule, c, chunk, radius):
    return float(np.sum(dout * O.branch_forward(inp, F, S, rule, c, chunk, radius)))


def _check(inp, rule, c, chunk, radius, seed, eps=1e-5, rtol=1e-6):
    rng = np.random.default_rng(seed)
    dout = rng.normal(size=np.shape(inp["q"]))
    g = BW.branch_backward(inp, dout, F, S, rule, c, chunk, radius)
    bad = []
    for name in INPUTS:
        if inp.get(name) is None:
            assert g["d" + name] is None
            continue
        for _ in range(2):
            U = rng.normal(size=np.shape(inp[name]))
            if name in ("beta", "alpha", "gate"):
                U *= 0.1                                   # stay inside (0, 1)
            plus = dict(inp)
            minus = dict(inp)
            plus[name] = inp[name] + eps * U
            minus[name] = inp[name] - eps * U
            fd = (_loss(plus, dout, rule, c, chunk, radius) - _loss(minus, dout, rule, c, chunk, radius)) / (2 * eps)
            an = float(np.sum(g["d" + name] * U))
            if abs(fd - an) > rtol * (1.0 + abs(fd)):
                bad.append((name, fd, an))
    return bad


RULES = [("vdn_solve", 1.0), ("vdn_scaled", 0.7), ("sana_scaled", 0.5), ("additive", 1.0)]


@pytest.mark.parametrize("rule,c", RULES, ids=[r for r, _ in RULES])
def test_gradients_match_central_differences(rule, c):
    assert _check(_inputs(1), rule, c, chunk=2, radius=1, seed=11) == []


@pytest.mark.parametrize("conv,text", [(False, False), (True, False), (False, True)])
def test_gradients_without_taps_or_text_state(conv, text):
    assert _check(_inputs(2, conv, text), "vdn_solve", 1.0, chunk=3, radius=0, seed=12) == []


def test_gradients_with_a_window_wider_than_the_clip():
    # radius 3 chunks of 2: every window reaches both clip ends, so only the seeds feed W_t
    assert _check(_inputs(3), "vdn_scaled", 0.5, chunk=2, radius=3, seed=13) == []


def test_gate_and_rms_weight_gradients_in_closed_form():
    # dL/dgate = dout * y and dL/drms_w = sum dout * gate * o r: the readout's own outputs
    inp = _inputs(4)
    rng = np.random.default_rng(14)
    dout = rng.normal(size=np.shape(inp["q"]))
    g = BW.branch_backward(inp, dout, F, S, "vdn_solve", 1.0, 2, 1)
    y = O.branch_forward(inp, F, S, "vdn_solve", 1.0, 2, 1) / inp["gate"]
    np.testing.assert_allclose(g["dgate"], dout * y, rtol=1e-12, atol=1e-12)
    yn = y / inp["rms_w"]
    np.testing.assert_allclose(g["drms_w"], np.sum(dout * inp["gate"] * yn, axis=(0, 1, 2)), rtol=1e-11)


def test_zero_upstream_gradient_gives_zero_gradients():
    inp = _inputs(5)
    g = BW.branch_backward(inp, np.zeros(np.shape(inp["q"])), F, S, "vdn_solve", 1.0, 2, 1)
    for name in INPUTS:
        assert np.all(g["d" + name] == 0.0)


# ----------------------------------------------------------------------------- planted mistakes
_orig = {n: getattr(BW, n) for n in ("rule_step_grad", "frame_statistics_grad", "readout_grad",
                                     "l2_normalize_grad", "short_conv_frame_grad", "gather_grad", "silu_grad")}


def _m_dA_sign(*a):
    dS_in, dA, dB, dal = _orig["rule_step_grad"](*a)
    return dS_in, -dA, dB, dal


def _m_dS_in_untransposed(S_in, A_f, B_f, alpha_f, rule, c, dS_out):
    dS_in, dA, dB, dal = _orig["rule_step_grad"](S_in, A_f, B_f, alpha_f, rule, c, dS_out)
    return dS_in.T, dA, dB, dal


def _m_stats_no_symmetric(kf, vf, beta, dA, dB):
    return _orig["frame_statistics_grad"](kf, vf, beta, 2 * np.triu(dA), dB)


def _m_stats_dB_transposed(kf, vf, beta, dA, dB):
    return _orig["frame_statistics_grad"](kf, vf, beta, dA, np.transpose(dB, (0, 2, 1)))


def _m_readout_no_r3(W_t, qf, gate, rms_w, dout):
    o = qf @ W_t.T
    r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + O.RMS_EPS)
    dW, dqf, dgate, drms = _orig["readout_grad"](W_t, qf, gate, rms_w, dout)
    do = dout * gate * rms_w * r
    return do.T @ qf, do @ W_t, dgate, drms


def _m_l2_no_projection(x, g, eps=O.L2_EPS):
    return g / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def _m_conv_flipped(x, w, g):
    return _orig["short_conv_frame_grad"](x, None if w is None else w[:, ::-1], g)


def _m_silu_as_sigmoid(x, g):
    return g / (1.0 + np.exp(-x))


def _m_gather_prefix_one_late(P, Q, seed, alpha_h, t, chunk, radius, dW, acc):
    lo, _ = O.window_bounds(t, P.shape[0], chunk, radius)
    saved = acc["dP"].copy()
    _orig["gather_grad"](P, Q, seed, alpha_h, t, chunk, radius, dW, acc)
    if lo > 1:                                    # the prefix gradient lands one frame early
        moved = acc["dP"][lo - 1] - saved[lo - 1]
        acc["dP"][lo - 1] = saved[lo - 1]
        acc["dP"][lo - 2] += moved


MUTANTS = {
    "dA_sign": ("rule_step_grad", _m_dA_sign),
    "dS_in_transposed": ("rule_step_grad", _m_dS_in_untransposed),
    "stats_dA_not_symmetrised": ("frame_statistics_grad", _m_stats_no_symmetric),
    "stats_dB_transposed": ("frame_statistics_grad", _m_stats_dB_transposed),
    "rmsnorm_r3_term_dropped": ("readout_grad", _m_readout_no_r3),
    "l2_projection_dropped": ("l2_normalize_grad", _m_l2_no_projection),
    "conv_taps_flipped": ("short_conv_frame_grad", _m_conv_flipped),
    "silu_derivative_as_sigmoid": ("silu_grad", _m_silu_as_sigmoid),
    "gather_prefix_one_frame_early": ("gather_grad", _m_gather_prefix_one_late),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_backward_mistake_is_caught(name, monkeypatch):
    fn_name, fn = MUTANTS[name]
    monkeypatch.setattr(BW, fn_name, fn)
    inp = _inputs(6)
    found = _check(inp, "vdn_solve", 1.0, chunk=2, radius=1, seed=16) + \
        _check(inp, "sana_scaled", 0.5, chunk=2, radius=0, seed=17)
    assert found, f"planted mistake {name} went unnoticed"
