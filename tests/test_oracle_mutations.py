"""Plants plausible mistakes in the oracle (CPU only, via monkeypatch) and checks
that at least one pin in test_oracle_pins.py fails for each of them."""
import numpy as np
import pytest

from oracle import vdn_oracle as O
import test_oracle_pins as pins

_orig = {name: getattr(O, name) for name in
         ("window_bounds", "frame_statistics", "rule_step", "gather_state", "seed_state",
          "prepare_features", "readout", "short_conv_frame", "sampled_outputs")}


def _window_hi_plus_one(t, F, chunk, radius):
    c = t // chunk
    return max(0, chunk * (c - radius)), min(F - 1, chunk * (c + radius + 1))


def _stats_B_transposed(kf, vf, beta):
    A, Bm = _orig["frame_statistics"](kf, vf, beta)
    return A, np.swapaxes(Bm, -1, -2)


def _stats_no_beta(kf, vf, beta):
    return _orig["frame_statistics"](kf, vf, np.ones_like(beta))


def _rule_D_on_left(S_in, A_f, B_f, alpha_f, rule, c=1.0):
    return _orig["rule_step"](np.diag(alpha_f) @ S_in @ np.diag(1 / alpha_f), A_f, B_f, alpha_f, rule, c)


def _rule_sana_sign(S_in, A_f, B_f, alpha_f, rule, c=1.0):
    if rule == "sana_scaled":
        return (S_in @ np.diag(alpha_f)) @ (np.eye(A_f.shape[0]) + c * c * A_f) + c * B_f
    return _orig["rule_step"](S_in, A_f, B_f, alpha_f, rule, c)


def _rule_solve_transposed(S_in, A_f, B_f, alpha_f, rule, c=1.0):
    if rule in ("vdn_solve", "vdn_scaled"):
        cc = 1.0 if rule == "vdn_solve" else c
        X = S_in @ np.diag(alpha_f) + cc * B_f
        return np.linalg.solve(np.eye(A_f.shape[0]) + cc * cc * A_f + 0.01 * np.triu(A_f, 1), X)
    return _orig["rule_step"](S_in, A_f, B_f, alpha_f, rule, c)


def _rule_c_dropped(S_in, A_f, B_f, alpha_f, rule, c=1.0):
    if rule == "vdn_scaled":
        return _orig["rule_step"](S_in, A_f, B_f, alpha_f, "vdn_solve")
    return _orig["rule_step"](S_in, A_f, B_f, alpha_f, rule, c)


def _gather_whole_window(P, Q, seed, alpha_h, t, chunk, radius, bridge="to_query"):
    return _orig["gather_state"](P, Q, seed, alpha_h, t, chunk, radius, "window")


def _gather_no_bridge(P, Q, seed, alpha_h, t, chunk, radius, bridge="to_query"):
    F = P.shape[0]
    lo, hi = O.window_bounds(t, F, chunk, radius)
    pre = seed if lo == 0 else P[lo - 1]
    suf = seed if hi == F - 1 else Q[hi + 1]
    return pre + suf


def _seed_full(text_state_h, d):
    return 2.0 * _orig["seed_state"](text_state_h, d)


def _features_no_silu_k(qh, kh, vh, F, S, wk=None, wv=None, silu_v=True, causal=False):
    d = qh.shape[-1]
    qf, _, vf = _orig["prepare_features"](qh, kh, vh, F, S, wk, wv, silu_v, causal)
    k = kh.reshape(F, S, d)
    kc = np.stack([O.short_conv_frame(k[f], wk, causal) for f in range(F)])
    return qf, O.l2_normalize(kc), vf


def _conv_flipped(x, w, causal=False):
    return _orig["short_conv_frame"](x, None if w is None else w[:, ::-1], causal)


def _readout_no_gate(W_t, qf_tokens, gate_tokens, rms_w, prenorm=False):
    return _orig["readout"](W_t, qf_tokens, np.ones_like(gate_tokens), rms_w, prenorm)


def _readout_W_transposed(W_t, qf_tokens, gate_tokens, rms_w, prenorm=False):
    return _orig["readout"](W_t.T, qf_tokens, gate_tokens, rms_w, prenorm)


def _sampled_with(frame_of, gate_row):
    """sampled_outputs with its token -> (frame, gate row) indexing replaced."""
    def mutant(inp, F, S, rule, c, chunk, radius, b, h, tokens, prenorm=False):
        st = O.head_state(inp, b, h, F, S, rule, c, chunk, radius)
        rms_w = np.asarray(inp["rms_w"], dtype=np.float64)
        g = np.asarray(inp["gate"][b, :, h, :], dtype=np.float64)
        res = np.empty((len(tokens), st["qf"].shape[-1]))
        for i, n in enumerate(np.asarray(tokens)):
            t, s = frame_of(int(n), S, F), int(n) % S
            res[i] = O.readout(st["W"][t], st["qf"][t, s][None, :], g[gate_row(int(n), S)][None, :], rms_w,
                               prenorm)[0]
        return res
    return mutant


# the last token of a frame read with the next frame's state
_sampled_frame_off_by_one = _sampled_with(lambda n, S, F: min((n + 1) // S, F - 1), lambda n, S: n)
# the gate row taken frame-local (token s of frame 0) instead of clip-wide
_sampled_gate_frame_local = _sampled_with(lambda n, S, F: n // S, lambda n, S: n % S)


MUTANTS = {
    "window_hi_plus_one": ("window_bounds", _window_hi_plus_one),
    "stats_B_transposed": ("frame_statistics", _stats_B_transposed),
    "stats_no_beta": ("frame_statistics", _stats_no_beta),
    "rule_D_on_left": ("rule_step", _rule_D_on_left),
    "rule_sana_sign": ("rule_step", _rule_sana_sign),
    "rule_solve_wrong_matrix": ("rule_step", _rule_solve_transposed),
    "rule_c_dropped": ("rule_step", _rule_c_dropped),
    "gather_whole_window": ("gather_state", _gather_whole_window),
    "gather_no_bridge": ("gather_state", _gather_no_bridge),
    "seed_full_text": ("seed_state", _seed_full),
    "features_no_silu_k": ("prepare_features", _features_no_silu_k),
    "conv_flipped": ("short_conv_frame", _conv_flipped),
    "readout_no_gate": ("readout", _readout_no_gate),
    "readout_W_transposed": ("readout", _readout_W_transposed),
    "sampled_frame_off_by_one": ("sampled_outputs", _sampled_frame_off_by_one),
    "sampled_gate_frame_local": ("sampled_outputs", _sampled_gate_frame_local),
}

PINS = [
    lambda: pins.test_window_partitions_frames(3, 1),
    lambda: pins.test_window_page_geometry(),
    lambda: pins.test_short_conv_is_numpy_convolve_same(3),
    lambda: pins.test_frame_statistics_is_sum_of_outer_products(),
    lambda: pins.test_solve_is_ridge_regression_least_squares(0.5),
    lambda: pins.test_sana_vs_vdn_scaled_small_c(),
    lambda: pins.test_one_token_per_frame_is_gated_delta_rule("vdn_solve"),
    lambda: pins.test_one_token_per_frame_is_gated_delta_rule("sana_scaled"),
    lambda: pins.test_text_state_only_decays_to_half_prompt("vdn_solve"),
    lambda: pins.test_additive_unit_alpha_is_bruteforce_far_field_attention(2, 1),
    lambda: pins.test_bridge_decays_across_exactly_the_frames_between(),
    lambda: pins.test_rmsnorm_gate_readout(),
    lambda: pins.test_prepare_features_from_library_routines(),
    lambda: pins.test_sampled_outputs_are_rows_of_the_whole_branch("vdn_solve", True),
    lambda: pins.test_sampled_outputs_prenorm_is_bruteforce_far_field_attention(),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    fn, mutant = MUTANTS[name]
    monkeypatch.setattr(O, fn, mutant)
    caught = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, np.linalg.LinAlgError, ValueError):
            caught += 1
    assert caught > 0, f"no pin fails with mutant {name}"


# ----------------------------------------------------------------------------- windowed softmax branch
import test_oracle_softmax_pins as spins  # noqa: E402

_orig_soft = {name: getattr(O, name) for name in ("window_softmax_frame", "window_bounds")}


def _soft_scale_over_d(qr_t, kr_win, v_win, scale):
    return _orig_soft["window_softmax_frame"](qr_t, kr_win, v_win, scale * scale)   # 1/d instead of 1/sqrt(d)


def _soft_no_max_shift(qr_t, kr_win, v_win, scale):
    with np.errstate(over="ignore", invalid="ignore"):
        w = np.exp((qr_t @ kr_win.T) * scale)
        return (w / w.sum(axis=1, keepdims=True)) @ v_win


def _soft_columns_normalised(qr_t, kr_win, v_win, scale):
    sc = (qr_t @ kr_win.T) * scale
    w = np.exp(sc - sc.max())
    with np.errstate(invalid="ignore", divide="ignore"):
        return (w / w.sum(axis=0, keepdims=True)) @ v_win / max(1, w.shape[0])


def _soft_keys_as_values(qr_t, kr_win, v_win, scale):
    return _orig_soft["window_softmax_frame"](qr_t, kr_win, kr_win, scale)


def _soft_window_short(t, F, chunk, radius):
    lo, hi = _orig_soft["window_bounds"](t, F, chunk, radius)
    return lo, max(lo, hi - 1)


SOFT_MUTANTS = {
    "softmax_scale_over_d": ("window_softmax_frame", _soft_scale_over_d),
    "softmax_no_max_shift": ("window_softmax_frame", _soft_no_max_shift),
    "softmax_columns_normalised": ("window_softmax_frame", _soft_columns_normalised),
    "softmax_keys_as_values": ("window_softmax_frame", _soft_keys_as_values),
    "softmax_window_one_frame_short": ("window_bounds", _soft_window_short),
}


@pytest.mark.parametrize("name", sorted(SOFT_MUTANTS))
def test_planted_softmax_mistake_is_caught(name, monkeypatch):
    fn, mutant = SOFT_MUTANTS[name]
    monkeypatch.setattr(O, fn, mutant)
    tests = [getattr(spins, n) for n in dir(spins) if n.startswith("test_")]
    caught = 0
    for t in tests:
        args = []
        if getattr(t, "pytestmark", None):
            params = [m for m in t.pytestmark if m.name == "parametrize"]
            if params:
                args = list(params[0].args[1][0]) if isinstance(params[0].args[1][0], tuple) else [params[0].args[1][0]]
        try:
            t(*args)
        except (AssertionError, ValueError, FloatingPointError):
            caught += 1
    assert caught > 0, f"no pin fails with mutant {name}"
