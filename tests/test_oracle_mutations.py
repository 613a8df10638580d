"""Plant plausible mistakes in the oracle (CPU only) and check that the pins
in ``test_oracle_pins`` catch every one of them."""

import numpy as np
import pytest

import oracle.moe_oracle as om
from tests import test_oracle_fp8 as fp8_pins
from tests import test_oracle_pins as pins


def _route_weights_from_c(x, Wr, bias, cfg):
    _, s, c = om.router_scores(x, Wr, bias)
    ids, margin = om.group_limited_topk(c, cfg.n_group, cfg.topk_group, cfg.top_k)
    return ids, om.routing_weights(c, ids, cfg.routed_scaling_factor), margin, s


def _double_scaling(s, ids, rsf, norm=True):
    sel = np.take_along_axis(s.astype(np.float64), ids.astype(np.int64), axis=1)
    return rsf * rsf * sel / sel.sum(axis=1, keepdims=True)


def _no_group_step(c, n_group, topk_group, top_k):
    return _ORIG_GLT(c, n_group, n_group, top_k)


def _group_score_max(c, n_group, topk_group, top_k):
    T, E = c.shape
    gs = E // n_group
    G = c.reshape(T, n_group, gs).max(axis=2)
    kept = np.argsort(-G, axis=1, kind="stable")[:, :topk_group]
    mask = np.zeros((T, n_group), bool)
    np.put_along_axis(mask, kept, True, axis=1)
    cand = np.where(np.repeat(mask, gs, axis=1), c.astype(np.float64), -np.inf)
    ids = np.argsort(-cand, axis=1, kind="stable")[:, :top_k].astype(np.int32)
    return ids, np.full(T, np.inf)


def _gate_up_swapped(x, w13, w2):
    I = w13.shape[0] // 2
    return _ORIG_SWIGLU(x, np.concatenate([w13[I:], w13[:I]]), w2)


def _w2_transposed_use(x, w13, w2):
    # uses w2 as if it were stored [I, H] (wrong orientation), only meaningful when square
    I = w13.shape[0] // 2
    xd = x.astype(np.float64)
    h = om._silu(xd @ w13[:I].T) * (xd @ w13[I:].T)
    return h @ (w2.reshape(w2.shape[1], w2.shape[0]).astype(np.float64))


_ORIG_GLT = om.group_limited_topk
_ORIG_SWIGLU = om.swiglu_mlp


def _scaled_shared(*args, **kw):
    out, ids, w, m = _ORIG_FWD(*args, **kw)
    x, ws13, ws2, cfg = args[0], args[5], args[6], args[7]
    if ws13 is not None:
        out = out + (cfg.routed_scaling_factor - 1.0) * _ORIG_SWIGLU(x, ws13, ws2)
    return out, ids, w, m


_ORIG_FWD = om.moe_forward
_ORIG_MASK = om.apply_token_mask


def _mask_ignored(ids, w, margin, token_mask):
    return ids, w, margin


def _forward_mask_kills_shared(*args, **kw):
    out, ids, w, m = _ORIG_FWD(*args, **kw)
    mask = kw.get("token_mask")
    if mask is not None:
        res = kw.get("residual")
        pad = np.asarray(mask).reshape(-1) == 0
        out = out.copy()
        out[pad] = 0.0 if res is None else np.asarray(res, dtype=np.float64)[pad]
    return out, ids, w, m

def _e4m3_bias_8(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e, m = (c >> 3) & 0xF, c & 7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -7, (1.0 + m / 8.0) * np.exp2(e - 8.0))
    val = np.where(c >> 7 == 1, -mag, mag)
    return np.where((e == 15) & (m == 7), np.nan, val)


def _e4m3_subnormals_as_normals(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e, m = (c >> 3) & 0xF, c & 7
    mag = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    val = np.where(c >> 7 == 1, -mag, mag)
    return np.where((e == 15) & (m == 7), np.nan, val)


def _ue8m0_bias_128(exps):
    s = np.asarray(exps, dtype=np.uint8).astype(np.float64)
    return np.where(s == 255, np.nan, np.exp2(s - 128.0))


def _block_index_transposed(codes, scale_exp, block=128):
    # row block and column block swapped in the scale lookup (on a non-square
    # block grid this reads the wrong scales or runs off the grid)
    codes = np.asarray(codes, dtype=np.uint8)
    scale = om.ue8m0_decode(scale_exp)
    rows = np.arange(codes.shape[-2]) // block
    cols = np.arange(codes.shape[-1]) // block
    return om.fp8_e4m3_decode(codes) * scale[..., cols[None, :], rows[:, None]]


def _rms_gamma_divided(x, eps=1e-6, gamma=None):
    xd = x.astype(np.float64)
    r = xd / np.sqrt(np.mean(xd * xd, axis=1, keepdims=True) + eps)
    return r if gamma is None else r / gamma.astype(np.float64)[None, :]


def _rms_gamma_reversed(x, eps=1e-6, gamma=None):
    xd = x.astype(np.float64)
    r = xd / np.sqrt(np.mean(xd * xd, axis=1, keepdims=True) + eps)
    return r if gamma is None else r * gamma.astype(np.float64)[::-1][None, :]


def _rms_eps_outside_root(x, eps=1e-6, gamma=None):
    xd = x.astype(np.float64)
    r = xd / (np.sqrt(np.mean(xd * xd, axis=1, keepdims=True)) + eps)
    return r if gamma is None else r * gamma.astype(np.float64)[None, :]


def _always_renormalise(s, ids, rsf, norm_topk_prob=True):
    sel = np.take_along_axis(s.astype(np.float64), ids.astype(np.int64), axis=1)
    return rsf * sel / sel.sum(axis=1, keepdims=True)


def _never_renormalise(s, ids, rsf, norm_topk_prob=True):
    sel = np.take_along_axis(s.astype(np.float64), ids.astype(np.int64), axis=1)
    return rsf * sel


PIN_TESTS = [
    lambda: pins.test_hand_worked_golden_example(),
    lambda: [pins.test_selection_matches_brute_force(*a) for a in
             [(8, 4, 2, 2), (16, 4, 2, 4), (12, 3, 2, 3)]],
    lambda: pins.test_bias_forces_selection_but_not_weights(),
    lambda: pins.test_weights_sum_to_scaling_factor_once(),
    lambda: pins.test_identical_experts_give_scaled_dense_mlp(),
    lambda: pins.test_single_expert_is_textbook_swiglu_plus_shared(),
    lambda: pins.test_swiglu_gate_up_order_and_w2_orientation(),
    lambda: pins.test_padding_mask_keeps_only_the_shared_expert(),
    lambda: pins.test_hand_worked_golden_example_without_renormalisation(),
    lambda: pins.test_rmsnorm_gamma_multiplies_each_channel(),
    lambda: pins.test_rmsnorm_eps_inside_the_square_root(),
    lambda: fp8_pins.test_e4m3_decode_matches_torch_float8_on_every_code(),
    lambda: fp8_pins.test_ue8m0_scales(),
    lambda: fp8_pins.test_block_scales_land_on_their_blocks_ragged_non_square(),
]

MUTATIONS = {
    "weights_from_bias_corrected_scores": [(pins, "route", _route_weights_from_c),
                                           (om, "route", _route_weights_from_c)],
    "scaling_applied_twice": [(om, "routing_weights", _double_scaling),
                              (pins, "routing_weights", _double_scaling)],
    "group_step_dropped": [(om, "group_limited_topk", _no_group_step),
                           (pins, "group_limited_topk", _no_group_step)],
    "group_score_is_max": [(om, "group_limited_topk", _group_score_max),
                           (pins, "group_limited_topk", _group_score_max)],
    "gate_up_swapped": [(om, "swiglu_mlp", _gate_up_swapped),
                        (pins, "swiglu_mlp", _gate_up_swapped)],
    "w2_misoriented": [(om, "swiglu_mlp", _w2_transposed_use),
                       (pins, "swiglu_mlp", _w2_transposed_use)],
    "shared_expert_scaled": [(pins, "moe_forward", _scaled_shared)],
    "rmsnorm_gamma_divided": [(om, "rmsnorm", _rms_gamma_divided),
                              (pins, "rmsnorm", _rms_gamma_divided)],
    "rmsnorm_gamma_wrong_channel": [(om, "rmsnorm", _rms_gamma_reversed),
                                    (pins, "rmsnorm", _rms_gamma_reversed)],
    "rmsnorm_eps_outside_root": [(om, "rmsnorm", _rms_eps_outside_root),
                                 (pins, "rmsnorm", _rms_eps_outside_root)],
    "norm_topk_prob_ignored": [(om, "routing_weights", _always_renormalise),
                               (pins, "routing_weights", _always_renormalise)],
    "renormalisation_dropped": [(om, "routing_weights", _never_renormalise),
                                (pins, "routing_weights", _never_renormalise)],
    "padding_mask_ignored": [(om, "apply_token_mask", _mask_ignored)],
    "padding_drops_shared_expert": [(pins, "moe_forward", _forward_mask_kills_shared)],
    "e4m3_exponent_bias_8": [(om, "fp8_e4m3_decode", _e4m3_bias_8),
                             (fp8_pins, "fp8_e4m3_decode", _e4m3_bias_8)],
    "e4m3_subnormals_as_normals": [(om, "fp8_e4m3_decode", _e4m3_subnormals_as_normals),
                                   (fp8_pins, "fp8_e4m3_decode", _e4m3_subnormals_as_normals)],
    "ue8m0_bias_128": [(om, "ue8m0_decode", _ue8m0_bias_128),
                       (fp8_pins, "ue8m0_decode", _ue8m0_bias_128)],
    "fp8_block_index_transposed": [(om, "fp8_block_dequant", _block_index_transposed),
                                   (fp8_pins, "fp8_block_dequant", _block_index_transposed)],
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    for mod, attr, fn in MUTATIONS[name]:
        monkeypatch.setattr(mod, attr, fn)
    failures = 0
    for pin in PIN_TESTS:
        try:
            pin()
        except Exception:  # AssertionError, or a shape error from a wrong layout
            failures += 1
    assert failures >= 1, f"no pin caught the planted mistake {name!r}"


def test_unmutated_oracle_passes_every_pin():
    for pin in PIN_TESTS:
        pin()
