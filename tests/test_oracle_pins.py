"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test would fail under a plausible mistake in the oracle: a dropped group
step, group scores from the wrong scores, weights from the bias-corrected
scores, a second application of the routed scaling factor, gate/up swapped,
a transposed w2, a scaled shared expert, or a token that leaks into another.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import (MoeConfig, bf16_round, group_limited_topk, moe_forward,
                    moe_forward_tokens, permutation, rmsnorm, route, router_scores,
                    routing_weights, swiglu_mlp)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_c(rng, T, E):
    # distinct fp32 values (ties have probability ~0 at this size)
    return rng.standard_normal((T, E)).astype(np.float32)


# ----------------------------------------------------------------------------
# Selection: brute force on tiny inputs
# ----------------------------------------------------------------------------
def _brute_force_select(c_row, n_group, topk_group, top_k):
    """Max-sum subsets: the best group subset by summed group scores (each the
    best pair sum inside the group), then the best expert subset by summed c."""
    E = c_row.size
    gs = E // n_group
    gscore = []
    for g in range(n_group):
        vals = c_row[g * gs:(g + 1) * gs]
        gscore.append(max(np.float32(vals[i]) + np.float32(vals[j])
                          for i, j in itertools.combinations(range(gs), 2)))
    best_groups = max(itertools.combinations(range(n_group), topk_group),
                      key=lambda sub: sum(float(gscore[g]) for g in sub))
    cand = [e for g in best_groups for e in range(g * gs, (g + 1) * gs)]
    best = max(itertools.combinations(cand, top_k),
               key=lambda sub: sum(float(c_row[e]) for e in sub))
    return set(best)


@pytest.mark.parametrize("E,G,g,k", [(8, 4, 2, 2), (16, 4, 2, 4), (12, 3, 2, 3), (16, 4, 3, 5)])
def test_selection_matches_brute_force(E, G, g, k):
    rng = np.random.default_rng(1234 + E + k)
    c = _rand_c(rng, 200, E)
    ids, margin = group_limited_topk(c, G, g, k)
    for t in range(c.shape[0]):
        assert set(ids[t].tolist()) == _brute_force_select(c[t], G, g, k), t
    assert np.all(margin > 0)


def test_selection_order_is_descending_c():
    rng = np.random.default_rng(7)
    c = _rand_c(rng, 100, 128)
    ids, _ = group_limited_topk(c, 4, 2, 8)
    sel = np.take_along_axis(c, ids.astype(np.int64), axis=1)
    assert np.all(np.diff(sel, axis=1) <= 0)


def test_single_group_reduces_to_plain_topk():
    rng = np.random.default_rng(11)
    c = _rand_c(rng, 300, 64)
    ids, _ = group_limited_topk(c, 1, 1, 6)
    ref = np.argpartition(-c, 6, axis=1)[:, :6]
    for t in range(c.shape[0]):
        assert set(ids[t].tolist()) == set(ref[t].tolist())


def test_exact_tie_goes_to_lower_index():
    # reading: ties resolve to the lower index, in groups and in experts
    c = np.array([[0.5, 0.5, 0.1, 0.1, 0.3, 0.7, 0.2, 0.0]], dtype=np.float32)
    # group scores [1.0, 0.2, 1.0, 0.2] -> groups 0 and 2 (0 and 2 tie with each other)
    ids, margin = group_limited_topk(c, 4, 2, 3)
    assert ids[0].tolist() == [5, 0, 1]
    c2 = np.array([[0.5, 0.5, 0.5, 0.5]], dtype=np.float32)
    ids2, m2 = group_limited_topk(c2, 2, 1, 1)
    assert ids2[0].tolist() == [0] and m2[0] == 0.0


def test_margin_is_distance_to_another_choice():
    c = np.array([[0.9, 0.1, 0.8, 0.2, 0.5, 0.45, 0.3, 0.29]], dtype=np.float32)
    # G = [1.0, 1.0, 0.95, 0.59]: groups 0 and 1 kept, group margin 0.05
    # candidates [0.9, 0.1, 0.8, 0.2] -> top-2 [0, 2], c margin 0.8 - 0.2 = 0.6
    ids, margin = group_limited_topk(c, 4, 2, 2)
    assert ids[0].tolist() == [0, 2]
    assert margin[0] == pytest.approx(float(np.float32(1.0) - np.float32(0.95)), abs=1e-7)


# ----------------------------------------------------------------------------
# Bias semantics and scaling (sglang PR #32341 report, router bias test name;
# xxqk.cn vLLM-Omni article, asymmetric routing)
# ----------------------------------------------------------------------------
def _small_router_inputs(T=300, H=64, E=32, seed=3):
    rng = np.random.default_rng(seed)
    x = bf16_round(rng.standard_normal((T, H)).astype(np.float32))
    Wr = (0.3 * rng.standard_normal((E, H))).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    return x, Wr, bias


def test_constant_bias_shift_changes_nothing():
    x, Wr, bias = _small_router_inputs()
    cfg = MoeConfig(E=32, top_k=4, n_group=4, topk_group=2)
    ids0, w0, m0, _ = route(x, Wr, bias, cfg)
    ids1, w1, m1, _ = route(x, Wr, bias + np.float32(0.25), cfg)
    ok = (m0 > 1e-5) & (m1 > 1e-5)
    assert ok.sum() > 250
    assert np.array_equal(ids0[ok], ids1[ok])
    assert np.array_equal(w0[ok], w1[ok])  # bit-identical: weights never see the bias


def test_bias_forces_selection_but_not_weights():
    x, Wr, bias = _small_router_inputs()
    cfg = MoeConfig(E=32, top_k=4, n_group=4, topk_group=2)
    forced = [1, 5, 17, 20]  # two experts in each of groups 0 and 2
    b = bias.copy()
    b[forced] += 10.0
    ids, w, _, s = route(x, Wr, b, cfg)
    for t in range(x.shape[0]):
        assert set(ids[t].tolist()) == set(forced)
    sel = np.take_along_axis(s.astype(np.float64), ids.astype(np.int64), axis=1)
    np.testing.assert_allclose(w, 2.5 * sel / sel.sum(axis=1, keepdims=True), rtol=1e-15)
    # the same ids without a bias give bit-identical weights
    w_nobias = routing_weights(s, ids, 2.5)
    assert np.array_equal(w, w_nobias)


def test_weights_sum_to_scaling_factor_once():
    x, Wr, bias = _small_router_inputs()
    cfg = MoeConfig(E=32, top_k=4, n_group=4, topk_group=2)
    _, w, _, _ = route(x, Wr, bias, cfg)
    np.testing.assert_allclose(w.sum(axis=1), 2.5, rtol=1e-12)


def test_router_logits_are_fp32_rounded_dot_products():
    x, Wr, bias = _small_router_inputs(T=20, H=64, E=8)
    logits, s, c = router_scores(x, Wr, bias)
    assert logits.dtype == np.float32 and s.dtype == np.float32 and c.dtype == np.float32
    # exact dot product with Python's correctly rounded fsum, then to fp32
    for t in range(5):
        for e in range(8):
            exact = math.fsum(float(a) * float(b) for a, b in zip(x[t], Wr[e]))
            assert logits[t, e] == np.float32(exact)
    # sigmoid and bias add, scalar reference
    for t in range(5):
        for e in range(8):
            sv = np.float32(1.0 / (1.0 + math.exp(-float(logits[t, e]))))
            assert s[t, e] == sv
            assert c[t, e] == np.float32(sv + bias[e])


# ----------------------------------------------------------------------------
# Hand-worked golden example
# ----------------------------------------------------------------------------
def _golden_inputs():
    with open(os.path.join(GOLDEN, "hand_worked_two_tokens.json")) as f:
        g = json.load(f)
    names = {"0": 0.0, "ln3": math.log(3), "-ln3": -math.log(3),
             "ln7": math.log(7), "-ln7": -math.log(7)}
    Wr = np.zeros((8, 2), dtype=np.float32)
    Wr[:, 0] = [names[v] for v in g["router_logits_token0"]]
    Wr[:, 1] = [names[v] for v in g["router_logits_token1"]]
    x = np.array(g["x"], dtype=np.float32)
    bias = np.array(g["bias"], dtype=np.float32)
    l3, l7 = math.log(3), math.log(7)
    w13 = np.array([[[l3, l3], [1.0, 2.0]] for _ in range(8)])
    w2 = np.array([[[e + 1.0], [1.0]] for e in range(8)])
    ws13 = np.array([[l7, l7], [1.0, 1.0]])
    ws2 = np.array([[1.0], [2.0]])
    cfg = MoeConfig(E=8, I=1, I_shared=1, top_k=2, n_group=4, topk_group=2)
    return g, x, Wr, bias, w13, w2, ws13, ws2, cfg


def test_hand_worked_golden_example():
    g, x, Wr, bias, w13, w2, ws13, ws2, cfg = _golden_inputs()
    out, ids, w, margin = moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg)
    assert ids.tolist() == g["expected_ids"]
    np.testing.assert_allclose(w, g["expected_weights"], rtol=1e-6)
    np.testing.assert_allclose(out, g["expected_out"], rtol=1e-6)
    assert np.all(margin > 0.09)


def test_hand_worked_golden_example_without_renormalisation():
    """norm_topk_prob off: the same experts, each weighted by 2.5 times its raw
    score (hand-worked values in the golden file)."""
    g, x, Wr, bias, w13, w2, ws13, ws2, cfg = _golden_inputs()
    cfg = MoeConfig(E=8, I=1, I_shared=1, top_k=2, n_group=4, topk_group=2,
                    norm_topk_prob=False)
    out, ids, w, _ = moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg)
    assert ids.tolist() == g["expected_ids"]
    np.testing.assert_allclose(w, g["expected_weights_no_renorm"], rtol=1e-6)
    np.testing.assert_allclose(out, g["expected_out_no_renorm"], rtol=1e-6)
    ids_r, w_r, _, _ = route(x, Wr, bias, cfg)
    assert ids_r.tolist() == g["expected_ids"]
    np.testing.assert_allclose(w_r, g["expected_weights_no_renorm"], rtol=1e-6)


# ----------------------------------------------------------------------------
# Expert math: closed forms and special cases
# ----------------------------------------------------------------------------
def _block(T=64, H=64, E=16, I=32, Is=32, seed=5, k=4, G=4, g=2):
    rng = np.random.default_rng(seed)
    x = bf16_round(rng.standard_normal((T, H)).astype(np.float32))
    Wr = (0.2 * rng.standard_normal((E, H))).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    w13 = bf16_round((0.1 * rng.standard_normal((E, 2 * I, H))).astype(np.float32))
    w2 = bf16_round((0.1 * rng.standard_normal((E, H, I))).astype(np.float32))
    ws13 = bf16_round((0.1 * rng.standard_normal((2 * Is, H))).astype(np.float32))
    ws2 = bf16_round((0.1 * rng.standard_normal((H, Is))).astype(np.float32))
    cfg = MoeConfig(E=E, I=I, I_shared=Is, top_k=k, n_group=G, topk_group=g)
    return x, Wr, bias, w13, w2, ws13, ws2, cfg


def test_identical_experts_give_scaled_dense_mlp():
    x, Wr, bias, w13, w2, ws13, ws2, cfg = _block()
    w13s = np.repeat(w13[:1], cfg.E, axis=0)
    w2s = np.repeat(w2[:1], cfg.E, axis=0)
    out, _, _, _ = moe_forward(x, Wr, bias, w13s, w2s, None, None,
                               MoeConfig(**{**cfg.__dict__, "I_shared": 0}))
    # closed form: routed output = (sum of weights) * MLP = 2.5 * MLP, whatever the routing
    ref = 2.5 * torch.nn.functional.linear(
        torch.nn.functional.silu(torch.from_numpy(x).double() @ torch.from_numpy(w13[0, :cfg.I]).double().T)
        * (torch.from_numpy(x).double() @ torch.from_numpy(w13[0, cfg.I:]).double().T),
        torch.from_numpy(w2[0]).double()).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_single_expert_is_textbook_swiglu_plus_shared():
    # E=1, k=1, one group: out = 2.5 * SwiGLU(x) + shared(x); the packed w13 is
    # the concatenation of separately drawn gate (w1) and up (w3) projections
    rng = np.random.default_rng(9)
    T, H, I = 16, 32, 24
    x = torch.from_numpy(rng.standard_normal((T, H))).double()
    w1 = torch.from_numpy(0.1 * rng.standard_normal((I, H))).double()
    w3 = torch.from_numpy(0.1 * rng.standard_normal((I, H))).double()
    w2 = torch.from_numpy(0.1 * rng.standard_normal((H, I))).double()
    v1 = torch.from_numpy(0.1 * rng.standard_normal((I, H))).double()
    v3 = torch.from_numpy(0.1 * rng.standard_normal((I, H))).double()
    v2 = torch.from_numpy(0.1 * rng.standard_normal((H, I))).double()
    w13 = torch.cat((w1, w3), dim=0)[None]  # [1, 2I, H]
    ws13 = torch.cat((v1, v3), dim=0)
    Wr = np.zeros((1, H), dtype=np.float32)
    bias = np.zeros(1, dtype=np.float32)
    cfg = MoeConfig(E=1, I=I, I_shared=I, top_k=1, n_group=1, topk_group=1)
    out, ids, w, _ = moe_forward(x.numpy(), Wr, bias, w13.numpy(), w2[None].numpy(),
                                 ws13.numpy(), v2.numpy(), cfg)
    F = torch.nn.functional
    mlp = lambda a, g, u, d: F.linear(F.silu(F.linear(a, g)) * F.linear(a, u), d)
    ref = 2.5 * mlp(x, w1, w3, w2) + mlp(x, v1, v3, v2)
    assert np.all(ids == 0) and np.allclose(w, 2.5)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_swiglu_gate_up_order_and_w2_orientation():
    rng = np.random.default_rng(21)
    H, I = 8, 4
    x = rng.standard_normal((3, H))
    w13 = rng.standard_normal((2 * I, H))
    w2 = rng.standard_normal((H, I))
    y = swiglu_mlp(x, w13, w2)
    # elementwise scalar loops
    ref = np.zeros((3, H))
    for t in range(3):
        for j in range(I):
            gte = sum(x[t, h] * w13[j, h] for h in range(H))
            upv = sum(x[t, h] * w13[I + j, h] for h in range(H))
            hj = gte / (1 + math.exp(-gte)) * upv
            for o in range(H):
                ref[t, o] += hj * w2[o, j]
    np.testing.assert_allclose(y, ref, rtol=1e-12)


def test_batch_isolation_and_permutation():
    x, Wr, bias, w13, w2, ws13, ws2, cfg = _block(T=96)
    full, ids, _, _ = moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg)
    a, _, _, _ = moe_forward(x[:40], Wr, bias, w13, w2, ws13, ws2, cfg)
    b, _, _, _ = moe_forward(x[40:], Wr, bias, w13, w2, ws13, ws2, cfg)
    np.testing.assert_allclose(np.concatenate([a, b]), full, rtol=1e-13, atol=1e-14)
    perm = np.random.default_rng(0).permutation(96)
    p, _, _, _ = moe_forward(x[perm], Wr, bias, w13, w2, ws13, ws2, cfg)
    np.testing.assert_allclose(p, full[perm], rtol=1e-13, atol=1e-14)
    sub, _, _, _ = moe_forward_tokens([5, 70, 3], x, Wr, bias, w13, w2, ws13, ws2, cfg)
    np.testing.assert_allclose(sub, full[[5, 70, 3]], rtol=1e-13, atol=1e-14)


def test_residual_and_given_ids():
    x, Wr, bias, w13, w2, ws13, ws2, cfg = _block(T=32)
    out, ids, w, _ = moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg)
    res = np.ones_like(x)
    out_r, _, _, _ = moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg, residual=res)
    np.testing.assert_allclose(out_r, out + 1.0, rtol=1e-14)
    # reversing each token's id order changes nothing (the restore is a sum)
    out_g, _, w_g, _ = moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg, ids=ids[:, ::-1])
    np.testing.assert_allclose(out_g, out, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(w_g, w[:, ::-1], rtol=1e-15)


def test_padding_mask_keeps_only_the_shared_expert():
    # [S2] "MoE 实现的源码级要点": the padding mask acts on the routing scores, which
    # are renormalised.  A padding token takes no routed expert (id -1, weight 0)
    # and keeps the dense shared expert; real tokens are untouched.
    x, Wr, bias, w13, w2, ws13, ws2, cfg = _block(T=48)
    mask = np.ones(48, dtype=np.uint8)
    mask[[0, 7, 8, 30, 47]] = 0
    res = np.full_like(x, 0.25)
    full, ids0, w0, m0 = moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg, residual=res)
    out, ids, w, margin = moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg, residual=res,
                                      token_mask=mask)
    pad = mask == 0
    # padding tokens: a textbook SwiGLU MLP of the shared weights, plus the residual
    F = torch.nn.functional
    xt = torch.from_numpy(x[pad]).double()
    Is = cfg.I_shared
    g = torch.from_numpy(ws13[:Is]).double()
    u = torch.from_numpy(ws13[Is:]).double()
    sh = F.linear(F.silu(F.linear(xt, g)) * F.linear(xt, u), torch.from_numpy(ws2).double())
    np.testing.assert_allclose(out[pad], sh.numpy() + 0.25, rtol=1e-12, atol=1e-12)
    assert np.all(ids[pad] == -1) and np.all(w[pad] == 0) and np.all(np.isinf(margin[pad]))
    # real tokens: bit for bit what the unmasked block gives
    assert np.array_equal(out[~pad], full[~pad])
    assert np.array_equal(ids[~pad], ids0[~pad]) and np.array_equal(w[~pad], w0[~pad])
    # all padding: only the shared expert anywhere; no padding: the unmasked block
    out_all, ids_all, _, _ = moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg,
                                         token_mask=np.zeros(48, dtype=np.uint8))
    assert np.all(ids_all == -1)
    np.testing.assert_allclose(out_all, swiglu_mlp(x, ws13, ws2), rtol=1e-14)
    out_none, _, _, _ = moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg, residual=res,
                                    token_mask=np.ones(48, dtype=np.uint8))
    assert np.array_equal(out_none, full)
    # the sampled form gives the same rows
    sub, _, _, _ = moe_forward_tokens([7, 9, 30], x, Wr, bias, w13, w2, ws13, ws2, cfg,
                                      residual=res, token_mask=mask)
    np.testing.assert_allclose(sub, out[[7, 9, 30]], rtol=1e-13, atol=1e-14)


def test_rmsnorm_unit_rms_and_bf16_rounding():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((10, 256)) * 3.0
    r = rmsnorm(x, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(r * r, axis=1)), 1.0, rtol=1e-12)
    # bf16 rounding: ties to even and exact values
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5], dtype=np.float32)
    exp = np.array([1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5], dtype=np.float32)
    np.testing.assert_array_equal(bf16_round(vals), exp)
    t = torch.from_numpy(rng.standard_normal(4096).astype(np.float32))
    np.testing.assert_array_equal(bf16_round(t.numpy()), t.to(torch.bfloat16).float().numpy())


def test_rmsnorm_gamma_multiplies_each_channel():
    """Rows whose mean square is a perfect square, with eps = 0, and a gamma of
    distinct powers of two: every output is a short binary fraction written out
    by hand.  A gamma divided instead of multiplied, or read at the wrong
    channel, changes them."""
    x = np.array([[3.0, -3.0, 3.0, -3.0],     # mean square 9 -> x / 3
                  [0.0, 4.0, 0.0, 0.0],       # mean square 4 -> x / 2
                  [1.0, 1.0, 1.0, 1.0]])      # mean square 1 -> x
    gamma = np.array([2.0, 0.5, 4.0, 0.25])
    exp = np.array([[2.0, -0.5, 4.0, -0.25],
                    [0.0, 1.0, 0.0, 0.0],
                    [2.0, 0.5, 4.0, 0.25]])
    np.testing.assert_array_equal(rmsnorm(x, eps=0.0, gamma=gamma), exp)
    # no gamma is gamma = 1
    np.testing.assert_array_equal(rmsnorm(x, eps=0.0), exp / gamma[None, :])


def test_rmsnorm_eps_inside_the_square_root():
    """A constant row a with a^2 = eps: a / sqrt(a^2 + eps) = 1 / sqrt(2)
    exactly in real arithmetic.  eps outside the root would give
    a / (|a| + eps) (~0.999), a dropped eps 1."""
    a, eps = 1e-3, 1e-6
    x = np.full((2, 64), a)
    x[1] = -a
    r = rmsnorm(x, eps=eps)
    np.testing.assert_allclose(r[0], 1.0 / math.sqrt(2.0), rtol=1e-12)
    np.testing.assert_allclose(r[1], -1.0 / math.sqrt(2.0), rtol=1e-12)
    # eps only matters relative to the mean square: a large row is unaffected
    np.testing.assert_allclose(rmsnorm(np.full((1, 64), 1e3), eps=eps), 1.0, rtol=1e-12)


def test_invalid_configs_raise():
    c = np.zeros((1, 10), dtype=np.float32)
    with pytest.raises(ValueError):
        group_limited_topk(c, 4, 2, 2)  # 10 % 4 != 0
    with pytest.raises(ValueError):
        group_limited_topk(np.zeros((1, 8), np.float32), 4, 1, 3)  # 2 candidates < 3


def test_permutation_matches_counting_definition():
    # row(t, j) = offset[e] + #{t' < t : e in ids[t']}, e = ids[t, j]; offsets = prefix counts
    rng = np.random.default_rng(17)
    T, E, k = 57, 12, 3
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    offsets, row_of, tok_of = permutation(ids, E)
    counts = [int((ids == e).sum()) for e in range(E)]
    assert offsets.tolist() == [sum(counts[:e]) for e in range(E + 1)]
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            before = sum(1 for tp in range(t) if e in ids[tp])
            r = offsets[e] + before
            assert row_of[t * k + j] == r and tok_of[r] == t
    assert sorted(row_of.tolist()) == list(range(T * k))
