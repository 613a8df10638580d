"""CUDA path (through the C ABI) against the CPU oracle.

Sizes span several 128-row tiles with ragged tails, experts with no tokens,
N tails (I and H not multiples of the tile), T = 1, the skewed (hot expert)
case, the named workloads (the two small ones in full, the large ones on a
seeded token sample), determinism and batch isolation.
"""

import numpy as np
import pytest
import torch

import oracle
from routed_moe_layer_b200 import inputs, ops
from routed_moe_layer_b200.ops import BlockConfig
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _dev(d):
    return {k: (None if v is None else v.to(DEV)) for k, v in d.items()}


def _run(d, cfg, residual=None, token_mask=None):
    ids = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device=DEV)
    w = torch.empty((cfg.T, cfg.top_k), dtype=torch.float32, device=DEV)
    ws = ops.alloc_workspace(ops.workspace_bytes(cfg), DEV)
    out = ops.forward(d["x"], d["Wr"], d["bias"], d["w13"], d["w2"], d.get("ws13"), d.get("ws2"),
                      cfg, residual=residual, workspace=ws, topk_ids=ids, topk_w=w,
                      token_mask=token_mask)
    torch.cuda.synchronize()
    code, site = ops.read_device_status(ws)
    assert code == 0, (ops.status_string(code), site)
    return out, ids, w


# ------------------------------------------------------------------ router
@pytest.mark.parametrize("T,H,E,k,G,g", [
    (1, 64, 8, 2, 4, 2), (37, 128, 16, 4, 4, 2), (300, 256, 128, 8, 4, 2),
    (1000, 1024, 128, 8, 4, 2), (129, 2048, 64, 6, 8, 3), (50, 512, 32, 4, 1, 1),
    (65, 192, 96, 16, 4, 4),
])
def test_router_matches_oracle(T, H, E, k, G, g):
    cfg = BlockConfig(T=T, H=H, E=E, top_k=k, n_group=G, topk_group=g)
    d = inputs.make_block_inputs(T, H, seed=T + E, E=E, I=64, I_shared=0, unit_scale=True)
    dd = _dev(d)
    ids, w = ops.route(dd["x"], dd["Wr"], dd["bias"], cfg)
    torch.cuda.synchronize()
    rep = parity.check_routing(ids, w, *[parity.to_np(d[n]) for n in ("x", "Wr", "bias")], cfg)
    assert rep["near_ties"] <= max(2, T // 20)


@pytest.mark.parametrize("wid", [0, 1, 2, 3])
def test_router_on_workloads(wid):
    wl = inputs.WORKLOADS[wid]
    d = inputs.workload_inputs(wid)
    cfg = BlockConfig(T=wl.T, H=wl.H)
    dd = {k: d[k].to(DEV) for k in ("x", "Wr", "bias")}
    ids, w = ops.route(dd["x"], dd["Wr"], dd["bias"], cfg)
    torch.cuda.synchronize()
    rep = parity.check_routing(ids, w, *[parity.to_np(d[n]) for n in ("x", "Wr", "bias")], cfg)
    print(f"workload {wl.name}: {rep}")
    # weights sum to the scaling factor on every token
    np.testing.assert_allclose(w.sum(1).cpu().numpy(), 2.5, rtol=1e-5)


@pytest.mark.parametrize("H,E,k,G,g", [(1024, 128, 8, 4, 2), (512, 64, 6, 8, 3),
                                       (256, 96, 16, 4, 4), (256, 32, 4, 1, 1)])
def test_router_batch_isolation(H, E, k, G, g):
    """A token's routing does not depend on the other tokens of the call: the
    first tokens of a large batch, routed alone, give the same bits (and the
    large batch matches the oracle)."""
    T, n = 4133, 777
    cfg = BlockConfig(T=T, H=H, E=E, top_k=k, n_group=G, topk_group=g)
    d = inputs.make_block_inputs(T, H, seed=E + k, E=E, I=64, I_shared=0, unit_scale=True)
    dd = _dev(d)
    ids, w = ops.route(dd["x"], dd["Wr"], dd["bias"], cfg)
    ids_s, w_s = ops.route(dd["x"][:n].contiguous(), dd["Wr"], dd["bias"], cfg.with_tokens(n))
    torch.cuda.synchronize()
    assert torch.equal(ids_s, ids[:n]) and torch.equal(w_s, w[:n])
    rep = parity.check_routing(ids, w, *[parity.to_np(d[m]) for m in ("x", "Wr", "bias")], cfg)
    assert rep["near_ties"] <= max(2, T // 20)


@pytest.mark.parametrize("T,H,k,G,g,norm,masked", [
    (20000, 2048, 8, 4, 2, True, False),  # the block's shape
    (4500, 1024, 8, 8, 3, True, True),    # groups of 16, padding tokens
    (4500, 512, 6, 2, 1, False, False),   # groups of 64, no renormalisation
    (4500, 256, 16, 4, 4, True, False),   # every group kept: no group step, top-16
    (9000, 768, 1, 2, 2, True, True),     # top-1
])
def test_large_batch_router_matches_small_batch_router(T, H, k, G, g, norm, masked):
    """Above 4096 tokens the selection runs 16 lanes per token, below it one
    warp per token; a token's ids and weights are the same bits either way (128
    experts in groups of 16, 32 or 64, with and without the group step, top-1
    to top-16, with and without renormalisation and padding), and match the
    oracle."""
    n = 700
    cfg = BlockConfig(T=T, H=H, E=128, top_k=k, n_group=G, topk_group=g,
                      norm_topk_prob=norm, routed_scaling_factor=2.5 if norm else 0.3)
    d = inputs.make_block_inputs(T, H, seed=H + k, E=128, I=64, I_shared=0, unit_scale=True)
    dd = _dev(d)
    mask = None
    if masked:
        gen = torch.Generator().manual_seed(H)
        mask = (torch.rand(T, generator=gen) > 0.25).to(torch.uint8).to(DEV)
    ids, w = ops.route(dd["x"], dd["Wr"], dd["bias"], cfg, token_mask=mask)
    ids_s, w_s = ops.route(dd["x"][:n].contiguous(), dd["Wr"], dd["bias"], cfg.with_tokens(n),
                           token_mask=None if mask is None else mask[:n].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(ids_s, ids[:n]) and torch.equal(w_s, w[:n])
    rep = parity.check_routing(ids, w, *[parity.to_np(d[m]) for m in ("x", "Wr", "bias")], cfg,
                               token_mask=None if mask is None else mask.cpu().numpy())
    assert rep["near_ties"] <= max(2, T // 20)


def test_router_bias_forces_selection_not_weights():
    T, H = 200, 512
    cfg = BlockConfig(T=T, H=H)
    d = _dev(inputs.make_block_inputs(T, H, seed=5, I=64, I_shared=0, unit_scale=True))
    forced = [3, 7, 40, 41, 44, 60, 61, 63]  # groups 0 and 1 only
    b = d["bias"].clone()
    b[forced] += 10.0
    ids, w = ops.route(d["x"], d["Wr"], b, cfg)
    ids0, w0 = ops.route(d["x"], d["Wr"], d["bias"], cfg)
    assert all(sorted(r) == forced for r in ids.cpu().tolist())
    # same ids -> bitwise the same weights whatever the bias
    same = (torch.sort(ids, 1).values == torch.sort(ids0, 1).values).all(1)
    for t in torch.nonzero(same).flatten().tolist():
        o, o0 = torch.argsort(ids[t]), torch.argsort(ids0[t])
        assert torch.equal(w[t][o], w0[t][o0])


@pytest.mark.parametrize("T,H,I", [(1, 256, 128), (300, 512, 256), (2048, 1024, 768),
                                   (5000, 256, 128)])
def test_routing_without_renormalisation(T, H, I):
    """norm_topk_prob off: weights are rsf x the raw scores of the chosen
    experts (no renormalisation); the router (one warp per token up to 4096
    tokens, half warps above) and the whole block (swapped and tiled GEMMs)
    against the oracle with the same option.  rsf = 0.3 keeps the weights'
    sum near 2 (eight sigmoids of about 0.85): with 2.5 it would be about 17,
    routed outputs some 7x those of the renormalised block, and the
    tolerance's absolute floor (2e-2) would no longer match the outputs' scale."""
    cfg = BlockConfig(T=T, H=H, I=I, I_shared=I, norm_topk_prob=False,
                      routed_scaling_factor=0.3)
    d = inputs.make_block_inputs(T, H, seed=31 + T, I=I, I_shared=I, unit_scale=True)
    dd = _dev(d)
    dn = parity.np_inputs(d)
    ids_r, w_r = ops.route(dd["x"], dd["Wr"], dd["bias"], cfg)
    torch.cuda.synchronize()
    parity.check_routing(ids_r, w_r, dn["x"], dn["Wr"], dn["bias"], cfg)
    # not renormalised: the sums are rsf x (sum of 8 sigmoids), not rsf
    assert not np.allclose(w_r.sum(1).cpu().numpy(), 0.3, rtol=1e-3)
    if T > 2048:
        return
    out, ids, w = _run(dd, cfg)
    assert torch.equal(ids, ids_r) and torch.equal(w, w_r)
    rep = parity.check_output(out, ids, dn, cfg)
    assert rep["rms_rel"] < 1e-2, rep


# ------------------------------------------------------------------ permutation
# T <= 1024 runs the single-CTA path, larger T the three-kernel path
@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (255, 128, 8), (256, 128, 8), (257, 128, 8),
                                   (1000, 16, 4), (1024, 128, 8), (1025, 128, 8), (3000, 64, 6),
                                   (19412, 128, 8)])
def test_permute_bit_exact(T, E, k):
    g = torch.Generator().manual_seed(T * 7 + E)
    ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    w = torch.rand((T, k), generator=g)
    H = 128
    x = torch.randn((T, H), generator=g).to(torch.bfloat16)
    cfg = BlockConfig(T=T, H=H, E=E, top_k=k, n_group=1, topk_group=1)
    r = ops.permute(ids.to(DEV), cfg, topk_w=w.to(DEV), x=x.to(DEV))
    torch.cuda.synchronize()
    code, _ = ops.read_device_status(r["workspace"])
    assert code == 0
    off, row_of, tok_of = oracle.permutation(ids.numpy(), E)
    assert np.array_equal(r["expert_offsets"].cpu().numpy(), off)
    assert np.array_equal(r["row_of"].cpu().numpy(), row_of)
    assert np.array_equal(r["tok_of"].cpu().numpy(), tok_of)
    assert torch.equal(r["w_of"].cpu(), w.reshape(-1)[torch.as_tensor(np.argsort(row_of))])
    assert torch.equal(r["xp"].cpu(), x[torch.as_tensor(tok_of)])


@pytest.mark.parametrize("T", [64, 2000])
def test_permute_reports_bad_expert_id(T):
    E, k = 16, 2
    ids = torch.tensor([[i % E, (i + 1) % E] for i in range(T)], dtype=torch.int32)
    ids[5, 1] = E  # out of range: skipped and reported
    cfg = BlockConfig(T=T, H=64, E=E, top_k=k, n_group=1, topk_group=1)
    r = ops.permute(ids.to(DEV), cfg)
    torch.cuda.synchronize()
    code, site = ops.read_device_status(r["workspace"])
    assert code == 6  # MOE_ERR_DEVICE_INDEX
    assert r["row_of"][5 * k + 1].item() == -1


# ------------------------------------------------------------------ forward
# up to 64 rows per expert on average (T*k <= 64*E) the expert GEMMs run with
# swapped operands (32-row chunks up to 20 rows per expert, else 128-row
# chunks), above it on 256-row tiles: the cases cover all three
FORWARD_CASES = [
    # T, H, E, I, I_shared, k, G, g
    (1, 256, 16, 128, 128, 4, 4, 2),
    (129, 256, 128, 192, 192, 8, 4, 2),     # swapped: I tail inside a 128-row weight tile
    (64, 320, 64, 128, 64, 6, 8, 3),        # swapped: H tail, separate shared-expert GEMMs
    (100, 256, 16, 128, 128, 4, 4, 2),
    (300, 512, 32, 192, 64, 8, 4, 2),       # I not a multiple of 128: SwiGLU N tail
    (700, 320, 16, 128, 128, 4, 4, 2),      # H not a multiple of 256: down/combine N tail
    (1000, 1024, 128, 768, 768, 8, 4, 2),   # several tiles per expert, ragged tails
    (2048, 2048, 128, 768, 768, 8, 4, 2),
    (300, 256, 64, 128, 128, 12, 4, 4),     # top-12 + shared: 13 slots per token
    (200, 512, 32, 128, 0, 16, 2, 2),       # top-16, no shared expert: 16 slots per token
]


@pytest.mark.parametrize("T,H,E,I,Is,k,G,g", FORWARD_CASES)
def test_forward_matches_oracle(T, H, E, I, Is, k, G, g):
    cfg = BlockConfig(T=T, H=H, E=E, I=I, I_shared=Is, top_k=k, n_group=G, topk_group=g)
    d = inputs.make_block_inputs(T, H, seed=11 + T, E=E, I=I, I_shared=Is, unit_scale=True)
    out, ids, w = _run(_dev(d), cfg)
    dn = parity.np_inputs(d)
    parity.check_routing(ids, w, dn["x"], dn["Wr"], dn["bias"], cfg)
    rep = parity.check_output(out, ids, dn, cfg)
    assert rep["rms_rel"] < 1e-2, rep  # bf16 storage of h and Y: a few 1e-3


@pytest.mark.parametrize("T,H,E,I,Is,k,G,g", [
    (40, 16384, 8, 128, 128, 2, 1, 1),      # H at the limit; swapped GEMMs (10 rows per expert)
    (600, 16384, 8, 128, 128, 2, 1, 1),     # H at the limit; pair GEMMs (150 rows per expert)
    (64, 256, 8, 16384, 16384, 2, 1, 1),    # I at the limit; swapped GEMMs
    (400, 256, 8, 16384, 0, 2, 1, 1),       # I at the limit; pair GEMMs, no shared expert
    (300, 512, 128, 128, 128, 16, 16, 2),   # 128 experts in 16 groups of 8, top-16
])
def test_forward_at_size_limits(T, H, E, I, Is, k, G, g):
    """The largest H and I the library accepts (16384), and the most groups
    and experts per token, against the oracle."""
    cfg = BlockConfig(T=T, H=H, E=E, I=I, I_shared=Is, top_k=k, n_group=G, topk_group=g)
    d = inputs.make_block_inputs(T, H, seed=5 + T, E=E, I=I, I_shared=Is, unit_scale=True)
    out, ids, w = _run(_dev(d), cfg)
    dn = parity.np_inputs(d)
    parity.check_routing(ids, w, dn["x"], dn["Wr"], dn["bias"], cfg)
    rep = parity.check_output(out, ids, dn, cfg)
    assert rep["rms_rel"] < 1e-2, rep


@pytest.mark.parametrize("T,E,k,Is", [
    (50, 1, 1, 128),    # one expert: out = 2.5 * SwiGLU(x) + shared(x); swapped GEMMs
    (500, 1, 1, 128),   # the same on the pair GEMMs
    (300, 4, 4, 0),     # every token to every expert (top-k = E), no shared expert
])
def test_forward_degenerate_routing(T, E, k, Is):
    """Routing with no choice left (a single expert, or top-k = E) against the oracle."""
    H, I = 256, 128
    cfg = BlockConfig(T=T, H=H, E=E, I=I, I_shared=Is, top_k=k, n_group=1, topk_group=1)
    d = inputs.make_block_inputs(T, H, seed=17 + T + E, E=E, I=I, I_shared=Is, unit_scale=True)
    out, ids, w = _run(_dev(d), cfg)
    assert torch.equal(torch.sort(ids, 1).values.cpu(),
                       torch.arange(E, dtype=torch.int32).expand(T, E)[:, :k])
    np.testing.assert_allclose(w.sum(1).cpu().numpy(), 2.5, rtol=1e-5)
    dn = parity.np_inputs(d)
    rep = parity.check_output(out, ids, dn, cfg)
    assert rep["rms_rel"] < 1e-2, rep


def test_identical_tokens_give_identical_rows():
    """1000 copies of one token route to the same experts and fill whole and
    partial tiles at every position: every output row has the same bits (each
    row's arithmetic does not depend on where it sits), and the row matches the
    oracle."""
    T, H = 1000, 512
    cfg = BlockConfig(T=T, H=H, I=256, I_shared=256)
    d = inputs.make_block_inputs(T, H, seed=23, I=256, I_shared=256, unit_scale=True)
    d["x"] = d["x"][:1].expand(T, H).contiguous()
    out, ids, w = _run(_dev(d), cfg)
    assert torch.equal(ids, ids[:1].expand(T, -1)) and torch.equal(w, w[:1].expand(T, -1))
    assert torch.equal(out, out[:1].expand(T, H))
    dn = parity.np_inputs({k: v[:1] if k == "x" else v for k, v in d.items()})
    rep = parity.check_output(out[:1], ids[:1], dn, cfg.with_tokens(1))
    assert rep["rms_rel"] < 1e-2, rep


def test_forward_residual_and_no_shared_expert():
    T, H, E, I = 513, 512, 32, 128
    for Is in (0, 128):
        cfg = BlockConfig(T=T, H=H, E=E, I=I, I_shared=Is)
        d = inputs.make_block_inputs(T, H, seed=3, E=E, I=I, I_shared=Is, unit_scale=True)
        dd = _dev(d)
        res = torch.randn((T, H), generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
        out, ids, _ = _run(dd, cfg, residual=res.to(DEV))
        rep = parity.check_output(out, ids, parity.np_inputs(d), cfg,
                                  residual_np=parity.to_np(res))
        assert rep["rms_rel"] < 1e-2, rep


def test_forward_in_place_residual():
    T, H = 300, 256
    cfg = BlockConfig(T=T, H=H, E=16, I=128, I_shared=128, top_k=4)
    d = _dev(inputs.make_block_inputs(T, H, seed=8, E=16, I=128, I_shared=128, unit_scale=True))
    res = torch.randn((T, H), device=DEV).to(torch.bfloat16)
    ref = ops.forward(d["x"], d["Wr"], d["bias"], d["w13"], d["w2"], d["ws13"], d["ws2"], cfg,
                      residual=res)
    buf = res.clone()
    ops.forward(d["x"], d["Wr"], d["bias"], d["w13"], d["w2"], d["ws13"], d["ws2"], cfg,
                residual=buf, out=buf)
    torch.cuda.synchronize()
    assert torch.equal(buf, ref)


@pytest.mark.parametrize("T", [300, 1000, 1500])
def test_forward_hot_experts_many_tiles(T):
    # a bias of +10 on 8 experts (2 groups) sends every token to them: those
    # experts get T rows (many full tiles or chunks + a tail), the other 120
    # get none; T = 300 runs the swapped GEMMs with 32-row chunks, 1000 with
    # 128-row chunks, 1500 the tiled GEMMs
    H = 512
    cfg = BlockConfig(T=T, H=H, I=256, I_shared=128)
    d = inputs.make_block_inputs(T, H, seed=21, I=256, I_shared=128, unit_scale=True)
    hot = [0, 5, 9, 31, 64, 70, 80, 95]
    d["bias"][hot] += 10.0
    out, ids, w = _run(_dev(d), cfg)
    assert all(sorted(r) == hot for r in ids.cpu().tolist())
    rep = parity.check_output(out, ids, parity.np_inputs(d), cfg)
    assert rep["rms_rel"] < 1e-2, rep


@pytest.mark.parametrize("T", [300, 1000, 2048])
def test_forward_padding_mask(T):
    """Padding tokens (mask 0) take no routed expert and keep the shared
    expert and the residual; real tokens give bit for bit the unmasked output.
    T = 300 / 1000 run the swapped GEMMs (32 / 128-row chunks), 2048 the tiled."""
    H = 512
    cfg = BlockConfig(T=T, H=H, I=256, I_shared=256)
    d = inputs.make_block_inputs(T, H, seed=60 + T, I=256, I_shared=256, unit_scale=True)
    dd = _dev(d)
    g = torch.Generator().manual_seed(T)
    mask = (torch.rand(T, generator=g) > 0.2).to(torch.uint8)
    mask[-37:] = 0  # a padded tail, as in a varlen batch
    res = torch.randn((T, H), generator=g).to(torch.bfloat16)
    ref_out, ref_ids, _ = _run(dd, cfg, residual=res.to(DEV))
    ids = torch.empty((T, cfg.top_k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, cfg.top_k), dtype=torch.float32, device=DEV)
    ws = ops.alloc_workspace(ops.workspace_bytes(cfg), DEV)
    out = ops.forward(dd["x"], dd["Wr"], dd["bias"], dd["w13"], dd["w2"], dd["ws13"], dd["ws2"],
                      cfg, residual=res.to(DEV), workspace=ws, topk_ids=ids, topk_w=w,
                      token_mask=mask.to(DEV))
    torch.cuda.synchronize()
    code, site = ops.read_device_status(ws)
    assert code == 0, (ops.status_string(code), site)
    real = mask.bool().to(DEV)
    assert torch.equal(out[real], ref_out[real]) and torch.equal(ids[real], ref_ids[real])
    dn = parity.np_inputs(d)
    parity.check_routing(ids, w, dn["x"], dn["Wr"], dn["bias"], cfg, token_mask=mask.numpy())
    rep = parity.check_output(out, ids, dn, cfg, residual_np=parity.to_np(res),
                              token_mask=mask.numpy())
    assert rep["rms_rel"] < 1e-2, rep
    # the router alone, and the extremes: every token padding / none
    ids_r, w_r = ops.route(dd["x"], dd["Wr"], dd["bias"], cfg, token_mask=mask.to(DEV))
    assert torch.equal(ids_r, ids) and torch.equal(w_r, w)
    none = torch.zeros(T, dtype=torch.uint8, device=DEV)
    out0 = ops.forward(dd["x"], dd["Wr"], dd["bias"], dd["w13"], dd["w2"], dd["ws13"], dd["ws2"],
                       cfg, token_mask=none)
    torch.cuda.synchronize()
    parity.check_output(out0, torch.full((T, cfg.top_k), -1, dtype=torch.int32), dn, cfg,
                        token_mask=np.zeros(T, dtype=np.uint8))
    all_real = torch.ones(T, dtype=torch.uint8, device=DEV)
    out1 = ops.forward(dd["x"], dd["Wr"], dd["bias"], dd["w13"], dd["w2"], dd["ws13"], dd["ws2"],
                       cfg, residual=res.to(DEV), token_mask=all_real)
    assert torch.equal(out1, ref_out)


def test_swapped_and_tiled_gemms_agree():
    """The same tokens through the swapped GEMMs (a small batch) and through
    the 256-row tiles (inside a large batch) give the same bits: both add the
    K steps in the same order and apply the same epilogue arithmetic."""
    T, H = 2048, 1024
    cfg = BlockConfig(T=T, H=H)
    d = _dev(inputs.make_block_inputs(T, H, seed=41, unit_scale=True))
    big, ids_big, _ = _run(d, cfg)  # 128 rows per expert: tiled
    n = 300                          # 18.75 rows per expert: swapped
    small, ids_small, _ = _run(dict(d, x=d["x"][:n].contiguous()), cfg.with_tokens(n))
    assert torch.equal(ids_small, ids_big[:n])
    diff = (small.float() - big[:n].float()).abs()
    assert torch.equal(small, big[:n]), f"max diff {diff.max().item()}, {int((diff > 0).sum())} differ"


@pytest.mark.parametrize("wid", [0, 1])
def test_forward_small_workloads_in_full(wid):
    wl = inputs.WORKLOADS[wid]
    cfg = BlockConfig(T=wl.T, H=wl.H)
    d = inputs.workload_inputs(wid)
    out, ids, w = _run(_dev(d), cfg)
    dn = parity.np_inputs(d)
    rrep = parity.check_routing(ids, w, dn["x"], dn["Wr"], dn["bias"], cfg)
    orep = parity.check_output(out, ids, dn, cfg)
    print(f"{wl.name}: routing {rrep} output {orep}")
    assert orep["rms_rel"] < 1e-2


@pytest.mark.parametrize("wid", [2, 3, 5])
def test_forward_large_workloads_sampled(wid):
    wl = inputs.WORKLOADS[wid]
    cfg = BlockConfig(T=wl.T, H=wl.H)
    d = inputs.workload_inputs(wid)
    mask = inputs.token_mask(wl)
    mask_np = None if mask is None else mask.numpy()
    out, ids, w = _run(_dev(d), cfg, token_mask=None if mask is None else mask.to(DEV))
    dn = parity.np_inputs(d)
    rrep = parity.check_routing(ids, w, dn["x"], dn["Wr"], dn["bias"], cfg, token_mask=mask_np)
    rng = np.random.default_rng(wid)
    sample = np.concatenate([[0, wl.T - 1, wl.T - 441], rng.choice(wl.T, 253, replace=False)])
    orep = parity.check_output(out, ids, dn, cfg, tokens=sample, token_mask=mask_np)
    ids_np = ids.cpu().numpy()
    counts = np.bincount(ids_np[ids_np >= 0].ravel(), minlength=128)
    print(f"{wl.name}: routing {rrep} output {orep} rows/expert min {counts.min()} "
          f"max {counts.max()}")
    assert orep["rms_rel"] < 1e-2
    if wl.hot_experts is not None:
        frac = counts[list(wl.hot_experts)].sum() / counts.sum()
        print(f"hot-expert share of selections: {frac:.3f}")


def test_forward_deterministic_and_isolated():
    T, H = 1000, 1024
    cfg = BlockConfig(T=T, H=H)
    d = _dev(inputs.make_block_inputs(T, H, seed=99, unit_scale=True))
    a, ids_a, _ = _run(d, cfg)
    b, ids_b, _ = _run(d, cfg)
    assert torch.equal(a, b) and torch.equal(ids_a, ids_b)
    # each token's output does not depend on the other tokens of the call
    split = 371
    for lo, hi in ((0, split), (split, T)):
        part = dict(d, x=d["x"][lo:hi].contiguous())
        p, _, _ = _run(part, cfg.with_tokens(hi - lo))
        assert torch.equal(p, a[lo:hi])


@pytest.mark.parametrize("T,H", [(240, 1024), (784, 2048), (1000, 1024)])
def test_small_batch_fused_projections_repeatable(T, H):
    """Few rows per expert: both expert projections run as one launch whose down
    items read the h rows that other CTAs' up items write.  Ten runs give the
    same bits (a missing wait or an overwritten input would show up as a
    difference between runs), with a residual as in the stacked model."""
    cfg = BlockConfig(T=T, H=H)
    d = _dev(inputs.make_block_inputs(T, H, seed=T + 7, unit_scale=True))
    res = inputs.make_tokens(T, H, seed=5).to(DEV)
    first = None
    for _ in range(10):
        out, ids, _ = _run(d, cfg, residual=res)
        if first is None:
            first = out.clone()
        else:
            assert torch.equal(out, first)


@pytest.mark.parametrize("overlap", [True, False])
def test_forward_host_batches_match_device_forward(overlap):
    """Host-resident batches streamed through the block give, bit for bit, the
    device entry point's output for each batch (and the oracle's, to tolerance)."""
    T, H = 700, 512
    cfg = BlockConfig(T=T, H=H, I=256, I_shared=256)
    d = inputs.make_block_inputs(T, H, seed=21, I=256, I_shared=256, unit_scale=True)
    dd = _dev(d)
    n = 5
    g = torch.Generator().manual_seed(77)
    xs = [torch.randn((T, H), generator=g).to(torch.bfloat16) for _ in range(n - 1)]
    xs.append(xs[0])  # a repeated input pointer is allowed
    if overlap:
        xs = [x.pin_memory() for x in xs]
    outs = [torch.zeros((T, H), dtype=torch.bfloat16) for _ in range(n)]
    if overlap:
        outs = [o.pin_memory() for o in outs]
    streams = (torch.cuda.Stream(), torch.cuda.Stream()) if overlap else None
    ws = ops.forward_host(xs, outs, dd["Wr"], dd["bias"], dd["w13"], dd["w2"], dd["ws13"],
                          dd["ws2"], cfg, copy_streams=streams)
    torch.cuda.current_stream().synchronize()
    code, site = ops.read_device_status(ws)
    assert code == 0, (ops.status_string(code), site)
    for b in range(n):
        ref, _, _ = _run(dict(dd, x=xs[b].to(DEV)), cfg)
        assert torch.equal(outs[b], ref.cpu()), b
    ids_b = _run(dict(dd, x=xs[1].to(DEV)), cfg)[1]
    d_np = {k: parity.to_np(v) for k, v in dict(d, x=xs[1]).items() if v is not None}
    parity.check_output(outs[1], ids_b, d_np, cfg)


@pytest.mark.parametrize("T,H,I", [(1, 256, 128), (40, 512, 192), (64, 320, 256),
                                   (300, 512, 256), (1000, 1024, 768), (2048, 2048, 1536)])
def test_dense_ffn_matches_oracle(T, H, I):
    """Dense feed-forward layer (up to 64 rows: swapped GEMMs, else tiled), with
    and without a residual (also in place)."""
    g = torch.Generator().manual_seed(T + I)
    x = torch.randn((T, H), generator=g).to(torch.bfloat16)
    w13 = (torch.randn((2 * I, H), generator=g) * H ** -0.5).to(torch.bfloat16)
    w2 = (torch.randn((H, I), generator=g) * I ** -0.5).to(torch.bfloat16)
    res = torch.randn((T, H), generator=g).to(torch.bfloat16)
    xd, w13d, w2d, resd = (t.to(DEV) for t in (x, w13, w2, res))
    out = ops.dense_ffn(xd, w13d, w2d)
    out_r = ops.dense_ffn(xd, w13d, w2d, residual=resd)
    buf = resd.clone()
    ops.dense_ffn(xd, w13d, w2d, residual=buf, out=buf)
    torch.cuda.synchronize()
    assert torch.equal(buf, out_r)
    xn, w13n, w2n, resn = (parity.to_np(t) for t in (x, w13, w2, res))
    for got, ref in ((out, oracle.dense_ffn(xn, w13n, w2n)),
                     (out_r, oracle.dense_ffn(xn, w13n, w2n, residual=resn))):
        g_np = parity.to_np(got).astype(np.float64)
        err = np.abs(g_np - ref)
        assert np.all(err <= parity.OUT_RTOL * (1 + np.abs(ref))), err.max()
        assert np.sqrt(np.mean(err ** 2) / np.mean(ref ** 2)) < 1e-2


# ------------------------------------------------------------------ RMSNorm, residual stack
def test_rmsnorm_matches_oracle():
    T, H = 333, 2048
    x = (3.0 * torch.randn((T, H), generator=torch.Generator().manual_seed(4))).to(torch.bfloat16)
    gamma = torch.rand(H, generator=torch.Generator().manual_seed(5)) + 0.5
    for g in (None, gamma):
        y = ops.rmsnorm(x.to(DEV), None if g is None else g.to(DEV), eps=1e-6)
        ref = oracle.rmsnorm(parity.to_np(x), 1e-6, None if g is None else g.numpy())
        got = parity.to_np(y)
        # one bf16 rounding of an fp32 result
        assert np.max(np.abs(got - ref) / (np.abs(ref) + 1e-3)) < 8e-3


def test_residual_stack_teacher_forced():
    # x <- x + block_l(RMSNorm(x)) for 3 layers; each layer is checked against
    # the oracle on the GPU's own bf16 input to that layer
    T, H, L = 700, 1024, 3
    cfg = BlockConfig(T=T, H=H)
    x = inputs.make_tokens(T, H, seed=4).to(DEV)
    for layer in range(L):
        wts = inputs.make_weights(H, seed=4, layer=layer)
        dw = _dev(wts)
        xin = x.clone()
        xn = ops.rmsnorm(x, eps=1e-6)
        out, ids, w = _run(dict(dw, x=xn), cfg, residual=x)
        dn = parity.np_inputs(dict(wts, x=xn.cpu()))
        parity.check_routing(ids, w, dn["x"], dn["Wr"], dn["bias"], cfg)
        rep = parity.check_output(out, ids, dn, cfg, residual_np=parity.to_np(xin))
        assert rep["rms_rel"] < 1e-2
        x = out


# ------------------------------------------------------------------ failure detection
def test_bounded_wait_times_out_and_context_survives():
    code, site = ops.selftest_wait_timeout(timeout_ns=50_000_000)  # 50 ms
    assert code == 5 and site == 99
    # the context is still usable
    T, H = 64, 256
    cfg = BlockConfig(T=T, H=H, E=16, I=128, I_shared=128, top_k=4)
    d = _dev(inputs.make_block_inputs(T, H, seed=1, E=16, I=128, I_shared=128, unit_scale=True))
    out, ids, _ = _run(d, cfg)
    assert torch.isfinite(out.float()).all()
