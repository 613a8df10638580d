"""FP8 expert weights (weight-only: E4M3 codes, one power-of-two scale per
128 x 128 block) through the C ABI.

Two gates: the FP8 block must give exactly the bits of the bf16 block run on
the dequantised weights (the oracle dequantises them; with power-of-two
scales they are bf16 values), and it must meet the block's parity contract
against the float64 oracle's FP8 forward.  Shapes cover both token-chunk
sizes, the fused and the separate shared expert, no shared expert, the
240-token workload's shape and a batch above the bf16 path's swapped range.
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

FP8_CASES = [
    # T, H, E, I, I_shared, k, G, g
    (1, 256, 16, 128, 128, 4, 4, 2),        # 32-row chunks, fused shared expert
    (100, 256, 16, 128, 128, 4, 4, 2),      # 128-row chunks, several per expert
    (64, 256, 64, 128, 256, 6, 8, 3),       # separate shared-expert GEMMs
    (300, 512, 32, 256, 0, 8, 4, 2),        # no shared expert, two weight tiles per N
    (240, 1024, 128, 768, 768, 8, 4, 2),    # the 240-token workload's shape
    (2048, 2048, 128, 768, 768, 8, 4, 2),   # bf16 path tiled here; FP8 stays swapped
]


def _fp8(H, E, I, Is, seed):
    return inputs.make_fp8_weights(H, seed, E=E, I=I, I_shared=Is, w13_std=H ** -0.5,
                                   w2_std=I ** -0.5)


def _dequantised(q):
    """bf16 weights written out by the oracle from the codes and scales."""
    out = {}
    for name in ("w13", "w2", "ws13", "ws2"):
        if q[name + "_q"] is None:
            out[name] = None
            continue
        deq = oracle.fp8_block_dequant(q[name + "_q"].numpy(), q[name + "_s"].numpy())
        t = torch.from_numpy(deq).to(torch.bfloat16)
        assert torch.equal(t.double(), torch.from_numpy(deq))  # exact bf16 values
        out[name] = t
    return out


def _status_ok(ws):
    code, site = ops.read_device_status(ws)
    assert code == 0, (ops.status_string(code), site)


@pytest.mark.parametrize("T,H,E,I,Is,k,G,g", FP8_CASES)
def test_fp8_block_is_the_bf16_block_on_dequantised_weights(T, H, E, I, Is, k, G, g):
    cfg = BlockConfig(T=T, H=H, E=E, I=I, I_shared=Is, top_k=k, n_group=G, topk_group=g)
    d = inputs.make_block_inputs(T, H, seed=5 + T, E=E, I=I, I_shared=Is, unit_scale=True)
    q = _fp8(H, E, I, Is, seed=5 + T)
    deq = _dequantised(q)
    x, Wr, bias = (d[n].to(DEV) for n in ("x", "Wr", "bias"))
    qd = {n: (None if v is None else v.to(DEV)) for n, v in q.items()}
    ws = ops.alloc_workspace(ops.workspace_bytes(cfg), DEV)
    out8 = ops.forward_fp8(x, Wr, bias, qd, cfg, workspace=ws)
    torch.cuda.synchronize()
    _status_ok(ws)
    dd = {n: (None if v is None else v.to(DEV)) for n, v in deq.items()}
    out16 = ops.forward(x, Wr, bias, dd["w13"], dd["w2"], dd["ws13"], dd["ws2"], cfg)
    torch.cuda.synchronize()
    diff = (out8.float() - out16.float()).abs()
    assert torch.equal(out8, out16), f"max diff {diff.max().item()}, {int((diff > 0).sum())} differ"


@pytest.mark.parametrize("T,H,E,I,Is,k,G,g", FP8_CASES[:5])
def test_fp8_block_matches_oracle(T, H, E, I, Is, k, G, g):
    cfg = BlockConfig(T=T, H=H, E=E, I=I, I_shared=Is, top_k=k, n_group=G, topk_group=g)
    d = inputs.make_block_inputs(T, H, seed=9 + T, E=E, I=I, I_shared=Is, unit_scale=True)
    q = _fp8(H, E, I, Is, seed=9 + T)
    x, Wr, bias = (d[n].to(DEV) for n in ("x", "Wr", "bias"))
    qd = {n: (None if v is None else v.to(DEV)) for n, v in q.items()}
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    ws = ops.alloc_workspace(ops.workspace_bytes(cfg), DEV)
    out = ops.forward_fp8(x, Wr, bias, qd, cfg, workspace=ws, topk_ids=ids, topk_w=w)
    torch.cuda.synchronize()
    _status_ok(ws)
    dn = parity.np_inputs(dict(x=d["x"], Wr=d["Wr"], bias=d["bias"]))
    parity.check_routing(ids, w, dn["x"], dn["Wr"], dn["bias"], cfg)
    # reference: the oracle's FP8 forward under the GPU's expert choice
    qn = {n: (None if v is None else v.numpy()) for n, v in q.items()}
    ref, _, _, _ = oracle.moe_forward_fp8(
        dn["x"], dn["Wr"], dn["bias"], qn["w13_q"], qn["w13_s"], qn["w2_q"], qn["w2_s"],
        qn["ws13_q"], qn["ws13_s"], qn["ws2_q"], qn["ws2_s"], parity.oracle_cfg(cfg),
        ids=ids.cpu().numpy())
    got = parity.to_np(out).astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= parity.OUT_RTOL * (1.0 + np.abs(ref))), err.max()
    assert np.sqrt(np.mean(err ** 2) / np.mean(ref ** 2)) < 1e-2


def test_fp8_padding_mask_and_residual():
    T, H, E, I = 300, 256, 32, 128
    cfg = BlockConfig(T=T, H=H, E=E, I=I, I_shared=I)
    d = inputs.make_block_inputs(T, H, seed=21, E=E, I=I, I_shared=I, unit_scale=True)
    q = _fp8(H, E, I, I, seed=21)
    deq = _dequantised(q)
    x, Wr, bias = (d[n].to(DEV) for n in ("x", "Wr", "bias"))
    qd = {n: (None if v is None else v.to(DEV)) for n, v in q.items()}
    mask = torch.ones(T, dtype=torch.uint8)
    mask[200:260] = 0
    res = torch.randn((T, H), generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    out8 = ops.forward_fp8(x, Wr, bias, qd, cfg, residual=res.to(DEV),
                           token_mask=mask.to(DEV))
    dd = {n: v.to(DEV) for n, v in deq.items()}
    out16 = ops.forward(x, Wr, bias, dd["w13"], dd["w2"], dd["ws13"], dd["ws2"], cfg,
                        residual=res.to(DEV), token_mask=mask.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(out8, out16)
