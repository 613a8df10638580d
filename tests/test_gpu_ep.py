"""Expert parallelism's device steps on one GPU (one rank holds every expert,
so both exchanges are the identity): route, permute, the rows' expert ids, the
receiver's sort by expert, the experts on grouped rows, the shared expert and
the restore through row_of.  Two gates: the output meets the block's parity
contract against the float64 oracle (evaluated under the GPU's expert choice),
and it is exactly the bits of moe_forward.  The exchange itself is covered on
gloo ranks (tests/test_ep_gloo.py); one GPU is all a run gets here, so the
multi-rank device path is not run."""

import pytest
import torch

from routed_moe_layer_b200 import inputs, ops
from routed_moe_layer_b200.dist import ep_forward
from routed_moe_layer_b200.ops import BlockConfig
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("T,H,E,I,k", [
    (1, 256, 16, 128, 4),
    (240, 1024, 128, 768, 8),      # swapped GEMMs on the received rows
    (2048, 1024, 128, 768, 8),     # tiled GEMMs (tile prefix from the row offsets)
    (700, 320, 16, 128, 4),        # H not a multiple of 256
])
def test_one_rank_ep_matches_oracle_and_the_block(T, H, E, I, k):
    cfg = BlockConfig(T=T, H=H, E=E, I=I, I_shared=I, top_k=k, n_group=4, topk_group=2)
    host = inputs.make_block_inputs(T, H, seed=3 + T, E=E, I=I, I_shared=I, unit_scale=True)
    d = {n: (None if v is None else v.to(DEV)) for n, v in host.items()}
    res_h = inputs.make_tokens(T, H, seed=99)
    res = res_h.to(DEV)
    ref = ops.forward(d["x"], d["Wr"], d["bias"], d["w13"], d["w2"], d["ws13"], d["ws2"], cfg,
                      residual=res)
    out = ep_forward(d["x"], d["Wr"], d["bias"], d["w13"], d["w2"], d["ws13"], d["ws2"], cfg,
                     residual=res)
    ids, w = ops.route(d["x"], d["Wr"], d["bias"], cfg)
    torch.cuda.synchronize()
    # against the oracle: routing gate, then the output under the GPU's ids
    dn = parity.np_inputs(host)
    parity.check_routing(ids, w, dn["x"], dn["Wr"], dn["bias"], cfg)
    rep = parity.check_output(out, ids, dn, cfg, residual_np=parity.to_np(res_h))
    assert rep["rms_rel"] < 1e-2, rep
    # against the block: bit for bit
    diff = (out.float() - ref.float()).abs()
    assert torch.equal(out, ref), f"max diff {diff.max().item()}, {int((diff > 0).sum())} differ"


def test_combine_rows_skips_rows_outside_y():
    """moe_combine_rows: a row_of entry at or beyond y's row count, or negative,
    adds 0 (like a rejected expert id); the rest is the fp32 sum in slot order."""
    T, H, k, R = 50, 256, 4, 120
    g = torch.Generator().manual_seed(7)
    y = torch.randn((R, H), generator=g).to(torch.bfloat16)
    row_of = torch.randint(0, R, (T, k), generator=g, dtype=torch.int32)
    row_of[3, 1] = R           # one past the end
    row_of[10, 0] = R + 1000   # far beyond
    row_of[20, 2] = -1         # rejected
    res = torch.randn((T, H), generator=g).to(torch.bfloat16)
    out = ops.combine_rows(y.to(DEV), row_of.reshape(-1).to(DEV), k, residual=res.to(DEV))
    torch.cuda.synchronize()
    ref = torch.zeros((T, H), dtype=torch.float32)
    for j in range(k):
        r = row_of[:, j].long()
        ok = (r >= 0) & (r < R)
        ref[ok] += y[r[ok]].float()
    ref += res.float()
    assert torch.equal(out.cpu(), ref.to(torch.bfloat16))
