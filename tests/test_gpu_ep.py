"""Expert parallelism's device steps on one GPU (one rank holds every expert,
so both exchanges are the identity): route, permute, the rows' expert ids, the
receiver's sort by expert, the experts on grouped rows, the shared expert and
the restore through row_of must give exactly the bits of moe_forward.  The
exchange itself is covered on gloo ranks (tests/test_ep_gloo.py); one GPU is
all a run gets here, so the multi-rank device path is not run."""

import pytest
import torch

from routed_moe_layer_b200 import inputs, ops
from routed_moe_layer_b200.dist import ep_forward
from routed_moe_layer_b200.ops import BlockConfig

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("T,H,E,I,k", [
    (1, 256, 16, 128, 4),
    (240, 1024, 128, 768, 8),      # swapped GEMMs on the received rows
    (2048, 1024, 128, 768, 8),     # tiled GEMMs (tile prefix from the row offsets)
    (700, 320, 16, 128, 4),        # H not a multiple of 256
])
def test_one_rank_ep_equals_the_block(T, H, E, I, k):
    cfg = BlockConfig(T=T, H=H, E=E, I=I, I_shared=I, top_k=k, n_group=4, topk_group=2)
    d = {n: (None if v is None else v.to(DEV)) for n, v in
         inputs.make_block_inputs(T, H, seed=3 + T, E=E, I=I, I_shared=I, unit_scale=True).items()}
    res = inputs.make_tokens(T, H, seed=99).to(DEV)
    ref = ops.forward(d["x"], d["Wr"], d["bias"], d["w13"], d["w2"], d["ws13"], d["ws2"], cfg,
                      residual=res)
    out = ep_forward(d["x"], d["Wr"], d["bias"], d["w13"], d["w2"], d["ws13"], d["ws2"], cfg,
                     residual=res)
    torch.cuda.synchronize()
    diff = (out.float() - ref.float()).abs()
    assert torch.equal(out, ref), f"max diff {diff.max().item()}, {int((diff > 0).sum())} differ"
