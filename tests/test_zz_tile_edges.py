"""Row counts at the tile and chunk boundaries of the grouped GEMMs.

A correction bias of +100 on experts 0..7 makes every token select exactly
those eight experts (the bias acts on selection only; the gating weights come
from the raw scores), so each of them holds exactly T rows and every other
expert none.  T is then chosen at the boundaries of the 256-row pair tiles
(tiled GEMMs) and of the 32- and 128-row token chunks (swapped GEMMs): one
row short of a tile, exactly a tile, one row over.
"""

import numpy as np
import pytest
import torch

from routed_moe_layer_b200 import inputs, ops
from routed_moe_layer_b200.ops import BlockConfig
from tests import parity

pytestmark = pytest.mark.gpu

DEV = "cuda"
FORCED = list(range(8))


@pytest.mark.parametrize("E,T", [
    (16, 255), (16, 256), (16, 257), (16, 513),     # tiled: T*8 > 64*16
    (128, 31), (128, 32), (128, 33),                # swapped, 32-row chunks (T*8 <= 20*128)
    (128, 383), (128, 384), (128, 385),             # swapped, 128-row chunks
])
def test_forced_experts_at_tile_boundaries(E, T):
    H, I = 256, 128
    cfg = BlockConfig(T=T, H=H, E=E, I=I, I_shared=I, top_k=8, n_group=4, topk_group=2)
    d = inputs.make_block_inputs(T, H, seed=E + T, E=E, I=I, I_shared=I, unit_scale=True)
    d["bias"][FORCED] = 100.0
    dd = {n: (None if v is None else v.to(DEV)) for n, v in d.items()}
    ids = torch.empty((T, 8), dtype=torch.int32, device=DEV)
    w = torch.empty((T, 8), dtype=torch.float32, device=DEV)
    ws = ops.alloc_workspace(ops.workspace_bytes(cfg), DEV)
    out = ops.forward(dd["x"], dd["Wr"], dd["bias"], dd["w13"], dd["w2"], dd["ws13"],
                      dd["ws2"], cfg, workspace=ws, topk_ids=ids, topk_w=w)
    torch.cuda.synchronize()
    code, site = ops.read_device_status(ws)
    assert code == 0, (ops.status_string(code), site)
    # every token took exactly the forced experts
    assert torch.equal(torch.sort(ids, dim=1).values.cpu(),
                       torch.tensor(FORCED, dtype=torch.int32).repeat(T, 1))
    dn = parity.np_inputs(d)
    parity.check_routing(ids, w, dn["x"], dn["Wr"], dn["bias"], cfg)
    rep = parity.check_output(out, ids, dn, cfg)
    assert rep["rms_rel"] < 1e-2, rep
    assert np.isfinite(rep["max_abs_err"])
