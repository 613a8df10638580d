"""Guard words around every buffer a call writes, and untouched inputs.

Each output and the workspace are views into a larger allocation whose bytes
before and after the view are filled with a pattern; after the call the
pattern must be intact (no write past either end), and the inputs must be
bit-identical to copies taken before the call.  Shapes cover the tiled and
the swapped GEMMs, the fused and the separate shared expert, no shared
expert, the padding mask, the dense FFN and the permutation.
"""

import pytest
import torch

from routed_moe_layer_b200 import inputs, ops
from routed_moe_layer_b200.ops import BlockConfig

GUARD = 4096          # bytes on each side (a multiple of the 256-byte workspace alignment)
PATTERN = 0xA5


def guarded(shape, dtype, device):
    """A tensor of ``shape`` inside a byte buffer with GUARD pattern bytes on
    both sides; returns (tensor, check) where check() asserts both guards
    are intact."""
    nbytes = int(torch.Size(shape).numel()) * torch.empty((), dtype=dtype).element_size()
    raw = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device=device)
    view = raw[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def check():
        head = raw[:GUARD]
        tail = raw[GUARD + nbytes:]
        assert bool((head == PATTERN).all()), "write before the start of the buffer"
        assert bool((tail == PATTERN).all()), "write past the end of the buffer"
    return view, check


def test_guard_helper_detects_writes_on_cpu():
    t, check = guarded((3, 5), torch.float32, "cpu")
    t.fill_(1.0)
    check()
    t.view(-1)[:0].fill_(0)  # empty write: still fine
    check()
    raw = t.view(torch.uint8).view(-1)
    base = raw.untyped_storage().data_ptr()
    assert raw.data_ptr() - base == GUARD
    # a write one element past the end is caught
    full = torch.empty(0, dtype=torch.uint8).set_(raw.untyped_storage())
    full[GUARD + raw.numel()] = 0
    with pytest.raises(AssertionError):
        check()


DEV = "cuda"

CASES = [
    # T, H, E, I, I_shared, k, G, g, masked
    (100, 256, 16, 128, 128, 4, 4, 2, False),      # swapped GEMMs (chunks of 128 rows)
    (300, 512, 128, 192, 64, 8, 4, 2, False),      # swapped (32-row chunks), separate shared
    (1000, 512, 16, 128, 0, 4, 4, 2, False),       # tiled, no shared expert
    (1500, 256, 32, 128, 128, 8, 4, 2, True),      # tiled, fused shared expert, padding mask
]


@pytest.mark.gpu
@pytest.mark.parametrize("T,H,E,I,Is,k,G,g,masked", CASES)
def test_forward_writes_only_its_buffers(T, H, E, I, Is, k, G, g, masked):
    cfg = BlockConfig(T=T, H=H, E=E, I=I, I_shared=Is, top_k=k, n_group=G, topk_group=g)
    d = {n: (None if v is None else v.to(DEV)) for n, v in
         inputs.make_block_inputs(T, H, seed=T, E=E, I=I, I_shared=Is, unit_scale=True).items()}
    before = {n: (None if v is None else v.clone()) for n, v in d.items()}
    mask = None
    if masked:
        mask = torch.ones(T, dtype=torch.uint8, device=DEV)
        mask[T // 2: T // 2 + 100] = 0
    out, c_out = guarded((T, H), torch.bfloat16, DEV)
    ids, c_ids = guarded((T, k), torch.int32, DEV)
    w, c_w = guarded((T, k), torch.float32, DEV)
    ws, c_ws = guarded((ops.workspace_bytes(cfg),), torch.uint8, DEV)
    ops.forward(d["x"], d["Wr"], d["bias"], d["w13"], d["w2"], d["ws13"], d["ws2"], cfg,
                out=out, workspace=ws, topk_ids=ids, topk_w=w, token_mask=mask)
    torch.cuda.synchronize()
    code, site = ops.read_device_status(ws)
    assert code == 0, (ops.status_string(code), site)
    for check in (c_out, c_ids, c_w, c_ws):
        check()
    for n, v in d.items():
        if v is not None:
            assert torch.equal(v, before[n]), f"input {n} was modified"


@pytest.mark.gpu
@pytest.mark.parametrize("T", [40, 700])  # swapped, tiled
def test_dense_ffn_writes_only_its_buffers(T):
    H, I = 256, 384
    x = inputs.make_tokens(T, H, seed=2).to(DEV)
    wd = {n: v.to(DEV) for n, v in inputs.make_dense_weights(H, I, seed=2, std=H ** -0.5).items()}
    res = inputs.make_tokens(T, H, seed=3).to(DEV)
    before = [t.clone() for t in (x, wd["w13"], wd["w2"], res)]
    out, c_out = guarded((T, H), torch.bfloat16, DEV)
    ws, c_ws = guarded((ops.lib().moe_dense_ffn_workspace_bytes(T, H, I),), torch.uint8, DEV)
    ops.dense_ffn(x, wd["w13"], wd["w2"], residual=res, out=out, workspace=ws)
    torch.cuda.synchronize()
    c_out()
    c_ws()
    for a, b in zip((x, wd["w13"], wd["w2"], res), before):
        assert torch.equal(a, b)


@pytest.mark.gpu
def test_permute_writes_only_its_buffers():
    T, E, k, H = 777, 64, 6, 256
    cfg = BlockConfig(T=T, H=H, E=E, top_k=k, n_group=8, topk_group=3)
    g = torch.Generator().manual_seed(4)
    ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    tw = torch.rand((T, k), generator=g)
    x = inputs.make_tokens(T, H, seed=4)
    ids, tw, x = ids.to(DEV), tw.to(DEV), x.to(DEV)
    ws, c_ws = guarded((ops.permute_workspace_bytes(cfg),), torch.uint8, DEV)
    res = ops.permute(ids, cfg, topk_w=tw, x=x, workspace=ws)
    torch.cuda.synchronize()
    c_ws()
    # the outputs are fresh tensors of their exact sizes: their contents are checked
    # bit for bit by the parity tests; here the row table must be a permutation
    assert torch.equal(torch.sort(res["row_of"].long()).values,
                       torch.arange(T * k, device=DEV))
