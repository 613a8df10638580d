"""The product path has no CPU fallback: without the CUDA library, or given
host tensors, every entry point raises instead of computing anything."""

import pytest
import torch

from routed_moe_layer_b200 import ops
from routed_moe_layer_b200.ops import BlockConfig


def test_missing_library_raises(monkeypatch):
    monkeypatch.setattr(ops, "_lib", None)
    monkeypatch.setattr(ops, "LIB_PATH", "/nonexistent/libroutedmoe.so")
    with pytest.raises(RuntimeError, match="missing"):
        ops.lib()


def _cpu_block(T=4, H=64, E=8, I=64):
    x = torch.zeros((T, H), dtype=torch.bfloat16)
    return dict(x=x, Wr=torch.zeros((E, H)), bias=torch.zeros(E),
                w13=torch.zeros((E, 2 * I, H), dtype=torch.bfloat16),
                w2=torch.zeros((E, H, I), dtype=torch.bfloat16),
                ws13=torch.zeros((2 * I, H), dtype=torch.bfloat16),
                ws2=torch.zeros((H, I), dtype=torch.bfloat16))


def test_host_tensors_are_rejected():
    cfg = BlockConfig(T=4, H=64, E=8, I=64, I_shared=64, top_k=2, n_group=2, topk_group=1)
    d = _cpu_block()
    with pytest.raises(ValueError, match="CUDA"):
        ops.forward(d["x"], d["Wr"], d["bias"], d["w13"], d["w2"], d["ws13"], d["ws2"], cfg)
    with pytest.raises(ValueError, match="CUDA"):
        ops.route(d["x"], d["Wr"], d["bias"], cfg)
    with pytest.raises(ValueError, match="CUDA"):
        ops.dense_ffn(d["x"], d["ws13"], d["ws2"])
    with pytest.raises(ValueError, match="CUDA"):
        ops.rmsnorm(d["x"])


def test_wrong_dtypes_and_shapes_are_rejected():
    d = _cpu_block()
    with pytest.raises(ValueError):
        ops._need(d["x"].float(), "x", torch.bfloat16, (4, 64))
    with pytest.raises(ValueError):
        ops._need(d["x"], "x", torch.bfloat16, (4, 128))
    with pytest.raises(TypeError):
        ops._need(None, "x", torch.bfloat16, (4, 64))
    # the host-batch entry point wants host tensors and checks them first
    with pytest.raises(ValueError, match="host"):
        ops._need_host(torch.zeros((4, 64), dtype=torch.bfloat16, device="meta"), "x_host",
                       (4, 64))
