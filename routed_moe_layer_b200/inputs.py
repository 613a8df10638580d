"""Seeded synthetic inputs for the routed MoE block.

This module holds no arithmetic of the method: it only draws tensors.  It is
the one module that both the CUDA path (tests, bench) and the CPU oracle
(through the tests) receive their inputs from.

Recipe.  One ``torch.Generator`` per tensor, seeded ``seed*1000 + idx`` (for
layer ``l`` of a residual stack ``seed*1000 + 100*l + idx``), tensor indices
0 x, 1 Wr, 2 bias, 3 w13, 4 w2, 5 ws13, 6 ws2.  Draws are fp32; bf16 tensors
are the fp32 draw rounded to nearest-even by ``Tensor.to(torch.bfloat16)``.
  x     ~ N(0, 1)          bf16 [T, H]
  Wr    ~ N(0, 0.02)       fp32 [E, H]
  bias  ~ U(-0.1, 0.1)     fp32 [E]     (hot experts, if any, set to +hot_bias)
  w13   ~ N(0, 0.02)       bf16 [E, 2I, H]   (gate rows, then up rows)
  w2    ~ N(0, 0.02)       bf16 [E, H, I]
  ws13  ~ N(0, 0.02)       bf16 [2I_s, H]
  ws2   ~ N(0, 0.02)       bf16 [H, I_s]
"""

from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch

# Named workloads: shapes and seeds of the benchmark / parity configurations.
#   0: one layer, 240 tokens, H=1024
#   1: one layer, 784 tokens (720 video = 3 latent frames x 12x20 patches + 64 text), H=2048
#   2: one layer, 19412 tokens (18900 video = 21 x 30x30 + 512 text), H=2048
#   3: CFG batch 2 x 19412 = 38824 rows, H=2048, bias +0.5 on 8 hot experts
#   4: 48 residual layers x (RMSNorm -> block) at 19412 tokens, H=2048
#   5: CFG batch 2 x 19412 rows with padded text: the second prompt has 64 real
#      text tokens, its other 448 text rows are padding (token mask 0)
#   6: dense feed-forward layer (a block without experts), 19412 tokens, H=2048,
#      intermediate 6912 = 9 x 768 (the active width of one token of the MoE block)
HOT_EXPERTS = tuple(range(0, 128, 16))  # two per group of 32


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    seed: int
    layers: int = 1
    hot_experts: Optional[Sequence[int]] = None
    hot_bias: float = 0.5
    padding: Optional[Sequence[tuple]] = None  # [start, stop) row ranges of padding tokens
    dense_I: int = 0  # > 0: a dense feed-forward layer of this intermediate size


WORKLOADS = {
    0: Workload("moe_layer_T240_H1024", 240, 1024, 0),
    1: Workload("moe_layer_T784_H2048", 784, 2048, 1),
    2: Workload("moe_layer_T19412_H2048", 19412, 2048, 2),
    3: Workload("moe_layer_cfg2x19412_H2048_skewed", 38824, 2048, 3, hot_experts=HOT_EXPERTS),
    4: Workload("moe_stack48_T19412_H2048", 19412, 2048, 4, layers=48),
    5: Workload("moe_layer_cfg2x19412_H2048_padded", 38824, 2048, 5,
                padding=((19412 + 18900 + 64, 38824),)),
    6: Workload("dense_ffn_T19412_H2048_I6912", 19412, 2048, 6, dense_I=6912),
}


def token_mask(w: Workload, device="cpu") -> Optional[torch.Tensor]:
    """uint8 [T] mask of a workload (1 = real token, 0 = padding), or None."""
    if not w.padding:
        return None
    m = torch.ones(w.T, dtype=torch.uint8)
    for a, b in w.padding:
        m[a:b] = 0
    return m.to(device)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, std, seed, device, dtype):
    t = torch.randn(shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _uniform(shape, lo, hi, seed, device):
    t = torch.rand(shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return t.mul_(hi - lo).add_(lo)


def make_tokens(T: int, H: int, seed: int, device="cpu") -> torch.Tensor:
    return _normal((T, H), 1.0, seed * 1000 + 0, device, torch.bfloat16)


def make_weights(H: int, seed: int, E: int = 128, I: int = 768, I_shared: int = 768,
                 device="cpu", layer: int = 0, hot_experts=None, hot_bias: float = 0.5,
                 wr_std: float = 0.02, w13_std: float = 0.02, w2_std: float = 0.02):
    """Returns dict(Wr, bias, w13, w2, ws13, ws2) for one block."""
    base = seed * 1000 + 100 * layer
    Wr = _normal((E, H), wr_std, base + 1, device, torch.float32)
    bias = _uniform((E,), -0.1, 0.1, base + 2, device)
    if hot_experts is not None:
        bias[list(hot_experts)] = hot_bias
    w13 = _normal((E, 2 * I, H), w13_std, base + 3, device, torch.bfloat16)
    w2 = _normal((E, H, I), w2_std, base + 4, device, torch.bfloat16)
    if I_shared > 0:
        ws13 = _normal((2 * I_shared, H), w13_std, base + 5, device, torch.bfloat16)
        ws2 = _normal((H, I_shared), w2_std, base + 6, device, torch.bfloat16)
    else:
        ws13 = ws2 = None
    return dict(Wr=Wr, bias=bias, w13=w13, w2=w2, ws13=ws13, ws2=ws2)


def make_dense_weights(H: int, I: int, seed: int, device="cpu", std: float = 0.02):
    """Returns dict(w13 [2I,H], w2 [H,I]) of a dense feed-forward layer
    (tensor indices 3 and 4 of the recipe)."""
    base = seed * 1000
    return dict(w13=_normal((2 * I, H), std, base + 3, device, torch.bfloat16),
                w2=_normal((H, I), std, base + 4, device, torch.bfloat16))


def make_block_inputs(T: int, H: int, seed: int, E: int = 128, I: int = 768,
                      I_shared: int = 768, device="cpu", hot_experts=None,
                      hot_bias: float = 0.5, unit_scale: bool = False):
    """Tokens + weights of one block: dict(x, Wr, bias, w13, w2, ws13, ws2).

    unit_scale: draw every weight with std 1/sqrt(fan_in) (router included),
    so that logits, activations and outputs are O(1) at any size."""
    stds = {}
    if unit_scale:
        stds = dict(wr_std=H ** -0.5, w13_std=H ** -0.5, w2_std=I ** -0.5)
    d = make_weights(H, seed, E=E, I=I, I_shared=I_shared, device=device,
                     hot_experts=hot_experts, hot_bias=hot_bias, **stds)
    d["x"] = make_tokens(T, H, seed, device=device)
    return d


def workload_inputs(cfg_id: int, device="cpu", layer: int = 0):
    """Inputs of a named workload (for a stack: the tokens and layer ``layer``)."""
    w = WORKLOADS[cfg_id]
    if w.dense_I:
        d = make_dense_weights(w.H, w.dense_I, w.seed, device=device)
    else:
        d = make_weights(w.H, w.seed, device=device, layer=layer,
                         hot_experts=w.hot_experts, hot_bias=w.hot_bias)
    d["x"] = make_tokens(w.T, w.H, w.seed, device=device)
    return d
