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
FP8 expert weights (``make_fp8_weights``): the same normal draws as w13..ws2,
stored as E4M3 codes with one power-of-two scale per 128 x 128 block
(scale exponents: tensor indices 7-10).
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


FP8_BLOCK = 128  # rows and columns of one scale block of an FP8 weight matrix


def _fp8_matrix(shape, std, seed, scale_seed, device):
    """E4M3 codes (uint8, ``shape``) and UE8M0 scale exponents (uint8, one per
    128 x 128 block of the last two dimensions): exponents ~ U{118, 119, 120}
    (scales 2^-9 .. 2^-7); codes = the N(0, std) draw of seed ``seed`` divided by
    its block's scale, clamped to +-448 and cast by ``Tensor.to(float8_e4m3fn)``."""
    N, K = shape[-2], shape[-1]
    nb, kb = -(-N // FP8_BLOCK), -(-K // FP8_BLOCK)
    sexp = torch.randint(118, 121, (*shape[:-2], nb, kb), generator=_gen(scale_seed, device),
                         device=device, dtype=torch.int32)
    scale = torch.exp2(sexp.to(torch.float32) - 127.0)
    scale = scale.repeat_interleave(FP8_BLOCK, -2)[..., :N, :]
    scale = scale.repeat_interleave(FP8_BLOCK, -1)[..., :K]
    draw = _normal(shape, std, seed, device, torch.float32)
    codes = (draw / scale).clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, sexp.to(torch.uint8)


def make_fp8_weights(H: int, seed: int, E: int = 128, I: int = 768, I_shared: int = 768,
                     device="cpu", layer: int = 0, w13_std: float = 0.02,
                     w2_std: float = 0.02):
    """FP8 expert weights of one block: dict(w13_q, w13_s, w2_q, w2_s, ws13_q,
    ws13_s, ws2_q, ws2_s); ``*_q`` E4M3 codes shaped like the bf16 weights of
    ``make_weights``, drawn from the same normal draws (tensor indices 3-6),
    ``*_s`` their UE8M0 block scale exponents (tensor indices 7-10)."""
    base = seed * 1000 + 100 * layer
    d = {}
    d["w13_q"], d["w13_s"] = _fp8_matrix((E, 2 * I, H), w13_std, base + 3, base + 7, device)
    d["w2_q"], d["w2_s"] = _fp8_matrix((E, H, I), w2_std, base + 4, base + 8, device)
    if I_shared > 0:
        d["ws13_q"], d["ws13_s"] = _fp8_matrix((2 * I_shared, H), w13_std, base + 5, base + 9,
                                               device)
        d["ws2_q"], d["ws2_s"] = _fp8_matrix((H, I_shared), w2_std, base + 6, base + 10, device)
    else:
        d["ws13_q"] = d["ws13_s"] = d["ws2_q"] = d["ws2_s"] = None
    return d


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
