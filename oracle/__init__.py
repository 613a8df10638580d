"""CPU oracle for the routed MoE block forward pass.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it.  It shares no code with the CUDA library (no
kernels, headers, helpers or constant tables); both sides receive the same
seeded inputs from ``routed_moe_layer_b200.inputs`` and nothing else.

The oracle is written for a reader checking it against the sources by eye:
plain NumPy, float64 arithmetic wherever the sources do not fix a precision,
no blocking, fusion or reordering.  See ``moe_oracle`` for the per-step
citations.
"""

from .moe_oracle import (  # noqa: F401
    MoeConfig,
    bf16_round,
    router_scores,
    group_limited_topk,
    route,
    routing_weights,
    swiglu_mlp,
    dense_ffn,
    apply_token_mask,
    moe_forward,
    moe_forward_tokens,
    permutation,
    rmsnorm,
    FP8_BLOCK,
    fp8_e4m3_decode,
    ue8m0_decode,
    fp8_block_dequant,
    moe_forward_fp8,
)
