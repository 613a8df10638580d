"""The seeded input generator (no method arithmetic): determinism and the
structure of the named workloads."""

import torch

from routed_moe_layer_b200 import inputs


def test_tokens_and_weights_are_seeded():
    a = inputs.make_block_inputs(8, 64, seed=3, E=8, I=64, I_shared=64)
    b = inputs.make_block_inputs(8, 64, seed=3, E=8, I=64, I_shared=64)
    c = inputs.make_block_inputs(8, 64, seed=4, E=8, I=64, I_shared=64)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert not torch.equal(a["x"], c["x"])


def test_workload_shapes_and_padding():
    w = inputs.WORKLOADS
    assert w[2].T == 18900 + 512 and w[3].T == 2 * w[2].T and w[5].T == 2 * w[2].T
    assert inputs.token_mask(w[2]) is None
    m = inputs.token_mask(w[5])
    assert m.dtype == torch.uint8 and m.shape == (w[5].T,)
    # the second prompt keeps 64 of its 512 text tokens; the rest is padding
    assert int((m == 0).sum()) == 448 and bool(m[: w[5].T - 448].all())
    assert not bool(m[-448:].any())
