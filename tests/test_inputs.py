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


def test_fp8_weights_are_seeded_and_shaped():
    a = inputs.make_fp8_weights(256, 2, E=2, I=192, I_shared=192)
    b = inputs.make_fp8_weights(256, 2, E=2, I=192, I_shared=192)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert a["w13_q"].dtype == torch.uint8 and a["w13_q"].shape == (2, 384, 256)
    assert a["w13_s"].shape == (2, 3, 2) and a["w2_s"].shape == (2, 2, 2)
    assert int(a["w2_s"].min()) >= 118 and int(a["w2_s"].max()) <= 120
    # no NaN codes (S.1111.111)
    assert not bool(((a["w13_q"] & 0x7F) == 0x7F).any())
    assert inputs.make_fp8_weights(256, 2, E=2, I=192, I_shared=0)["ws13_q"] is None
