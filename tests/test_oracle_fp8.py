"""Pins of the oracle's FP8 expert-weight functions against facts that do not
come from the oracle: the E4M3 and UE8M0 definitions (values the formats fix,
and PyTorch's own float8_e4m3fn conversion), the block layout of the scales on
a ragged, non-square matrix, and the rounding bound of the generator's cast."""

import numpy as np
import torch

from oracle import (MoeConfig, bf16_round, fp8_block_dequant, fp8_e4m3_decode,
                    moe_forward, moe_forward_fp8, ue8m0_decode)
from routed_moe_layer_b200 import inputs


def test_e4m3_decode_matches_torch_float8_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = fp8_e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    fin = ~np.isnan(lib)
    assert np.array_equal(ours[fin], lib[fin])
    assert np.array_equal(np.signbit(ours[fin]), np.signbit(lib[fin]))


def test_e4m3_decode_values_fixed_by_the_format():
    # sign | exponent (bias 7) | 3-bit mantissa; exponent 0 = subnormal; S.1111.111 = NaN
    table = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
             0x38: 1.0, 0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0,
             0xB8: -1.0, 0xFE: -448.0, 0x81: -(2.0 ** -9)}
    got = fp8_e4m3_decode(np.array(list(table), dtype=np.uint8))
    assert np.array_equal(got, np.array(list(table.values())))
    assert np.signbit(fp8_e4m3_decode(np.array([0x80], np.uint8)))[0]
    assert np.isnan(fp8_e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()
    # positive codes increase with the code and every value is a bf16 value
    pos = fp8_e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(bf16_round(pos).astype(np.float64), pos)


def test_ue8m0_scales():
    got = ue8m0_decode(np.array([127, 128, 126, 0, 254], np.uint8))
    assert np.array_equal(got, [1.0, 2.0, 0.5, 2.0 ** -127, 2.0 ** 127])
    assert np.isnan(ue8m0_decode(np.array([255], np.uint8)))[0]


def test_block_scales_land_on_their_blocks_ragged_non_square():
    # 2 matrices of 300 x 200: blocks rows [0,128) [128,256) [256,300), cols [0,128) [128,200)
    E, N, K = 2, 300, 200
    codes = np.full((E, N, K), 0x38, np.uint8)  # every code 1.0
    sexp = np.zeros((E, 3, 2), np.uint8)
    for e in range(E):
        for i in range(3):
            for j in range(2):
                sexp[e, i, j] = 100 + 10 * e + 3 * i + j
    deq = fp8_block_dequant(codes, sexp)
    assert deq.shape == (E, N, K)
    row_blocks = [(0, 128), (128, 256), (256, 300)]
    col_blocks = [(0, 128), (128, 200)]
    for e in range(E):
        for i, (r0, r1) in enumerate(row_blocks):
            for j, (c0, c1) in enumerate(col_blocks):
                want = 2.0 ** (100 + 10 * e + 3 * i + j - 127)
                assert np.all(deq[e, r0:r1, c0:c1] == want), (e, i, j)


def test_one_scale_step_doubles_exactly_its_block():
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 0x7F, size=(260, 140)).astype(np.uint8)  # finite codes
    sexp = rng.integers(110, 130, size=(3, 2)).astype(np.uint8)
    base = fp8_block_dequant(codes, sexp)
    sexp2 = sexp.copy()
    sexp2[2, 1] += 1
    bumped = fp8_block_dequant(codes, sexp2)
    changed = np.zeros_like(base, bool)
    changed[256:, 128:] = True
    assert np.array_equal(bumped[changed], 2 * base[changed])
    assert np.array_equal(bumped[~changed], base[~changed])


def test_dequantised_generator_weights_within_the_e4m3_rounding_bound():
    # the generator casts (draw / block scale) to E4M3 with PyTorch; decoding and
    # rescaling must give the draw back within half an E4M3 step at its binade
    H, I, E, seed = 256, 192, 3, 11
    q = inputs.make_fp8_weights(H, seed, E=E, I=I, I_shared=I)
    ref = inputs.make_weights(H, seed, E=E, I=I, I_shared=I)
    for name in ("w13", "w2", "ws13", "ws2"):
        deq = fp8_block_dequant(q[name + "_q"].numpy(), q[name + "_s"].numpy())
        # the generator's fp32 draw, before its bf16 rounding in make_weights
        shape = tuple(ref[name].shape)
        idx = {"w13": 3, "w2": 4, "ws13": 5, "ws2": 6}[name]
        g = torch.Generator().manual_seed(seed * 1000 + idx)
        draw = (torch.randn(shape, generator=g) * 0.02).numpy().astype(np.float64)
        sc = fp8_block_dequant(np.full(shape, 0x38, np.uint8), q[name + "_s"].numpy())
        bound = np.maximum(np.abs(draw) * 2.0 ** -4, sc * 2.0 ** -10)
        assert np.all(np.abs(deq - draw) <= bound * (1 + 1e-12)), name
        # and every dequantised weight is a bf16 value
        assert np.array_equal(bf16_round(deq).astype(np.float64), deq), name


def test_fp8_forward_is_the_bf16_forward_on_block_constant_weights():
    # weights with a single code per block: the FP8 block must equal the bf16
    # block on the matrices written out by hand from the scales
    T, H, I, E = 6, 256, 128, 4
    cfg = MoeConfig(E=E, I=I, I_shared=I, top_k=2, n_group=2, topk_group=1)
    rng = np.random.default_rng(3)
    x = bf16_round(rng.standard_normal((T, H)))
    Wr = rng.standard_normal((E, H)).astype(np.float32) * 0.05
    bias = np.zeros(E, np.float32)

    def const_blocks(shape, code, exps):
        q = np.full(shape, code, np.uint8)
        dense = np.empty(shape, np.float64)
        nb, kb = exps.shape[-2], exps.shape[-1]
        for i in range(nb):
            for j in range(kb):
                dense[..., i * 128:(i + 1) * 128, j * 128:(j + 1) * 128] = \
                    np.exp2(exps[..., i, j].astype(np.float64) - 127)[..., None, None] * \
                    (1.0 if code == 0x38 else -1.5)
        return q, dense

    e13 = rng.integers(118, 122, size=(E, 2, 2)).astype(np.uint8)
    e2 = rng.integers(118, 122, size=(E, 2, 1)).astype(np.uint8)
    es13 = rng.integers(118, 122, size=(2, 2)).astype(np.uint8)
    es2 = rng.integers(118, 122, size=(2, 1)).astype(np.uint8)
    w13_q, w13 = const_blocks((E, 2 * I, H), 0x38, e13)
    w2_q, w2 = const_blocks((E, H, I), 0xBC, e2)  # 0xBC = -1.5
    ws13_q, ws13 = const_blocks((2 * I, H), 0x38, es13)
    ws2_q, ws2 = const_blocks((H, I), 0xBC, es2)
    got = moe_forward_fp8(x, Wr, bias, w13_q, e13, w2_q, e2, ws13_q, es13, ws2_q, es2, cfg)[0]
    want = moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg)[0]
    assert np.array_equal(got, want)
