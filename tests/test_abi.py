"""C-ABI checks that need no GPU: the library builds and loads, exports every
entry point that include/routed_moe.h declares, and rejects bad arguments on
the host (these paths return before any CUDA call)."""

import ctypes
import glob
import os
import re

import pytest

from routed_moe_layer_b200 import build, ops
from routed_moe_layer_b200.ops import BlockConfig

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    if build.needs_build():
        build.build_library()
    return ops.lib()


def _declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = _declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n


def test_library_does_not_link_the_driver_directly():
    # the driver API is reached through cudaGetDriverEntryPoint, so the
    # library loads on hosts without libcuda
    import subprocess
    out = subprocess.run(["ldd", ops.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out


def test_status_strings(L):
    for code in range(8):
        assert ops.status_string(code).startswith(ops.STATUS_NAMES[code])
    assert ops.status_string(99) == "unknown moe_status_t"


DEFAULT = BlockConfig(T=19412, H=2048)


@pytest.mark.parametrize("change,expect", [
    ({}, 0),
    ({"E": 130, "n_group": 5}, 2),          # E above 128
    ({"E": 128, "n_group": 3}, 1),          # E not divisible by n_group
    ({"topk_group": 5}, 1),                 # more kept groups than groups
    ({"n_group": 64, "topk_group": 2}, 1),  # 2 experts per group * 2 groups < top_k
    ({"n_group": 128, "topk_group": 64}, 1),  # groups of one expert cannot give a top-2
    ({"n_group": 128, "topk_group": 128}, 2),  # no group step, but n_group > 16
    ({"n_group": 32, "topk_group": 8}, 2),     # more groups than a half warp ranks
    ({"top_k": 17, "topk_group": 4}, 2),
    ({"H": 1000}, 2),
    ({"I": 96}, 2),
    ({"I_shared": 32}, 2),
    ({"T": -1}, 1),
    ({"top_k": 0}, 1),
])
def test_config_checks(L, change, expect):
    import dataclasses
    cfg = dataclasses.replace(DEFAULT, **change)
    c = cfg.c()
    assert L.moe_check_config(ctypes.byref(c)) == expect
    if expect != 0:
        assert L.moe_workspace_bytes(ctypes.byref(c)) == 0


def test_null_and_nan_configs(L):
    assert L.moe_check_config(None) == 1
    c = DEFAULT.c()
    c.routed_scaling_factor = float("nan")
    assert L.moe_check_config(ctypes.byref(c)) == 1
    c = DEFAULT.c()
    c.flags = 1
    assert L.moe_check_config(ctypes.byref(c)) == 1
    c = DEFAULT.c()
    c.norm_topk_prob = 2
    assert L.moe_check_config(ctypes.byref(c)) == 1


def test_workspace_sizes_grow_with_tokens(L):
    a = ops.workspace_bytes(BlockConfig(T=240, H=1024))
    b = ops.workspace_bytes(BlockConfig(T=19412, H=2048))
    assert 0 < a < b
    # gathered rows + intermediate + shared intermediate dominate
    R = 19412 * 8
    assert b >= R * 2048 * 2 + R * 768 * 2 + 19412 * 768 * 2
    assert ops.permute_workspace_bytes(BlockConfig(T=19412, H=2048)) < 2 << 20


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below fails its host checks


def test_forward_rejects_bad_arguments_on_the_host(L):
    c = BlockConfig(T=64, H=256, I=128, I_shared=128).c()
    need = L.moe_workspace_bytes(ctypes.byref(c))
    args = [FAKE] * 7
    # null x
    assert L.moe_forward(None, *args[1:], ctypes.byref(c), FAKE, None, FAKE, need, None) == 1
    # shared weights missing while I_shared > 0
    assert L.moe_forward(*args[:5], None, None, ctypes.byref(c), FAKE, None, FAKE, need,
                         None) == 1
    # out aliases x
    assert L.moe_forward(*args, ctypes.byref(c), FAKE, None, FAKE, need, None) == 1
    out = ctypes.c_void_p(0x20000)
    # workspace too small, missing, misaligned
    assert L.moe_forward(*args, ctypes.byref(c), out, None, FAKE, need - 1, None) == 3
    assert L.moe_forward(*args, ctypes.byref(c), out, None, None, need, None) == 3
    assert L.moe_forward(*args, ctypes.byref(c), out, None, ctypes.c_void_p(0x10010), need,
                         None) == 3
    # invalid configuration is reported before anything else
    bad = BlockConfig(T=64, H=250).c()
    assert L.moe_forward(*args, ctypes.byref(bad), out, None, FAKE, need, None) == 2
    # T = 0 is a no-op
    z = BlockConfig(T=0, H=256, I=128, I_shared=128).c()
    assert L.moe_forward(None, None, None, None, None, None, None, ctypes.byref(z), None, None,
                         None, 0, None) == 0


def test_route_permute_rmsnorm_reject_bad_arguments(L):
    c = BlockConfig(T=64, H=256).c()
    assert L.moe_route(None, FAKE, FAKE, ctypes.byref(c), FAKE, FAKE, None, 0, None) == 1
    assert L.moe_route(FAKE, FAKE, FAKE, None, FAKE, FAKE, None, 0, None) == 1
    need = L.moe_permute_workspace_bytes(ctypes.byref(c))
    assert L.moe_permute(FAKE, None, None, ctypes.byref(c), FAKE, FAKE, FAKE, None, None, FAKE,
                         need - 1, None) == 3
    assert L.moe_permute(FAKE, None, None, ctypes.byref(c), FAKE, FAKE, FAKE, None, FAKE, FAKE,
                         need, None) == 1  # xp without x
    assert L.moe_rmsnorm(FAKE, None, ctypes.c_float(1e-6), 4, 100, FAKE, None) == 1
    assert L.moe_rmsnorm(FAKE, None, ctypes.c_float(-1.0), 4, 128, FAKE, None) == 1
    assert L.moe_selftest_wait_timeout(FAKE, 0, None) == 1


def test_forward_host_rejects_bad_arguments_on_the_host(L):
    c = BlockConfig(T=64, H=256, I=128, I_shared=128).c()
    need = L.moe_forward_host_workspace_bytes(ctypes.byref(c))
    assert need == L.moe_workspace_bytes(ctypes.byref(c)) + 4 * 64 * 256 * 2
    P = ctypes.c_void_p * 2
    xs = P(0x100000, 0x100000)          # one input buffer used twice: allowed
    outs = P(0x200000, 0x200000)        # one output buffer reused: allowed
    w = [FAKE] * 6

    def call(x, o, n, cfg=c, ws=FAKE, nbytes=need, weights=w):
        return L.moe_forward_host(x, o, n, *weights, ctypes.byref(cfg), ws, nbytes, None, None,
                                  None)

    assert call(xs, outs, -1) == 1
    assert call(None, outs, 2) == 1
    assert call(xs, None, 2) == 1
    assert call(P(0x100000, 0), outs, 2) == 1                   # NULL batch pointer
    assert call(xs, P(0x200000, 0x100000 + 64 * 256), 2) == 1  # out overlaps an input's tail
    assert call(xs, outs, 2, nbytes=need - 1) == 3
    assert call(xs, outs, 2, ws=ctypes.c_void_p(0x10010)) == 3
    assert call(xs, outs, 2, weights=[FAKE] * 4 + [None, None]) == 1  # shared weights missing
    assert call(xs, outs, 2, cfg=BlockConfig(T=64, H=250).c()) == 2
    # nothing to do: no batches, or T = 0
    assert call(None, None, 0) == 0
    z = BlockConfig(T=0, H=256, I=128, I_shared=128).c()
    assert call(None, None, 3, cfg=z) == 0


def test_dense_ffn_rejects_bad_arguments_on_the_host(L):
    need = L.moe_dense_ffn_workspace_bytes(64, 256, 128)
    assert need >= 64 * 128 * 2 + 64 * 256 * 2
    assert L.moe_dense_ffn_workspace_bytes(64, 250, 128) == 0
    out = ctypes.c_void_p(0x20000)
    args = lambda **k: [k.get("x", FAKE), FAKE, FAKE, k.get("T", 64), k.get("H", 256),
                        k.get("I", 128), None, k.get("out", out), k.get("ws", FAKE),
                        k.get("nbytes", need), None]
    assert L.moe_dense_ffn(*args(x=None)) == 1
    assert L.moe_dense_ffn(*args(out=FAKE)) == 1          # out aliases x
    assert L.moe_dense_ffn(*args(T=-1)) == 1
    assert L.moe_dense_ffn(*args(H=250)) == 2
    assert L.moe_dense_ffn(*args(I=16384 + 64)) == 2
    assert L.moe_dense_ffn(*args(nbytes=need - 1)) == 3
    assert L.moe_dense_ffn(*args(ws=ctypes.c_void_p(0x10010))) == 3
    assert L.moe_dense_ffn(*args(T=0, x=None, out=None)) == 0


def test_forward_fp8_rejects_bad_arguments_on_the_host(L):
    c = BlockConfig(T=64, H=256, I=128, I_shared=128).c()
    need = L.moe_workspace_bytes(ctypes.byref(c))
    out = ctypes.c_void_p(0x20000)

    def call(cfg=c, x=FAKE, q=(FAKE,) * 8, o=out, ws=FAKE, nbytes=need):
        return L.moe_forward_fp8(x, FAKE, FAKE, *q, ctypes.byref(cfg), o, None, ws, nbytes,
                                 None)

    assert call(x=None) == 1
    assert call(q=(FAKE, None) + (FAKE,) * 6) == 1            # w13 scales missing
    assert call(q=(FAKE,) * 4 + (None,) * 4) == 1             # shared weights missing
    assert call(q=(FAKE,) * 6 + (None, FAKE)) == 1            # shared w2 codes missing
    assert call(o=FAKE) == 1                                  # out aliases x
    assert call(nbytes=need - 1) == 3
    assert call(ws=ctypes.c_void_p(0x10010)) == 3
    # H, I and I_shared must be multiples of the 128-wide scale blocks
    for bad in (BlockConfig(T=64, H=320, I=128, I_shared=128),
                BlockConfig(T=64, H=256, I=192, I_shared=192),
                BlockConfig(T=64, H=256, I=128, I_shared=64)):
        assert call(cfg=bad.c()) == 2
    assert call(cfg=BlockConfig(T=64, H=250).c()) == 2
    z = BlockConfig(T=0, H=256, I=128, I_shared=128).c()
    assert call(cfg=z, x=None, q=(None,) * 8, o=None, ws=None, nbytes=0) == 0


def test_expert_parallel_entries_reject_bad_arguments_on_the_host(L):
    # moe_rows_expert_ids
    assert L.moe_rows_expert_ids(FAKE, 0, 10, FAKE, None) == 1
    assert L.moe_rows_expert_ids(FAKE, 129, 10, FAKE, None) == 1
    assert L.moe_rows_expert_ids(None, 8, 10, FAKE, None) == 1
    assert L.moe_rows_expert_ids(None, 8, 0, None, None) == 0
    # moe_expert_rows
    need = L.moe_expert_rows_workspace_bytes(100, 256, 8, 128)
    assert need >= 100 * 128 * 2
    assert L.moe_expert_rows_workspace_bytes(100, 250, 8, 128) == 0
    y = ctypes.c_void_p(0x20000)
    args = lambda **k: [k.get("xr", FAKE), FAKE, k.get("R", 100), k.get("E", 8), k.get("H", 256),
                        k.get("I", 128), FAKE, FAKE, None, k.get("dest", FAKE), k.get("y", y),
                        k.get("ws", FAKE), k.get("nbytes", need), None]
    assert L.moe_expert_rows(*args(xr=None)) == 1
    assert L.moe_expert_rows(*args(dest=None)) == 1
    assert L.moe_expert_rows(*args(y=FAKE)) == 1            # y aliases xr
    assert L.moe_expert_rows(*args(E=129)) == 2
    assert L.moe_expert_rows(*args(H=250)) == 2
    assert L.moe_expert_rows(*args(nbytes=need - 1)) == 3
    assert L.moe_expert_rows(*args(ws=ctypes.c_void_p(0x10010))) == 3
    assert L.moe_expert_rows(*args(R=0, xr=None, y=None)) == 0
    # moe_combine_rows
    out = ctypes.c_void_p(0x30000)
    assert L.moe_combine_rows(None, 80, FAKE, 10, 256, 8, None, None, out, None) == 1
    assert L.moe_combine_rows(FAKE, 80, FAKE, 10, 256, 8, None, None, FAKE, None) == 1  # out is y
    assert L.moe_combine_rows(FAKE, -1, FAKE, 10, 256, 8, None, None, out, None) == 1  # R < 0
    assert L.moe_combine_rows(FAKE, 80, FAKE, 10, 250, 8, None, None, out, None) == 2
    assert L.moe_combine_rows(FAKE, 80, FAKE, 10, 256, 17, None, None, out, None) == 2
    assert L.moe_combine_rows(None, 0, None, 0, 256, 8, None, None, None, None) == 0


def test_public_header_is_plain_c():
    """include/*.h is a C ABI: it must compile as C99 (and as C++) with no torch types."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        for lang, std in (("c", "c99"), ("c++", "c++17")):
            r = subprocess.run(["gcc", "-fsyntax-only", f"-std={std}", "-Wall", "-Werror", "-x",
                                lang, h], capture_output=True, text=True)
            assert r.returncode == 0, (h, lang, r.stderr)
        src = open(h).read()
        assert "#include <torch" not in src and "torch::" not in src and "at::" not in src
