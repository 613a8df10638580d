"""Thin ctypes binding of libroutedmoe.so (declared in include/routed_moe.h).

Argument marshalling only: every step of the block runs in the library's
CUDA kernels.  PyTorch provides device memory (outputs and workspace are
allocated with torch) and the current CUDA stream.  There is no fallback:
if the library is missing or a call fails, a RuntimeError is raised.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Sequence

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libroutedmoe.so")

MOE_OK = 0
STATUS_NAMES = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
    3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_TIMEOUT",
    6: "MOE_ERR_DEVICE_INDEX", 7: "MOE_ERR_NO_DEVICE",
}
STAGES = ("router", "permute", "expert_up", "expert_down", "shared_expert", "combine")
NUM_STAGES = len(STAGES)


class MoeCfg(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int32), ("H", ctypes.c_int32), ("E", ctypes.c_int32),
        ("I", ctypes.c_int32), ("I_shared", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32),
        ("routed_scaling_factor", ctypes.c_float), ("norm_topk_prob", ctypes.c_int32),
        ("flags", ctypes.c_int32),
    ]


class MoeForwardOpts(ctypes.Structure):
    _fields_ = [
        ("residual", ctypes.c_void_p), ("topk_ids", ctypes.c_void_p),
        ("topk_w", ctypes.c_void_p), ("stage_events", ctypes.POINTER(ctypes.c_void_p)),
        ("wait_timeout_ns", ctypes.c_int64), ("token_mask", ctypes.c_void_p),
    ]


@dataclasses.dataclass
class BlockConfig:
    """Hyper-parameters of the block (LingBot-Video MoE defaults)."""

    T: int
    H: int
    E: int = 128
    I: int = 768
    I_shared: int = 768
    top_k: int = 8
    n_group: int = 4
    topk_group: int = 2
    routed_scaling_factor: float = 2.5
    norm_topk_prob: bool = True

    def c(self) -> MoeCfg:
        return MoeCfg(self.T, self.H, self.E, self.I, self.I_shared, self.top_k, self.n_group,
                      self.topk_group, float(self.routed_scaling_factor),
                      1 if self.norm_topk_prob else 0, 0)

    def with_tokens(self, T: int) -> "BlockConfig":
        return dataclasses.replace(self, T=T)


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libroutedmoe.so once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m routed_moe_layer_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    cfgp = ctypes.POINTER(MoeCfg)
    sig = {
        "moe_status_string": (ctypes.c_char_p, [i32]),
        "moe_check_config": (i32, [cfgp]),
        "moe_route_workspace_bytes": (sz, [cfgp]),
        "moe_permute_workspace_bytes": (sz, [cfgp]),
        "moe_workspace_bytes": (sz, [cfgp]),
        "moe_route": (i32, [vp, vp, vp, cfgp, vp, vp, vp, sz, vp]),
        "moe_route_masked": (i32, [vp, vp, vp, vp, cfgp, vp, vp, vp, sz, vp]),
        "moe_permute": (i32, [vp, vp, vp, cfgp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "moe_forward": (i32, [vp, vp, vp, vp, vp, vp, vp, cfgp, vp,
                              ctypes.POINTER(MoeForwardOpts), vp, sz, vp]),
        "moe_forward_fp8": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, cfgp, vp,
                                  ctypes.POINTER(MoeForwardOpts), vp, sz, vp]),
        "moe_forward_host_workspace_bytes": (sz, [cfgp]),
        "moe_forward_host": (i32, [ctypes.POINTER(vp), ctypes.POINTER(vp), i32, vp, vp, vp, vp,
                                   vp, vp, cfgp, vp, sz, vp, vp, vp]),
        "moe_dense_ffn_workspace_bytes": (sz, [i32, i32, i32]),
        "moe_dense_ffn": (i32, [vp, vp, vp, i32, i32, i32, vp, vp, vp, sz, vp]),
        "moe_rows_expert_ids": (i32, [vp, i32, i32, vp, vp]),
        "moe_expert_rows_workspace_bytes": (sz, [i32, i32, i32, i32]),
        "moe_expert_rows": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]),
        "moe_combine_rows": (i32, [vp, i32, vp, i32, i32, i32, vp, vp, vp, vp]),
        "moe_rmsnorm": (i32, [vp, vp, ctypes.c_float, i32, i32, vp, vp]),
        "moe_read_device_status": (i32, [vp, ctypes.POINTER(i32), vp]),
        "moe_selftest_wait_timeout": (i32, [vp, i64, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().moe_status_string(int(code)).decode()


def _check(code: int, what: str):
    if code != MOE_OK:
        raise RuntimeError(f"{what}: {status_string(code)}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, shape: Sequence[int]):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def check_config(cfg: BlockConfig) -> int:
    c = cfg.c()
    return int(lib().moe_check_config(ctypes.byref(c)))


def workspace_bytes(cfg: BlockConfig) -> int:
    c = cfg.c()
    return int(lib().moe_workspace_bytes(ctypes.byref(c)))


def permute_workspace_bytes(cfg: BlockConfig) -> int:
    c = cfg.c()
    return int(lib().moe_permute_workspace_bytes(ctypes.byref(c)))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns blocks aligned to at least 512 bytes
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def route(x: torch.Tensor, Wr: torch.Tensor, bias: torch.Tensor, cfg: BlockConfig,
          token_mask: Optional[torch.Tensor] = None):
    """Router: returns (topk_ids int32 [T,k], topk_w fp32 [T,k]); with a uint8
    token_mask [T], padding tokens (0) get ids -1 and weights 0."""
    T, H = cfg.T, cfg.H
    _need(x, "x", torch.bfloat16, (T, H))
    _need(Wr, "Wr", torch.float32, (cfg.E, H))
    _need(bias, "bias", torch.float32, (cfg.E,))
    if token_mask is not None:
        _need(token_mask, "token_mask", torch.uint8, (T,))
    ids = torch.empty((T, cfg.top_k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, cfg.top_k), dtype=torch.float32, device=x.device)
    c = cfg.c()
    ws = alloc_workspace(lib().moe_route_workspace_bytes(ctypes.byref(c)), x.device)
    if token_mask is None:
        _check(lib().moe_route(_ptr(x), _ptr(Wr), _ptr(bias), ctypes.byref(c), _ptr(ids),
                               _ptr(w), _ptr(ws), ws.numel(), _stream_ptr()), "moe_route")
    else:
        _check(lib().moe_route_masked(_ptr(x), _ptr(Wr), _ptr(bias), _ptr(token_mask),
                                      ctypes.byref(c), _ptr(ids), _ptr(w), _ptr(ws), ws.numel(),
                                      _stream_ptr()), "moe_route_masked")
    return ids, w


def permute(topk_ids: torch.Tensor, cfg: BlockConfig, topk_w: Optional[torch.Tensor] = None,
            x: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """Token->expert permutation; returns dict(expert_offsets, row_of, tok_of, w_of, xp, workspace)."""
    T, k, E = cfg.T, cfg.top_k, cfg.E
    _need(topk_ids, "topk_ids", torch.int32, (T, k))
    dev = topk_ids.device
    if topk_w is not None:
        _need(topk_w, "topk_w", torch.float32, (T, k))
    if x is not None:
        _need(x, "x", torch.bfloat16, (T, cfg.H))
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty(T * k, dtype=torch.int32, device=dev)
    tok_of = torch.empty(T * k, dtype=torch.int32, device=dev)
    w_of = torch.empty(T * k, dtype=torch.float32, device=dev) if topk_w is not None else None
    xp = torch.empty((T * k, cfg.H), dtype=torch.bfloat16, device=dev) if x is not None else None
    need = permute_workspace_bytes(cfg)
    if workspace is None:
        workspace = alloc_workspace(need, dev)
    c = cfg.c()
    _check(lib().moe_permute(_ptr(topk_ids), _ptr(topk_w), _ptr(x), ctypes.byref(c),
                             _ptr(offsets), _ptr(row_of), _ptr(tok_of), _ptr(w_of), _ptr(xp),
                             _ptr(workspace), workspace.numel(), _stream_ptr()), "moe_permute")
    return dict(expert_offsets=offsets, row_of=row_of, tok_of=tok_of, w_of=w_of, xp=xp,
                workspace=workspace)


class StageTimer:
    """CUDA events recorded by moe_forward around stages, on its stream.

    ``stages`` selects the stages to time (default: all).  Every recorded
    event serialises the kernels around it, so time only what is needed."""

    def __init__(self, stages=STAGES):
        idx = sorted({i for name in stages for i in (STAGES.index(name), STAGES.index(name) + 1)})
        self.events = [torch.cuda.Event(enable_timing=True) if i in idx else None
                       for i in range(NUM_STAGES + 1)]
        for e in self.events:  # torch creates the CUDA event on its first record
            if e is not None:
                e.record()
        handles = [e.cuda_event if e is not None else None for e in self.events]
        if not all(h for h, e in zip(handles, self.events) if e is not None):
            raise RuntimeError("could not create CUDA events for stage timing")
        self.stages = tuple(stages)
        self._arr = (ctypes.c_void_p * (NUM_STAGES + 1))(*handles)

    def as_ptr(self):
        return ctypes.cast(self._arr, ctypes.POINTER(ctypes.c_void_p))

    def stage_ms(self):
        return {name: self.events[STAGES.index(name)].elapsed_time(
                    self.events[STAGES.index(name) + 1]) for name in self.stages}


def forward(x: torch.Tensor, Wr: torch.Tensor, bias: torch.Tensor, w13: torch.Tensor,
            w2: torch.Tensor, ws13: Optional[torch.Tensor], ws2: Optional[torch.Tensor],
            cfg: BlockConfig, residual: Optional[torch.Tensor] = None,
            out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
            topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
            timer: Optional[StageTimer] = None, wait_timeout_ns: int = 0,
            token_mask: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Block forward; returns out bf16 [T,H] (written in place when ``out`` is given).
    token_mask: uint8 [T] padding mask (0 = padding: shared expert only)."""
    T, H, E, I, Is, k = cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared, cfg.top_k
    _need(x, "x", torch.bfloat16, (T, H))
    _need(Wr, "Wr", torch.float32, (E, H))
    _need(bias, "bias", torch.float32, (E,))
    _need(w13, "w13", torch.bfloat16, (E, 2 * I, H))
    _need(w2, "w2", torch.bfloat16, (E, H, I))
    if Is > 0:
        _need(ws13, "ws13", torch.bfloat16, (2 * Is, H))
        _need(ws2, "ws2", torch.bfloat16, (H, Is))
    if residual is not None:
        _need(residual, "residual", torch.bfloat16, (T, H))
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    else:
        _need(out, "out", torch.bfloat16, (T, H))
    if topk_ids is not None:
        _need(topk_ids, "topk_ids", torch.int32, (T, k))
    if topk_w is not None:
        _need(topk_w, "topk_w", torch.float32, (T, k))
    if token_mask is not None:
        _need(token_mask, "token_mask", torch.uint8, (T,))
    if workspace is None:
        workspace = alloc_workspace(workspace_bytes(cfg), x.device)
    opts = MoeForwardOpts(
        residual=None if residual is None else residual.data_ptr(),
        topk_ids=None if topk_ids is None else topk_ids.data_ptr(),
        topk_w=None if topk_w is None else topk_w.data_ptr(),
        stage_events=timer.as_ptr() if timer is not None else None,
        wait_timeout_ns=int(wait_timeout_ns),
        token_mask=None if token_mask is None else token_mask.data_ptr())
    c = cfg.c()
    _check(lib().moe_forward(_ptr(x), _ptr(Wr), _ptr(bias), _ptr(w13), _ptr(w2), _ptr(ws13),
                             _ptr(ws2), ctypes.byref(c), _ptr(out), ctypes.byref(opts),
                             _ptr(workspace), workspace.numel(), _stream_ptr()), "moe_forward")
    return out


def forward_fp8(x: torch.Tensor, Wr: torch.Tensor, bias: torch.Tensor, fp8: dict,
                cfg: BlockConfig, residual: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                topk_ids: Optional[torch.Tensor] = None, topk_w: Optional[torch.Tensor] = None,
                timer: Optional[StageTimer] = None, wait_timeout_ns: int = 0,
                token_mask: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Block forward with FP8 expert weights (E4M3 codes, one power-of-two
    scale per 128 x 128 block); returns out bf16 [T,H].  ``fp8`` holds uint8
    tensors w13_q [E,2I,H], w13_s [E,2I/128,H/128], w2_q [E,H,I],
    w2_s [E,H/128,I/128] and, with a shared expert, ws13_q, ws13_s, ws2_q,
    ws2_s (the layouts of moe_forward_fp8)."""
    T, H, E, I, Is = cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared
    u8 = torch.uint8
    _need(x, "x", torch.bfloat16, (T, H))
    _need(Wr, "Wr", torch.float32, (E, H))
    _need(bias, "bias", torch.float32, (E,))
    blk = lambda n: -(-n // 128)
    _need(fp8["w13_q"], "w13_q", u8, (E, 2 * I, H))
    _need(fp8["w13_s"], "w13_s", u8, (E, blk(2 * I), blk(H)))
    _need(fp8["w2_q"], "w2_q", u8, (E, H, I))
    _need(fp8["w2_s"], "w2_s", u8, (E, blk(H), blk(I)))
    shared = [None] * 4
    if Is > 0:
        _need(fp8["ws13_q"], "ws13_q", u8, (2 * Is, H))
        _need(fp8["ws13_s"], "ws13_s", u8, (blk(2 * Is), blk(H)))
        _need(fp8["ws2_q"], "ws2_q", u8, (H, Is))
        _need(fp8["ws2_s"], "ws2_s", u8, (blk(H), blk(Is)))
        shared = [fp8["ws13_q"], fp8["ws13_s"], fp8["ws2_q"], fp8["ws2_s"]]
    if residual is not None:
        _need(residual, "residual", torch.bfloat16, (T, H))
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    else:
        _need(out, "out", torch.bfloat16, (T, H))
    if topk_ids is not None:
        _need(topk_ids, "topk_ids", torch.int32, (T, cfg.top_k))
    if topk_w is not None:
        _need(topk_w, "topk_w", torch.float32, (T, cfg.top_k))
    if token_mask is not None:
        _need(token_mask, "token_mask", torch.uint8, (T,))
    if workspace is None:
        workspace = alloc_workspace(workspace_bytes(cfg), x.device)
    opts = MoeForwardOpts(
        residual=None if residual is None else residual.data_ptr(),
        topk_ids=None if topk_ids is None else topk_ids.data_ptr(),
        topk_w=None if topk_w is None else topk_w.data_ptr(),
        stage_events=timer.as_ptr() if timer is not None else None,
        wait_timeout_ns=int(wait_timeout_ns),
        token_mask=None if token_mask is None else token_mask.data_ptr())
    c = cfg.c()
    _check(lib().moe_forward_fp8(
        _ptr(x), _ptr(Wr), _ptr(bias), _ptr(fp8["w13_q"]), _ptr(fp8["w13_s"]),
        _ptr(fp8["w2_q"]), _ptr(fp8["w2_s"]), *[_ptr(t) for t in shared], ctypes.byref(c),
        _ptr(out), ctypes.byref(opts), _ptr(workspace), workspace.numel(), _stream_ptr()),
        "moe_forward_fp8")
    return out


def forward_host_workspace_bytes(cfg: BlockConfig) -> int:
    c = cfg.c()
    return int(lib().moe_forward_host_workspace_bytes(ctypes.byref(c)))


def _need_host(t: torch.Tensor, name: str, shape: Sequence[int]):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be torch.bfloat16, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def forward_host(x_host: Sequence[torch.Tensor], out_host: Sequence[torch.Tensor],
                 Wr: torch.Tensor, bias: torch.Tensor, w13: torch.Tensor, w2: torch.Tensor,
                 ws13: Optional[torch.Tensor], ws2: Optional[torch.Tensor], cfg: BlockConfig,
                 workspace: Optional[torch.Tensor] = None,
                 copy_streams: Optional[Sequence[torch.cuda.Stream]] = None):
    """Block forward over host-resident batches (moe_forward_host).

    x_host[b] / out_host[b]: CPU bf16 [T,H] tensors (pin them for overlap).
    Kernels run on the current stream; copy_streams = (h2d, d2h) run the copies
    (None: the current stream, no overlap).  Returns once queued: synchronise
    the current stream before reading out_host."""
    n = len(x_host)
    if len(out_host) != n:
        raise ValueError("x_host and out_host must have the same length")
    T, H, E, I, Is = cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared
    for b in range(n):
        _need_host(x_host[b], f"x_host[{b}]", (T, H))
        _need_host(out_host[b], f"out_host[{b}]", (T, H))
    _need(Wr, "Wr", torch.float32, (E, H))
    _need(bias, "bias", torch.float32, (E,))
    _need(w13, "w13", torch.bfloat16, (E, 2 * I, H))
    _need(w2, "w2", torch.bfloat16, (E, H, I))
    if Is > 0:
        _need(ws13, "ws13", torch.bfloat16, (2 * Is, H))
        _need(ws2, "ws2", torch.bfloat16, (H, Is))
    if workspace is None:
        workspace = alloc_workspace(forward_host_workspace_bytes(cfg), Wr.device)
    xs = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in x_host])
    os_ = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in out_host])
    h2d = d2h = None
    if copy_streams is not None:
        h2d = ctypes.c_void_p(copy_streams[0].cuda_stream)
        d2h = ctypes.c_void_p(copy_streams[1].cuda_stream)
    c = cfg.c()
    _check(lib().moe_forward_host(xs, os_, n, _ptr(Wr), _ptr(bias), _ptr(w13), _ptr(w2),
                                  _ptr(ws13), _ptr(ws2), ctypes.byref(c), _ptr(workspace),
                                  workspace.numel(), _stream_ptr(), h2d, d2h),
           "moe_forward_host")
    return workspace


def dense_ffn(x: torch.Tensor, w13: torch.Tensor, w2: torch.Tensor,
              residual: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Dense SwiGLU feed-forward layer (moe_dense_ffn): out = [residual +] SwiGLU(x)."""
    T, H = x.shape
    I = w13.shape[0] // 2
    _need(x, "x", torch.bfloat16, (T, H))
    _need(w13, "w13", torch.bfloat16, (2 * I, H))
    _need(w2, "w2", torch.bfloat16, (H, I))
    if residual is not None:
        _need(residual, "residual", torch.bfloat16, (T, H))
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    else:
        _need(out, "out", torch.bfloat16, (T, H))
    if workspace is None:
        workspace = alloc_workspace(lib().moe_dense_ffn_workspace_bytes(T, H, I), x.device)
    _check(lib().moe_dense_ffn(_ptr(x), _ptr(w13), _ptr(w2), T, H, I, _ptr(residual), _ptr(out),
                               _ptr(workspace), workspace.numel(), _stream_ptr()), "moe_dense_ffn")
    return out


def rows_expert_ids(offsets: torch.Tensor, E: int) -> torch.Tensor:
    """Expert id of every row of an expert-sorted row list (moe_rows_expert_ids):
    int32 [offsets[E] - offsets[0]] from device offsets int32 [E+1]."""
    _need(offsets, "offsets", torch.int32, (E + 1,))
    R = int(offsets[E].item() - offsets[0].item())
    ids = torch.empty(R, dtype=torch.int32, device=offsets.device)
    _check(lib().moe_rows_expert_ids(_ptr(offsets), E, R, _ptr(ids), _stream_ptr()),
           "moe_rows_expert_ids")
    return ids


def expert_rows(xr: torch.Tensor, offsets: torch.Tensor, w13: torch.Tensor, w2: torch.Tensor,
                row_dest: torch.Tensor, row_w: Optional[torch.Tensor] = None,
                y: Optional[torch.Tensor] = None, y_rows: Optional[int] = None,
                workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Routed experts on rows grouped by expert (moe_expert_rows):
    y[row_dest[r]] = row_w[r] * SwiGLU_e(xr[r]) for r in [offsets[e], offsets[e+1]).
    ``offsets`` may be a view into a longer offsets tensor (the local experts'
    slice).  Returns y bf16 [y_rows (default R), H]."""
    R, H = xr.shape
    E = w13.shape[0]
    I = w13.shape[1] // 2
    _need(xr, "xr", torch.bfloat16, (R, H))
    _need(offsets, "offsets", torch.int32, (E + 1,))
    _need(w13, "w13", torch.bfloat16, (E, 2 * I, H))
    _need(w2, "w2", torch.bfloat16, (E, H, I))
    _need(row_dest, "row_dest", torch.int32, (R,))
    if row_w is not None:
        _need(row_w, "row_w", torch.float32, (R,))
    if y is None:
        y = torch.empty((R if y_rows is None else y_rows, H), dtype=torch.bfloat16,
                        device=xr.device)
    elif y.dtype != torch.bfloat16 or y.dim() != 2 or y.shape[1] != H or not y.is_contiguous():
        raise ValueError("y must be a contiguous bf16 [rows, H] tensor")
    if workspace is None:
        workspace = alloc_workspace(lib().moe_expert_rows_workspace_bytes(R, H, E, I), xr.device)
    _check(lib().moe_expert_rows(_ptr(xr), _ptr(offsets), R, E, H, I, _ptr(w13), _ptr(w2),
                                 _ptr(row_w), _ptr(row_dest), _ptr(y), _ptr(workspace),
                                 workspace.numel(), _stream_ptr()), "moe_expert_rows")
    return y


def combine_rows(y: torch.Tensor, row_of: torch.Tensor, top_k: int,
                 shared: Optional[torch.Tensor] = None, residual: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The restore through row_of (moe_combine_rows): out[t] = bf16(sum_j y[row_of[t, j]]
    + shared[t] + residual[t]) in fp32, slot order, one rounding; a row_of entry
    outside [0, y.shape[0]) adds 0."""
    H = y.shape[1]
    T = row_of.numel() // top_k
    if y.dtype != torch.bfloat16 or y.dim() != 2 or not y.is_cuda or not y.is_contiguous():
        raise ValueError("y must be a contiguous CUDA bf16 [rows, H] tensor")
    _need(row_of, "row_of", torch.int32, (T * top_k,))
    for name, t in (("shared", shared), ("residual", residual)):
        if t is not None:
            _need(t, name, torch.bfloat16, (T, H))
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=y.device)
    else:
        _need(out, "out", torch.bfloat16, (T, H))
    _check(lib().moe_combine_rows(_ptr(y), y.shape[0], _ptr(row_of), T, H, top_k, _ptr(shared),
                                  _ptr(residual), _ptr(out), _stream_ptr()), "moe_combine_rows")
    return out


def rmsnorm(x: torch.Tensor, gamma: Optional[torch.Tensor] = None, eps: float = 1e-6,
            out: Optional[torch.Tensor] = None) -> torch.Tensor:
    T, H = x.shape
    _need(x, "x", torch.bfloat16, (T, H))
    if gamma is not None:
        _need(gamma, "gamma", torch.float32, (H,))
    if out is None:
        out = torch.empty_like(x)
    _check(lib().moe_rmsnorm(_ptr(x), _ptr(gamma), float(eps), T, H, _ptr(out), _stream_ptr()),
           "moe_rmsnorm")
    return out


def read_device_status(workspace: torch.Tensor):
    """Synchronises the current stream; returns (code, site) and clears the word."""
    site = ctypes.c_int32(0)
    code = lib().moe_read_device_status(_ptr(workspace), ctypes.byref(site), _stream_ptr())
    return int(code), int(site.value)


def selftest_wait_timeout(timeout_ns: int, workspace: Optional[torch.Tensor] = None):
    """Runs the bounded-wait self test; returns (code, site) read back from the device."""
    if workspace is None:
        workspace = alloc_workspace(256, torch.device("cuda"))
    _check(lib().moe_selftest_wait_timeout(_ptr(workspace), int(timeout_ns), _stream_ptr()),
           "moe_selftest_wait_timeout")
    return read_device_status(workspace)
