"""Benchmark of the routed MoE block forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step = one full block forward (router, permutation, grouped SwiGLU
experts, shared expert and combine) over one batch of seeded synthetic
tokens, inputs resident in HBM.  The default workload is the 19,412-token
layer (21 latent frames x 30x30 patches + 512 text tokens, H=2048, 128
experts, top-8).  Under torchrun every rank runs its own batch of the same
size on its own GPU (token data parallelism: no collective on the data path;
weak scaling); the timed region is bracketed by a barrier and a device
synchronise on both sides and the slowest rank's time is reported.

``--impl reference`` times the CPU oracle (the only reference
implementation: the source pages ship no code) on a bounded token sample of
the same workload, on rank 0 only.

Prints one JSON line (rank 0).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from routed_moe_layer_b200 import inputs, ops  # noqa: E402
from routed_moe_layer_b200.dist import max_over_ranks, rank_token_seed  # noqa: E402
from routed_moe_layer_b200.ops import BlockConfig  # noqa: E402

METRIC = "MoE-layer tokens/s and TFLOP/s at T~19.4k bf16; % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
def kernels_per_step(cfg: BlockConfig, fp8: bool = False) -> int:
    """Launches of one block forward: router 3 (Wr split, GEMM, selection), permutation
    and gather (one kernel up to 1024 tokens, else three and a gather), expert up and
    down (one launch for small batches; the shared expert folded into both), combine."""
    return 3 + (1 if cfg.T <= 1024 else 4) + (1 if fused_small_batch(cfg, fp8) else 2) + 1


def flops_per_token(cfg: BlockConfig) -> float:
    """Algorithmic FLOPs of one token: router GEMM, top_k SwiGLU experts, shared expert."""
    return (2.0 * cfg.E * cfg.H + cfg.top_k * 6.0 * cfg.H * cfg.I + 6.0 * cfg.H * cfg.I_shared)


DATASHEET_HBM_GBS = 8000.0  # B200 HBM3e, nominal


def weight_bytes_per_element(fp8: bool) -> float:
    """bf16: 2 bytes; FP8: one E4M3 byte plus one scale byte per 128 x 128 block."""
    return 1.0 + 1.0 / (128 * 128) if fp8 else 2.0


def algorithmic_bytes(cfg: BlockConfig, experts_used: int, fp8: bool = False) -> float:
    """Weights of the experts that receive a token + shared + router + x in + out
    (no implementation intermediates: gathered rows, h and expert outputs are not counted)."""
    b = weight_bytes_per_element(fp8)
    per_expert = 3.0 * cfg.I * cfg.H * b
    return (experts_used * per_expert + 3.0 * cfg.I_shared * cfg.H * b + cfg.E * cfg.H * 4 +
            cfg.E * 4 + 2.0 * cfg.T * cfg.H * 2)


def up_launch_bytes(cfg: BlockConfig, experts_used: int, fp8: bool = False,
                    both: bool = False) -> float:
    """The expert-up launch's share of the algorithmic bytes: w13 of the used
    experts, ws13 and the tokens x once (no intermediates); with ``both`` (one
    launch runs both projections) also w2 of the used experts and ws2."""
    b = weight_bytes_per_element(fp8)
    k = 3.0 if both else 2.0
    return (experts_used * k * cfg.I * cfg.H * b + k * cfg.I_shared * cfg.H * b +
            cfg.T * cfg.H * 2.0)


def fused_small_batch(cfg: BlockConfig, fp8: bool) -> bool:
    """The library runs both swapped projections as one launch: few rows per
    expert and the shared expert, if any, a group of the routed GEMMs."""
    return (not fp8 and cfg.T * cfg.top_k <= 64 * cfg.E and
            (cfg.I_shared == cfg.I or cfg.I_shared == 0))


class CallTimer:
    """Two CUDA events around one call on the current stream (created and
    recorded once up front so that their handles exist)."""

    def __init__(self):
        self.begin = torch.cuda.Event(enable_timing=True)
        self.end = torch.cuda.Event(enable_timing=True)
        self.begin.record()
        self.end.record()

    def stage_ms(self):
        return {"expert_up": self.begin.elapsed_time(self.end)}


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of ``kernel`` from the committed ncu summary, or None when the
    kernel's source has changed since the counters were taken (or none were taken)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("workload") != workload:
        return None
    with open(os.path.join(ROOT, rec["source"]), "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    if not sha.startswith(rec["source_sha256_prefix"]):
        return None
    return float(rec["dram_bytes_read"] + rec["dram_bytes_write"])


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()

    def stop(self):
        if self._thr is not None:
            self._stop.set()
            self._thr.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def _dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    return world, rank, local


def _barrier(world):
    if world > 1:
        torch.distributed.barrier()


def _max_over_ranks(v: float, world: int) -> float:
    return max_over_ranks(v) if world > 1 else v


def cpu_oracle_sample(cfg_id: int, target_s: float = 12.0, d_cpu=None):
    """Times the CPU oracle on a bounded sample of the workload's tokens.
    Returns (tokens_per_s, cores, sample description)."""
    import oracle
    from tests import parity

    wl = inputs.WORKLOADS[cfg_id]
    cfg = BlockConfig(T=wl.T, H=wl.H)
    if d_cpu is None:
        d_cpu = inputs.workload_inputs(cfg_id)
    dn = parity.np_inputs(d_cpu)
    ocfg = parity.oracle_cfg(cfg)
    m = inputs.token_mask(wl)
    mask_np = None if m is None else m.numpy()
    rng = np.random.default_rng(0)
    n = 16
    t_used = 0.0
    done = 0
    while True:
        toks = rng.choice(wl.T, n, replace=False)
        t0 = time.perf_counter()
        if wl.dense_I:
            oracle.dense_ffn(dn["x"][toks], dn["w13"], dn["w2"])
        else:
            oracle.moe_forward_tokens(toks, dn["x"], dn["Wr"], dn["bias"], dn["w13"], dn["w2"],
                                      dn["ws13"], dn["ws2"], ocfg, token_mask=mask_np)
        dt = time.perf_counter() - t0
        t_used += dt
        done += n
        if t_used >= target_s or done >= wl.T:
            break
        n = int(min(wl.T - done, max(n, n * max(1.0, (target_s - t_used) / max(dt, 1e-3)))))
        n = max(1, min(n, 4096))
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    return done / t_used, int(cores), (f"{done} tokens of {wl.name} drawn at random, "
                                       f"float64 NumPy oracle, {t_used:.1f} s")


def run_reference(args, world, rank):
    """CPU oracle arm: bounded token sample per step, rank 0 only."""
    if rank != 0:
        return
    wl = inputs.WORKLOADS[args.config]
    cfg = BlockConfig(T=wl.T, H=wl.H)
    import oracle
    from tests import parity
    d_cpu = inputs.workload_inputs(args.config)
    dn = parity.np_inputs(d_cpu)
    ocfg = parity.oracle_cfg(cfg)
    per_step = max(1, min(wl.T, args.ref_tokens))
    m = inputs.token_mask(wl)
    mask_np = None if m is None else m.numpy()
    rng = np.random.default_rng(1)
    def one(toks):
        if wl.dense_I:
            oracle.dense_ffn(dn["x"][toks], dn["w13"], dn["w2"])
        else:
            oracle.moe_forward_tokens(toks, dn["x"], dn["Wr"], dn["bias"], dn["w13"], dn["w2"],
                                      dn["ws13"], dn["ws2"], ocfg, token_mask=mask_np)

    for _ in range(args.warmup if args.ref_warmup else 0):
        one(rng.choice(wl.T, per_step, replace=False))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one(rng.choice(wl.T, per_step, replace=False))
    dt = time.perf_counter() - t0
    tps = per_step * args.steps / dt
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    line = {
        "impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "E": 128, "I": 768,
                   "top_k": 8, "tokens_per_step_sampled": per_step},
        "tflops": tps * (6.0 * wl.H * wl.dense_I if wl.dense_I else flops_per_token(cfg)) / 1e12,
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": int(cores), "kind": "oracle",
                         "sample": f"{per_step} random tokens of {wl.name} per step"},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    wl = inputs.WORKLOADS[args.config]
    cfg = BlockConfig(T=wl.T, H=wl.H)
    layers = wl.layers
    # weights: identical on every rank; tokens: a different batch per rank
    gen_dev = dev if layers > 1 else "cpu"
    dense = wl.dense_I > 0  # a dense feed-forward layer instead of the MoE block
    fp8 = bool(args.fp8)
    if fp8 and (dense or layers > 1):
        raise SystemExit("--fp8 applies to the single-layer MoE workloads")
    weights = []
    for l in range(layers):
        if dense:
            wd = inputs.make_dense_weights(wl.H, wl.dense_I, wl.seed, device=gen_dev)
        else:
            wd = inputs.make_weights(wl.H, wl.seed, device=gen_dev, layer=l,
                                     hot_experts=wl.hot_experts, hot_bias=wl.hot_bias)
        if fp8:  # E4M3 expert weights from the same normal draws, router unchanged
            wd = dict(Wr=wd["Wr"], bias=wd["bias"],
                      **inputs.make_fp8_weights(wl.H, wl.seed, device=dev, layer=l))
        weights.append({k: (None if v is None else v.to(dev)) for k, v in wd.items()})
    x_host = inputs.make_tokens(wl.T, wl.H, rank_token_seed(wl.seed, rank)).pin_memory()
    x = x_host.to(dev)
    ws = ops.alloc_workspace(ops.workspace_bytes(cfg) if not dense else
                             ops.lib().moe_dense_ffn_workspace_bytes(wl.T, wl.H, wl.dense_I), dev)
    out = torch.empty_like(x)
    xn_buf = torch.empty_like(x)
    ids = torch.empty((wl.T, cfg.top_k), dtype=torch.int32, device=dev)

    mask_dev = inputs.token_mask(wl, dev)  # padding mask of the workload, or None

    def step(xin, timer=None):
        if dense:  # the whole layer is timed: both GEMMs (no stage events inside)
            w = weights[0]
            if timer is not None:
                timer.begin.record(torch.cuda.current_stream())
            ops.dense_ffn(xin, w["w13"], w["w2"], out=out, workspace=ws)
            if timer is not None:
                timer.end.record(torch.cuda.current_stream())
            return out
        if fp8:
            w = weights[0]
            return ops.forward_fp8(xin, w["Wr"], w["bias"], w, cfg, out=out, workspace=ws,
                                   timer=timer, topk_ids=ids, token_mask=mask_dev)
        if layers == 1:
            w = weights[0]
            return ops.forward(xin, w["Wr"], w["bias"], w["w13"], w["w2"], w["ws13"], w["ws2"],
                               cfg, out=out, workspace=ws, timer=timer, topk_ids=ids,
                               token_mask=mask_dev)
        # residual stack: x <- x + block_l(RMSNorm(x)), updated in place in `out`
        out.copy_(xin)
        for l, w in enumerate(weights):
            ops.rmsnorm(out, eps=1e-6, out=xn_buf)
            ops.forward(xn_buf, w["Wr"], w["bias"], w["w13"], w["w2"], w["ws13"], w["ws2"], cfg,
                        residual=out, out=out, workspace=ws, timer=timer if l == 0 else None,
                        topk_ids=ids)
        return out

    for _ in range(args.warmup):
        step(x)
    torch.cuda.synchronize()
    code, site = ops.read_device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {ops.status_string(code)} at {site}")

    stream = torch.cuda.current_stream()
    # only the dominant kernel is timed inside the headline region: every
    # recorded event orders the chained kernels around it
    timers = [(CallTimer() if dense else ops.StageTimer(stages=("expert_up",)))
              for _ in range(args.steps)]
    sampler = ClockSampler(local)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    ev0.record(stream)
    for i in range(args.steps):
        step(x, timer=timers[i])
    ev1.record(stream)
    torch.cuda.synchronize()
    sampler.stop()
    _barrier(world)
    ms_local = ev0.elapsed_time(ev1) / args.steps
    ms = _max_over_ranks(ms_local, world)
    code, site = ops.read_device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {ops.status_string(code)} at {site}")

    # the expert-up stage is exactly one kernel launch
    up_ms_live = float(np.mean([t.stage_ms()["expert_up"] for t in timers]))
    # stage split, from a separate pass with every stage boundary recorded
    if dense:
        per_stage = {"dense_ffn": up_ms_live}
        experts_used = 0
    else:
        split_timers = [ops.StageTimer() for _ in range(min(args.steps, 10))]
        for t in split_timers:
            step(x, timer=t)
        torch.cuda.synchronize()
        per_stage = {k: float(np.mean([t.stage_ms()[k] for t in split_timers]))
                     for k in ops.STAGES}
        flat = ids.reshape(-1).long()
        counts = torch.bincount(flat[flat >= 0], minlength=cfg.E)  # padding tokens have ids -1
        experts_used = int((counts > 0).sum().item())

    # end to end: pinned host tokens -> device -> block -> host, every step.
    # Serial: one batch at a time, the copies on the compute stream.
    out_host = torch.empty_like(x_host).pin_memory()
    x_dev = torch.empty_like(x)

    def serial_steps(n):
        for _ in range(n):
            x_dev.copy_(x_host, non_blocking=True)
            y = step(x_dev)
            out_host.copy_(y, non_blocking=True)

    serial_steps(2)
    _barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    serial_steps(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    e2e_serial_ms = _max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    e2e_ms, e2e_mode = e2e_serial_ms, "serial: copy in, block, copy out, one batch at a time"
    if layers == 1 and mask_dev is None and not dense and not fp8:
        # the library's host-batch entry point: every step's batch is copied in
        # and its output copied out, the copies of the neighbouring batches
        # overlapping each batch's kernels (two copy streams)
        w = weights[0]
        copy_streams = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
        hws = ops.alloc_workspace(ops.forward_host_workspace_bytes(cfg), dev)

        def host_steps(n):
            ops.forward_host([x_host] * n, [out_host] * n, w["Wr"], w["bias"], w["w13"], w["w2"],
                             w["ws13"], w["ws2"], cfg, workspace=hws, copy_streams=copy_streams)

        host_steps(2)
        _barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        host_steps(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        _barrier(world)
        code, site = ops.read_device_status(hws)
        if code != 0:
            raise RuntimeError(f"device status {ops.status_string(code)} at {site}")
        e2e_ms = _max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
        e2e_mode = ("moe_forward_host: batch b+1 copied in and b-1 copied out while b computes "
                    "(pinned host buffers, two copy streams)")

    if rank == 0:
        peaks, peak_src = load_peaks()
        tok_per_step = wl.T * layers
        total_tokens = tok_per_step * world
        value = total_tokens / (ms * 1e-3)
        fpt = flops_per_token(cfg) if not dense else 6.0 * wl.H * wl.dense_I
        # padding tokens (token mask 0) run only the router and the shared expert
        n_pad = 0 if mask_dev is None else int((mask_dev == 0).sum().item())
        n_real = wl.T - n_pad
        fpt_pad = 2.0 * cfg.E * cfg.H + 6.0 * cfg.H * cfg.I_shared
        flops_per_step = n_real * fpt + n_pad * fpt_pad  # one layer, one rank
        tflops = flops_per_step * layers * world / (ms * 1e-3) / 1e12
        # the expert-up launch also runs the shared expert as one more group
        # when its intermediate size equals the experts' (the model's case)
        R = n_real * cfg.top_k
        up_rows = R + (wl.T if cfg.I_shared == cfg.I else 0)
        up_flops = 2.0 * up_rows * cfg.H * (2 * cfg.I)
        both = not dense and fused_small_batch(cfg, fp8)
        if both:  # the timed launch also runs the down projection
            up_flops += 2.0 * up_rows * cfg.I * cfg.H
        if dense:  # the timed launch pair is the whole layer: both GEMMs
            up_rows, up_flops = wl.T, flops_per_step
        up_ms = up_ms_live
        # a kernel inside a long timed region runs at the power-capped sustained
        # clock: compare it with the sustained peak there, with the burst peak otherwise
        long_region = ms * args.steps > 200.0
        peak_key = "bf16_tflops_sustained" if long_region else "bf16_tflops"
        peak_tf = peaks.get(peak_key, peaks["bf16_tflops"])
        achieved = up_flops / (up_ms * 1e-3) / 1e12
        layer_ms = ms / layers
        hbm_bytes = (algorithmic_bytes(cfg, experts_used, fp8) if not dense else
                     3.0 * wl.dense_I * wl.H * 2 + 2.0 * wl.T * wl.H * 2)
        t_flop = flops_per_step / peak_tf / 1e12
        t_hbm = hbm_bytes / peaks["hbm_gbs"] / 1e9
        swapped = wl.T * cfg.top_k <= 64 * cfg.E  # the kernel the library picks for this shape
        kernel = ("grouped_gemm_swap_kernel<SwiGLU> (expert up, shared expert folded in)"
                  if swapped else
                  "grouped_gemm_kernel<SwiGLU> (expert up, shared expert folded in)")
        if both:
            kernel = "swap_fused_kernel (expert up then down in one launch, shared expert folded in)"
        if fp8:
            swapped = True  # FP8 weights: the dequantising swapped kernel at every size
            kernel = "grouped_gemm_swap_fp8_kernel<SwiGLU> (expert up, E4M3 weights, shared folded in)"
        if dense:
            swapped = wl.T <= 64
            kernel = "grouped_gemm_kernel<SwiGLU> + <RowScale> (dense layer: both GEMMs)"
        if t_hbm > t_flop:
            # HBM-bound layer: the expert-up launch's algorithmic bytes are w13 of the
            # used experts, ws13 and the tokens once (the gathered rows it reads and
            # the h it writes are intermediates and are not counted)
            up_bytes = up_launch_bytes(cfg, experts_used, fp8, both)
            ach = up_bytes / (up_ms * 1e-3) / 1e9
            rf = {"bound": "hbm", "kernel": kernel, "achieved": ach, "peak": peaks["hbm_gbs"],
                  "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
                  "peak_source": f"{peak_src} HBM copy bandwidth",
                  "frac_of_datasheet_8000_gbs": ach / DATASHEET_HBM_GBS,
                  "algorithmic_bytes_per_launch": up_bytes, "flops_per_launch": up_flops}
        else:
            rf = {"bound": "tensor", "kernel": kernel,
                  "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                  "frac": achieved / peak_tf,
                  "peak_source": f"{peak_src} bf16 dense {'sustained' if long_region else 'burst'}"}
        rf["traffic"] = (None if swapped or dense else
                         measured_traffic("grouped_gemm_kernel<EPI_SWIGLU>", wl.name))
        rf["traffic_unit"] = "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"
        rf["layer_roofline_frac"] = max(t_flop, t_hbm) / (layer_ms * 1e-3)
        if t_hbm > t_flop:
            rf["layer_hbm_frac_of_datasheet_8000_gbs"] = (
                hbm_bytes / (DATASHEET_HBM_GBS * 1e9) / (layer_ms * 1e-3))
        cpu_tps, cores, sample = (None, None, None)
        if world == 1 and not args.no_cpu_baseline:
            cpu_tps, cores, sample = cpu_oracle_sample(args.config, target_s=args.cpu_seconds)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal/uniform tensors of the workload's shapes)",
            "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "E": cfg.E, "I": cfg.I,
                       "I_shared": cfg.I_shared, "top_k": cfg.top_k, "n_group": cfg.n_group,
                       "topk_group": cfg.topk_group, "layers": layers,
                       "tokens_per_gpu_per_step": tok_per_step,
                       "padding_tokens_per_layer": n_pad,
                       "dense_intermediate": wl.dense_I or None,
                       "expert_weights": ("fp8 e4m3, one power-of-two scale per 128x128 block"
                                          if fp8 else "bf16"),
                       "l2": ("inputs larger than L2: " +
                              ("the layer's 85 MB of weights, 80 MB of tokens in and out"
                               if dense else "1.2 GB of expert weights read per layer"))},
            "tflops": tflops,
            "roofline": rf,
            "stage_ms": per_stage,
            "stage_ms_note": ("the timed calls themselves" if dense else
                              "separate pass with an event at every stage boundary"),
            "experts_used": experts_used,
            "cpu_baseline": None if cpu_tps is None else {
                "value": cpu_tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                "sample": sample},
            "e2e": {"value": total_tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(x_host.numel() * 2),
                    "d2h_bytes_per_step": int(out_host.numel() * 2),
                    "mode": e2e_mode,
                    "serial_value": total_tokens / (e2e_serial_ms * 1e-3)},
            "gpu_launches": ((2 if dense else kernels_per_step(cfg, fp8) + (1 if layers > 1 else 0)) *
                             layers * args.steps),
            "clocks": sampler.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=2, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-tokens", type=int, default=64,
                    help="tokens per step for --impl reference (bounded CPU sample)")
    ap.add_argument("--ref-warmup", action="store_true")
    ap.add_argument("--fp8", action="store_true",
                    help="FP8 (E4M3, block-scaled) expert weights (single-layer MoE workloads)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        raise SystemExit("--warmup must be >= 3")
    world, rank, local = _dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
