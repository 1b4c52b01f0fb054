#!/usr/bin/env python3
"""Benchmark of the Agent Attention forward pass on B200.

One step = one whole forward pass (pool -> aggregate -> merge -> broadcast)
over one batch of the synthetic workload, through the C ABI.  Prints ONE JSON
line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...     (the fp64 CPU oracle as the reference arm)

For N > 1 it is launched by torch.distributed.run; every rank runs the full
workload on its own GPU with its own seed (weak scaling, no collective on the
data path); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "agent-attn tokens·heads/s; achieved HBM GB/s vs B200 peak (1 GPU)"
UNIT = "tokens*heads/s"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_bytes(w, batch):
    """Algorithmic HBM bytes of one pass: Q, K, V read once and O written once."""
    return 4 * batch * w.H * w.N * w.d * w.elem_bytes


class ClockSampler:
    """Samples SM clocks and clock-event (throttle) reasons through NVML in a
    background thread while the timed region runs (read-only queries)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int, enabled: bool):
        import threading
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.error = None
        self._stop = threading.Event()
        self._thread = None
        if not enabled:
            return
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[gpu_index]) if vis and vis.split(",")[0].isdigit() \
                else gpu_index
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: leave the record empty
            self.error = repr(e)
            return
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception as e:
                self.error = repr(e)
                return
            self._stop.wait(0.005)

    def stop(self):
        if self._thread is None:
            return None if self.error is None else {"error": self.error}
        self._stop.set()
        self._thread.join(timeout=5)
        if not self.samples:
            return {"error": self.error or "no samples"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": sorted(self.reasons)}


# Sources of each kernel the roofline reports; a recorded DRAM-traffic figure
# applies only while its kernel's sources hash the same.
_TC_COMMON = ("common.cuh", "tc_primitives.cuh", "kernels_tc.cuh")
ROOFLINE_SOURCES = {
    "agent_aggregate+agent_merge": _TC_COMMON + ("kernels_merge.cuh",),
    "agent_broadcast": _TC_COMMON,
    "agent_fused_small": _TC_COMMON + ("kernels_fused.cuh",),
}


def kernel_source_sha(kernel: str):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "efficient_vision_attention_b200", "csrc")
    for name in ROOFLINE_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel's current sources."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    if kernel not in ROOFLINE_SOURCES:
        return None
    for r in rec.get("records", []):
        if (r.get("kernel") == kernel and r.get("workload") == workload
                and r.get("source_sha") == kernel_source_sha(kernel)):
            return r.get("dram_bytes_per_launch")
    return None


# ex2.approx.f32 results per clock per SM (measured on B200 with a
# micro-benchmark; the packed bf16x2 / f16x2 forms give no more per clock).
SFU_EXP_PER_CLK_PER_SM = 16


def sfu_roofline(n_exp: int, ms: float, sms: int, mhz: float) -> dict:
    """The exponential roofline of a softmax kernel: n_exp exponentials per
    launch in `ms` milliseconds against SFU_EXP_PER_CLK_PER_SM results per
    clock on each of `sms` SMs at `mhz`."""
    peak = SFU_EXP_PER_CLK_PER_SM * sms * mhz * 1e6
    achieved = n_exp / (ms * 1e-3)
    return {"bound": "sfu", "achieved": achieved, "peak": peak, "unit": "exp/s",
            "frac": achieved / peak, "exps_per_launch": n_exp, "sm_mhz": mhz}


def cpu_baseline(w, target_s=12.0):
    """The fp64 oracle, as it stands, on a bounded sample of the workload:
    whole (b, h) slices, as many as fit in about target_s seconds."""
    import numpy as np
    import oracle
    from efficient_vision_attention_b200.workloads import make_inputs
    inp = make_inputs(w, B=1)
    q, k, v, ag = inp["q"], inp["k"], inp["v"], inp["agents"]

    def one(h):
        f = lambda t: t[0, h:h + 1].double().numpy()
        a = None if ag is None else ag[h:h + 1].double().numpy()
        return oracle.agent_attn(f(q), f(k), f(v), w.grid_h, w.grid_w, w.pool_h, w.pool_w,
                                 w.scale, agents=a)

    oracle.build()
    t0 = time.perf_counter()
    done = 0
    while True:
        one(done % w.H)
        done += 1
        el = time.perf_counter() - t0
        if el >= target_s or (el / done) * (done + 1) > 3 * target_s:
            break
    el = time.perf_counter() - t0
    return {"value": done * w.N / el, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{done} whole (b,h) slice(s) of {w.name} (N={w.N}, k={w.n_agents}, "
                      f"d={w.d}), fp64, {el:.1f} s"}


def bench_config(w, world, set_bytes=None, n_sets=None):
    cfg = w.describe()
    cfg.update({"global_batch": world * w.B, "seq_len": w.N, "parallelism": f"replicas x{world}"})
    if set_bytes is not None:
        cfg["l2"] = (f"rotating {n_sets} input sets of {set_bytes / 2**20:.0f} MiB "
                     f"(> 3x the 126 MB L2)")
    return cfg


def input_sets(w):
    """Bytes of one input set and the number of sets the native arm rotates
    through so that consecutive steps' inputs together exceed L2."""
    set_bytes = workload_bytes(w, w.B)
    return set_bytes, max(2, math.ceil(3 * L2_BYTES / set_bytes))


def run_reference(args, w):
    from efficient_vision_attention_b200.replicas import dist_env
    world, rank, _ = dist_env()
    if rank != 0:
        return
    steps, warm = args.steps, args.warmup
    base = cpu_baseline(w, target_s=1.0)          # warm-up and sizing
    per_step = max(1.0, min(8.0, 150.0 / max(1, steps + warm)))
    for _ in range(max(0, warm - 1)):
        cpu_baseline(w, target_s=0.2)
    vals = []
    t0 = time.perf_counter()
    for _ in range(steps):
        vals.append(cpu_baseline(w, target_s=per_step / 2))
    el = time.perf_counter() - t0
    value = statistics.median(v["value"] for v in vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": warm, "ms_per_step": 1e3 * el / max(1, steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": bench_config(w, world, *input_sets(w)),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": base["cores"], "kind": "oracle",
                         "sample": vals[-1]["sample"] + " per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_native(args, w):
    import torch
    import efficient_vision_attention_b200 as eva
    from efficient_vision_attention_b200 import replicas
    from efficient_vision_attention_b200.workloads import make_inputs

    world, rank, local = replicas.dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = replicas.init("nccl", dev)
    eva.load_library()
    stream = torch.cuda.current_stream(dev)
    dt = eva.AA_FP32 if w.dtype == "fp32" else eva.AA_BF16
    B, H, N, d, nk = w.B, w.H, w.N, w.d, w.n_agents

    # Rotate input sets so that the inputs of consecutive steps together exceed L2.
    set_bytes, n_sets = input_sets(w)
    sets = []
    for i in range(n_sets):
        inp = make_inputs(w, seed=replicas.rank_seed(w.seed, rank) + i)
        s = {n: inp[n].to(dev) for n in "qkv"}
        s["agents"] = inp["agents"].to(dev) if inp["agents"] is not None else None
        s["out"] = torch.empty_like(s["q"])
        sets.append(s)
    ws_bytes = eva.agent_attn_workspace_bytes(B, H, N, d, nk, dt)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def step(i):
        s = sets[i % n_sets]
        if w.learnable_agents:
            eva.agent_attn_forward_agents(s["q"], s["k"], s["v"], s["agents"], nk, 0, s["out"],
                                          B, H, N, d, w.scale, dt, stream)
        else:
            eva.agent_attn_forward_ws(s["q"], s["k"], s["v"], None, s["out"], B, H, N, d,
                                      w.grid_h, w.grid_w, w.pool_h, w.pool_w, w.scale, dt, ws,
                                      ws_bytes, stream)

    fused = takes_fused_small_path(w)
    launches_per_step = 1 if fused else (3 if w.learnable_agents else 4)
    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()

    def barrier():
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()

    clocks = ClockSampler(local, enabled=(rank == 0 and not args.no_clocks))
    barrier()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    barrier()
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = replicas.max_over_ranks(ms, pg, dev)
    units = world * B * H * N
    value = units / (ms_max * 1e-3)

    # Per-stage durations, measured live with events on the launch stream:
    # each stage is launched `reps` times back to back (inputs rotating over
    # the same sets) between two events, so the device time per launch is
    # measured without host launch gaps.
    stage = {"pool": [], "aggregate": [], "broadcast": []}
    s0 = sets[0]
    a_low = torch.empty((B, H, nk, d), dtype=w.torch_dtype, device=dev)
    a32 = torch.empty((B, H, nk, d), dtype=torch.float32, device=dev)
    va_low = torch.empty((B, H, nk, d), dtype=w.torch_dtype, device=dev)
    va32 = torch.empty((B, H, nk, d), dtype=torch.float32, device=dev)
    if w.learnable_agents:
        agents, a_stride = s0["agents"], 0
    else:
        agents, a_stride = (a32 if dt == eva.AA_FP32 else a_low), H * nk * d
    va_in = va32 if dt == eva.AA_FP32 else va_low

    def run_pool(s):
        eva.agent_attn_stage_pool(s["q"], a32, a_low, B, H, N, d, w.grid_h, w.grid_w,
                                  w.pool_h, w.pool_w, dt, stream)

    def run_agg(s):
        eva.agent_attn_stage_aggregate(agents, a_stride, s["k"], s["v"], None if dt != eva.AA_FP32
                                       else va32, va_low if dt != eva.AA_FP32 else None, B, H,
                                       N, d, nk, w.scale, dt, stream)

    def run_bc(s):
        eva.agent_attn_stage_broadcast(s["q"], agents, a_stride, va_in, s["out"], B, H, N, d,
                                       nk, w.scale, dt, stream)

    if not w.learnable_agents:
        run_pool(s0)
    run_agg(s0)
    torch.cuda.synchronize()
    reps = max(10, min(args.steps, 50))
    for name, fn in (("pool", run_pool), ("aggregate", run_agg), ("broadcast", run_bc)):
        if name == "pool" and w.learnable_agents:
            stage[name].append(0.0)
            continue
        for r in range(3):
            fn(sets[r % n_sets])
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for r in range(reps):
            fn(sets[r % n_sets])
        e1.record(stream)
        torch.cuda.synchronize()
        stage[name].append(e0.elapsed_time(e1) / reps)
    stage_ms = {k: statistics.mean(v) for k, v in stage.items()}
    half_bytes = 2 * B * H * N * d * w.elem_bytes       # aggregate: K+V; broadcast: Q+O
    peak, peak_kind = peaks()
    dom = "aggregate" if stage_ms["aggregate"] >= stage_ms["broadcast"] else "broadcast"
    achieved = half_bytes / (stage_ms[dom] * 1e-3) / 1e9
    both = 2 * half_bytes / ((stage_ms["aggregate"] + stage_ms["broadcast"]) * 1e-3) / 1e9
    kernel_name = {"aggregate": "agent_aggregate+agent_merge", "broadcast": "agent_broadcast"}[dom]
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": f"of {peak_kind}",
                "kernel": kernel_name,
                "algorithmic_bytes_per_launch": half_bytes,
                "traffic": recorded_traffic(kernel_name, w.name)}
    if fused:
        # the whole pass is one kernel: Q, K, V read once, O written once per
        # launch, timed as the step itself (one launch per step)
        fused_bytes = 2 * half_bytes
        achieved = fused_bytes / (ms_max * 1e-3) / 1e9
        dom, kernel_name = None, "agent_fused_small"
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "peak_kind": f"of {peak_kind}",
                    "kernel": kernel_name, "algorithmic_bytes_per_launch": fused_bytes,
                    "traffic": recorded_traffic(kernel_name, w.name)}
    # The same kernel against its exponential bound (one exp per score: B*H*N*k
    # in either stage), at the SM clock the sampler saw as the maximum.
    clk_mhz = (clk or {}).get("sm_max_mhz") or 1965.0
    sfu = sfu_roofline((2 if fused else 1) * B * H * N * nk, ms_max if fused else stage_ms[dom],
                       torch.cuda.get_device_properties(dev).multi_processor_count,
                       float(clk_mhz))
    sfu["kernel"] = kernel_name

    # The DWC term of the full module (depth-wise 3x3 convolution of V added to
    # O) on the same workload: its own kernel, HBM-bound (V read, O read and
    # written), timed with back-to-back launches like the stages above.
    gw_ = torch.Generator().manual_seed(w.seed + 77)
    dwc_w = (torch.randn((H, d, 3, 3), generator=gw_) * 0.3).to(dev)
    dwc_b = (torch.randn((H, d), generator=gw_) * 0.1).to(dev)

    def run_dwc(s):
        eva.agent_attn_dwc(s["v"], dwc_w, dwc_b, s["out"], B, H, w.grid_h, w.grid_w, d, dt, True,
                           stream)

    for r in range(3):
        run_dwc(sets[r % n_sets])
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for r in range(reps):
        run_dwc(sets[r % n_sets])
    e1.record(stream)
    torch.cuda.synchronize()
    dwc_ms = e0.elapsed_time(e1) / reps
    dwc_bytes = 3 * B * H * N * d * w.elem_bytes
    dwc = {"kernel": "dwc", "ms": dwc_ms, "algorithmic_bytes_per_launch": dwc_bytes,
           "achieved_gbs": dwc_bytes / (dwc_ms * 1e-3) / 1e9,
           "frac": dwc_bytes / (dwc_ms * 1e-3) / 1e9 / peak}

    # The full module output (attention + DWC term) through its own entry
    # point: the forward pass, then the DWC kernel accumulating into its output
    # (chained by programmatic dependent launch).
    def run_fwd_dwc(s):
        eva.agent_attn_forward_dwc(s["q"], s["k"], s["v"], agents if w.learnable_agents else None,
                                   dwc_w, dwc_b, s["out"], B, H, N, d, w.grid_h, w.grid_w,
                                   w.pool_h, w.pool_w, w.scale, dt, stream)

    for r in range(3):
        run_fwd_dwc(sets[r % n_sets])
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for r in range(reps):
        run_fwd_dwc(sets[r % n_sets])
    e1.record(stream)
    torch.cuda.synchronize()
    fd_ms = e0.elapsed_time(e1) / reps
    fwd_dwc = {"ms_per_forward": fd_ms, "value": B * H * N / (fd_ms * 1e-3), "unit": UNIT,
               "vs_forward": fd_ms / ms_max}

    # The forward pass with agent bias (row, column and block components in
    # both softmaxes) on the same workload (bias added inside the score tiles).
    gb_ = torch.Generator().manual_seed(w.seed + 78)
    nb_ = w.pool_h * w.pool_w

    def bias_triple():
        return [(torch.randn((H, nk, n_), generator=gb_) * 0.5).to(dev)
                for n_ in (w.grid_h, w.grid_w, nb_)]

    b1_, b2_ = bias_triple(), bias_triple()

    def run_bias(s):
        eva.agent_attn_forward_bias(s["q"], s["k"], s["v"], None, b1_, b2_, s["out"], B, H, N, d,
                                    w.grid_h, w.grid_w, w.pool_h, w.pool_w, w.scale, dt, stream)

    bias_fwd = None
    if not w.learnable_agents:
        run_bias(sets[0])
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for r in range(3):
            run_bias(sets[r % n_sets])
        e1.record(stream)
        torch.cuda.synchronize()
        b_ms = e0.elapsed_time(e1) / 3
        bias_fwd = {"ms_per_forward": b_ms, "value": B * H * N / (b_ms * 1e-3), "unit": UNIT,
                    "path": "tcgen05" if (w.dtype == "bf16" and d <= 64) else "simt"}

    # The backward pass (gradients of Q, K, V for an output gradient) on the
    # same workload: the forward statistics recomputed on the tensor cores
    # (bf16, d <= 64), the gradient kernels SIMT with fp32 arithmetic.
    bwd = None
    if not w.learnable_agents:
        dout_ = torch.randn(sets[0]["q"].shape, generator=torch.Generator().manual_seed(5)).to(
            w.torch_dtype).to(dev)
        gq_, gk_, gv_ = (torch.empty_like(sets[0]["q"]) for _ in range(3))

        def run_bwd(s):
            eva.agent_attn_backward(s["q"], s["k"], s["v"], None, dout_, gq_, gk_, gv_, None, B, H,
                                    N, d, w.grid_h, w.grid_w, w.pool_h, w.pool_w, w.scale, dt,
                                    stream)

        for r in range(2):
            run_bwd(sets[r % n_sets])
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        bwd_reps = 5
        e0.record(stream)
        for r in range(bwd_reps):
            run_bwd(sets[r % n_sets])
        e1.record(stream)
        torch.cuda.synchronize()
        bwd_ms = e0.elapsed_time(e1) / bwd_reps
        bwd = {"ms_per_backward": bwd_ms, "value": B * H * N / (bwd_ms * 1e-3), "unit": UNIT,
               "path": ("forward statistics on tcgen05, gradients simt"
                        if (w.dtype == "bf16" and d <= 64) else "simt")}

    # End to end through the host-buffer entry point: pinned host inputs copied
    # in, result copied out, every step.
    hin = make_inputs(w, seed=replicas.rank_seed(w.seed, rank))
    hq, hk, hv = (hin[n].pin_memory() for n in "qkv")
    hag = hin["agents"].pin_memory() if hin["agents"] is not None else None
    hout = torch.empty_like(hq).pin_memory()
    e2e_steps = max(3, min(10, args.steps))

    def host_step():
        # learnable workloads: pool_h * pool_w equals the agent count, so the
        # host entry point takes the [H, k, d] agents through the same call
        eva.agent_attn_forward_host(hq, hk, hv, hag, hout, B, H, N, d, w.grid_h, w.grid_w,
                                    w.pool_h, w.pool_w, w.scale, dt, stream)

    assert w.pool_h * w.pool_w == nk
    if True:
        for _ in range(2):
            host_step()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            host_step()
        e1.record(stream)
        barrier()
        e_ms = replicas.max_over_ranks(e0.elapsed_time(e1) / e2e_steps, pg, dev)
        in_bytes = 3 * B * H * N * d * w.elem_bytes + (hag.numel() * hag.element_size()
                                                       if hag is not None else 0)
        e2e = {"value": units / (e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": in_bytes,
               "d2h_bytes_per_step": B * H * N * d * w.elem_bytes,
               "ms_per_step": e_ms}

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(w)

    replicas.finalize(pg)
    if rank != 0:
        return
    cfg = bench_config(w, world, set_bytes, n_sets)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": cfg,
        "hbm_gbs_aggregate_plus_broadcast": both,
        "hbm_frac_aggregate_plus_broadcast": both / peak,
        "stage_ms": stage_ms,
        "forward_path": "fused_small (one kernel)" if fused else
                        "pool + aggregate + merge + broadcast",
        "roofline": roofline,
        "sfu_roofline": sfu,
        "dwc_term": dwc,
        "forward_dwc": fwd_dwc,
        "agent_bias_forward": bias_fwd,
        "backward": bwd,
        "cpu_baseline": base,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def takes_fused_small_path(w) -> bool:
    """Whether the library runs this workload's forward pass as the single
    fused small-slice kernel: bf16, pooled agents, N <= 256, k <= 128,
    8 <= d <= 64 with d % 8 == 0, and the O staging tiles fitting the K and V
    buffers (the rule of fused_small_fits in kernels_fused.cuh)."""
    N, d, k = w.grid_h * w.grid_w, w.d, w.pool_h * w.pool_w
    if w.dtype != "bf16" or w.learnable_agents or not (1 <= N <= 256 and 1 <= k <= 128):
        return False
    if not (8 <= d <= 64 and d % 8 == 0):
        return False
    rows = (N + 15) // 16 * 16
    return 2 * rows * 128 >= ((N + 127) // 128) * 128 * 128


def main():
    args = parse()
    from efficient_vision_attention_b200.workloads import BENCH_WORKLOAD, WORKLOADS
    w = WORKLOADS[args.workload or BENCH_WORKLOAD]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_native(args, w)


if __name__ == "__main__":
    main()
