"""Benchmark: MoE dispatch + combine fused with layout on B200.

One step = the whole hot path over one batch: layout (histogram, scan, slot
assignment), fused dispatch (flat, or two-level through node staging for the
DeepSeek-V3-shaped workload) and fused combine.  The combine reads a separate
stand-in expert-output buffer (as it would after the expert GEMMs), so no
step reads rows the same step just wrote through L2.

Timing: W untimed warm-up steps, then exactly K timed steps, each replaying
the step's CUDA graph between CUDA events on the launching stream, with L2
flushed (a read of a buffer twice the L2 size) before every step, outside the
events.  A second pass of K steps replays layout, dispatch and combine as
three graphs with events between them for the per-kernel breakdown and the
roofline figure.  Multi-GPU runs are independent replicas (no collective on
the data path): value = bytes all ranks moved / the max over ranks of the
timed time.

Metric: achieved algorithmic HBM GB/s of dispatch + combine.  Algorithmic
bytes per step are T*H*2 + T*k*H*2 for dispatch (read each token row once,
write each destination row once) and the same for combine (read each expert
row once, write each output row once); layout metadata and node staging
traffic are not credited.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload olmoe]
                    [--impl reference] [--engine auto|vector|bulk]
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from combine_moe_layout_06_b200 import inputs  # noqa: E402

METRIC = "dispatch+combine achieved HBM GB/s, % of B200 peak, and tokens/s on 1 GPU"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = {
    "combine": ["combine.cu", "moe_common.cuh"],
    "dispatch": ["dispatch.cu", "moe_common.cuh"],
}


def kernel_source_sha(stage):
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[stage]:
        with open(os.path.join(ROOT, "combine_moe_layout_06_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(stage, workload):
    """DRAM bytes per launch (read + write) from the committed ncu summary of
    this kernel, or None when there is none or the kernel source changed
    since it was captured."""
    import glob
    import re
    want = kernel_source_sha(stage)
    pat = re.compile(r"<!-- roofline-traffic kernel=(\w+) workload=(\w+) bytes=(\d+) sources=(\w+) -->")
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        with open(path) as f:
            for m in pat.finditer(f.read()):
                if m.group(1) == stage and m.group(2) == workload and m.group(4) == want:
                    return int(m.group(3))
    return None


def algorithmic_bytes(wl, tokens=None):
    T = wl.T if tokens is None else tokens
    row = wl.H * 2
    dispatch = T * row + T * wl.k * row
    combine = T * wl.k * row + T * row
    return dispatch, combine


def workload_desc(wl):
    return {
        "workload": f"{wl.name}: {inputs.DESCRIPTIONS[wl.name]}",
        "tokens": wl.T, "hidden": wl.H, "experts": wl.E, "top_k": wl.k,
        "virtual_ranks": wl.R, "virtual_nodes": wl.N,
        "dispatch_mode": "two-level node staging" if wl.two_level else "flat",
    }


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every 10 ms
    while the timed region runs (read-only queries)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: report no samples
            self._nv = None

    def _run(self):
        nv = self._nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = get_reasons(self._h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.01)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "nvml" if self._nv else "unavailable"}


# ---------------------------------------------------------------- oracle leg

def oracle_step_time(d, tokens, reps, eo_bits):
    """Time the oracle (plain C loops, one thread) on the first `tokens`
    tokens of the workload: layout, dispatch, combine.  Best of `reps`."""
    import oracle
    wl = d["workload"]
    topk = np.ascontiguousarray(d["topk_idx"][:tokens])
    x = np.ascontiguousarray(d["x"][:tokens])
    w = np.ascontiguousarray(d["topk_w"][:tokens])
    eo = np.ascontiguousarray(eo_bits[: tokens * wl.k])
    best = float("inf")
    for _ in range(reps):
        t0 = time.perf_counter()
        lay = oracle.layout(topk, wl.E, wl.R, wl.N, nodes=wl.two_level)
        if wl.two_level:
            oracle.dispatch_two_level(x, lay, wl.R, wl.N)
        else:
            oracle.dispatch_flat(x, lay["slot"])
        oracle.combine(eo, w, lay["slot"])
        best = min(best, time.perf_counter() - t0)
    return best


def run_reference(args):
    """The comparison arm: the oracle, as it stands, on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    d = inputs.make(args.workload)
    wl = d["workload"]
    tokens = max(1, min(wl.T, args.ref_tokens or max(1, wl.T // 8)))
    eo = inputs.random_bf16_bits((tokens * wl.k, wl.H), seed=wl.seed + 7)
    for _ in range(args.warmup):
        oracle_step_time(d, tokens, 1, eo)
    times = [oracle_step_time(d, tokens, 1, eo) for _ in range(args.steps)]
    disp, comb = algorithmic_bytes(wl, tokens)
    total_t = sum(times)
    gbs = (disp + comb) * args.steps / total_t / 1e9
    sample = f"first {tokens} of {wl.T} tokens per step (layout+dispatch+combine), 1 thread"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 3), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total_t / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_desc(wl),
        "tokens_per_s": round(tokens * args.steps / total_t, 1),
        "cpu_baseline": {"value": round(gbs, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(gbs, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm

def main():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="olmoe", choices=sorted(inputs.WORKLOADS))
    p.add_argument("--engine", default="auto", choices=["auto", "vector", "bulk"])
    p.add_argument("--e2e-steps", type=int, default=0, help="end-to-end steps (0: min(K, 50))")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--ref-tokens", type=int, default=0)
    args = p.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    from combine_moe_layout_06_b200 import buffers, capi

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    d = inputs.make(args.workload)
    wl = d["workload"]
    flags = capi.MOE_FLAG_TWO_LEVEL if wl.two_level else 0
    flags |= {"auto": 0, "vector": capi.MOE_FLAG_COPY_VECTOR, "bulk": capi.MOE_FLAG_COPY_BULK}[args.engine]
    cfg = capi.config(wl.T, wl.H, wl.E, wl.k, wl.R, wl.N, flags)
    dev = torch.device("cuda", local)
    lay = buffers.DeviceLayout(cfg, dev)
    x_dev = buffers.bf16_from_bits(d["x"], dev)
    topk_dev = torch.from_numpy(d["topk_idx"]).to(dev)
    w_dev = torch.from_numpy(d["topk_w"]).to(dev)
    eo_bits = inputs.random_bf16_bits((wl.T * wl.k, wl.H), seed=wl.seed + 7)
    eo_dev = buffers.bf16_from_bits(eo_bits, dev)
    recv = torch.empty((wl.T * wl.k, wl.H), dtype=torch.bfloat16, device=dev)
    y = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
    staging = None
    if wl.two_level:
        staging = torch.empty((capi.moe_node_staging_rows(cfg), wl.H), dtype=torch.bfloat16,
                              device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.ones(max(2 * l2, 1 << 20) // 4, dtype=torch.float32, device=dev)

    def flush():
        flush_buf.sum()

    def do_layout():
        capi.moe_layout(cfg, topk_dev, lay.struct)

    def do_dispatch():
        capi.moe_dispatch(cfg, lay.struct, x_dev, recv, staging)

    def do_combine():
        capi.moe_combine(cfg, lay.struct, eo_dev, w_dev, y)

    def do_step():
        do_layout()
        do_dispatch()
        do_combine()

    launches_per_step = 3 + (2 if wl.two_level else 1) + 1

    for _ in range(args.warmup):
        flush()
        do_step()
    torch.cuda.synchronize()
    st = capi.moe_get_error(lay.struct)
    if st != capi.MOE_OK:
        raise SystemExit(f"device error after warm-up: {capi.moe_status_string(st)}")

    # graphs: one for the whole step, one per stage for the breakdown
    side = torch.cuda.Stream(dev)
    graphs = {}
    for name, fn in (("step", do_step), ("layout", do_layout), ("dispatch", do_dispatch),
                     ("combine", do_combine)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            fn()
        graphs[name] = g
    for _ in range(3):
        graphs["step"].replay()
    torch.cuda.synchronize()

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(K):
            flush()
            ev[i][0].record()
            graphs["step"].replay()
            ev[i][1].record()
        torch.cuda.synchronize()
    barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = float(sum(step_ms))
    if world > 1:
        t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())

    # per-kernel breakdown, same protocol
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    for i in range(K):
        flush()
        evk[i][0].record()
        graphs["layout"].replay()
        evk[i][1].record()
        graphs["dispatch"].replay()
        evk[i][2].record()
        graphs["combine"].replay()
        evk[i][3].record()
    torch.cuda.synchronize()
    barrier()
    t_layout = statistics.mean(e[0].elapsed_time(e[1]) for e in evk)
    t_dispatch = statistics.mean(e[1].elapsed_time(e[2]) for e in evk)
    t_combine = statistics.mean(e[2].elapsed_time(e[3]) for e in evk)
    st = capi.moe_get_error(lay.struct)
    if st != capi.MOE_OK:
        raise SystemExit(f"device error in the timed region: {capi.moe_status_string(st)}")

    disp_b, comb_b = algorithmic_bytes(wl)
    step_bytes = disp_b + comb_b
    ms_per_step = total_ms / K
    value = step_bytes * world * K / (total_ms * 1e-3) / 1e9
    peak, peak_src = measured_peak()
    dom = "dispatch" if t_dispatch >= t_combine else "combine"
    dom_bytes = disp_b if dom == "dispatch" else comb_b
    dom_ms = t_dispatch if dom == "dispatch" else t_combine
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9

    # end to end through the C ABI from pinned host buffers
    e2e_steps = args.e2e_steps or min(K, 50)
    x_h = torch.from_numpy(d["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    topk_h = torch.from_numpy(d["topk_idx"]).pin_memory()
    w_h = torch.from_numpy(d["topk_w"]).pin_memory()
    y_h = torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory()
    h2d = x_h.numel() * 2 + topk_h.numel() * 4 + w_h.numel() * 4
    d2h = y_h.numel() * 2
    torch.cuda.synchronize()
    barrier()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        x_dev.copy_(x_h, non_blocking=True)
        topk_dev.copy_(topk_h, non_blocking=True)
        w_dev.copy_(w_h, non_blocking=True)
        do_layout()
        do_dispatch()
        capi.moe_combine(cfg, lay.struct, recv, w_dev, y)   # identity expert
        y_h.copy_(y, non_blocking=True)
        torch.cuda.current_stream().synchronize()
    e2e_s = time.perf_counter() - t0
    if world > 1:
        t = torch.tensor([e2e_s], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_s = float(t.item())
    e2e_value = step_bytes * world * e2e_steps / e2e_s / 1e9

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        one = oracle_step_time(d, wl.T, 1, eo_bits)
        reps = max(1, min(30, int(args.cpu_seconds / max(one, 1e-3))))
        best = min(one, oracle_step_time(d, wl.T, reps, eo_bits))
        cpu = {"value": round(step_bytes / best / 1e9, 3), "unit": "GB/s", "cores": 1,
               "kind": "oracle",
               "sample": f"full workload ({wl.T} tokens: layout+dispatch+combine), best of "
                         f"{reps + 1} runs, single thread on {os.cpu_count()} host cores"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_desc(wl), parallelism=f"replicas x{world}" if world > 1 else "single GPU",
                           l2="flushed before every timed step (read of a 2xL2 buffer, outside the events)",
                           engine=args.engine, timing="CUDA graph per step, CUDA events"),
            "pct_of_peak": round(100 * value / world / peak, 2),
            "peak_gbs": peak, "peak_source": peak_src,
            "pct_of_nominal_8tbs": round(100 * value / world / NOMINAL_HBM_GBS, 2),
            "tokens_per_s": round(wl.T * world * K / (total_ms * 1e-3), 1),
            "dispatch_combine_only_gbs": round(step_bytes / ((t_dispatch + t_combine) * 1e-3) / 1e9, 2),
            "kernels_ms": {"layout": round(t_layout, 5), "dispatch": round(t_dispatch, 5),
                           "combine": round(t_combine, 5)},
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 2),
                         "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": profiled_traffic(dom, wl.name),
                         "peak_kind": f"{peak_src} copy bandwidth (burst: kernel timed alone)"},
            "clocks": clocks.summary(),
            "e2e": {"value": round(e2e_value, 3), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": launches_per_step * K,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    for g in graphs.values():
        del g
    graphs.clear()
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
