"""Benchmark: MoE dispatch + combine fused with layout on B200.

One step = the whole hot path over one batch: layout (histogram, scan, slot
assignment), fused dispatch (two-level through node staging for the
DeepSeek-V3-shaped workload, flat for the others) and fused combine.  The
combine reads a separate stand-in expert-output buffer (as it would after the
expert GEMMs), so no step reads rows the same step just wrote through L2.

One GPU (the default): the headline is the DeepSeek-V3-shaped workload
(T=16384 H=7168 E=256 k=8, R=8 ranks on N=2 nodes, two-level dispatch), the
largest of the five.  `per_workload` holds the same measurement of the other
four workloads, timed in the same process under the same protocol.

Timing: W untimed warm-up steps, then exactly K timed steps back to back,
bracketed by two CUDA events on the launching stream (and a barrier plus a
device synchronise on both sides).  Steps alternate between two independent
buffer sets (inputs, layout, outputs), so no step finds its inputs in L2: a
buffer is touched again only after about twice the step's traffic.  Steps
are replayed from CUDA graphs of GRAPH_STEPS (10) steps.  Stage costs come
from the same protocol applied to graphs of layout only and layout +
dispatch: dispatch = (layout + dispatch) - layout, combine = step - (layout
+ dispatch).  The decoupled pack -> copy -> unpack path is timed the same
way for comparison.

Several GPUs (torchrun, one rank per GPU): the headline is expert
parallelism over sharded sources across the processes.  Every rank routes a
batch of its own; the per-expert counts are all-gathered (NCCL); the
dispatch and combine kernels store to and load from every rank's receive and
expert-output buffers through CUDA IPC mappings; an NCCL all-reduce of one
word separates dispatch, the experts' slot and combine, as a barrier would.
value = bytes all ranks moved / the max over ranks of the timed time.  The
single-GPU step run on every rank at once (no collective on the data path)
is kept as `replicas`.

Metric: achieved algorithmic HBM GB/s of dispatch + combine.  Algorithmic
bytes per step are T*H*2 + T*k*H*2 for dispatch (read each token row once,
write each destination row once) and the same for combine (read each expert
row once, write each output row once); layout metadata and node staging
traffic are not credited.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload dsv3]
                    [--tokens T] [--impl reference] [--engine auto|vector|bulk]
"""
from __future__ import annotations

import argparse
import dataclasses
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
DEFAULT_WORKLOAD = "dsv3"
WORKLOAD_ORDER = ("tiny", "olmoe", "qwen3", "dsv3", "longctx")


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# Steps per CUDA graph replay in the timed loops.
GRAPH_STEPS = 10
# Fewest timed steps of each per-workload entry.
PER_WORKLOAD_MIN_STEPS = 100

KERNEL_SOURCES = {
    "combine": ["combine.cu", "moe_common.cuh"],
    "dispatch": ["bulk.cu", "dispatch.cu", "moe_common.cuh"],
    "layout_dispatch": ["fused.cu", "layout_common.cuh", "moe_common.cuh"],
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


def roofline_entry(kernel, achieved, peak, peak_src, ms, traffic):
    """The line's roofline object: algorithmic bytes per launch over the
    kernel's measured time against the measured copy peak; with the
    kernel's DRAM traffic per launch (ncu) known, also that traffic over the
    same time (what the kernel really moves, e.g. a two-level dispatch's
    staging writes, which the algorithmic bytes do not credit)."""
    out = {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 2), "peak": peak,
           "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
           "peak_kind": f"{peak_src} copy bandwidth"}
    if traffic:
        moved = traffic / (ms * 1e-3) / 1e9
        out["traffic_gbs"] = round(moved, 2)
        out["traffic_frac"] = round(moved / peak, 4)
    return out


def max_over_ranks(value, world, device):
    """The largest value over all ranks (each rank passes its own)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(bytes_per_step, world, steps, seconds):
    """Whole-job throughput: every rank moved bytes_per_step per step, and the
    job took the slowest rank's time."""
    return bytes_per_step * world * steps / seconds / 1e9


def algorithmic_bytes(wl, tokens=None):
    T = wl.T if tokens is None else tokens
    row = wl.H * 2
    dispatch = T * row + T * wl.k * row
    combine = T * wl.k * row + T * row
    return dispatch, combine


# One hot node: DeepSeek-V3-shaped rows (H=7168, E=256, k=8, R=8) over
# N=2 nodes, 90% of the tokens routing all k choices to node 0.
NODE_SKEW = dict(T=16384, H=7168, E=256, k=8, R=8, N=2, hot_frac=0.9, seed=1240)


def workload_inputs(name, tokens=0, source=0):
    d = inputs.make_source(name, source)
    return inputs.prefix(d, tokens) if tokens else d


def workload_desc(wl):
    full = inputs.WORKLOADS[wl.name].T
    name = wl.name if wl.T == full else f"{wl.name} (first {wl.T} of {full} tokens)"
    return {
        "workload": f"{name}: {inputs.DESCRIPTIONS[wl.name]}",
        "tokens": wl.T, "hidden": wl.H, "experts": wl.E, "top_k": wl.k,
        "virtual_ranks": wl.R, "virtual_nodes": wl.N,
        "dispatch_mode": "two-level node staging" if wl.two_level else "flat",
    }


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every 5 ms
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
            self._stop.wait(0.005)

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

def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform's."""
    import platform
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or platform.machine()


def oracle_step_time(d, tokens, reps, eo_bits, parallel=False):
    """Time the oracle (plain C loops, one thread) on the first `tokens`
    tokens of the workload: layout, dispatch, combine.  Best of `reps`.
    parallel: dispatch and combine through the oracle's OpenMP variants
    (token loops over all host threads; the layout stays serial)."""
    import oracle
    wl = d["workload"]
    topk = np.ascontiguousarray(d["topk_idx"][:tokens])
    x = np.ascontiguousarray(d["x"][:tokens])
    w = np.ascontiguousarray(d["topk_w"][:tokens])
    eo = np.ascontiguousarray(eo_bits[: tokens * wl.k])
    two = oracle.dispatch_two_level_par if parallel else oracle.dispatch_two_level
    flat = oracle.dispatch_flat_par if parallel else oracle.dispatch_flat
    comb = oracle.combine_par if parallel else oracle.combine
    best = float("inf")
    for _ in range(reps):
        t0 = time.perf_counter()
        lay = oracle.layout(topk, wl.E, wl.R, wl.N, nodes=wl.two_level)
        if wl.two_level:
            two(x, lay, wl.R, wl.N)
        else:
            flat(x, lay["slot"])
        comb(eo, w, lay["slot"])
        best = min(best, time.perf_counter() - t0)
    return best


# Bytes of dispatch + combine per reference-arm step: the sample is the first
# tokens of the workload whose step moves about this many bytes.
REF_SAMPLE_BYTES = 128 << 20


def reference_tokens(wl, requested=0):
    if requested:
        return max(1, min(wl.T, requested))
    per_token = sum(algorithmic_bytes(wl, 1))
    return max(1, min(wl.T, REF_SAMPLE_BYTES // per_token))


def run_reference(args):
    """The comparison arm: the oracle, as it stands, on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    d = workload_inputs(args.workload, args.tokens)
    wl = d["workload"]
    tokens = reference_tokens(wl, args.ref_tokens)
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


# ---------------------------------------------------------------- HBM probe

def hbm_probe():
    """Write-only (fill), read-only (sum) and copy bandwidth of 2 GiB bf16
    buffers with torch's own kernels: the ceilings a write-heavy dispatch and
    a read-heavy combine are bound by.  Best of 10, CUDA events."""
    import torch
    n = 1 << 30
    a = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    b = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    a.fill_(1.0)

    def best(fn, bytes_moved):
        for _ in range(3):
            fn()
        times = []
        for _ in range(10):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            fn()
            e.record()
            torch.cuda.synchronize()
            times.append(s.elapsed_time(e) * 1e-3)
        return round(bytes_moved / min(times) / 1e9, 1)

    out = {"probe": "hbm", "bytes": 2 * n,
           "write_only_gbs": best(lambda: b.fill_(2.0), 2 * n),
           "read_only_gbs": best(lambda: a.sum(dtype=torch.float32), 2 * n),
           "copy_gbs": best(lambda: b.copy_(a), 4 * n)}
    print(json.dumps(out), flush=True)
    return 0


# ---------------------------------------------------------------- our arm

@dataclasses.dataclass
class Ctx:
    world: int
    rank: int
    local: int
    dev: object

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()


def engine_flags(args):
    from combine_moe_layout_06_b200 import capi
    return {"auto": 0, "vector": capi.MOE_FLAG_COPY_VECTOR,
            "bulk": capi.MOE_FLAG_COPY_BULK}[args.engine]


def node_balance(args, ctx):
    """Two-level dispatch on a hot-node routing (NODE_SKEW), with the second
    phase walking (node, token) pairs (no node_src) and staging rows
    (node_src given).  Same protocol as the main step: two buffer sets,
    graphs of two steps, K steps between two events; dispatch = (layout +
    dispatch) - layout."""
    import torch

    from combine_moe_layout_06_b200 import buffers, capi
    dev, world = ctx.dev, ctx.world
    sk = NODE_SKEW
    T, H, E, k, R, N = (sk[c] for c in ("T", "H", "E", "k", "R", "N"))
    d = inputs.make_node_skewed(T, H, E, k, N, sk["hot_frac"], sk["seed"])
    # the expansion kernel is what is compared, so the split form
    cfg = capi.config(T, H, E, k, R, N, capi.MOE_FLAG_TWO_LEVEL | capi.MOE_FLAG_TWO_LEVEL_SPLIT |
                      engine_flags(args))
    bf16 = dict(dtype=torch.bfloat16, device=dev)
    rows = capi.moe_node_staging_rows(cfg)

    class Set:
        def __init__(self):
            self.x = buffers.bf16_from_bits(d["x"], dev)
            self.topk = torch.from_numpy(d["topk_idx"]).to(dev)
            self.recv = torch.empty((T * k, H), **bf16)
            self.staging = torch.empty((rows, H), **bf16)
            self.lay = {v: buffers.DeviceLayout(cfg, dev, node_src=v) for v in (False, True)}

    sets = [Set(), Set()]

    def ld(b, v):
        capi.moe_layout_dispatch(cfg, b.topk, b.lay[v].struct, b.x, b.recv, b.staging)

    def lo(b, v):
        capi.moe_layout(cfg, b.topk, b.lay[v].struct)

    for i in range(args.warmup):
        for v in (False, True):
            ld(sets[i % 2], v)
    torch.cuda.synchronize()
    side = torch.cuda.Stream(dev)
    A, B = sets
    graphs = {}
    for v in (False, True):
        for name, fn in (("LD", ld), ("L", lo)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side, capture_error_mode="thread_local"):
                fn(A, v)
                fn(B, v)
            graphs[(name, v)] = g
    for g in graphs.values():
        g.replay()
    torch.cuda.synchronize()
    K2 = max(args.steps // 2, 1)

    def timed(key):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ctx.barrier()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(K2):
            graphs[key].replay()
        e1.record()
        torch.cuda.synchronize()
        ctx.barrier()
        return max_over_ranks(e0.elapsed_time(e1), world, dev) / (2 * K2)

    out = {}
    disp_b = T * H * 2 + T * k * H * 2
    for v, name in ((False, "pairs"), (True, "rows")):
        t_ld, t_l = timed(("LD", v)), timed(("L", v))
        ms = t_ld - t_l
        out[name] = {"dispatch_ms": round(ms, 5), "layout_ms": round(t_l, 5),
                     "dispatch_gbs": round(disp_b * world / (ms * 1e-3) / 1e9, 2)}
    for b in sets:
        for v in (False, True):
            st = capi.moe_get_error(b.lay[v].struct)
            if st != capi.MOE_OK:
                raise SystemExit(f"device error in the node-balance run: {capi.moe_status_string(st)}")
    counts = sets[0].lay[True].node_counts.cpu().tolist()
    graphs.clear()
    return {"workload": f"DeepSeek-V3-shaped rows T={T} H={H} E={E} k={k} R={R} N={N}, "
                        f"{int(sk['hot_frac'] * 100)}% of tokens send all k choices to node 0",
            "node_counts": counts,
            "pairs": out["pairs"], "rows": out["rows"],
            "rows_speedup": round(out["pairs"]["dispatch_ms"] / out["rows"]["dispatch_ms"], 3),
            "path": "two-level dispatch (node pack + node expansion); pairs: the expansion "
                    "walks (node, token) pairs, rows: it walks staging rows (node_src)",
            "bytes_per_step": disp_b}


class StepBench:
    """One workload's step over two independent buffer sets: the buffers,
    the CUDA graphs of the step and of its stage prefixes, and the timed
    loops.  `extras` adds the comparison paths: "decoupled" (pack / copy /
    unpack), "agrs" (all-gather / reduce-scatter), "fp8" (e4m3 payload) and
    "ep" (sharded sources, the workload's R ranks on this GPU)."""

    def __init__(self, ctx, args, d, extras=()):
        import torch

        from combine_moe_layout_06_b200 import buffers, capi
        self.ctx, self.args, self.d = ctx, args, d
        wl = self.wl = d["workload"]
        dev = ctx.dev
        flags = capi.MOE_FLAG_TWO_LEVEL if wl.two_level else 0
        flags |= engine_flags(args)
        if args.layout == "cluster":
            flags |= capi.MOE_FLAG_LAYOUT_CLUSTER
        if args.layout == "fused":
            flags |= capi.MOE_FLAG_LAYOUT_FUSED
        if args.two_level_split:
            flags |= capi.MOE_FLAG_TWO_LEVEL_SPLIT
        self.flags = flags
        cfg = self.cfg = capi.config(wl.T, wl.H, wl.E, wl.k, wl.R, wl.N, flags)
        # the decoupled comparison path packs per rank: one "node" per rank
        copy_bits = flags & (capi.MOE_FLAG_COPY_VECTOR | capi.MOE_FLAG_COPY_BULK)
        dcfg = self.dcfg = capi.config(wl.T, wl.H, wl.E, wl.k, wl.R, wl.R,
                                       capi.MOE_FLAG_TWO_LEVEL | copy_bits)
        eo_bits = self.eo_bits = inputs.random_bf16_bits((wl.T * wl.k, wl.H), seed=wl.seed + 7)
        bf16 = dict(dtype=torch.bfloat16, device=dev)
        self.with_decoupled = "decoupled" in extras
        self.with_agrs = "agrs" in extras and wl.R <= capi.MOE_MAX_NODES
        self.with_fp8 = "fp8" in extras and wl.H % 8 == 0
        # sharded sources are flat (one NVSwitch domain), also for a two-level workload
        self.with_ep = "ep" in extras and wl.R <= capi.MOE_MAX_NODES

        # Expert parallelism over sharded sources with every rank on this
        # GPU: rank g routes tokens [sb[g], sb[g+1]); its receive and
        # expert-output buffers are the rank's rows of the set's recv / eo
        # (pointer tables).  The per-expert counts of each shard come from
        # the library's own layout, the rows per rank from its C ABI.
        G = self.G = wl.R
        sb = self.sb = (np.arange(G + 1, dtype=np.int64) * wl.T) // G
        if self.with_ep:
            ep_cfgs = self.ep_cfgs = [capi.config(int(sb[g + 1] - sb[g]), wl.H, wl.E, wl.k, wl.R, 1,
                                                  copy_bits) for g in range(G)]
            topk_all = torch.from_numpy(d["topk_idx"]).to(dev)
            counts = []
            for g in range(G):
                lay = buffers.DeviceLayout(ep_cfgs[g], dev)
                capi.moe_layout(ep_cfgs[g], topk_all[int(sb[g]):int(sb[g + 1])], lay.struct)
                counts.append(lay.expert_counts.cpu().numpy())
            ep_rows = self.ep_rows = np.array(capi.moe_ep_receive_rows(np.stack(counts), wl.R))
            ep_first = np.concatenate([[0], np.cumsum(ep_rows)])
            del topk_all

        outer = self

        class EpShards:
            """Per-rank layouts and sharded-source arrays of one buffer set."""

            def __init__(self, b):
                i32 = dict(dtype=torch.int32, device=dev)
                self.lays = [buffers.DeviceLayout(c, dev) for c in outer.ep_cfgs]
                self.counts_all = torch.zeros((G, wl.E), **i32)
                self.arrays = [(torch.zeros(wl.E + 1, **i32), torch.zeros(wl.R + 1, **i32),
                                torch.zeros(max(c.num_tokens * wl.k, 1), **i32))
                               for c in outer.ep_cfgs]
                self.structs = [capi.ep_layout_struct(*a) for a in self.arrays]
                row = wl.H * 2
                self.recv_bufs = [b.recv.data_ptr() + int(ep_first[r]) * row for r in range(wl.R)]
                self.eo_bufs = [b.eo.data_ptr() + int(ep_first[r]) * row for r in range(wl.R)]
                self.cap = int(ep_rows.max())

        class BufferSet:
            """One independent set of the step's inputs and outputs (the
            comparison paths' buffers are added by extras(), once both sets'
            step buffers exist)."""

            def __init__(self):
                self.lay = buffers.DeviceLayout(cfg, dev)
                self.x = buffers.bf16_from_bits(d["x"], dev)
                self.topk = torch.from_numpy(d["topk_idx"]).to(dev)
                self.w = torch.from_numpy(d["topk_w"]).to(dev)
                self.eo = buffers.bf16_from_bits(eo_bits, dev)
                self.recv = torch.empty((wl.T * wl.k, wl.H), **bf16)
                self.y = torch.empty((wl.T, wl.H), **bf16)
                self.staging = None
                if wl.two_level:
                    self.staging = torch.empty((capi.moe_node_staging_rows(cfg), wl.H), **bf16)

            def extras(self):
                if outer.with_decoupled:
                    self.dlay = buffers.DeviceLayout(dcfg, dev)
                    rows = capi.moe_node_staging_rows(dcfg)
                    self.dsend = torch.empty((rows, wl.H), **bf16)
                    self.dxfer = torch.empty((rows, wl.H), **bf16)
                    self.csend = torch.empty((wl.T * wl.k, wl.H), **bf16)
                    self.cxfer = torch.empty((wl.T * wl.k, wl.H), **bf16)
                if outer.with_fp8:
                    rows = wl.T * wl.k
                    self.recv_q = torch.empty((rows, wl.H), dtype=torch.uint8, device=dev)
                    self.recv_s = torch.empty(rows, dtype=torch.float32, device=dev)
                    self.eo_q = torch.empty((rows, wl.H), dtype=torch.uint8, device=dev)
                    self.eo_s = torch.empty(rows, dtype=torch.float32, device=dev)
                    # expert outputs as an fp8 producer would emit them
                    capi.moe_quantize_rows_fp8(self.eo, rows, wl.H, self.eo_q, self.eo_s)
                    if wl.two_level:
                        srows = capi.moe_node_staging_rows(cfg)
                        self.st_q = torch.empty((srows, wl.H), dtype=torch.uint8, device=dev)
                        self.st_s = torch.empty(srows, dtype=torch.float32, device=dev)
                if outer.with_agrs:
                    self.gathered = torch.empty((wl.R * wl.T, wl.H), **bf16)
                    self.partial = torch.empty((wl.R * wl.T, wl.H), dtype=torch.float32, device=dev)
                self.ep = EpShards(self) if outer.with_ep else None

        self.sets = [BufferSet(), BufferSet()]
        for b in self.sets:
            b.extras()
        self.ep_streams = [torch.cuda.Stream(dev) for _ in range(G)] if self.with_ep else []

        # one cluster launch when asked for, and always for one chunk of 256 tokens
        self.cluster_layout = (args.layout == "cluster" and wl.T <= 131072) or wl.T <= 256
        self.small_layout = wl.T <= 256 * 256      # count + assign (scan folded in)
        layout_launches = 1 if self.cluster_layout else (2 if self.small_layout else 3)
        # moe_layout_dispatch as the count + assign/dispatch pair (the
        # library's rule: flat, 16-byte rows, at most 256 experts, no engine
        # or layout override)
        self.ld_pair = (not args.unfused and not wl.two_level and args.layout == "fused"
                        and (wl.H * 2) % 16 == 0 and wl.E <= 256)
        # two-level: one kernel (16-byte rows, N + k <= 32), else or with
        # --two-level-split a pack kernel then an expansion kernel
        self.two_kernels = wl.two_level and (args.two_level_split or args.engine == "vector"
                                             or (wl.H * 2) % 16 or wl.N + wl.k > 32)
        self.launches_per_step = (2 if self.ld_pair else
                                  layout_launches + (2 if self.two_kernels else 1)) + 1
        self.graphs = {}

    # ---- the step and its parts
    def layout(self, b):
        from combine_moe_layout_06_b200 import capi
        capi.moe_layout(self.cfg, b.topk, b.lay.struct)

    def layout_dispatch(self, b):
        from combine_moe_layout_06_b200 import capi
        if self.args.unfused:
            self.layout(b)
            capi.moe_dispatch(self.cfg, b.lay.struct, b.x, b.recv, b.staging)
        else:
            capi.moe_layout_dispatch(self.cfg, b.topk, b.lay.struct, b.x, b.recv, b.staging)

    def step(self, b):
        from combine_moe_layout_06_b200 import capi
        self.layout_dispatch(b)
        capi.moe_combine(self.cfg, b.lay.struct, b.eo, b.w, b.y)

    def combine(self, b):
        from combine_moe_layout_06_b200 import capi
        capi.moe_combine(self.cfg, b.lay.struct, b.eo, b.w, b.y)

    def decoupled_step(self, b):
        from combine_moe_layout_06_b200 import capi
        capi.moe_layout(self.dcfg, b.topk, b.dlay.struct)
        capi.moe_dispatch_decoupled(self.dcfg, b.dlay.struct, b.x, b.dsend, b.dxfer, b.recv)
        capi.moe_combine_decoupled(self.dcfg, b.dlay.struct, b.eo, b.w, b.csend, b.cxfer, b.y)

    def fp8_layout_dispatch(self, b):
        from combine_moe_layout_06_b200 import capi
        self.layout(b)
        if self.wl.two_level:
            capi.moe_dispatch_fp8_two_level(self.cfg, b.lay.struct, b.x, b.st_q, b.st_s,
                                            b.recv_q, b.recv_s)
        else:
            capi.moe_dispatch_fp8(self.cfg, b.lay.struct, b.x, b.recv_q, b.recv_s)

    def fp8_step(self, b):
        from combine_moe_layout_06_b200 import capi
        self.fp8_layout_dispatch(b)
        capi.moe_combine_fp8(self.cfg, b.lay.struct, b.eo_q, b.eo_s, b.w, b.y)

    def ep_phase(self, fn):
        """Run fn(g) for every rank on its own stream, all after the work
        enqueued so far and before anything enqueued later (the ranks of a
        multi-GPU system run concurrently; the joins stand for its barriers)."""
        import torch
        cur = torch.cuda.current_stream()
        for st in self.ep_streams:
            st.wait_stream(cur)
        for g, st in enumerate(self.ep_streams):
            with torch.cuda.stream(st):
                fn(g)
        for st in self.ep_streams:
            cur.wait_stream(st)

    def ep_step(self, b):
        from combine_moe_layout_06_b200 import capi
        e, sb, G, cfgs = b.ep, self.sb, self.G, self.ep_cfgs

        def sh(t, g):
            return t[int(sb[g]):int(sb[g + 1])]

        def local(g):
            capi.moe_layout(cfgs[g], sh(b.topk, g), e.lays[g].struct)
            e.counts_all[g].copy_(e.lays[g].expert_counts)   # the count all-gather

        def send(g):
            capi.moe_ep_layout(cfgs[g], g, G, sh(b.topk, g), e.counts_all, e.lays[g].struct,
                               e.structs[g])
            capi.moe_ep_dispatch(cfgs[g], e.lays[g].struct, e.structs[g], sh(b.x, g),
                                 e.recv_bufs, e.cap)

        def gather(g):
            capi.moe_ep_combine(cfgs[g], e.lays[g].struct, e.structs[g], e.eo_bufs, e.cap,
                                sh(b.w, g), sh(b.y, g))

        self.ep_phase(local)
        self.ep_phase(send)
        self.ep_phase(gather)

    def agrs_step(self, b):
        from combine_moe_layout_06_b200 import capi
        self.layout(b)
        capi.moe_dispatch_allgather(self.cfg, b.lay.struct, b.x, b.gathered, b.recv)
        capi.moe_combine_reducescatter(self.cfg, b.lay.struct, b.eo, b.w, b.partial, b.y)

    # ---- running and timing
    def layouts(self):
        for b in self.sets:
            yield b.lay
            if self.with_decoupled:
                yield b.dlay
            if self.with_ep:
                yield from b.ep.lays

    def check_errors(self, where):
        from combine_moe_layout_06_b200 import capi
        for lay in self.layouts():
            st = capi.moe_get_error(lay.struct)
            if st != capi.MOE_OK:
                raise SystemExit(f"device error {where} ({self.wl.name}): {capi.moe_status_string(st)}")

    def prepare(self, warmup):
        """Warm-up steps of every path, then the CUDA graphs: GRAPH_STEPS steps
        alternating the two sets, a pair and a single step for the remainder
        of K, for the step and its stage prefixes.  Programmatic dependent
        launch overlaps consecutive kernels inside a graph but not across two
        replays, so longer graphs measure the steady state a model-level graph
        sees (one replay boundary costs about 2 us)."""
        import torch
        paths = [self.step]
        if self.with_decoupled:
            paths.append(self.decoupled_step)
        if self.with_agrs:
            paths.append(self.agrs_step)
        if self.with_fp8:
            paths.append(self.fp8_step)
        if self.with_ep:
            paths.append(self.ep_step)
        for i in range(warmup):
            for fn in paths:
                fn(self.sets[i % 2])
        torch.cuda.synchronize()
        self.check_errors("after warm-up")
        side = torch.cuda.Stream(self.ctx.dev)

        def capture(fn, n):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side, capture_error_mode="thread_local"):
                for i in range(n):
                    fn(self.sets[i % 2])
            return g

        def graph_set(fn):
            return capture(fn, GRAPH_STEPS), capture(fn, 2), capture(fn, 1)

        self.graphs = {"step": graph_set(self.step), "L": graph_set(self.layout),
                       "LD": graph_set(self.layout_dispatch), "C": graph_set(self.combine)}
        if self.with_decoupled:
            self.graphs["decoupled"] = graph_set(self.decoupled_step)
        if self.with_agrs:
            self.graphs["agrs"] = graph_set(self.agrs_step)
        if self.with_fp8:
            self.graphs["fp8"] = graph_set(self.fp8_step)
            self.graphs["fp8_LD"] = graph_set(self.fp8_layout_dispatch)
        if self.with_ep:
            self.graphs["ep"] = graph_set(self.ep_step)
        for gs in self.graphs.values():
            for g in gs:
                g.replay()
        torch.cuda.synchronize()

    def timed(self, name, K):
        """K steps back to back between two events on the stream (ms, max
        over ranks)."""
        import torch
        multi, pair, single = self.graphs[name]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        self.ctx.barrier()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(K // GRAPH_STEPS):
            multi.replay()
        rest = K % GRAPH_STEPS
        for _ in range(rest // 2):
            pair.replay()
        if rest % 2:
            single.replay()
        e1.record()
        torch.cuda.synchronize()
        self.ctx.barrier()
        return max_over_ranks(e0.elapsed_time(e1), self.ctx.world, self.ctx.dev)

    def flushed_steps(self, K):
        """One step at a time after writing a scratch buffer of twice the L2
        outside the timed region (the cold variant of the back-to-back
        measurement); per-step times, median and mean."""
        import torch
        dev, world = self.ctx.dev, self.ctx.world
        scratch = torch.empty(2 * torch.cuda.get_device_properties(dev).L2_cache_size // 4,
                              dtype=torch.float32, device=dev)
        single = self.graphs["step"][2]
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        self.ctx.barrier()
        torch.cuda.synchronize()
        for e0, e1 in evs:
            scratch.fill_(1.0)
            e0.record()
            single.replay()
            e1.record()
        torch.cuda.synchronize()
        self.ctx.barrier()
        ts = sorted(e0.elapsed_time(e1) for e0, e1 in evs)
        return {"median_ms": round(max_over_ranks(statistics.median(ts), world, dev), 5),
                "mean_ms": round(max_over_ranks(statistics.fmean(ts), world, dev), 5),
                "steps": K, "flush_bytes": scratch.numel() * 4}

    def measure(self, K, flushed=True):
        """Every timed loop of this workload, under one clock sampler."""
        raw = {}
        with ClockSampler(self.ctx.local) as clocks:
            raw["step"] = self.timed("step", K)
            raw["L"] = self.timed("L", K) / K
            raw["LD"] = self.timed("LD", K) / K
            raw["C"] = self.timed("C", K) / K
            for name in ("decoupled", "agrs", "fp8", "ep"):
                if name in self.graphs:
                    raw[name] = self.timed(name, K)
            if "fp8_LD" in self.graphs:
                raw["fp8_LD"] = self.timed("fp8_LD", K) / K
            if flushed:
                raw["flushed"] = self.flushed_steps(K)
        raw["clocks"] = clocks.summary()
        self.check_errors("in the timed region")
        return raw

    def report(self, raw, K):
        """The line's entries for this workload (headline or per-workload)."""
        import torch
        wl, world = self.wl, self.ctx.world
        total_ms = raw["step"]
        ms_per_step = total_ms / K
        t_l, t_ld = raw["L"], raw["LD"]
        # Stage costs by subtraction.  With the count + assign/dispatch pair
        # the assignment runs inside the dispatch kernel: the pair's whole
        # cost counts as dispatch (the layout alone, moe_layout's kernels, is
        # reported beside it).
        if self.ld_pair:
            t_layout, t_dispatch, t_combine = 0.0, t_ld, ms_per_step - t_ld
        else:
            t_layout, t_dispatch, t_combine = t_l, t_ld - t_l, ms_per_step - t_ld
        disp_b, comb_b = algorithmic_bytes(wl)
        step_bytes = disp_b + comb_b
        value = job_gbs(step_bytes, world, K, total_ms * 1e-3)
        peak, peak_src = measured_peak()
        dom = "dispatch" if t_dispatch >= t_combine else "combine"
        dom_kernel = "layout_dispatch" if dom == "dispatch" and self.ld_pair else dom
        dom_bytes = disp_b if dom == "dispatch" else comb_b
        dom_ms = t_dispatch if dom == "dispatch" else t_combine
        achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
        l2 = torch.cuda.get_device_properties(self.ctx.dev).L2_cache_size
        out = {
            "value": round(value, 2), "unit": "GB/s", "ms_per_step": round(ms_per_step, 5),
            "config": dict(
                workload_desc(wl),
                l2=("inputs larger than L2: steps alternate between two independent buffer "
                    "sets, each step moves %.1f MB (%.2fx L2)" % (step_bytes / 1e6, step_bytes / l2)),
                engine=self.args.engine,
                layout=("count kernel + assign/dispatch kernel" if self.ld_pair
                        else "one cluster launch" if self.cluster_layout else
                        ("count + assign kernels" if self.small_layout else "count/scan/assign kernels")),
                two_level_dispatch=(None if not wl.two_level else
                                    "node pack + node expansion" if self.two_kernels else
                                    "one kernel (staging rows read back from L2)"),
                entry="moe_layout + moe_dispatch" if self.args.unfused else "moe_layout_dispatch",
                timing=f"K steps back to back (CUDA graphs of {GRAPH_STEPS} steps) between two CUDA "
                       "events on the launching stream; stage costs from graphs of layout, "
                       "layout+dispatch and the full step"),
            "pct_of_peak": round(100 * value / world / peak, 2),
            "peak_gbs": peak, "peak_source": peak_src,
            "pct_of_nominal_8tbs": round(100 * value / world / NOMINAL_HBM_GBS, 2),
            "tokens_per_s": round(wl.T * world * K / (total_ms * 1e-3), 1),
            "tokens_per_s_dispatch_combine": round(wl.T * world / ((t_dispatch + t_combine) * 1e-3), 1),
            "dispatch_combine_only_gbs": round(step_bytes / ((t_dispatch + t_combine) * 1e-3) / 1e9, 2),
            "kernels_ms": ({"layout_dispatch": round(t_dispatch, 5), "combine": round(t_combine, 5),
                            "layout_kernels_alone": round(t_l, 5)} if self.ld_pair else
                           {"layout": round(t_layout, 5), "dispatch": round(t_dispatch, 5),
                            "combine": round(t_combine, 5),
                            # combines alone, back to back (layouts from the warm-up)
                            "combine_alone": round(raw["C"], 5)}),
            "roofline": roofline_entry(dom_kernel, achieved, peak, peak_src, dom_ms,
                                       profiled_traffic(dom_kernel, wl.name if wl.T == inputs.WORKLOADS[wl.name].T
                                                        else "none")),
            "clocks": raw["clocks"],
            "step_bytes": step_bytes,
        }
        if "flushed" in raw:
            out["flushed_step"] = raw["flushed"]
        if "decoupled" in raw:
            dec_value = job_gbs(step_bytes, world, K, raw["decoupled"] * 1e-3)
            out["decoupled_3pass"] = {
                "value": round(dec_value, 2), "unit": "GB/s",
                "ms_per_step": round(raw["decoupled"] / K, 5),
                "fused_speedup": round(value / dec_value, 3),
                "path": "layout (per-rank groups) + pack/copy/unpack dispatch + pack/copy/unpack combine"}
        if "agrs" in raw:
            ag_value = job_gbs(step_bytes, world, K, raw["agrs"] * 1e-3)
            out["allgather_reducescatter"] = {
                "value": round(ag_value, 2), "unit": "GB/s", "ms_per_step": round(raw["agrs"] / K, 5),
                "fused_speedup": round(value / ag_value, 3),
                "path": "layout + all-gather dispatch (R copies, per-rank select) + "
                        "reduce-scatter combine (per-rank fp32 partials, rank-order sum)"}
        if "fp8" in raw:
            fp8_ms = raw["fp8"]
            fp8_bytes = 2 * (wl.T * wl.H * 2 + wl.T * wl.k * (wl.H + 4))
            out["fp8_payload"] = {
                "value": round(job_gbs(fp8_bytes, world, K, fp8_ms * 1e-3), 2), "unit": "GB/s",
                "ms_per_step": round(fp8_ms / K, 5),
                "tokens_per_s": round(wl.T * world * K / (fp8_ms * 1e-3), 1),
                "speedup_vs_bf16_step": round(total_ms / fp8_ms, 3),
                "kernels_ms": {"dispatch": round(raw["fp8_LD"] - t_l, 5),
                               "combine": round(fp8_ms / K - raw["fp8_LD"], 5)},
                "bytes_per_step": fp8_bytes,
                "path": ("layout + fp8 two-level dispatch (each row quantized once, its codes and "
                         "scale staged once per node touched, read back from L2 and expanded to "
                         "the node's receive rows, one kernel; staging not credited) + "
                         if wl.two_level and not self.args.two_level_split else
                         "layout + fp8 two-level dispatch (quantize once into node staging, then "
                         "expand codes and scales; staging not credited) + " if wl.two_level else
                         "layout + fp8 dispatch (quantize once, k copies of e4m3 codes + scale) + ")
                        + "fp8 combine (expert rows already e4m3)"}
        if "ep" in raw:
            ep_value = job_gbs(step_bytes, world, K, raw["ep"] * 1e-3)
            out["expert_parallel_virtual_ranks"] = {
                "value": round(ep_value, 2), "unit": "GB/s", "ms_per_step": round(raw["ep"] / K, 5),
                "ranks": self.G, "vs_single_source": round(ep_value / value, 3),
                "receive_rows": [int(r) for r in self.ep_rows],
                "path": f"{self.G} source ranks on this GPU, one stream each, joined between "
                        "phases: layout of its shard and the count all-gather (device copies); "
                        "sharded-source layout and dispatch into every rank's receive buffer; "
                        "combine from every rank's expert outputs (pointer tables)"}
        return out

    def e2e(self, steps):
        """End to end through the C ABI from pinned host buffers, pipelined
        over the two buffer sets: step i's inputs go up on a copy stream
        while step i-1 computes, and step i's result comes down on another
        copy stream while step i+1 computes.  Every step still copies all its
        inputs in and its result out; the events only order each set's
        reuse.  Returns the entry of the line (wall clock, max over ranks)."""
        import torch

        from combine_moe_layout_06_b200 import capi
        d, wl, dev, world = self.d, self.wl, self.ctx.dev, self.ctx.world
        x_h = torch.from_numpy(d["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
        topk_h = torch.from_numpy(d["topk_idx"]).pin_memory()
        w_h = torch.from_numpy(d["topk_w"]).pin_memory()
        y_h = [torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory() for _ in self.sets]
        h2d = x_h.numel() * 2 + topk_h.numel() * 4 + w_h.numel() * 4
        d2h = y_h[0].numel() * 2
        s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        inputs_up = [torch.cuda.Event() for _ in self.sets]
        computed = [torch.cuda.Event() for _ in self.sets]
        result_down = [torch.cuda.Event() for _ in self.sets]

        def run(compute: bool) -> float:
            torch.cuda.synchronize()
            self.ctx.barrier()
            t0 = time.perf_counter()
            for i in range(steps):
                j = i % 2
                b = self.sets[j]
                if i >= 2:
                    s_in.wait_event(computed[j])        # step i-2 has read this set's inputs
                with torch.cuda.stream(s_in):
                    b.x.copy_(x_h, non_blocking=True)
                    b.topk.copy_(topk_h, non_blocking=True)
                    b.w.copy_(w_h, non_blocking=True)
                    inputs_up[j].record(s_in)
                s_comp.wait_event(inputs_up[j])
                if i >= 2:
                    s_comp.wait_event(result_down[j])   # step i-2's result has left this set's y
                with torch.cuda.stream(s_comp):
                    if compute:
                        capi.moe_layout_dispatch(self.cfg, b.topk, b.lay.struct, b.x, b.recv,
                                                 b.staging)
                        capi.moe_combine(self.cfg, b.lay.struct, b.recv, b.w, b.y)  # identity expert
                    computed[j].record(s_comp)
                s_out.wait_event(computed[j])
                with torch.cuda.stream(s_out):
                    y_h[j].copy_(b.y, non_blocking=True)
                    result_down[j].record(s_out)
            for s_ in (s_in, s_comp, s_out):
                s_.synchronize()
            return max_over_ranks(time.perf_counter() - t0, world, dev)

        copies_s = run(False)
        e2e_s = run(True)
        step_bytes = sum(algorithmic_bytes(wl))
        return {"value": round(job_gbs(step_bytes, world, steps, e2e_s), 3), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
                "copies_only_value": round(job_gbs(step_bytes, world, steps, copies_s), 3),
                "mode": "moe_layout_dispatch + moe_combine per step, host copies pipelined "
                        "on two copy streams over two buffer sets (wall clock)"}

    def release(self):
        import torch
        self.graphs.clear()
        self.sets = []
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def cpu_baselines(d, eo_bits, seconds):
    """The oracle as it stands on the host: single thread, then its OpenMP
    dispatch/combine variants on all host threads (full workload)."""
    import oracle
    wl = d["workload"]
    step_bytes = sum(algorithmic_bytes(wl))
    one = oracle_step_time(d, wl.T, 1, eo_bits)
    reps = max(1, min(30, int(seconds / max(one, 1e-3))))
    best = min(one, oracle_step_time(d, wl.T, reps, eo_bits))
    cpu = {"value": round(step_bytes / best / 1e9, 3), "unit": "GB/s", "cores": 1,
           "kind": "oracle",
           "sample": f"full workload ({wl.T} tokens: layout+dispatch+combine), best of "
                     f"{reps + 1} runs, single thread on {os.cpu_count()} host cores",
           "cpu_model": cpu_model()}
    threads = oracle.parallel_threads()
    one = oracle_step_time(d, wl.T, 1, eo_bits, parallel=True)
    reps = max(1, min(30, int(seconds / 2 / max(one, 1e-3))))
    best = min(one, oracle_step_time(d, wl.T, reps, eo_bits, parallel=True))
    cpu_par = {"value": round(step_bytes / best / 1e9, 3), "unit": "GB/s", "cores": threads,
               "kind": "oracle, dispatch and combine token loops over OpenMP threads "
                       "(layout serial)",
               "sample": f"full workload ({wl.T} tokens), best of {reps + 1} runs"}
    return cpu, cpu_par


# ---------------------------------------------------------------- several GPUs

def ep_plan(local_counts, num_ranks, group=None, out=None):
    """Host side of the sharded-source set-up on every rank: all-gather the
    per-expert counts (source-rank order), then the rows each expert rank
    receives (the library's moe_ep_receive_rows) and the buffer capacity
    every rank allocates (the largest).  Returns (counts_all, rows, cap)."""
    from combine_moe_layout_06_b200 import capi
    from combine_moe_layout_06_b200 import ep as epmod
    counts_all = epmod.gather_counts(local_counts, group, out=out)
    rows = capi.moe_ep_receive_rows(counts_all.cpu().numpy(), num_ranks)
    return counts_all, rows, max(max(rows), 1)


def ep_shuffle(args, ctx, d):
    """Expert parallelism over sharded sources across the processes (one
    rank per GPU, NCCL process group): see the module docstring."""
    import torch
    import torch.distributed as dist

    from combine_moe_layout_06_b200 import buffers, capi
    from combine_moe_layout_06_b200 import ep as epmod
    wl = d["workload"]
    G, g, dev = ctx.world, ctx.rank, ctx.dev
    cfg = capi.config(wl.T, wl.H, wl.E, wl.k, G, 1, engine_flags(args))
    me = epmod.ExpertParallelRank(cfg, g, G, dev)
    bf16 = dict(dtype=torch.bfloat16, device=dev)
    topk = torch.from_numpy(d["topk_idx"]).to(dev)
    x = buffers.bf16_from_bits(d["x"], dev)
    w = torch.from_numpy(d["topk_w"]).to(dev)
    y = torch.empty((wl.T, wl.H), **bf16)
    counts_all = torch.zeros((G, wl.E), dtype=torch.int32, device=dev)
    # set-up: one layout and count exchange sizes every rank's buffers
    capi.moe_layout(cfg, topk, me.local.struct)
    _, rows, cap = ep_plan(me.local.expert_counts, G, out=counts_all)
    recv = torch.empty((cap, wl.H), **bf16)
    eo = torch.empty((cap, wl.H), **bf16)
    recv_peers = epmod.share_buffer(recv)
    eo_peers = epmod.share_buffer(eo)
    recv_ptrs = [p for p, _ in recv_peers]
    eo_ptrs = [p for p, _ in eo_peers]
    fence_word = torch.zeros(1, dtype=torch.int32, device=dev)

    def fence():
        # every rank's work enqueued so far is complete before any rank's
        # later work starts (stream-ordered: an NCCL all-reduce of one word)
        dist.all_reduce(fence_word)

    def step(xb, topkb, wb, yb):
        capi.moe_layout(cfg, topkb, me.local.struct)
        epmod.gather_counts(me.local.expert_counts, out=counts_all)
        capi.moe_ep_layout(cfg, g, G, topkb, counts_all, me.local.struct, me.ep)
        capi.moe_ep_dispatch(cfg, me.local.struct, me.ep, xb, recv_ptrs, cap)
        fence()    # every row has landed: the experts would run here
        capi.moe_ep_combine(cfg, me.local.struct, me.ep, eo_ptrs, cap, wb, yb)
        fence()    # no rank's next dispatch overwrites rows a peer still reads

    # stand-in expert outputs: the received rows themselves (identity expert)
    step(x, topk, w, y)
    torch.cuda.synchronize()
    eo.copy_(recv)
    fence()
    for _ in range(args.warmup):
        step(x, topk, w, y)
    torch.cuda.synchronize()
    st = capi.moe_get_error(me.local.struct)
    if st != capi.MOE_OK:
        raise SystemExit(f"device error in the expert-parallel warm-up: {capi.moe_status_string(st)}")
    K = args.steps
    with ClockSampler(ctx.local) as clocks:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ctx.barrier()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(K):
            step(x, topk, w, y)
        e1.record()
        torch.cuda.synchronize()
        ctx.barrier()
        ms = max_over_ranks(e0.elapsed_time(e1), G, dev)
    st = capi.moe_get_error(me.local.struct)
    if st != capi.MOE_OK:
        raise SystemExit(f"device error in the expert-parallel run: {capi.moe_status_string(st)}")

    # end to end: this rank's inputs up from pinned host memory, the step,
    # its output down, every step (wall clock, max over ranks)
    steps_e2e = args.e2e_steps or min(K, 20)
    x_h = torch.from_numpy(d["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    topk_h = torch.from_numpy(d["topk_idx"]).pin_memory()
    w_h = torch.from_numpy(d["topk_w"]).pin_memory()
    y_h = torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory()
    x2, topk2, w2 = torch.empty_like(x), torch.empty_like(topk), torch.empty_like(w)
    torch.cuda.synchronize()
    ctx.barrier()
    t0 = time.perf_counter()
    for _ in range(steps_e2e):
        x2.copy_(x_h, non_blocking=True)
        topk2.copy_(topk_h, non_blocking=True)
        w2.copy_(w_h, non_blocking=True)
        step(x2, topk2, w2, y)
        y_h.copy_(y, non_blocking=True)
    torch.cuda.synchronize()
    e2e_s = max_over_ranks(time.perf_counter() - t0, G, dev)
    step_bytes = sum(algorithmic_bytes(wl))
    out = {
        "value": round(job_gbs(step_bytes, G, K, ms * 1e-3), 2), "ms_per_step": round(ms / K, 5),
        "receive_rows": [int(r) for r in rows], "capacity_rows": int(cap),
        "clocks": clocks.summary(),
        "e2e": {"value": round(job_gbs(step_bytes, G, steps_e2e, e2e_s), 3), "unit": "GB/s",
                "h2d_bytes_per_step": x_h.numel() * 2 + topk_h.numel() * 4 + w_h.numel() * 4,
                "d2h_bytes_per_step": y_h.numel() * 2, "steps": steps_e2e,
                "mode": "per rank: host copies of its inputs, the expert-parallel step, its "
                        "output back (wall clock, max over ranks)"},
        "launches_per_step": 5,
    }
    # unmap the peers' buffers only once no rank still writes to them
    torch.cuda.synchronize()
    ctx.barrier()
    del recv_peers, eo_peers, recv_ptrs, eo_ptrs
    torch.cuda.synchronize()
    torch.cuda.ipc_collect()
    ctx.barrier()
    return out


def run_several(args, ctx):
    import torch
    d = workload_inputs(args.workload, args.tokens, source=ctx.rank)
    wl = d["workload"]
    shuffle = ep_shuffle(args, ctx, d)
    torch.cuda.empty_cache()
    replicas = StepBench(ctx, args, d)
    replicas.prepare(args.warmup)
    rep = replicas.report(replicas.measure(args.steps, flushed=False), args.steps)
    replicas.release()
    if ctx.rank == 0:
        K = args.steps
        line = {
            "metric": METRIC, "value": shuffle["value"], "unit": "GB/s", "n_gpus": ctx.world,
            "steps": K, "warmup": args.warmup, "ms_per_step": shuffle["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_desc(wl),
                           dispatch_mode="flat, one expert rank per GPU (sharded sources)",
                           parallelism=f"expert parallelism over {ctx.world} processes, one rank "
                                       "per GPU, every rank routing a batch of its own",
                           l2="inputs larger than L2: each rank's step moves %.0f MB"
                              % (sum(algorithmic_bytes(wl)) / 1e6),
                           timing="K eager steps between two CUDA events on the launching stream, "
                                  "max over ranks"),
            "tokens_per_s": round(wl.T * ctx.world * K / (shuffle["ms_per_step"] * K * 1e-3), 1),
            "expert_parallel": {k: v for k, v in shuffle.items() if k not in ("e2e", "clocks")},
            "replicas": {k: rep[k] for k in ("value", "ms_per_step", "kernels_ms", "roofline",
                                             "pct_of_peak", "config")},
            "clocks": shuffle["clocks"],
            "e2e": shuffle["e2e"],
            "gpu_launches": shuffle["launches_per_step"] * K,
            "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- one GPU

def run_one(args, ctx):
    import torch
    d = workload_inputs(args.workload, args.tokens)
    wl = d["workload"]
    K = args.steps
    main = StepBench(ctx, args, d, extras=[e for e, off in (
        ("decoupled", args.no_decoupled), ("agrs", args.no_agrs), ("fp8", args.no_fp8),
        ("ep", args.no_ep)) if not off])
    main.prepare(args.warmup)
    head = main.report(main.measure(K), K)
    e2e = main.e2e(args.e2e_steps or min(K, 50))
    launches = main.launches_per_step * K
    eo_bits = main.eo_bits
    main.release()
    del main

    per = {}
    names = [] if args.no_per_workload else [n for n in (args.per_workload.split(",")
                                                         if args.per_workload else WORKLOAD_ORDER)
                                             if n and n != args.workload]
    # the other workloads are extra entries, timed over at least PER_WORKLOAD_MIN_STEPS
    # steps (the headline keeps exactly K): a few hundred microseconds of steps
    # would leave one disturbance too much weight
    K_pw = max(K, PER_WORKLOAD_MIN_STEPS)
    for name in names:
        pd = workload_inputs(name)
        sb = StepBench(ctx, args, pd, extras=[] if args.no_decoupled else ["decoupled"])
        sb.prepare(args.warmup)
        per[name] = sb.report(sb.measure(K_pw, flushed=False), K_pw)
        per[name]["steps"] = K_pw
        sb.release()
        del sb

    balance = None
    if not args.no_node_balance:
        with ClockSampler(ctx.local) as nb_clocks:
            balance = node_balance(args, ctx)
        balance["clocks"] = nb_clocks.summary()
        torch.cuda.empty_cache()

    cpu = cpu_par = None
    if ctx.rank == 0 and not args.no_cpu_baseline:
        cpu, cpu_par = cpu_baselines(d, eo_bits, args.cpu_seconds)

    line = {"metric": METRIC, "value": head["value"], "unit": "GB/s", "n_gpus": ctx.world,
            "steps": K, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic"}
    head["config"]["parallelism"] = "single GPU"
    for key, val in head.items():
        if key not in ("value", "unit", "ms_per_step"):
            line[key] = val
    line.update({
        "node_balance": balance,
        "e2e": e2e,
        "gpu_launches": launches,
        "cpu_baseline": cpu,
        "cpu_baseline_parallel": cpu_par,
        "per_workload": per or None,
    })
    print(json.dumps(line), flush=True)
    return 0


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(inputs.WORKLOADS))
    p.add_argument("--tokens", type=int, default=0,
                   help="time only the first T tokens of the workload (a scaled-down case of "
                        "the same shape and routing, e.g. for ncu captures)")
    p.add_argument("--per-workload", default="",
                   help="comma-separated workloads for per_workload (default: every other one)")
    p.add_argument("--no-per-workload", action="store_true")
    p.add_argument("--engine", default="auto", choices=["auto", "vector", "bulk"])
    p.add_argument("--layout", default="kernels", choices=["kernels", "fused", "cluster"],
                   help="kernels: layout kernels then the dispatch kernel; fused: a count kernel "
                        "then an assign/dispatch kernel (flat); cluster: one-cluster layout")
    p.add_argument("--two-level-split", action="store_true",
                   help="two-level dispatch as a pack kernel then an expansion kernel (default: "
                        "one kernel, staging rows read back from L2)")
    p.add_argument("--unfused", action="store_true",
                   help="moe_layout + moe_dispatch instead of moe_layout_dispatch")
    p.add_argument("--e2e-steps", type=int, default=0, help="end-to-end steps (0: min(K, 50))")
    p.add_argument("--no-decoupled", action="store_true",
                   help="skip timing the pack/copy/unpack comparison path")
    p.add_argument("--no-fp8", action="store_true",
                   help="skip timing the fp8 (e4m3) payload path")
    p.add_argument("--no-agrs", action="store_true",
                   help="skip timing the all-gather / reduce-scatter comparison path")
    p.add_argument("--no-node-balance", action="store_true",
                   help="skip timing the two node expansions on a hot-node routing")
    p.add_argument("--no-ep", action="store_true",
                   help="skip timing expert parallelism over sharded sources (virtual ranks)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--ref-tokens", type=int, default=0)
    p.add_argument("--hbm-probe", action="store_true",
                   help="measure write-only / read-only / copy HBM bandwidth and exit")
    p.add_argument("--ep-processes", action="store_true",
                   help="time the multi-process expert-parallel step even on one GPU (a process "
                        "group of one rank; torchrun with several GPUs always takes it)")
    args = p.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    return args


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.hbm_probe:
        return hbm_probe()

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    several = world > 1 or args.ep_processes
    if several:
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            if "MASTER_PORT" not in os.environ:
                import socket
                with socket.socket() as sk:
                    sk.bind(("127.0.0.1", 0))
                    os.environ["MASTER_PORT"] = str(sk.getsockname()[1])
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    ctx = Ctx(world, rank, local, dev)
    try:
        return run_several(args, ctx) if several else run_one(args, ctx)
    finally:
        if several:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
