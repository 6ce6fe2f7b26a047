"""Seeded synthetic inputs for MoE dispatch / combine.

This module only draws inputs: token activations ``x`` and a router's top-k
choice ``topk_idx`` with gate weights ``topk_w``.  It holds none of the
dispatch, layout or combine arithmetic, and both the CUDA path and the oracle
take their inputs from it.

The workload shapes follow the models the pages name (OLMoE, Qwen3-235B,
DeepSeek-V3) and the non-divisible expert-parallel case of TensorRT-LLM PR
#13888 ("support non-divisible EP in MoE alltoall and slurm benchmark").  The
router is simulated on the host: logits are drawn, biased per workload,
passed through a softmax, the k largest are kept (ties go to the lower expert
index) in descending order, and the weights are optionally renormalised to
sum to one.  The hot path never sees logits.
"""
from __future__ import annotations

import dataclasses
import functools

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int           # tokens
    H: int           # hidden size (bf16 elements per row)
    E: int           # experts
    k: int           # experts per token
    R: int           # virtual expert-parallel ranks
    N: int           # virtual nodes (R/N ranks each)
    seed: int
    renorm: bool     # renormalise the kept softmax weights to sum 1
    zipf_s: float = 0.0      # per-expert bias coef*ln((e+1)^-s); 0 = none
    zipf_coef: float = 1.0
    home_frac: float = 0.0   # target share of a token's k experts on one node
    two_level: bool = False  # the workload is timed with node staging

    @property
    def recv_rows(self) -> int:
        return self.T * self.k


# The five workloads.  Seeds are 1234 + position.
WORKLOADS = {
    "tiny": Workload("tiny", T=256, H=128, E=8, k=2, R=2, N=1, seed=1234,
                     renorm=True),
    "olmoe": Workload("olmoe", T=4096, H=2048, E=64, k=8, R=4, N=1, seed=1235,
                      renorm=False),
    "qwen3": Workload("qwen3", T=8192, H=4096, E=128, k=8, R=8, N=1, seed=1236,
                      renorm=True, zipf_s=1.2, zipf_coef=2.0),
    "dsv3": Workload("dsv3", T=16384, H=7168, E=256, k=8, R=8, N=2, seed=1237,
                     renorm=True, home_frac=0.80, two_level=True),
    "longctx": Workload("longctx", T=65536, H=2048, E=60, k=4, R=7, N=1,
                        seed=1238, renorm=True, zipf_s=1.0, zipf_coef=1.0),
}

DESCRIPTIONS = {
    "tiny": "T=256 H=128 E=8 k=2 R=2, N(0,1) router, renormalised",
    "olmoe": "OLMoE-shaped: T=4096 H=2048 E=64 k=8 R=4, uniform N(0,1) router, softmax weights",
    "qwen3": "Qwen3-235B-shaped: T=8192 H=4096 E=128 k=8 R=8, Zipf(1.2) expert bias",
    "dsv3": "DeepSeek-V3-shaped: T=16384 H=7168 E=256 k=8 R=8 N=2, ~80% home-node routing, two-level",
    "longctx": "long-context non-divisible EP: T=65536 H=2048 E=60 k=4 R=7, Zipf(1.0) bias",
}


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _streams(seed: int):
    """Two independent PCG64 streams from one seed: activations, router."""
    xs, rs = np.random.SeedSequence(seed).spawn(2)
    return (np.random.Generator(np.random.PCG64(xs)),
            np.random.Generator(np.random.PCG64(rs)))


def _topk_desc(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest per row, descending, ties to the lower index."""
    order = np.argsort(-logits, axis=1, kind="stable")
    return np.ascontiguousarray(order[:, :k]).astype(np.int32)


def _softmax(logits: np.ndarray) -> np.ndarray:
    z = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(z)
    return p / p.sum(axis=1, keepdims=True)


def _home_fraction(logits: np.ndarray, home_mask: np.ndarray, k: int) -> float:
    part = np.argpartition(-logits, k - 1, axis=1)[:, :k]
    return float(np.take_along_axis(home_mask, part, axis=1).mean())


@functools.lru_cache(maxsize=None)
def home_bias(name: str) -> float:
    """Logit bias on each token's home node, found by bisection on the fixed
    seed so the mean share of its top-k experts on that node is home_frac."""
    wl = WORKLOADS[name]
    _, rng = _streams(wl.seed)
    logits = rng.standard_normal((wl.T, wl.E))
    home = rng.integers(0, wl.N, size=wl.T)
    per_node = wl.E // wl.N
    home_mask = (np.arange(wl.E)[None, :] // per_node) == home[:, None]
    lo, hi = 0.0, 8.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if _home_fraction(logits + mid * home_mask, home_mask, wl.k) < wl.home_frac:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def router_logits(wl: Workload, rng: np.random.Generator):
    logits = rng.standard_normal((wl.T, wl.E))
    extra = {}
    if wl.zipf_s:
        w = (np.arange(wl.E) + 1.0) ** (-wl.zipf_s)
        logits = logits + wl.zipf_coef * np.log(w)[None, :]
    if wl.home_frac:
        home = rng.integers(0, wl.N, size=wl.T)
        per_node = wl.E // wl.N
        home_mask = (np.arange(wl.E)[None, :] // per_node) == home[:, None]
        b = home_bias(wl.name)
        logits = logits + b * home_mask
        extra["home_bias"] = b
        extra["home_node"] = home
    return logits, extra


def route(logits: np.ndarray, k: int, renorm: bool):
    idx = _topk_desc(logits, k)
    p = _softmax(logits)
    w = np.take_along_axis(p, idx, axis=1)
    if renorm:
        w = w / w.sum(axis=1, keepdims=True)
    return idx, np.ascontiguousarray(w, dtype=np.float32)


def x_bf16_bits(x_f32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns by round-to-nearest-even, using torch's CPU
    conversion (input preparation only)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x_f32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


@functools.lru_cache(maxsize=8)
def make(name: str) -> dict:
    """Inputs of a named workload: x (uint16 bf16 bits [T,H]), topk_idx
    (int32 [T,k]), topk_w (float32 [T,k]) and routing metadata."""
    return _generate(WORKLOADS[name])


def make_source(name: str, source: int) -> dict:
    """Inputs of source rank `source` of a named workload when every rank
    routes a batch of its own (same shape and routing recipe, the seed moved
    by 1000 per rank; rank 0 gets the workload's own inputs)."""
    if source == 0:
        return make(name)
    return _generate(dataclasses.replace(WORKLOADS[name], seed=WORKLOADS[name].seed + 1000 * source))


def prefix(d: dict, tokens: int) -> dict:
    """The first `tokens` tokens of a workload's inputs (same rows, same
    routes and weights) as a scaled-down case of the same shape; the
    workload record's T becomes `tokens`."""
    wl = d["workload"]
    tokens = max(1, min(int(tokens), wl.T))
    out = dict(d)
    out["workload"] = dataclasses.replace(wl, T=tokens)
    for key in ("x", "topk_idx", "topk_w"):
        out[key] = np.ascontiguousarray(d[key][:tokens])
    if "home_node" in d:
        out["home_node"] = d["home_node"][:tokens]
    return out


def _generate(wl: Workload) -> dict:
    xrng, rrng = _streams(wl.seed)
    x = xrng.standard_normal((wl.T, wl.H), dtype=np.float32)
    logits, extra = router_logits(wl, rrng)
    idx, w = route(logits, wl.k, wl.renorm)
    out = {"workload": wl, "x": x_bf16_bits(x), "topk_idx": idx, "topk_w": w}
    out.update(extra)
    return out


def make_random(T: int, H: int, E: int, k: int, seed: int, renorm: bool = True,
                zipf_s: float = 0.0) -> dict:
    """Small random case (parity sweeps): N(0,1) x, N(0,1) logits with an
    optional Zipf bias."""
    xrng, rng = _streams(seed)
    x = xrng.standard_normal((T, H), dtype=np.float32)
    logits = rng.standard_normal((T, E))
    if zipf_s:
        logits = logits + np.log((np.arange(E) + 1.0) ** (-zipf_s))[None, :]
    idx, w = route(logits, k, renorm)
    return {"x": x_bf16_bits(x), "topk_idx": idx, "topk_w": w}


def make_node_skewed(T: int, H: int, E: int, k: int, N: int, hot_frac: float, seed: int) -> dict:
    """Routing with one hot node: each token, with probability hot_frac,
    sends all k choices to the first E//N experts (which sit on node 0 under
    a contiguous expert partition); the others route uniformly.  Node 0 then
    stages far more rows than the rest (the load imbalance a load-aware
    forwarder is meant to absorb)."""
    xrng, rng = _streams(seed)
    x = xrng.standard_normal((T, H), dtype=np.float32)
    logits = rng.standard_normal((T, E))
    hot = rng.random(T) < hot_frac
    logits[np.ix_(hot, np.arange(E) < E // N)] += 50.0
    idx, w = route(logits, k, True)
    return {"x": x_bf16_bits(x), "topk_idx": idx, "topk_w": w}


def random_bf16(shape, seed: int, scale: float = 1.0) -> np.ndarray:
    """N(0, scale^2) values as bf16 bit patterns (e.g. stand-in expert outputs)."""
    rng = _rng(seed)
    return x_bf16_bits(scale * rng.standard_normal(shape, dtype=np.float32))


def random_bf16_bits(shape, seed: int) -> np.ndarray:
    """Fast stand-in expert outputs: bf16 bit patterns with a random sign, a
    biased exponent in [120, 130] (magnitudes 2^-7 .. 2^4) and a uniform
    7-bit mantissa.  16-bit integer draws only, so multi-GB buffers are
    cheap."""
    rng = _rng(seed)
    r = rng.integers(0, 1 << 16, size=int(np.prod(shape)), dtype=np.uint16)
    out = (r & np.uint16(1)) << np.uint16(15)
    out |= (np.uint16(120) + (r >> np.uint16(1)) % np.uint16(11)) << np.uint16(7)
    out |= (r >> np.uint16(8)) & np.uint16(0x7F)
    return out.reshape(shape)
