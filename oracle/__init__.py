"""Oracle for MoE dispatch / combine with layout: plain CPU loops in C.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA
library never loads it and shares no code with it.

``moe_oracle.c`` holds the arithmetic (each function cites the passage it
follows); this module compiles it with gcc on first use and marshals numpy
arrays through ctypes.  bf16 arrays are carried as ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

# Same meanings as the library's status codes; kept separate on purpose.
OK, INVALID_ARG, EMPTY_RANK, BAD_NODES, EXPERT_OOB, DUP_EXPERT = range(6)
STATUS_NAMES = {
    OK: "OK",
    INVALID_ARG: "INVALID_ARG",
    EMPTY_RANK: "EMPTY_RANK",
    BAD_NODES: "BAD_NODES",
    EXPERT_OOB: "EXPERT_OOB",
    DUP_EXPERT: "DUP_EXPERT",
}


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"oracle refused: {STATUS_NAMES.get(code, code)}")
        self.code = code
        self.name = STATUS_NAMES.get(code, str(code))


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so (gcc, no fused contraction)."""
    with _lock:
        fresh = os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)
        if fresh and not force:
            return _LIB
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
        return _LIB


def _load():
    """Bind the oracle library.  ``MOE_ORACLE_LIB`` names another build of it
    (the mutation tests use this to check that the pins catch planted
    mistakes)."""
    global _lib
    if _lib is None:
        _lib = _bind(os.environ.get("MOE_ORACLE_LIB") or build())
    return _lib


def _bind(path: str):
    lib = ctypes.CDLL(path)
    i32, i64, p = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
    lib.oracle_partition.argtypes = [i32, i32, p]
    lib.oracle_partition.restype = ctypes.c_int
    lib.oracle_validate_config.argtypes = [i64, i32, i32, i32, i32, i32]
    lib.oracle_validate_config.restype = ctypes.c_int
    lib.oracle_validate_topk.argtypes = [i64, i32, i32, p]
    lib.oracle_validate_topk.restype = ctypes.c_int
    lib.oracle_layout.argtypes = [i64, i32, i32, i32, i32, p, p, p, p, p, p, p, p]
    lib.oracle_layout.restype = ctypes.c_int
    lib.oracle_node_sources.argtypes = [i64, i32, p, p, p]
    lib.oracle_node_sources.restype = None
    lib.oracle_ep_layout.argtypes = [i64, i32, i32, i32, i32, p, p, p, p, p, p]
    lib.oracle_ep_layout.restype = ctypes.c_int
    lib.oracle_dispatch_flat.argtypes = [i64, i32, i32, p, p, p]
    lib.oracle_dispatch_flat.restype = None
    lib.oracle_dispatch_two_level.argtypes = [i64, i32, i32, i32, i32, p, p, p, p, p, p, p]
    lib.oracle_dispatch_two_level.restype = None
    lib.oracle_combine.argtypes = [i64, i32, i32, p, p, p, p]
    lib.oracle_combine.restype = None
    lib.oracle_parallel_threads.argtypes = []
    lib.oracle_parallel_threads.restype = ctypes.c_int
    lib.oracle_dispatch_flat_par.argtypes = [i64, i32, i32, p, p, p]
    lib.oracle_dispatch_flat_par.restype = None
    lib.oracle_dispatch_two_level_par.argtypes = [i64, i32, i32, i32, i32, p, p, p, p, p, p, p]
    lib.oracle_dispatch_two_level_par.restype = None
    lib.oracle_combine_par.argtypes = [i64, i32, i32, p, p, p, p]
    lib.oracle_combine_par.restype = None
    lib.oracle_combine_tokens.argtypes = [i64, p, i32, i32, p, p, p, p]
    lib.oracle_combine_tokens.restype = None
    lib.oracle_combine_rank_partials.argtypes = [i64, i32, i32, i32, p, p, p, p, p]
    lib.oracle_combine_rank_partials.restype = None
    lib.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_to_f32.restype = ctypes.c_float
    lib.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_e4m3.restype = ctypes.c_uint8
    lib.oracle_e4m3_to_f32_array.argtypes = [p, p, i64]
    lib.oracle_e4m3_to_f32_array.restype = None
    lib.oracle_f32_to_e4m3_array.argtypes = [p, p, i64]
    lib.oracle_f32_to_e4m3_array.restype = None
    lib.oracle_quantize_rows_fp8.argtypes = [i64, i32, p, p, p]
    lib.oracle_quantize_rows_fp8.restype = None
    lib.oracle_dispatch_fp8.argtypes = [i64, i32, i32, p, p, p, p]
    lib.oracle_dispatch_fp8.restype = None
    lib.oracle_combine_fp8.argtypes = [i64, i32, i32, p, p, p, p, p]
    lib.oracle_combine_fp8.restype = None
    lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
    lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_f32.restype = ctypes.c_float
    lib.oracle_f32_to_bf16_array.argtypes = [p, p, i64]
    lib.oracle_f32_to_bf16_array.restype = None
    lib.oracle_bf16_to_f32_array.argtypes = [p, p, i64]
    lib.oracle_bf16_to_f32_array.restype = None
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- bf16

def f32_to_bf16(a) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even."""
    a = _c(a, np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    _load().oracle_f32_to_bf16_array(_ptr(a), _ptr(out), a.size)
    return out


def bf16_to_f32(a) -> np.ndarray:
    a = _c(a, np.uint16)
    out = np.empty(a.shape, dtype=np.float32)
    _load().oracle_bf16_to_f32_array(_ptr(a), _ptr(out), a.size)
    return out


# ---------------------------------------------------------------- partition

def partition(E: int, R: int) -> np.ndarray:
    """First expert of each rank, int32 [R+1] (last entry = E)."""
    out = np.zeros(max(R, 0) + 1, dtype=np.int32)
    st = _load().oracle_partition(E, R, _ptr(out))
    if st != OK:
        raise OracleError(st)
    return out


def validate_config(T, H, E, k, R, N) -> int:
    return _load().oracle_validate_config(T, H, E, k, R, N)


def validate_topk(topk: np.ndarray, E: int) -> int:
    topk = _c(topk, np.int32)
    T, k = topk.shape
    return _load().oracle_validate_topk(T, k, E, _ptr(topk))


# ---------------------------------------------------------------- layout

def layout(topk: np.ndarray, E: int, R: int, N: int = 1, nodes: bool = False) -> dict:
    """Layout metadata.  ``nodes`` also computes the node staging map and its
    inverse ``node_src`` (staging row -> token)."""
    topk = _c(topk, np.int32)
    T, k = topk.shape
    out = {
        "expert_counts": np.zeros(E, np.int32),
        "expert_offsets": np.zeros(E + 1, np.int32),
        "rank_offsets": np.zeros(R + 1, np.int32),
        "slot": np.zeros((T, k), np.int32),
    }
    null = ctypes.c_void_p(0)
    if nodes:
        out["node_counts"] = np.zeros(N, np.int32)
        out["node_offsets"] = np.zeros(N + 1, np.int32)
        out["node_slot"] = np.zeros((T, N), np.int32)
        nc, no, ns = (_ptr(out["node_counts"]), _ptr(out["node_offsets"]),
                      _ptr(out["node_slot"]))
    else:
        nc = no = ns = null
    st = _load().oracle_layout(T, k, E, R, N, _ptr(topk),
                               _ptr(out["expert_counts"]), _ptr(out["expert_offsets"]),
                               _ptr(out["rank_offsets"]), _ptr(out["slot"]), nc, no, ns)
    if st != OK:
        raise OracleError(st)
    if nodes:
        out["node_src"] = np.zeros(int(out["node_offsets"][N]), np.int32)
        _load().oracle_node_sources(T, N, _ptr(out["node_offsets"]), _ptr(out["node_slot"]),
                                    _ptr(out["node_src"]))
    return out


def ep_layout(topk: np.ndarray, E: int, R: int, shard_begin) -> dict:
    """Layout with the tokens sharded over source ranks (shard g = tokens
    [shard_begin[g], shard_begin[g+1])): per-source counts [G, E], expert and
    rank offsets, and slot [T, k] as rows of the concatenated receive
    buffers."""
    topk = _c(topk, np.int32)
    T, k = topk.shape
    sb = _c(shard_begin, np.int64)
    G = sb.size - 1
    out = {
        "counts": np.zeros((G, E), np.int32),
        "expert_offsets": np.zeros(E + 1, np.int32),
        "rank_offsets": np.zeros(R + 1, np.int32),
        "slot": np.zeros((T, k), np.int32),
    }
    st = _load().oracle_ep_layout(T, k, E, R, G, _ptr(sb), _ptr(topk), _ptr(out["counts"]),
                                  _ptr(out["expert_offsets"]), _ptr(out["rank_offsets"]),
                                  _ptr(out["slot"]))
    if st != OK:
        raise OracleError(st)
    return out


# ---------------------------------------------------------------- dispatch

def dispatch_flat(x_bits: np.ndarray, slot: np.ndarray) -> np.ndarray:
    """x_bits uint16 [T, H]; returns recv uint16 [T*k, H]."""
    x_bits = _c(x_bits, np.uint16)
    slot = _c(slot, np.int32)
    T, H = x_bits.shape
    k = slot.shape[1]
    recv = np.zeros((T * k, H), np.uint16)
    _load().oracle_dispatch_flat(T, H, k, _ptr(slot), _ptr(x_bits), _ptr(recv))
    return recv


def dispatch_two_level(x_bits: np.ndarray, lay: dict, R: int, N: int):
    """Returns (staging uint16 [U, H], recv uint16 [T*k, H])."""
    x_bits = _c(x_bits, np.uint16)
    T, H = x_bits.shape
    slot = _c(lay["slot"], np.int32)
    k = slot.shape[1]
    U = int(lay["node_offsets"][N])
    staging = np.zeros((max(U, 1), H), np.uint16)
    recv = np.zeros((T * k, H), np.uint16)
    _load().oracle_dispatch_two_level(
        T, H, k, R, N, _ptr(slot), _ptr(_c(lay["rank_offsets"], np.int32)),
        _ptr(_c(lay["node_offsets"], np.int32)), _ptr(_c(lay["node_slot"], np.int32)),
        _ptr(x_bits), _ptr(staging), _ptr(recv))
    return staging[:U], recv


# ---------------------------------------------------------------- combine

def combine(eo_bits: np.ndarray, w: np.ndarray, slot: np.ndarray) -> np.ndarray:
    """eo_bits uint16 [T*k, H], w float32 [T, k]; returns y uint16 [T, H]."""
    eo_bits = _c(eo_bits, np.uint16)
    w = _c(w, np.float32)
    slot = _c(slot, np.int32)
    T, k = slot.shape
    H = eo_bits.shape[1]
    y = np.zeros((T, H), np.uint16)
    _load().oracle_combine(T, H, k, _ptr(slot), _ptr(w), _ptr(eo_bits), _ptr(y))
    return y


# ------------------------------------------- token loops over host threads
# The same results as dispatch_flat / dispatch_two_level / combine, with the
# token loops split over OpenMP threads (timing only; the layout stays serial).

def parallel_threads() -> int:
    """Threads the parallel variants use (OMP_NUM_THREADS, else all cores)."""
    return int(_load().oracle_parallel_threads())


def dispatch_flat_par(x_bits: np.ndarray, slot: np.ndarray) -> np.ndarray:
    x_bits = _c(x_bits, np.uint16)
    slot = _c(slot, np.int32)
    T, H = x_bits.shape
    k = slot.shape[1]
    recv = np.zeros((T * k, H), np.uint16)
    _load().oracle_dispatch_flat_par(T, H, k, _ptr(slot), _ptr(x_bits), _ptr(recv))
    return recv


def dispatch_two_level_par(x_bits: np.ndarray, lay: dict, R: int, N: int):
    x_bits = _c(x_bits, np.uint16)
    T, H = x_bits.shape
    slot = _c(lay["slot"], np.int32)
    k = slot.shape[1]
    U = int(lay["node_offsets"][N])
    staging = np.zeros((max(U, 1), H), np.uint16)
    recv = np.zeros((T * k, H), np.uint16)
    _load().oracle_dispatch_two_level_par(
        T, H, k, R, N, _ptr(slot), _ptr(_c(lay["rank_offsets"], np.int32)),
        _ptr(_c(lay["node_offsets"], np.int32)), _ptr(_c(lay["node_slot"], np.int32)),
        _ptr(x_bits), _ptr(staging), _ptr(recv))
    return staging[:U], recv


def combine_par(eo_bits: np.ndarray, w: np.ndarray, slot: np.ndarray) -> np.ndarray:
    eo_bits = _c(eo_bits, np.uint16)
    w = _c(w, np.float32)
    slot = _c(slot, np.int32)
    T, k = slot.shape
    H = eo_bits.shape[1]
    y = np.zeros((T, H), np.uint16)
    _load().oracle_combine_par(T, H, k, _ptr(slot), _ptr(w), _ptr(eo_bits), _ptr(y))
    return y


def combine_tokens(eo_bits: np.ndarray, w: np.ndarray, slot: np.ndarray,
                   tokens) -> np.ndarray:
    """Combine for the listed tokens only; returns uint16 [len(tokens), H]."""
    eo_bits = _c(eo_bits, np.uint16)
    w = _c(w, np.float32)
    slot = _c(slot, np.int32)
    tokens = _c(tokens, np.int64)
    k = slot.shape[1]
    H = eo_bits.shape[1]
    y = np.zeros((tokens.size, H), np.uint16)
    _load().oracle_combine_tokens(tokens.size, _ptr(tokens), H, k, _ptr(slot),
                                  _ptr(w), _ptr(eo_bits), _ptr(y))
    return y


def combine_rank_partials(eo_bits: np.ndarray, w: np.ndarray, slot: np.ndarray,
                          rank_offsets: np.ndarray) -> np.ndarray:
    """Combine in the reduce-scatter order: per-rank fp32 partial sums, added
    in rank order, one bf16 rounding."""
    eo_bits = _c(eo_bits, np.uint16)
    w = _c(w, np.float32)
    slot = _c(slot, np.int32)
    ro = _c(rank_offsets, np.int32)
    T, k = slot.shape
    H = eo_bits.shape[1]
    y = np.zeros((T, H), np.uint16)
    _load().oracle_combine_rank_partials(T, H, k, ro.size - 1, _ptr(slot), _ptr(ro), _ptr(w),
                                         _ptr(eo_bits), _ptr(y))
    return y


# ---------------------------------------------------------------- fp8 payload

def e4m3_to_f32(codes) -> np.ndarray:
    """Decode e4m3 codes (flat result)."""
    codes = _c(codes, np.uint8).ravel()
    out = np.empty(codes.size, np.float32)
    _load().oracle_e4m3_to_f32_array(_ptr(codes), _ptr(out), codes.size)
    return out


def f32_to_e4m3(vals) -> np.ndarray:
    """Encode to e4m3 codes (flat result)."""
    vals = _c(vals, np.float32).ravel()
    out = np.empty(vals.size, np.uint8)
    _load().oracle_f32_to_e4m3_array(_ptr(vals), _ptr(out), vals.size)
    return out


def quantize_rows_fp8(src_bits: np.ndarray):
    """bf16 rows -> (e4m3 codes uint8 [rows, H], fp32 scale [rows])."""
    src_bits = _c(src_bits, np.uint16)
    rows, H = src_bits.shape
    q = np.zeros((rows, H), np.uint8)
    scale = np.zeros(rows, np.float32)
    _load().oracle_quantize_rows_fp8(rows, H, _ptr(src_bits), _ptr(q), _ptr(scale))
    return q, scale


def dispatch_fp8(x_bits: np.ndarray, slot: np.ndarray):
    x_bits = _c(x_bits, np.uint16)
    slot = _c(slot, np.int32)
    T, H = x_bits.shape
    k = slot.shape[1]
    q = np.zeros((T * k, H), np.uint8)
    scale = np.zeros(T * k, np.float32)
    _load().oracle_dispatch_fp8(T, H, k, _ptr(slot), _ptr(x_bits), _ptr(q), _ptr(scale))
    return q, scale


def combine_fp8(eo_q: np.ndarray, eo_scale: np.ndarray, w: np.ndarray, slot: np.ndarray):
    eo_q = _c(eo_q, np.uint8)
    eo_scale = _c(eo_scale, np.float32)
    w = _c(w, np.float32)
    slot = _c(slot, np.int32)
    T, k = slot.shape
    H = eo_q.shape[1]
    y = np.zeros((T, H), np.uint16)
    _load().oracle_combine_fp8(T, H, k, _ptr(slot), _ptr(w), _ptr(eo_q), _ptr(eo_scale), _ptr(y))
    return y
