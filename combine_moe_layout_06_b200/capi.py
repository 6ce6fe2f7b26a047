"""Python binding of libmoe_layout.so (include/moe_layout.h).

Argument marshalling only: every entry point forwards to the C function of
the same name, and all device work runs in the library's CUDA kernels.
Tensors (anything with ``data_ptr()``) or raw integer addresses may be passed
where the C ABI takes a pointer; ``stream`` may be a ``torch.cuda.Stream``,
a raw ``cudaStream_t`` integer, or ``None`` for torch's current stream.

If the shared library has not been built this module raises on first use;
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_LAYOUT_LIB names another build of the library (e.g. a test build with
# shortened device waits); the in-tree build is the default.
LIB_PATH = os.environ.get("MOE_LAYOUT_LIB") or os.path.join(_HERE, "libmoe_layout.so")

MOE_MAX_EXPERTS = 1024
MOE_MAX_TOPK = 32
MOE_MAX_NODES = 32

MOE_FLAG_TWO_LEVEL = 0x1
MOE_FLAG_COPY_VECTOR = 0x2
MOE_FLAG_COPY_BULK = 0x4
MOE_FLAG_LAYOUT_CLUSTER = 0x8
MOE_FLAG_LAYOUT_FUSED = 0x10
MOE_FLAG_TWO_LEVEL_FUSED = 0x20
MOE_FLAG_TWO_LEVEL_SPLIT = 0x40

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_EMPTY_RANK = 2
MOE_ERR_BAD_NODES = 3
MOE_ERR_EXPERT_OOB = 4
MOE_ERR_DUP_EXPERT = 5
MOE_ERR_TIMEOUT = 6
MOE_ERR_CUDA = 7
MOE_ERR_BAD_LAYOUT = 8

STATUS_NAMES = {
    MOE_OK: "OK", MOE_ERR_INVALID_ARG: "INVALID_ARG", MOE_ERR_EMPTY_RANK: "EMPTY_RANK",
    MOE_ERR_BAD_NODES: "BAD_NODES", MOE_ERR_EXPERT_OOB: "EXPERT_OOB",
    MOE_ERR_DUP_EXPERT: "DUP_EXPERT", MOE_ERR_TIMEOUT: "TIMEOUT", MOE_ERR_CUDA: "CUDA",
    MOE_ERR_BAD_LAYOUT: "BAD_LAYOUT",
}

# Every entry point the header declares.
ENTRY_POINTS = (
    "moe_status_string", "moe_check_config", "moe_expert_partition",
    "moe_layout_workspace_bytes", "moe_node_staging_rows", "moe_layout", "moe_dispatch",
    "moe_combine", "moe_get_error", "moe_dispatch_decoupled", "moe_combine_decoupled",
    "moe_layout_noalloc", "moe_layout_dispatch", "moe_dispatch_allgather",
    "moe_combine_reducescatter", "moe_quantize_rows_fp8", "moe_dispatch_fp8", "moe_combine_fp8",
    "moe_ep_layout", "moe_ep_dispatch", "moe_ep_combine", "moe_dispatch_fp8_two_level",
    "moe_ep_receive_rows", "moe_enable_peer_access",
)

MOE_LAYOUT_NOALLOC_SCRATCH_BYTES = 4 << 20


class MoeConfig(ctypes.Structure):
    _fields_ = [("num_tokens", ctypes.c_int64), ("hidden", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("num_ranks", ctypes.c_int32), ("num_nodes", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


class MoeLayout(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in (
        "expert_counts", "expert_offsets", "rank_offsets", "slot", "node_counts",
        "node_offsets", "node_slot", "error_word", "workspace", "node_src")]


class MoeEpLayout(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in ("expert_offsets", "rank_offsets", "slot")]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{where}: {moe_status_string(status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library.  Raises if it was never built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m combine_moe_layout_06_b200.build` "
            "(there is no fallback implementation)")
    L = ctypes.CDLL(LIB_PATH)
    P, C, S = ctypes.c_void_p, ctypes.POINTER(MoeConfig), ctypes.c_int
    L.moe_status_string.argtypes = [S]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_check_config.argtypes = [C]
    L.moe_expert_partition.argtypes = [ctypes.c_int32, ctypes.c_int32, P]
    L.moe_layout_workspace_bytes.argtypes = [C, ctypes.POINTER(ctypes.c_size_t)]
    L.moe_node_staging_rows.argtypes = [C, ctypes.POINTER(ctypes.c_int64)]
    LP = ctypes.POINTER(MoeLayout)
    L.moe_layout.argtypes = [C, P, LP, P]
    L.moe_dispatch.argtypes = [C, LP, P, P, P, P]
    L.moe_combine.argtypes = [C, LP, P, P, P, P]
    L.moe_get_error.argtypes = [LP, P]
    L.moe_dispatch_decoupled.argtypes = [C, LP, P, P, P, P, P]
    L.moe_combine_decoupled.argtypes = [C, LP, P, P, P, P, P, P]
    L.moe_layout_noalloc.argtypes = [C, P, LP, P]
    L.moe_layout_dispatch.argtypes = [C, P, LP, P, P, P, P]
    L.moe_dispatch_allgather.argtypes = [C, LP, P, P, P, P]
    L.moe_combine_reducescatter.argtypes = [C, LP, P, P, P, P, P]
    L.moe_quantize_rows_fp8.argtypes = [P, ctypes.c_int64, ctypes.c_int32, P, P, P]
    L.moe_dispatch_fp8.argtypes = [C, LP, P, P, P, P]
    L.moe_combine_fp8.argtypes = [C, LP, P, P, P, P, P]
    L.moe_dispatch_fp8_two_level.argtypes = [C, LP, P, P, P, P, P, P]
    EP = ctypes.POINTER(MoeEpLayout)
    PP = ctypes.POINTER(ctypes.c_void_p)
    L.moe_ep_layout.argtypes = [C, ctypes.c_int32, ctypes.c_int32, P, P, LP, EP, P]
    L.moe_ep_dispatch.argtypes = [C, LP, EP, P, PP, ctypes.c_int64, P]
    L.moe_ep_combine.argtypes = [C, LP, EP, PP, ctypes.c_int64, P, P, P]
    L.moe_ep_receive_rows.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P]
    L.moe_enable_peer_access.argtypes = [ctypes.c_int32, ctypes.c_int32]
    for name in ENTRY_POINTS[1:]:
        getattr(L, name).restype = S
    _lib = L
    return L


def _ptr(x):
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return x.data_ptr() or None
    return int(x)


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream or None
    if hasattr(stream, "cuda_stream"):
        return stream.cuda_stream or None
    return int(stream) or None


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def config(T, H, E, k, R, N=1, flags=0) -> MoeConfig:
    return MoeConfig(int(T), int(H), int(E), int(k), int(R), int(N), int(flags))


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def moe_check_config(cfg: MoeConfig) -> int:
    return lib().moe_check_config(ctypes.byref(cfg))


def moe_expert_partition(num_experts: int, num_ranks: int) -> list:
    out = (ctypes.c_int32 * (max(num_ranks, 0) + 1))()
    _check(lib().moe_expert_partition(num_experts, num_ranks, out), "moe_expert_partition")
    return list(out)


def moe_layout_workspace_bytes(cfg: MoeConfig) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_layout_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)),
           "moe_layout_workspace_bytes")
    return n.value


def moe_node_staging_rows(cfg: MoeConfig) -> int:
    n = ctypes.c_int64(0)
    _check(lib().moe_node_staging_rows(ctypes.byref(cfg), ctypes.byref(n)), "moe_node_staging_rows")
    return n.value


def layout_struct(expert_counts, expert_offsets, rank_offsets, slot, error_word, workspace,
                  node_counts=None, node_offsets=None, node_slot=None,
                  node_src=None) -> MoeLayout:
    return MoeLayout(_ptr(expert_counts), _ptr(expert_offsets), _ptr(rank_offsets), _ptr(slot),
                     _ptr(node_counts), _ptr(node_offsets), _ptr(node_slot), _ptr(error_word),
                     _ptr(workspace), _ptr(node_src))


def moe_layout(cfg: MoeConfig, topk_idx, layout: MoeLayout, stream=None) -> None:
    _check(lib().moe_layout(ctypes.byref(cfg), _ptr(topk_idx), ctypes.byref(layout),
                            _stream(stream)), "moe_layout")


def moe_dispatch(cfg: MoeConfig, layout: MoeLayout, x, recv, node_staging=None,
                 stream=None) -> None:
    _check(lib().moe_dispatch(ctypes.byref(cfg), ctypes.byref(layout), _ptr(x), _ptr(recv),
                              _ptr(node_staging), _stream(stream)), "moe_dispatch")


def moe_layout_dispatch(cfg: MoeConfig, topk_idx, layout: MoeLayout, x, recv, node_staging=None,
                        stream=None) -> None:
    _check(lib().moe_layout_dispatch(ctypes.byref(cfg), _ptr(topk_idx), ctypes.byref(layout),
                                     _ptr(x), _ptr(recv), _ptr(node_staging), _stream(stream)),
           "moe_layout_dispatch")


def moe_combine(cfg: MoeConfig, layout: MoeLayout, expert_out, topk_weights, y,
                stream=None) -> None:
    _check(lib().moe_combine(ctypes.byref(cfg), ctypes.byref(layout), _ptr(expert_out),
                             _ptr(topk_weights), _ptr(y), _stream(stream)), "moe_combine")


def moe_get_error(layout: MoeLayout, stream=None) -> int:
    """Status recorded on the device since the last call (waits for stream)."""
    return lib().moe_get_error(ctypes.byref(layout), _stream(stream))


def moe_dispatch_decoupled(cfg: MoeConfig, layout: MoeLayout, x, send, xfer, recv,
                           stream=None) -> None:
    _check(lib().moe_dispatch_decoupled(ctypes.byref(cfg), ctypes.byref(layout), _ptr(x),
                                        _ptr(send), _ptr(xfer), _ptr(recv), _stream(stream)),
           "moe_dispatch_decoupled")


def moe_combine_decoupled(cfg: MoeConfig, layout: MoeLayout, expert_out, topk_weights, send,
                          xfer, y, stream=None) -> None:
    _check(lib().moe_combine_decoupled(ctypes.byref(cfg), ctypes.byref(layout), _ptr(expert_out),
                                       _ptr(topk_weights), _ptr(send), _ptr(xfer), _ptr(y),
                                       _stream(stream)), "moe_combine_decoupled")


def moe_layout_noalloc(cfg: MoeConfig, topk_idx, layout: MoeLayout, stream=None) -> None:
    """moe_layout() with the library's fixed device scratch instead of
    layout.workspace (for callers that cannot allocate device memory)."""
    _check(lib().moe_layout_noalloc(ctypes.byref(cfg), _ptr(topk_idx), ctypes.byref(layout),
                                    _stream(stream)), "moe_layout_noalloc")


def ep_layout_struct(expert_offsets, rank_offsets, slot) -> MoeEpLayout:
    return MoeEpLayout(_ptr(expert_offsets), _ptr(rank_offsets), _ptr(slot))


def _ptr_array(bufs):
    """Host array of device pointers (tensors or integers)."""
    return (ctypes.c_void_p * len(bufs))(*[_ptr(b) for b in bufs])


def moe_ep_layout(cfg: MoeConfig, source_rank: int, num_sources: int, topk_idx, counts_all,
                  local: MoeLayout, ep: MoeEpLayout, stream=None) -> None:
    _check(lib().moe_ep_layout(ctypes.byref(cfg), source_rank, num_sources, _ptr(topk_idx),
                               _ptr(counts_all), ctypes.byref(local), ctypes.byref(ep),
                               _stream(stream)), "moe_ep_layout")


def moe_ep_receive_rows(counts_all, num_ranks: int):
    """Rows each of `num_ranks` expert ranks receives, from every source's
    expert counts (host int32 [num_sources][num_experts]) -> list of int."""
    import numpy as np
    c = np.ascontiguousarray(np.asarray(counts_all), dtype=np.int32)
    if c.ndim != 2:
        raise ValueError("counts_all must be [num_sources][num_experts]")
    out = (ctypes.c_int64 * max(int(num_ranks), 1))()
    _check(lib().moe_ep_receive_rows(c.shape[1], int(num_ranks), c.shape[0],
                                     c.ctypes.data_as(ctypes.c_void_p), out),
           "moe_ep_receive_rows")
    return list(out)[: int(num_ranks)]


def moe_enable_peer_access(device: int, peer_device: int) -> None:
    """Let kernels on `device` reach memory on `peer_device` (host call)."""
    _check(lib().moe_enable_peer_access(int(device), int(peer_device)), "moe_enable_peer_access")


def moe_ep_dispatch(cfg: MoeConfig, local: MoeLayout, ep: MoeEpLayout, x, recv_bufs,
                    capacity_rows: int, stream=None) -> None:
    arr = _ptr_array(recv_bufs)
    _check(lib().moe_ep_dispatch(ctypes.byref(cfg), ctypes.byref(local), ctypes.byref(ep), _ptr(x),
                                 arr, capacity_rows, _stream(stream)), "moe_ep_dispatch")


def moe_ep_combine(cfg: MoeConfig, local: MoeLayout, ep: MoeEpLayout, expert_out_bufs,
                   capacity_rows: int, topk_weights, y, stream=None) -> None:
    arr = _ptr_array(expert_out_bufs)
    _check(lib().moe_ep_combine(ctypes.byref(cfg), ctypes.byref(local), ctypes.byref(ep), arr,
                                capacity_rows, _ptr(topk_weights), _ptr(y), _stream(stream)),
           "moe_ep_combine")


def moe_dispatch_allgather(cfg: MoeConfig, layout: MoeLayout, x, gathered, recv,
                           stream=None) -> None:
    _check(lib().moe_dispatch_allgather(ctypes.byref(cfg), ctypes.byref(layout), _ptr(x),
                                        _ptr(gathered), _ptr(recv), _stream(stream)),
           "moe_dispatch_allgather")


def moe_combine_reducescatter(cfg: MoeConfig, layout: MoeLayout, expert_out, topk_weights,
                              partial, y, stream=None) -> None:
    _check(lib().moe_combine_reducescatter(ctypes.byref(cfg), ctypes.byref(layout),
                                           _ptr(expert_out), _ptr(topk_weights), _ptr(partial),
                                           _ptr(y), _stream(stream)),
           "moe_combine_reducescatter")


def moe_quantize_rows_fp8(src, rows: int, hidden: int, q, scale, stream=None) -> None:
    """bf16 rows -> e4m3 codes (uint8) plus one fp32 scale per row."""
    _check(lib().moe_quantize_rows_fp8(_ptr(src), int(rows), int(hidden), _ptr(q), _ptr(scale),
                                       _stream(stream)), "moe_quantize_rows_fp8")


def moe_dispatch_fp8(cfg: MoeConfig, layout: MoeLayout, x, recv_q, recv_scale,
                     stream=None) -> None:
    _check(lib().moe_dispatch_fp8(ctypes.byref(cfg), ctypes.byref(layout), _ptr(x), _ptr(recv_q),
                                  _ptr(recv_scale), _stream(stream)), "moe_dispatch_fp8")


def moe_dispatch_fp8_two_level(cfg: MoeConfig, layout: MoeLayout, x, staging_q, staging_scale,
                               recv_q, recv_scale, stream=None) -> None:
    _check(lib().moe_dispatch_fp8_two_level(ctypes.byref(cfg), ctypes.byref(layout), _ptr(x),
                                            _ptr(staging_q), _ptr(staging_scale), _ptr(recv_q),
                                            _ptr(recv_scale), _stream(stream)),
           "moe_dispatch_fp8_two_level")


def moe_combine_fp8(cfg: MoeConfig, layout: MoeLayout, eo_q, eo_scale, topk_weights, y,
                    stream=None) -> None:
    _check(lib().moe_combine_fp8(ctypes.byref(cfg), ctypes.byref(layout), _ptr(eo_q),
                                 _ptr(eo_scale), _ptr(topk_weights), _ptr(y), _stream(stream)),
           "moe_combine_fp8")
