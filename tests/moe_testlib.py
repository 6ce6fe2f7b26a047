"""Helpers shared by the GPU parity tests: run the CUDA path through the C
ABI on seeded inputs and bring results back as numpy arrays."""
import numpy as np
import torch

from combine_moe_layout_06_b200 import build, buffers, capi  # noqa: F401  (buffers re-exported)

_built = False


def ensure_lib():
    global _built
    if not _built:
        assert torch.cuda.is_available(), "GPU tests need a CUDA device"
        build.build()
        capi.lib()
        _built = True


def cfg_of(T, H, E, k, R, N=1, flags=0):
    return capi.config(T, H, E, k, R, N, flags)


def gpu_layout(cfg, topk_np, node_src=True):
    """Run moe_layout; returns (DeviceLayout, device topk).  node_src=False
    leaves the staging-row map out (pair-walking node expansion)."""
    ensure_lib()
    lay = buffers.DeviceLayout(cfg, node_src=node_src)
    topk = torch.from_numpy(np.ascontiguousarray(topk_np, np.int32)).cuda()
    capi.moe_layout(cfg, topk, lay.struct)
    return lay, topk


def staging_buffer(cfg, fill=None):
    rows = capi.moe_node_staging_rows(cfg)
    buf = torch.empty((max(rows, 1), cfg.hidden), dtype=torch.bfloat16, device="cuda")
    if fill is not None:
        buf.view(torch.int16).fill_(fill)
    return buf


def gpu_dispatch(cfg, lay, x_dev, fill=None):
    recv = torch.empty((cfg.num_tokens * cfg.top_k, cfg.hidden), dtype=torch.bfloat16, device="cuda")
    if fill is not None:
        recv.view(torch.int16).fill_(fill)
    staging = staging_buffer(cfg, fill) if cfg.flags & capi.MOE_FLAG_TWO_LEVEL else None
    capi.moe_dispatch(cfg, lay.struct, x_dev, recv, staging)
    return recv, staging


def gpu_combine(cfg, lay, eo_dev, w_np):
    w = torch.from_numpy(np.ascontiguousarray(w_np, np.float32)).cuda()
    y = torch.empty((cfg.num_tokens, cfg.hidden), dtype=torch.bfloat16, device="cuda")
    capi.moe_combine(cfg, lay.struct, eo_dev, w, y)
    return y


def to_dev(bits):
    return buffers.bf16_from_bits(bits)


def bits(t):
    return buffers.bits_of(t)


def assert_layout_equal(got: dict, ref: dict):
    for key, want in ref.items():
        have = got[key]
        assert have.shape == np.asarray(want).shape, key
        if not np.array_equal(have, want):
            bad = np.argwhere(np.asarray(have) != np.asarray(want))[:5]
            raise AssertionError(f"{key} differs at {bad.tolist()}")


def bf16_bits_to_f64(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_combine_close(y_bits, ref_bits, rtol=1e-2, atol=1e-3):
    """The combine contract: within 1e-2 relative / 1e-3 absolute of the
    oracle in bf16."""
    y = bf16_bits_to_f64(y_bits)
    r = bf16_bits_to_f64(ref_bits)
    ok = np.abs(y - r) <= atol + rtol * np.abs(r)
    if not ok.all():
        i = np.argwhere(~ok)[:5]
        raise AssertionError(f"combine outside tolerance at {i.tolist()}")
