"""GPU parity of the fp8 (e4m3) payload against the oracle: codes and scales
bit for bit (quantization, fp8 dispatch) and fp8 combine bit for bit (same
FMA order).  Against the bf16 combine of the unquantized rows, the fp8
result stays within e4m3's quantization bound for any magnitudes, and for
unit-scale expert outputs within rtol 0.02 / atol 0.15, the tolerance
TensorRT-LLM PR #13888 validates its fp8 combine with."""
import numpy as np
import pytest
import torch

import moe_testlib as M
from combine_moe_layout_06_b200 import capi, inputs

pytestmark = pytest.mark.gpu

CASES = [
    # T, H, E, k, R
    (1, 8, 4, 1, 1),
    (33, 136, 13, 4, 5),
    (257, 72, 64, 8, 4),
    (300, 16, 32, 16, 8),      # k > 8, rows shorter than a warp's vectors
    (1000, 2048, 60, 4, 7),
    (64, 3088, 32, 6, 4),      # 193 16-value groups: a ragged last group per row
    (40, 4096, 16, 4, 2),      # 8 groups per lane, the most held in registers
    (24, 8208, 16, 4, 2),      # beyond the register-resident kernels
]


def _u8(t):
    return t.detach().cpu().contiguous().numpy().view(np.uint8)


def _assert_fp8_error_bound(y_bits, eo_bits, w, slot, scale_rows):
    """|fp8 combine - bf16 combine| within the e4m3 quantization bound: each
    term w_j x_j carries a relative error <= 2^-4 (3 mantissa bits, half an
    ulp) plus, below e4m3's normal range, an absolute error <= scale * 2^-10;
    both results carry a bf16 rounding (2^-8 relative) and fp32 sums."""
    y = M.bf16_bits_to_f64(y_bits)
    xf = M.bf16_bits_to_f64(eo_bits)
    wf = w.astype(np.float64)
    T, k = slot.shape
    terms = np.stack([wf[:, j:j + 1] * np.abs(xf[slot[:, j]]) for j in range(k)], -1)
    sub = np.stack([wf[:, j:j + 1] * scale_rows[slot[:, j]][:, None] for j in range(k)], -1)
    exact = np.stack([wf[:, j:j + 1] * xf[slot[:, j]] for j in range(k)], -1).sum(-1)
    bound = ((2.0 ** -4 + 2.0 ** -20) * terms.sum(-1) + 2.0 ** -10 * sub.sum(-1)
             + 2 * 2.0 ** -8 * (np.abs(exact) + 2.0 ** -4 * terms.sum(-1)) + 1e-30)
    ok = np.abs(y - exact) <= bound
    assert ok.all(), f"outside the e4m3 error bound at {np.argwhere(~ok)[:5].tolist()}"


def _run_fp8(cfg, lay, x_dev, eo_bits, w):
    T, H, k = cfg.num_tokens, cfg.hidden, cfg.top_k
    recv_q = torch.empty((T * k, H), dtype=torch.uint8, device="cuda")
    recv_s = torch.empty(T * k, dtype=torch.float32, device="cuda")
    capi.moe_dispatch_fp8(cfg, lay.struct, x_dev, recv_q, recv_s)
    eo_dev = M.to_dev(eo_bits)
    eo_q = torch.empty((T * k, H), dtype=torch.uint8, device="cuda")
    eo_s = torch.empty(T * k, dtype=torch.float32, device="cuda")
    capi.moe_quantize_rows_fp8(eo_dev, T * k, H, eo_q, eo_s)
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    capi.moe_combine_fp8(cfg, lay.struct, eo_q, eo_s, torch.from_numpy(w).cuda(), y)
    return recv_q, recv_s, eo_q, eo_s, y


@pytest.mark.parametrize("T,H,E,k,R", CASES)
def test_fp8_small(oracle_mod, T, H, E, k, R):
    d = inputs.make_random(T, H, E, k, seed=T + H + 5)
    x, topk, w = d["x"], d["topk_idx"], d["topk_w"]
    ref = oracle_mod.layout(topk, E, R)
    cfg = M.cfg_of(T, H, E, k, R)
    lay, _ = M.gpu_layout(cfg, topk)
    eo = inputs.random_bf16_bits((T * k, H), seed=3 * T + H)
    recv_q, recv_s, eo_q, eo_s, y = _run_fp8(cfg, lay, M.to_dev(x), eo, w)
    rq, rs = oracle_mod.dispatch_fp8(x, ref["slot"])
    assert np.array_equal(_u8(recv_q), rq)
    assert np.array_equal(recv_s.cpu().numpy(), rs)
    eq, es = oracle_mod.quantize_rows_fp8(eo)
    assert np.array_equal(_u8(eo_q), eq)
    assert np.array_equal(eo_s.cpu().numpy(), es)
    y_bits = M.bits(y)
    assert np.array_equal(y_bits, oracle_mod.combine_fp8(eq, es, w, ref["slot"]))
    _assert_fp8_error_bound(y_bits, eo, w, ref["slot"], es.astype(np.float64))
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK


def test_fp8_zero_and_extreme_rows(oracle_mod):
    T, H, E, k, R = 64, 32, 8, 2, 2
    d = inputs.make_random(T, H, E, k, seed=1)
    x = d["x"].copy()
    x[3] = 0                                     # zero row: scale 1, codes 0
    x[5, 7] = 0x7F7F                             # bf16 max: scale huge
    x[6] = 0x0001                                # a bf16 subnormal row
    x[8, 3] = 0x7FC0                             # NaNs among finite values: no magnitude
    x[8, 5] = 0xFFC0
    x[9, 0] = 0x7F80                             # +infinity: scale inf, the rest code 0
    ref = oracle_mod.layout(d["topk_idx"], E, R)
    cfg = M.cfg_of(T, H, E, k, R)
    lay, _ = M.gpu_layout(cfg, d["topk_idx"])
    eo = inputs.random_bf16_bits((T * k, H), seed=2)
    recv_q, recv_s, _, _, _ = _run_fp8(cfg, lay, M.to_dev(x), eo, d["topk_w"])
    rq, rs = oracle_mod.dispatch_fp8(x, ref["slot"])
    assert np.array_equal(_u8(recv_q), rq)
    assert np.array_equal(recv_s.cpu().numpy(), rs)


def test_fp8_workload_olmoe(oracle_mod):
    d = inputs.make("olmoe")
    wl = d["workload"]
    ref = oracle_mod.layout(d["topk_idx"], wl.E, wl.R)
    cfg = M.cfg_of(wl.T, wl.H, wl.E, wl.k, wl.R)
    lay, _ = M.gpu_layout(cfg, d["topk_idx"])
    eo = inputs.random_bf16_bits((wl.T * wl.k, wl.H), seed=wl.seed + 7)
    recv_q, recv_s, eo_q, eo_s, y = _run_fp8(cfg, lay, M.to_dev(d["x"]), eo, d["topk_w"])
    rq, rs = oracle_mod.dispatch_fp8(d["x"], ref["slot"])
    assert np.array_equal(_u8(recv_q), rq) and np.array_equal(recv_s.cpu().numpy(), rs)
    eq, es = oracle_mod.quantize_rows_fp8(eo)
    assert np.array_equal(_u8(eo_q), eq) and np.array_equal(eo_s.cpu().numpy(), es)
    y_bits = M.bits(y)
    assert np.array_equal(y_bits, oracle_mod.combine_fp8(eq, es, d["topk_w"], ref["slot"]))
    _assert_fp8_error_bound(y_bits, eo, d["topk_w"], ref["slot"], es.astype(np.float64))
    # unit-scale expert outputs: the pages' fp8 combine tolerance
    eo_n = inputs.random_bf16((wl.T * wl.k, wl.H), seed=wl.seed + 8)
    _, _, _, _, y_n = _run_fp8(cfg, lay, M.to_dev(d["x"]), eo_n, d["topk_w"])
    M.assert_combine_close(M.bits(y_n), oracle_mod.combine(eo_n, d["topk_w"], ref["slot"]),
                           rtol=0.02, atol=0.15)
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK


@pytest.mark.parametrize("form", [0, capi.MOE_FLAG_TWO_LEVEL_SPLIT])
@pytest.mark.parametrize("node_src", [True, False])
@pytest.mark.parametrize("T,H,E,k,R,N", [
    (33, 136, 13, 4, 5, 5),         # H % 16 != 0: the split form whatever the flag
    (257, 2048, 64, 8, 4, 2),
    (129, 1056, 32, 8, 8, 2),       # 66 groups: 32-byte accesses, a ragged last block of 64
    (97, 1040, 32, 6, 4, 2),        # 65 groups (odd): the 16-byte form
    (600, 7168, 32, 8, 8, 4),       # 14 groups of 16 values per lane
    (300, 8192, 64, 16, 16, 16),    # N + k = 32, the one-kernel limit
])
def test_fp8_two_level(oracle_mod, T, H, E, k, R, N, node_src, form):
    """Both fp8 two-level forms (one kernel: quantize, stage, read back,
    expand; split: quantizer then two expansions) give the oracle's staging
    and receive codes and scales."""
    d = inputs.make_random(T, H, E, k, seed=T + N)
    x, topk = d["x"], d["topk_idx"]
    ref = oracle_mod.layout(topk, E, R, N, nodes=True)
    cfg = M.cfg_of(T, H, E, k, R, N, capi.MOE_FLAG_TWO_LEVEL | form)
    lay, _ = M.gpu_layout(cfg, topk, node_src=node_src)
    rows = capi.moe_node_staging_rows(cfg)
    st_q = torch.full((rows, H), 0x55, dtype=torch.uint8, device="cuda")
    st_s = torch.zeros(rows, dtype=torch.float32, device="cuda")
    recv_q = torch.empty((T * k, H), dtype=torch.uint8, device="cuda")
    recv_s = torch.empty(T * k, dtype=torch.float32, device="cuda")
    capi.moe_dispatch_fp8_two_level(cfg, lay.struct, M.to_dev(x), st_q, st_s, recv_q, recv_s)
    rq, rs = oracle_mod.dispatch_fp8(x, ref["slot"])
    assert np.array_equal(_u8(recv_q), rq)
    assert np.array_equal(recv_s.cpu().numpy(), rs)
    # staging row u holds the codes of token node_src[u]; rows beyond U untouched
    xq, xs = oracle_mod.quantize_rows_fp8(x)
    U = int(ref["node_offsets"][-1])
    assert np.array_equal(_u8(st_q)[:U], xq[ref["node_src"]])
    assert np.array_equal(st_s.cpu().numpy()[:U], xs[ref["node_src"]])
    assert np.all(_u8(st_q)[U:] == 0x55)
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK


@pytest.mark.parametrize("form", [0, capi.MOE_FLAG_TWO_LEVEL_SPLIT])
def test_fp8_two_level_dsv3_workload(oracle_mod, form):
    """The DeepSeek-V3-shaped workload at full size through the fp8
    two-level dispatch: receive codes and scales as the oracle's fp8
    dispatch, staging rows as its quantizer of the staged tokens."""
    d = inputs.make("dsv3")
    wl = d["workload"]
    x, topk = d["x"], d["topk_idx"]
    ref = oracle_mod.layout(topk, wl.E, wl.R, wl.N, nodes=True)
    cfg = M.cfg_of(wl.T, wl.H, wl.E, wl.k, wl.R, wl.N, capi.MOE_FLAG_TWO_LEVEL | form)
    lay, _ = M.gpu_layout(cfg, topk)
    rows = capi.moe_node_staging_rows(cfg)
    st_q = torch.empty((rows, wl.H), dtype=torch.uint8, device="cuda")
    st_s = torch.empty(rows, dtype=torch.float32, device="cuda")
    recv_q = torch.empty((wl.T * wl.k, wl.H), dtype=torch.uint8, device="cuda")
    recv_s = torch.empty(wl.T * wl.k, dtype=torch.float32, device="cuda")
    capi.moe_dispatch_fp8_two_level(cfg, lay.struct, M.to_dev(x), st_q, st_s, recv_q, recv_s)
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK
    rq, rs = oracle_mod.dispatch_fp8(x, ref["slot"])
    assert np.array_equal(_u8(recv_q), rq)
    assert np.array_equal(recv_s.cpu().numpy(), rs)
    del recv_q
    xq, xs = oracle_mod.quantize_rows_fp8(x)
    U = int(ref["node_offsets"][-1])
    assert np.array_equal(_u8(st_q)[:U], xq[ref["node_src"]])
    assert np.array_equal(st_s.cpu().numpy()[:U], xs[ref["node_src"]])
    torch.cuda.empty_cache()


def test_fp8_refusals():
    cfg = M.cfg_of(4, 12, 8, 2, 2)                       # hidden % 8 != 0
    lay, _ = M.gpu_layout(cfg, np.array([[0, 1], [2, 3], [4, 5], [6, 7]], np.int32))
    x = torch.zeros((4, 12), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((8, 12), dtype=torch.uint8, device="cuda")
    s = torch.empty(8, dtype=torch.float32, device="cuda")
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_dispatch_fp8(cfg, lay.struct, x, q, s)
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG
    two = M.cfg_of(4, 16, 8, 2, 2, 2, capi.MOE_FLAG_TWO_LEVEL)
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_dispatch_fp8(two, lay.struct, x, q, s)
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG
    flat = M.cfg_of(4, 16, 8, 2, 2)
    with pytest.raises(capi.MoeError) as ei:                 # the staged form needs node staging
        capi.moe_dispatch_fp8_two_level(flat, lay.struct, x, q, s, q, s)
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG
