"""GPU parity: the CUDA path through the C ABI against the oracle.

Layout and dispatch must match bit for bit; combine must be within 1e-2
relative / 1e-3 absolute of the oracle (and is expected to be bit-exact,
since both sides use the same fp32 FMA order and one RNE store).  Small
shapes compare every value; the five named workloads run at full size in the
launch configuration bench.py times.
"""
import numpy as np
import pytest
import torch

import moe_testlib as M
from combine_moe_layout_06_b200 import capi, inputs

pytestmark = pytest.mark.gpu

TWO = capi.MOE_FLAG_TWO_LEVEL
VEC = capi.MOE_FLAG_COPY_VECTOR
BULK = capi.MOE_FLAG_COPY_BULK
CL = capi.MOE_FLAG_LAYOUT_CLUSTER
ONE = capi.MOE_FLAG_TWO_LEVEL_FUSED
SPLIT = capi.MOE_FLAG_TWO_LEVEL_SPLIT
CANARY = 0x7F81          # a signalling-NaN bf16 pattern no dispatched row holds

SMALL = [
    # T, H, E, k, R, N
    (1, 8, 4, 1, 1, 1),
    (7, 64, 8, 3, 4, 2),
    (33, 136, 13, 4, 5, 5),
    (255, 128, 16, 8, 8, 4),
    (256, 128, 8, 2, 2, 1),
    (257, 72, 64, 8, 4, 2),
    (1000, 256, 60, 4, 7, 7),
    (513, 9, 20, 6, 10, 5),      # odd row: 18 bytes -> 2-byte vectors
    (300, 10, 32, 16, 8, 8),     # 20-byte rows -> 4-byte vectors, k > 8
    (130, 64, 32, 32, 4, 2),     # k = E = 32
    (600, 16, 1024, 8, 32, 32),  # E at the library maximum
    (2049, 2048, 64, 8, 4, 1),
]


def _small_inputs(T, H, E, k, seed):
    d = inputs.make_random(T, H, E, k, seed=seed, zipf_s=0.7)
    return d["x"], d["topk_idx"], d["topk_w"]


@pytest.mark.parametrize("T,H,E,k,R,N", SMALL)
def test_layout_small(oracle_mod, T, H, E, k, R, N):
    _, topk, _ = _small_inputs(T, H, E, k, seed=T + E)
    for flags in (0, TWO, CL, TWO | CL):
        cfg = M.cfg_of(T, H, E, k, R, N, flags)
        lay, _ = M.gpu_layout(cfg, topk)
        ref = oracle_mod.layout(topk, E, R, N, nodes=bool(flags & TWO))
        M.assert_layout_equal(lay.host(), ref)
        assert capi.moe_get_error(lay.struct) == capi.MOE_OK


@pytest.mark.parametrize("T,H,E,k,R,N", SMALL)
def test_dispatch_and_combine_small(oracle_mod, T, H, E, k, R, N):
    x, topk, w = _small_inputs(T, H, E, k, seed=3 * T + H)
    ref = oracle_mod.layout(topk, E, R, N, nodes=True)
    recv_ref = oracle_mod.dispatch_flat(x, ref["slot"])
    staging_ref, recv2_ref = oracle_mod.dispatch_two_level(x, ref, R, N)
    assert np.array_equal(recv2_ref, recv_ref)
    eo = inputs.random_bf16_bits((T * k, H), seed=T * k + H)
    y_ref = oracle_mod.combine(eo, w, ref["slot"])
    x_dev = M.to_dev(x)
    # TWO: one kernel (node staging, then the staging row read back) where
    # N + k <= 32 and rows are 16-byte multiples, else pack + expansion;
    # TWO | SPLIT and TWO | VEC: pack + expansion
    runs = [(f, True) for f in (0, TWO, VEC, TWO | VEC, BULK, TWO | BULK, TWO | ONE,
                                TWO | SPLIT, TWO | SPLIT | BULK)]
    runs += [(f, False) for f in (TWO | SPLIT, TWO | VEC, TWO | SPLIT | BULK)]   # pair-walking expansion
    for flags, node_src in runs:
        cfg = M.cfg_of(T, H, E, k, R, N, flags)
        lay, _ = M.gpu_layout(cfg, topk, node_src=node_src)
        want = ref if flags & TWO else {k_: v for k_, v in ref.items() if not k_.startswith("node")}
        if not node_src:
            want = {k_: v for k_, v in want.items() if k_ != "node_src"}
        M.assert_layout_equal(lay.host(), want)
        recv, staging = M.gpu_dispatch(cfg, lay, x_dev, fill=CANARY)
        assert np.array_equal(M.bits(recv), recv_ref)
        lay2 = M.buffers.DeviceLayout(cfg, node_src=node_src)
        recv2 = torch.empty_like(recv)
        st2 = M.staging_buffer(cfg) if flags & TWO else None
        capi.moe_layout_dispatch(cfg, torch.from_numpy(topk).cuda(), lay2.struct, x_dev, recv2, st2)
        assert np.array_equal(M.bits(recv2), recv_ref), "fused layout + dispatch"
        if flags & TWO:
            U = int(ref["node_offsets"][-1])
            st = M.bits(staging)
            assert np.array_equal(st[:U], staging_ref)
            assert np.all(st[U:] == CANARY), "no stray staging writes"
        y = M.gpu_combine(cfg, lay, M.to_dev(eo), w)
        M.assert_combine_close(M.bits(y), y_ref)
        assert np.array_equal(M.bits(y), y_ref), "fixed-order fp32 FMA is bit-exact"
        assert capi.moe_get_error(lay.struct) == capi.MOE_OK


@pytest.mark.parametrize("T,E,k,R,N,shift", [
    (10240, 1024, 8, 8, 4, 0),    # histograms of 160 KB: read from global memory, 40 chunks
    (7000, 256, 8, 8, 2, 4),      # workspace off a 16-byte boundary, 28 chunks
    (60000, 256, 8, 8, 2, 4),     # workspace off a 16-byte boundary, 235 chunks
    (33 * 256, 96, 6, 6, 3, 0),   # 33 chunks, k not a multiple of 4 (scalar routes and slots)
])
def test_layout_histogram_paths(oracle_mod, T, E, k, R, N, shift):
    """The assign kernel's histogram paths: copied whole into shared memory
    (chunk-major, the default for 16-byte aligned workspaces up to 128 KB of
    histograms), or read from global memory (expert-major) when the
    histograms are larger or the workspace is not 16-byte aligned, with
    up to 32 chunks and beyond.  Each matches the oracle bit for bit."""
    d = inputs.make_random(T, 8, E, k, seed=T + E)
    topk = d["topk_idx"]
    ref = oracle_mod.layout(topk, E, R, N, nodes=True)
    for flags in (0, TWO):
        cfg = M.cfg_of(T, 8, E, k, R, N, flags)
        lay = M.buffers.DeviceLayout(cfg)
        ws = torch.zeros(capi.moe_layout_workspace_bytes(cfg) + 16, dtype=torch.uint8, device="cuda")
        struct = capi.layout_struct(lay.expert_counts, lay.expert_offsets, lay.rank_offsets, lay.slot,
                                    lay.error_word, ws.data_ptr() + shift, lay.node_counts,
                                    lay.node_offsets, lay.node_slot, lay.node_src)
        capi.moe_layout(cfg, torch.from_numpy(topk).cuda(), struct)
        want = ref if flags else {k_: v for k_, v in ref.items() if not k_.startswith("node")}
        M.assert_layout_equal(lay.host(), want)
        assert capi.moe_get_error(struct) == capi.MOE_OK


@pytest.mark.parametrize("T", [40000, 140001])
def test_large_batch_multi_kernel_layout(oracle_mod, T):
    """Above 16384 tokens the layout runs as count + assign kernels over a
    workspace (the scan folded into assign up to 65536 tokens, a separate
    scan kernel beyond)."""
    H, E, k, R, N = 8, 64, 4, 8, 2
    x, topk, w = _small_inputs(T, H, E, k, seed=77)
    ref = oracle_mod.layout(topk, E, R, N, nodes=True)
    for flags in (0, TWO):
        cfg = M.cfg_of(T, H, E, k, R, N, flags)
        lay, _ = M.gpu_layout(cfg, topk)
        want = ref if flags else {k_: v for k_, v in ref.items() if not k_.startswith("node")}
        M.assert_layout_equal(lay.host(), want)
        recv, _ = M.gpu_dispatch(cfg, lay, M.to_dev(x))
        assert np.array_equal(M.bits(recv), oracle_mod.dispatch_flat(x, ref["slot"]))
        y = M.gpu_combine(cfg, lay, recv, w)
        assert np.array_equal(M.bits(y), oracle_mod.combine(M.bits(recv), w, ref["slot"]))
        assert capi.moe_get_error(lay.struct) == capi.MOE_OK


@pytest.mark.parametrize("engine", [0, VEC, BULK, ONE, SPLIT, SPLIT | BULK])
@pytest.mark.parametrize("hot_frac", [0.0, 0.9, 1.0])
def test_skewed_node_loads(oracle_mod, engine, hot_frac):
    """One hot node (up to every token on node 0, the other nodes empty): the
    one-kernel two-level dispatch and, in the two-kernel form, the
    row-balanced and the pair-walking expansions all reproduce the oracle's
    staging and receive buffers bit for bit."""
    T, H, E, k, R, N = 5000, 264, 64, 6, 8, 4
    d = inputs.make_node_skewed(T, H, E, k, N, hot_frac, seed=int(hot_frac * 10) + 3)
    x, topk = d["x"], d["topk_idx"]
    ref = oracle_mod.layout(topk, E, R, N, nodes=True)
    staging_ref, recv_ref = oracle_mod.dispatch_two_level(x, ref, R, N)
    if hot_frac == 1.0:
        assert ref["node_counts"][1:].sum() == 0 and ref["node_counts"][0] == T
    x_dev = M.to_dev(x)
    cfg = M.cfg_of(T, H, E, k, R, N, TWO | engine)
    for node_src in (True, False):
        lay, _ = M.gpu_layout(cfg, topk, node_src=node_src)
        want = ref if node_src else {k_: v for k_, v in ref.items() if k_ != "node_src"}
        M.assert_layout_equal(lay.host(), want)
        recv, staging = M.gpu_dispatch(cfg, lay, x_dev, fill=CANARY)
        U = int(ref["node_offsets"][-1])
        assert np.array_equal(M.bits(staging)[:U], staging_ref)
        assert np.array_equal(M.bits(recv), recv_ref)
        assert capi.moe_get_error(lay.struct) == capi.MOE_OK


def test_combine_nan_and_infinity_propagate(oracle_mod):
    """Non-finite expert outputs: NaN where the oracle has NaN (any payload;
    the GPU stores bf16 NaNs in canonical form), every other value bit for
    bit, infinities included."""
    T, H, E, k, R = 300, 64, 16, 4, 4
    d = inputs.make_random(T, H, E, k, seed=12)
    ref = oracle_mod.layout(d["topk_idx"], E, R)
    eo = inputs.random_bf16_bits((T * k, H), seed=13)
    eo[5, 3] = 0x7FC0                                  # NaN
    eo[9, 0] = 0xFFC1                                  # negative NaN, odd payload
    eo[20, 7] = 0x7F80                                 # +inf
    eo[21, 7] = 0xFF80                                 # -inf (inf - inf where both meet)
    eo[40, 2] = 0x7F80
    cfg = M.cfg_of(T, H, E, k, R)
    lay, _ = M.gpu_layout(cfg, d["topk_idx"])
    y = M.bits(M.gpu_combine(cfg, lay, M.to_dev(eo), d["topk_w"]))
    want = oracle_mod.combine(eo, d["topk_w"], ref["slot"])
    nan = lambda b: (b & 0x7FFF) > 0x7F80
    assert np.array_equal(nan(y), nan(want)) and nan(want).any()
    assert np.array_equal(y[~nan(want)], want[~nan(want)])
    assert ((want & 0x7FFF) == 0x7F80).any(), "an infinity reaches the output"


def test_empty_batch(oracle_mod):
    cfg = M.cfg_of(0, 64, 8, 2, 2, 2, TWO)
    lay, _ = M.gpu_layout(cfg, np.zeros((0, 2), np.int32))
    h = lay.host()
    assert not h["expert_offsets"].any() and not h["rank_offsets"].any()
    assert not h["node_offsets"].any() and not h["expert_counts"].any()
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    capi.moe_dispatch(cfg, lay.struct, x, x, x)
    capi.moe_combine(cfg, lay.struct, x, torch.empty(0, device="cuda"), x)
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK


def test_k1_unit_weight_round_trip_is_identity():
    x, topk, _ = _small_inputs(777, 96, 12, 1, seed=5)
    cfg = M.cfg_of(777, 96, 12, 1, 3)
    lay, _ = M.gpu_layout(cfg, topk)
    x_dev = M.to_dev(x)
    recv, _ = M.gpu_dispatch(cfg, lay, x_dev)
    y = M.gpu_combine(cfg, lay, recv, np.ones((777, 1), np.float32))
    assert torch.equal(y.view(torch.int16), x_dev.view(torch.int16))


def test_round_trip_identity_expert_renormalised():
    x, topk, w = _small_inputs(1500, 512, 32, 6, seed=8)
    cfg = M.cfg_of(1500, 512, 32, 6, 4)
    lay, _ = M.gpu_layout(cfg, topk)
    recv, _ = M.gpu_dispatch(cfg, lay, M.to_dev(x))
    y = M.gpu_combine(cfg, lay, recv, w)
    M.assert_combine_close(M.bits(y), x)


def test_unaligned_buffers(oracle_mod):
    """Base addresses off the 16-byte grid take the narrow-vector kernels."""
    T, H, E, k, R = 300, 64, 16, 4, 4
    x, topk, w = _small_inputs(T, H, E, k, seed=21)
    ref = oracle_mod.layout(topk, E, R)
    cfg = M.cfg_of(T, H, E, k, R)
    lay, _ = M.gpu_layout(cfg, topk)
    for shift in (1, 2):   # elements: 2-byte and 4-byte offsets
        xs = torch.empty(T * H + 8, dtype=torch.bfloat16, device="cuda")
        xv = xs[shift:shift + T * H].view(T, H)
        xv.copy_(M.to_dev(x))
        rs = torch.empty(T * k * H + 8, dtype=torch.bfloat16, device="cuda")
        rv = rs[shift:shift + T * k * H].view(T * k, H)
        capi.moe_dispatch(cfg, lay.struct, xv, rv)
        assert np.array_equal(M.bits(rv), oracle_mod.dispatch_flat(x, ref["slot"]))
        ys = torch.empty(T * H + 8, dtype=torch.bfloat16, device="cuda")
        yv = ys[shift:shift + T * H].view(T, H)
        capi.moe_combine(cfg, lay.struct, rv, torch.from_numpy(w).cuda(), yv)
        assert np.array_equal(M.bits(yv), oracle_mod.combine(M.bits(rv), w, ref["slot"]))


# ---------------------------------------------------------------- workloads

NAMES = ["tiny", "olmoe", "qwen3", "dsv3", "longctx"]


def _workload_cfg(wl, two_level):
    return M.cfg_of(wl.T, wl.H, wl.E, wl.k, wl.R, wl.N, TWO if two_level else 0)


@pytest.mark.parametrize("name", NAMES)
def test_workload_layout_dispatch(oracle_mod, name):
    d = inputs.make(name)
    wl = d["workload"]
    x, topk = d["x"], d["topk_idx"]
    ref = oracle_mod.layout(topk, wl.E, wl.R, wl.N, nodes=True)
    x_dev = M.to_dev(x)
    modes = [False, True] if wl.two_level or wl.N > 1 else [False]
    for two in modes:
        cfg = _workload_cfg(wl, two)
        lay, _ = M.gpu_layout(cfg, topk)
        got = lay.host()
        want = ref if two else {k_: v for k_, v in ref.items() if not k_.startswith("node")}
        M.assert_layout_equal(got, want)
        recv, staging = M.gpu_dispatch(cfg, lay, x_dev)
        # the fused entry point gives the same layout and rows
        lay2 = M.buffers.DeviceLayout(cfg)
        recv2 = torch.empty_like(recv)
        st2 = M.staging_buffer(cfg) if two else None
        capi.moe_layout_dispatch(cfg, torch.from_numpy(topk).cuda(), lay2.struct, x_dev, recv2, st2)
        M.assert_layout_equal(lay2.host(), want)
        assert torch.equal(recv2.view(torch.int16), recv.view(torch.int16))
        del recv2, st2
        # every receive row equals its token's row (full check on the device)
        slot_dev = torch.from_numpy(ref["slot"].reshape(-1).astype(np.int64)).cuda()
        tok_dev = torch.arange(wl.T, device="cuda").repeat_interleave(wl.k)
        assert torch.equal(recv.view(torch.int16)[slot_dev], x_dev.view(torch.int16)[tok_dev])
        del slot_dev, tok_dev
        if wl.T * wl.k * wl.H <= 1 << 30:
            assert np.array_equal(M.bits(recv), oracle_mod.dispatch_flat(x, ref["slot"]))
        if two:
            U = int(ref["node_offsets"][-1])
            node_tok = np.concatenate([np.flatnonzero(ref["node_slot"][:, n] >= 0)
                                       for n in range(wl.N)])
            assert node_tok.size == U
            st = staging[:U].view(torch.int16)
            assert torch.equal(st, x_dev.view(torch.int16)[torch.from_numpy(node_tok).cuda()])
        assert capi.moe_get_error(lay.struct) == capi.MOE_OK
        del recv, staging
        torch.cuda.empty_cache()


@pytest.mark.parametrize("engine", [VEC, BULK], ids=["register", "bulk"])
@pytest.mark.parametrize("name", ["olmoe", "dsv3", "longctx"])
def test_workload_forced_engine(oracle_mod, name, engine):
    """Each copy engine, forced, on the full workloads."""
    d = inputs.make(name)
    wl = d["workload"]
    x, topk, w = d["x"], d["topk_idx"], d["topk_w"]
    ref = oracle_mod.layout(topk, wl.E, wl.R, wl.N, nodes=True)
    cfg = M.cfg_of(wl.T, wl.H, wl.E, wl.k, wl.R, wl.N, (TWO if wl.two_level else 0) | engine)
    lay, _ = M.gpu_layout(cfg, topk)
    x_dev = M.to_dev(x)
    recv, _ = M.gpu_dispatch(cfg, lay, x_dev)
    slot_dev = torch.from_numpy(ref["slot"].reshape(-1).astype(np.int64)).cuda()
    tok_dev = torch.arange(wl.T, device="cuda").repeat_interleave(wl.k)
    assert torch.equal(recv.view(torch.int16)[slot_dev], x_dev.view(torch.int16)[tok_dev])
    del slot_dev, tok_dev
    eo = inputs.random_bf16_bits((wl.T * wl.k, wl.H), seed=wl.seed + 9)
    y = M.bits(M.gpu_combine(cfg, lay, M.to_dev(eo), w))
    assert np.array_equal(y, oracle_mod.combine(eo, w, ref["slot"]))
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK


@pytest.mark.parametrize("form", [ONE, SPLIT])
def test_workload_two_level_forms(oracle_mod, form):
    """Both two-level dispatch forms (one kernel; pack then expansion) on the
    DeepSeek-V3-shaped workload at full size: staging rows and receive rows
    as the oracle has them."""
    d = inputs.make("dsv3")
    wl = d["workload"]
    x, topk = d["x"], d["topk_idx"]
    ref = oracle_mod.layout(topk, wl.E, wl.R, wl.N, nodes=True)
    cfg = M.cfg_of(wl.T, wl.H, wl.E, wl.k, wl.R, wl.N, TWO | form)
    lay, _ = M.gpu_layout(cfg, topk)
    x_dev = M.to_dev(x)
    recv, staging = M.gpu_dispatch(cfg, lay, x_dev)
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK
    slot_dev = torch.from_numpy(ref["slot"].reshape(-1).astype(np.int64)).cuda()
    tok_dev = torch.arange(wl.T, device="cuda").repeat_interleave(wl.k)
    assert torch.equal(recv.view(torch.int16)[slot_dev], x_dev.view(torch.int16)[tok_dev])
    del slot_dev, tok_dev, recv
    U = int(ref["node_offsets"][-1])
    node_tok = np.concatenate([np.flatnonzero(ref["node_slot"][:, n] >= 0) for n in range(wl.N)])
    assert node_tok.size == U
    assert torch.equal(staging[:U].view(torch.int16),
                       x_dev.view(torch.int16)[torch.from_numpy(node_tok).cuda()])
    del staging
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", NAMES)
def test_workload_layout_cluster(oracle_mod, name):
    """The single-cluster layout kernel against the oracle at full size."""
    d = inputs.make(name)
    wl = d["workload"]
    topk = d["topk_idx"]
    ref = oracle_mod.layout(topk, wl.E, wl.R, wl.N, nodes=True)
    cfg = M.cfg_of(wl.T, wl.H, wl.E, wl.k, wl.R, wl.N, TWO | CL)
    lay, _ = M.gpu_layout(cfg, topk)
    M.assert_layout_equal(lay.host(), ref)
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK


@pytest.mark.parametrize("name", NAMES)
def test_workload_combine(oracle_mod, name):
    d = inputs.make(name)
    wl = d["workload"]
    topk, w = d["topk_idx"], d["topk_w"]
    ref = oracle_mod.layout(topk, wl.E, wl.R)
    eo = inputs.random_bf16_bits((wl.T * wl.k, wl.H), seed=wl.seed + 7)
    y_ref = oracle_mod.combine(eo, w, ref["slot"])
    cfg = _workload_cfg(wl, wl.two_level)
    lay, _ = M.gpu_layout(cfg, topk)
    y = M.bits(M.gpu_combine(cfg, lay, M.to_dev(eo), w))
    M.assert_combine_close(y, y_ref)
    assert np.array_equal(y, y_ref)
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK


@pytest.mark.parametrize("H", [1040, 1520, 1032])
def test_combine_many_waves_ragged_chunks(oracle_mod, H):
    """Combines of at least 8 resident waves of (token, 1 KB chunk) items take
    the 32-byte-per-lane form when the row has an even number of 16-byte
    vectors: rows ending 2 (H = 1040) and 62 (H = 1520) vectors into their
    last chunk.  An odd vector count (H = 1032) keeps the 16-byte form at the
    same size.  Bit for bit against the oracle."""
    T, E, k, R = 50001, 32, 4, 4
    _, topk, w = _small_inputs(T, 8, E, k, seed=H)
    ref = oracle_mod.layout(topk, E, R)
    eo = inputs.random_bf16_bits((T * k, H), seed=H + 1)
    cfg = M.cfg_of(T, H, E, k, R)
    lay, _ = M.gpu_layout(cfg, topk)
    y = M.bits(M.gpu_combine(cfg, lay, M.to_dev(eo), w))
    y_ref = oracle_mod.combine(eo, w, ref["slot"])
    M.assert_combine_close(y, y_ref)
    assert np.array_equal(y, y_ref)
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK


# ---------------------------------------------------------------- decoupled

@pytest.mark.parametrize("name", NAMES)
def test_decoupled_matches_oracle(oracle_mod, name):
    """The pack -> copy -> unpack comparison path against the oracle at full
    size: its receive rows equal the oracle's flat dispatch and its combine
    (of those rows, an identity expert) the oracle's combine, bit for bit
    and within the combine tolerance; and both equal the fused path."""
    d = inputs.make(name)
    wl = d["workload"]
    x, topk, w = d["x"], d["topk_idx"], d["topk_w"]
    ref = oracle_mod.layout(topk, wl.E, wl.R)
    recv_ref = oracle_mod.dispatch_flat(x, ref["slot"])
    y_ref = oracle_mod.combine(recv_ref, w, ref["slot"])
    x_dev = M.to_dev(x)
    dcfg = M.cfg_of(wl.T, wl.H, wl.E, wl.k, wl.R, wl.R, TWO)
    dlay, _ = M.gpu_layout(dcfg, topk)
    rows = capi.moe_node_staging_rows(dcfg)
    send = torch.empty((rows, wl.H), dtype=torch.bfloat16, device="cuda")
    xfer = torch.empty_like(send)
    recv_d = torch.full((wl.T * wl.k, wl.H), CANARY, dtype=torch.int16,
                        device="cuda").view(torch.bfloat16)
    capi.moe_dispatch_decoupled(dcfg, dlay.struct, x_dev, send, xfer, recv_d)
    del send, xfer
    assert np.array_equal(M.bits(recv_d), recv_ref)
    send2 = torch.empty_like(recv_d)
    xfer2 = torch.empty_like(recv_d)
    y_d = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    wd = torch.from_numpy(w).cuda()
    capi.moe_combine_decoupled(dcfg, dlay.struct, recv_d, wd, send2, xfer2, y_d)
    del send2, xfer2
    y_bits = M.bits(y_d)
    M.assert_combine_close(y_bits, y_ref)
    assert np.array_equal(y_bits, y_ref)
    assert capi.moe_get_error(dlay.struct) == capi.MOE_OK
    # the fused path on the same inputs gives the same bits
    fused_cfg = _workload_cfg(wl, False)
    flay, _ = M.gpu_layout(fused_cfg, topk)
    recv_f, _ = M.gpu_dispatch(fused_cfg, flay, x_dev)
    assert torch.equal(recv_f.view(torch.int16), recv_d.view(torch.int16))
    del recv_f
    y_f = M.gpu_combine(fused_cfg, flay, recv_d, w)
    assert torch.equal(y_f.view(torch.int16), y_d.view(torch.int16))
    del recv_d
    torch.cuda.empty_cache()


# ---------------------------------------------------------------- errors

def test_device_data_errors_are_reported():
    T, H, E, k, R = 64, 32, 8, 2, 2
    _, topk, w = _small_inputs(T, H, E, k, seed=1)
    bad = topk.copy()
    bad[5, 1] = E          # out of range
    cfg = M.cfg_of(T, H, E, k, R, 2, TWO)
    lay, _ = M.gpu_layout(cfg, bad)
    assert capi.moe_get_error(lay.struct) == capi.MOE_ERR_EXPERT_OOB
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK, "reading clears the word"
    dup = topk.copy()
    dup[9, 1] = dup[9, 0]
    lay, _ = M.gpu_layout(cfg, dup)
    assert capi.moe_get_error(lay.struct) == capi.MOE_ERR_DUP_EXPERT
    neg = topk.copy()
    neg[0, 0] = -3
    neg[1, 1] = neg[1, 0]
    lay, _ = M.gpu_layout(cfg, neg)
    assert capi.moe_get_error(lay.struct) == capi.MOE_ERR_EXPERT_OOB, "out-of-range wins"
    # the layout of the valid entries still only names rows inside the buffer
    h = lay.host()
    s = h["slot"]
    assert s[0, 0] == -1 and s[1, 1] == -1
    valid = s[s >= 0]
    assert valid.max() < T * k and np.unique(valid).size == valid.size


def test_bad_slot_is_reported_and_skipped():
    T, H, E, k, R = 40, 64, 8, 2, 2
    x, topk, w = _small_inputs(T, H, E, k, seed=2)
    cfg = M.cfg_of(T, H, E, k, R)
    lay, _ = M.gpu_layout(cfg, topk)
    lay.slot[3] = T * k + 5          # corrupt one slot
    recv = torch.zeros((T * k, H), dtype=torch.bfloat16, device="cuda")
    capi.moe_dispatch(cfg, lay.struct, M.to_dev(x), recv)
    assert capi.moe_get_error(lay.struct) == capi.MOE_ERR_BAD_LAYOUT
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    capi.moe_combine(cfg, lay.struct, recv, torch.from_numpy(w).cuda(), y)
    assert capi.moe_get_error(lay.struct) == capi.MOE_ERR_BAD_LAYOUT


# ---------------------------------------------------------- all-gather / reduce-scatter

@pytest.mark.parametrize("name", ["tiny", "olmoe", "longctx", "small"])
def test_allgather_reducescatter(oracle_mod, name):
    if name == "small":
        T, H, E, k, R = 333, 72, 24, 5, 6
        x, topk, w = _small_inputs(T, H, E, k, seed=12)
    else:
        d = inputs.make(name)
        wl = d["workload"]
        T, H, E, k, R = wl.T, wl.H, wl.E, wl.k, wl.R
        x, topk, w = d["x"], d["topk_idx"], d["topk_w"]
    ref = oracle_mod.layout(topk, E, R)
    cfg = M.cfg_of(T, H, E, k, R)
    lay, _ = M.gpu_layout(cfg, topk)
    x_dev = M.to_dev(x)
    gathered = torch.empty((R * T, H), dtype=torch.bfloat16, device="cuda")
    recv = torch.empty((T * k, H), dtype=torch.bfloat16, device="cuda")
    capi.moe_dispatch_allgather(cfg, lay.struct, x_dev, gathered, recv)
    assert torch.equal(gathered.view(R, T, H).view(torch.int16),
                       x_dev.view(torch.int16).unsqueeze(0).expand(R, T, H))
    if T * k * H <= 1 << 28:
        assert np.array_equal(M.bits(recv), oracle_mod.dispatch_flat(x, ref["slot"]))
    else:
        slot_dev = torch.from_numpy(ref["slot"].reshape(-1).astype(np.int64)).cuda()
        tok_dev = torch.arange(T, device="cuda").repeat_interleave(k)
        assert torch.equal(recv.view(torch.int16)[slot_dev], x_dev.view(torch.int16)[tok_dev])
    eo = inputs.random_bf16_bits((T * k, H), seed=T + H + 1)
    partial = torch.empty((R * T, H), dtype=torch.float32, device="cuda")
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    capi.moe_combine_reducescatter(cfg, lay.struct, M.to_dev(eo), torch.from_numpy(w).cuda(),
                                   partial, y)
    y_bits = M.bits(y)
    assert np.array_equal(y_bits, oracle_mod.combine_rank_partials(eo, w, ref["slot"],
                                                                   ref["rank_offsets"]))
    M.assert_combine_close(y_bits, oracle_mod.combine(eo, w, ref["slot"]))
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK
