"""moe_layout_dispatch() with MOE_FLAG_LAYOUT_FUSED: a count kernel plus an
assign/dispatch kernel (the per-CTA histograms meet in the workspace, where
the count kernel's last CTA turns them into prefixes; the dispatch kernel
ranks its own tokens).

Its layout arrays and receive rows must equal the oracle's bit for bit, on
ragged token counts (CTA ranges of unequal length), several token blocks per
CTA, k above 8, the expert-count limit of the pair and the configurations that
fall back to the layout kernels; back-to-back calls of different sizes must
reuse the ticket counter (it resets itself), and the pair must replay inside a
CUDA graph.
"""
import numpy as np
import pytest
import torch

import moe_testlib as M
from combine_moe_layout_06_b200 import buffers, capi, inputs

pytestmark = pytest.mark.gpu

FUSED = capi.MOE_FLAG_LAYOUT_FUSED

CASES = [
    # T, H, E, k, R
    (1, 8, 4, 1, 1),            # one token, one CTA
    (17, 64, 8, 3, 4),          # two CTAs of 8 and 9 tokens
    (1000, 136, 13, 4, 5),      # 272-byte rows, E not a multiple of R
    (4097, 2048, 64, 8, 4),     # OLMoE-shaped rows, 148 ragged CTAs
    (3001, 2056, 64, 8, 4),     # 4112-byte rows: a 4096-byte chunk and a 16-byte tail
    (2500, 64, 64, 16, 8),      # k > 8
    (700, 32, 256, 8, 8),       # the pair's expert limit
    (5000, 16, 1, 1, 1),        # one expert
    (200000, 8, 64, 2, 8),      # several 384-token blocks per CTA
]


def _inputs(T, H, E, k, seed):
    d = inputs.make_random(T, H, E, k, seed=seed, zipf_s=0.9)
    return d["x"], d["topk_idx"]


def _run(cfg, topk, x_dev, lay=None, recv=None):
    lay = lay or buffers.DeviceLayout(cfg)
    if recv is None:
        recv = torch.empty((cfg.num_tokens * cfg.top_k, cfg.hidden), dtype=torch.bfloat16,
                           device="cuda")
    capi.moe_layout_dispatch(cfg, torch.from_numpy(np.ascontiguousarray(topk)).cuda(), lay.struct,
                             x_dev, recv)
    return lay, recv


def _flat(ref):
    return {k_: v for k_, v in ref.items() if not k_.startswith("node")}


@pytest.mark.parametrize("T,H,E,k,R", CASES)
def test_pair_matches_oracle(oracle_mod, T, H, E, k, R):
    M.ensure_lib()
    x, topk = _inputs(T, H, E, k, seed=T + 31 * E + k)
    ref = oracle_mod.layout(topk, E, R, 1, nodes=False)
    x_dev = M.to_dev(x)
    cfg = M.cfg_of(T, H, E, k, R, 1, FUSED)
    lay, recv = _run(cfg, topk, x_dev)
    M.assert_layout_equal(lay.host(), _flat(ref))
    slot_dev = torch.from_numpy(ref["slot"].reshape(-1).astype(np.int64)).cuda()
    tok_dev = torch.arange(T, device="cuda").repeat_interleave(k)
    assert torch.equal(recv.view(torch.int16)[slot_dev], x_dev.view(torch.int16)[tok_dev])
    if T * k * H <= 1 << 24:
        assert np.array_equal(M.bits(recv), oracle_mod.dispatch_flat(x, ref["slot"]))
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK
    # the default path (layout kernels, then the dispatch kernel) agrees
    lay2, recv2 = _run(M.cfg_of(T, H, E, k, R), topk, x_dev)
    M.assert_layout_equal(lay2.host(), _flat(ref))
    assert torch.equal(recv2.view(torch.int16), recv.view(torch.int16))


def _barrier_words(lay, cfg):
    """The ticket counter (and the word after it): at the end of the layout
    kernels' chunk histograms (E * ceil(T/256) int32, rounded up to 256
    bytes)."""
    C = (cfg.num_tokens + 255) // 256
    off = (cfg.num_experts * C * 4 + 255) // 256 * 256
    return lay.workspace[off:off + 8].view(torch.int32).cpu().numpy()


def test_back_to_back_calls_reuse_the_counter(oracle_mod):
    """One workspace, calls of different grid sizes in a row: every token
    count up to 256 puts the counter at the same place (one histogram chunk)
    while the grid runs from 1 to 16 CTAs.  Each result is right and the
    counter is zero after every call."""
    M.ensure_lib()
    H, E, k, R = 64, 32, 4, 4
    shared = buffers.DeviceLayout(M.cfg_of(256, H, E, k, R))
    for i, T in enumerate([256, 17, 200, 1, 256, 100, 256]):
        x, topk = _inputs(T, H, E, k, seed=100 + i)
        cfg = M.cfg_of(T, H, E, k, R, 1, FUSED)
        sub = buffers.DeviceLayout(cfg)
        sub.workspace = shared.workspace
        sub.struct = capi.layout_struct(sub.expert_counts, sub.expert_offsets, sub.rank_offsets,
                                        sub.slot, sub.error_word, shared.workspace)
        _, recv = _run(cfg, topk, M.to_dev(x), lay=sub)
        ref = oracle_mod.layout(topk, E, R, 1, nodes=False)
        M.assert_layout_equal(sub.host(), _flat(ref))
        assert np.array_equal(M.bits(recv), oracle_mod.dispatch_flat(x, ref["slot"]))
        assert capi.moe_get_error(sub.struct) == capi.MOE_OK
        assert np.array_equal(_barrier_words(sub, cfg), [0, 0])
    # and a large grid, several calls on one layout
    T = 60000
    cfg = M.cfg_of(T, H, E, k, R, 1, FUSED)
    lay = buffers.DeviceLayout(cfg)
    x, topk = _inputs(T, H, E, k, seed=7)
    ref = oracle_mod.layout(topk, E, R, 1, nodes=False)
    x_dev = M.to_dev(x)
    for _ in range(3):
        _, recv = _run(cfg, topk, x_dev, lay=lay)
        M.assert_layout_equal(lay.host(), _flat(ref))
        assert np.array_equal(M.bits(recv), oracle_mod.dispatch_flat(x, ref["slot"]))
        assert np.array_equal(_barrier_words(lay, cfg), [0, 0])


def test_invalid_routes_match_the_layout_kernels():
    """Out-of-range and repeated expert ids: the pair drops them
    exactly as moe_layout() does (slot -1, not counted) and reports the same
    error."""
    M.ensure_lib()
    T, H, E, k, R = 3000, 64, 16, 4, 4
    x, topk = _inputs(T, H, E, k, seed=9)
    x_dev = M.to_dev(x)
    for mutate, status in ((lambda t: t.__setitem__((5, 1), E), capi.MOE_ERR_EXPERT_OOB),
                           (lambda t: t.__setitem__((2999, 3), t[2999, 0]), capi.MOE_ERR_DUP_EXPERT),
                           (lambda t: t.__setitem__((0, 0), -7), capi.MOE_ERR_EXPERT_OOB)):
        bad = topk.copy()
        mutate(bad)
        cfg = M.cfg_of(T, H, E, k, R, 1, FUSED)
        lay, recv = _run(cfg, bad, x_dev)
        ref, _ = M.gpu_layout(M.cfg_of(T, H, E, k, R), bad)
        M.assert_layout_equal(lay.host(), ref.host())
        assert capi.moe_get_error(lay.struct) == status
        assert capi.moe_get_error(ref.struct) == status
        s = lay.host()["slot"].reshape(-1)
        ok = s >= 0
        rows = recv.view(torch.int16)[torch.from_numpy(s[ok].astype(np.int64)).cuda()]
        toks = torch.from_numpy(np.repeat(np.arange(T), k)[ok]).cuda()
        assert torch.equal(rows, x_dev.view(torch.int16)[toks])


def test_fallbacks_give_the_same_results(oracle_mod):
    """Configurations the pair does not take (more than 256
    experts, rows that are not 16-byte multiples, unaligned x) run the layout
    kernels and the dispatch kernel, with the same results."""
    M.ensure_lib()
    for T, H, E, k, R, shift in ((900, 32, 300, 8, 10, 0), (900, 9, 32, 4, 4, 0),
                                 (900, 32, 32, 4, 4, 2)):
        x, topk = _inputs(T, H, E, k, seed=T + H + shift)
        ref = oracle_mod.layout(topk, E, R, 1, nodes=False)
        cfg = M.cfg_of(T, H, E, k, R, 1, FUSED)
        flat = torch.empty(T * H + shift, dtype=torch.bfloat16, device="cuda")
        x_dev = flat[shift:].view(T, H)
        x_dev.copy_(M.to_dev(x))
        lay, recv = _run(cfg, topk, x_dev)
        M.assert_layout_equal(lay.host(), _flat(ref))
        assert np.array_equal(M.bits(recv), oracle_mod.dispatch_flat(x, ref["slot"]))
        assert capi.moe_get_error(lay.struct) == capi.MOE_OK


def test_pair_replays_in_a_cuda_graph(oracle_mod):
    M.ensure_lib()
    T, H, E, k, R = 4096, 2048, 64, 8, 4
    x, topk = _inputs(T, H, E, k, seed=4)
    ref = oracle_mod.layout(topk, E, R, 1, nodes=False)
    cfg = M.cfg_of(T, H, E, k, R, 1, FUSED)
    lay = buffers.DeviceLayout(cfg)
    x_dev = M.to_dev(x)
    topk_dev = torch.from_numpy(topk).cuda()
    recv = torch.empty((T * k, H), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        capi.moe_layout_dispatch(cfg, topk_dev, lay.struct, x_dev, recv, stream=s.cuda_stream)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            capi.moe_layout_dispatch(cfg, topk_dev, lay.struct, x_dev, recv, stream=s.cuda_stream)
    for _ in range(3):
        recv.zero_()
        lay.slot.fill_(-5)
        g.replay()
        torch.cuda.synchronize()
        M.assert_layout_equal(lay.host(), _flat(ref))
        assert np.array_equal(M.bits(recv), oracle_mod.dispatch_flat(x, ref["slot"]))
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK
    assert np.array_equal(_barrier_words(lay, cfg), [0, 0])
