"""moe_layout_noalloc(): the layout for callers that cannot allocate device
memory (no cudaMalloc allowed where they run, e.g. inside a stream capture,
or under a framework that owns every allocation).  Its scratch is a fixed
array inside the library; its results must equal the oracle's layout, and
moe_layout()'s (which uses a caller-provided workspace), call after call.

This file is collected last on purpose: a run that stops at the first
failure has run every other test before it.  It passes alone in a fresh
process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

from combine_moe_layout_06_b200 import buffers, build, capi, inputs

pytestmark = pytest.mark.gpu

TWO = capi.MOE_FLAG_TWO_LEVEL


def _noalloc_struct(lay):
    """The layout arrays of `lay` with no workspace at all."""
    return capi.layout_struct(lay.expert_counts, lay.expert_offsets, lay.rank_offsets, lay.slot,
                              lay.error_word, None, lay.node_counts, lay.node_offsets,
                              lay.node_slot, lay.node_src)


def _check(cfg, topk_np, oracle_mod):
    """moe_layout_noalloc against the oracle and against moe_layout."""
    topk = torch.from_numpy(np.ascontiguousarray(topk_np, np.int32)).cuda()
    ref = buffers.DeviceLayout(cfg)
    capi.moe_layout(cfg, topk, ref.struct)
    got = buffers.DeviceLayout(cfg)
    got_struct = _noalloc_struct(got)
    capi.moe_layout_noalloc(cfg, topk, got_struct)
    torch.cuda.synchronize()
    assert capi.moe_get_error(ref.struct) == capi.MOE_OK
    assert capi.moe_get_error(got_struct) == capi.MOE_OK
    two = bool(cfg.flags & TWO)
    want = oracle_mod.layout(topk_np, cfg.num_experts, cfg.num_ranks, cfg.num_nodes, nodes=two)
    have, other = got.host(), ref.host()
    assert set(want) <= set(have)
    for key in want:
        assert np.array_equal(have[key], want[key]), ("oracle", key)
    for key in other:
        assert np.array_equal(have[key], other[key]), ("moe_layout", key)


def test_noalloc_layout_matches_oracle_twice(oracle_mod):
    build.build()
    assert torch.cuda.is_available()
    # two calls in a row with different problems: the second must not see
    # anything the first left in the shared scratch array
    for name, flags in [("dsv3", TWO), ("longctx", 0)]:
        d = inputs.make(name)
        wl = d["workload"]
        cfg = capi.config(wl.T, wl.H, wl.E, wl.k, wl.R, wl.N, flags)
        _check(cfg, d["topk_idx"], oracle_mod)
    # a batch above the single-cluster limit, whose layout uses the scratch
    big = inputs.make_random(140001, 8, 64, 4, seed=5)
    cfg = capi.config(140001, 8, 64, 4, 8, 2, TWO)
    for _ in range(2):
        _check(cfg, big["topk_idx"], oracle_mod)
    # and the same small problem twice in a row
    small = inputs.make_random(1000, 8, 60, 4, seed=3)
    cfg = capi.config(1000, 8, 60, 4, 7, 7, TWO)
    for _ in range(2):
        _check(cfg, small["topk_idx"], oracle_mod)


def test_noalloc_scratch_limit(oracle_mod):
    """A configuration whose histograms fill the fixed array exactly is
    taken; one more token is refused before anything runs, with every other
    argument valid, so only the size limit can refuse it."""
    build.build()
    E, k, R = 256, 1, 8
    T_max = capi.MOE_LAYOUT_NOALLOC_SCRATCH_BYTES // (4 * E) * 256   # 4096 chunks of 256 tokens
    rng = np.random.default_rng(11)
    topk_np = rng.integers(0, E, size=(T_max + 1, k), dtype=np.int32)

    over = capi.config(T_max + 1, 8, E, k, R)
    lay = buffers.DeviceLayout(over)
    topk = torch.from_numpy(topk_np).cuda()
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_layout_noalloc(over, topk, _noalloc_struct(lay))
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert int(lay.expert_counts.abs().sum()) == 0, "a refused call writes nothing"
    # the same arrays are fine for moe_layout (caller workspace), so the
    # refusal came from the scratch size alone
    capi.moe_layout(over, topk, lay.struct)
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK

    at = capi.config(T_max, 8, E, k, R)
    _check(at, topk_np[:T_max], oracle_mod)
