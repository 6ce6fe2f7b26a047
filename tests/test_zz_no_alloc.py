"""moe_layout_noalloc(): the layout for callers that cannot allocate device
memory (no cudaMalloc allowed where they run, e.g. inside a stream capture,
or under a framework that owns every allocation).  Its scratch is a fixed
array inside the library, so its results must equal moe_layout()'s, which
uses a caller-provided workspace, call after call.

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


def _both(cfg, topk_np):
    topk = torch.from_numpy(np.ascontiguousarray(topk_np, np.int32)).cuda()
    ref = buffers.DeviceLayout(cfg)
    capi.moe_layout(cfg, topk, ref.struct)
    got = buffers.DeviceLayout(cfg)
    got_struct = capi.layout_struct(got.expert_counts, got.expert_offsets, got.rank_offsets,
                                    got.slot, got.error_word, None, got.node_counts,
                                    got.node_offsets, got.node_slot,
                                    got.node_src)   # no workspace at all
    capi.moe_layout_noalloc(cfg, topk, got_struct)
    torch.cuda.synchronize()
    assert capi.moe_get_error(ref.struct) == capi.MOE_OK
    assert capi.moe_get_error(got_struct) == capi.MOE_OK
    return got.host(), ref.host()


def test_noalloc_layout_matches_allocating_layout_twice():
    build.build()
    assert torch.cuda.is_available()
    # two calls in a row with different problems: the second must not see
    # anything the first left in the shared scratch array
    cases = [("dsv3", TWO), ("longctx", 0)]
    for name, flags in cases:
        d = inputs.make(name)
        wl = d["workload"]
        cfg = capi.config(wl.T, wl.H, wl.E, wl.k, wl.R, wl.N, flags)
        assert capi.moe_layout_workspace_bytes(cfg) <= capi.MOE_LAYOUT_NOALLOC_SCRATCH_BYTES
        got, ref = _both(cfg, d["topk_idx"])
        assert got.keys() == ref.keys()
        for key in ref:
            assert np.array_equal(got[key], ref[key]), (name, key)
    # a batch above the single-cluster limit, whose layout uses the scratch
    big = inputs.make_random(140001, 8, 64, 4, seed=5)
    cfg = capi.config(140001, 8, 64, 4, 8, 2, TWO)
    assert capi.moe_layout_workspace_bytes(cfg) <= capi.MOE_LAYOUT_NOALLOC_SCRATCH_BYTES
    for _ in range(2):
        got, ref = _both(cfg, big["topk_idx"])
        for key in ref:
            assert np.array_equal(got[key], ref[key]), ("big", key)
    # and the same small problem twice in a row
    small = inputs.make_random(1000, 8, 60, 4, seed=3)
    cfg = capi.config(1000, 8, 60, 4, 7, 7, TWO)
    first, ref = _both(cfg, small["topk_idx"])
    second, _ = _both(cfg, small["topk_idx"])
    for key in ref:
        assert np.array_equal(first[key], ref[key]) and np.array_equal(second[key], ref[key])


def test_noalloc_refuses_problems_beyond_its_scratch():
    build.build()
    big = capi.config(1 << 20, 8, 1024, 8, 8)     # needs 16 MiB of histograms
    assert capi.moe_layout_workspace_bytes(big) > capi.MOE_LAYOUT_NOALLOC_SCRATCH_BYTES
    empty = capi.MoeLayout()
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_layout_noalloc(big, 0, empty, stream=0)
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG
