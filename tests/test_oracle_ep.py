"""Pins for the oracle's sharded-source layout (CPU only).

Expert parallelism over real GPUs shards the source tokens: rank g routes
tokens [shard_begin[g], shard_begin[g+1]) and every rank's receive buffer
holds its experts' rows ("[None][feat] support non-divisible EP in MoE
alltoall and slurm benchmark", TensorRT-LLM PR #13888; FUSCO article,
section "FUSCO 的核心创新").  The reading taken orders an expert's rows by
source rank, then by the source's token order.  The oracle builds it the way
a sharded system does (per-source counts, exchange, offsets, per-source
cursors); these tests pin it against an independent formulation (sort the
(expert, source, token, column) tuples and read off positions), against the
per-source histograms, and against the single-source layout, which it must
equal when the shards are contiguous and in rank order.
"""
import numpy as np
import pytest

from combine_moe_layout_06_b200 import inputs


def _random_topk(rng, T, E, k):
    if T == 0:
        return np.zeros((0, k), np.int32)
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)


def _brute(topk, E, shard_begin):
    T, k = topk.shape
    src = np.searchsorted(np.asarray(shard_begin), np.arange(T), side="right") - 1
    tuples = sorted((int(topk[t, j]), int(src[t]), t, j) for t in range(T) for j in range(k))
    slot = np.full((T, k), -1, np.int64)
    for pos, (_, _, t, j) in enumerate(tuples):
        slot[t, j] = pos
    return slot


CASES = [
    # T, E, k, R, shard sizes
    (10, 6, 2, 3, [4, 0, 6]),
    (33, 13, 4, 5, [7, 7, 7, 7, 5]),
    (40, 16, 8, 4, [0, 40, 0, 0]),
    (64, 60, 4, 7, [1, 2, 3, 4, 5, 6, 43]),
    (0, 8, 2, 2, [0, 0]),
    (19, 9, 9, 3, [10, 9, 0]),
]


@pytest.mark.parametrize("T,E,k,R,sizes", CASES)
def test_ep_layout_matches_sorted_tuples(oracle_mod, T, E, k, R, sizes):
    rng = np.random.default_rng(T * 7 + E)
    topk = _random_topk(rng, T, E, k)
    sb = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    got = oracle_mod.ep_layout(topk, E, R, sb)
    assert np.array_equal(got["slot"].astype(np.int64), _brute(topk, E, sb))
    for g in range(len(sizes)):
        part = topk[sb[g]:sb[g + 1]].ravel()
        assert np.array_equal(got["counts"][g], np.bincount(part, minlength=E))
    assert got["expert_offsets"][-1] == T * k


@pytest.mark.parametrize("T,E,k,R,sizes", CASES)
def test_contiguous_shards_equal_single_source(oracle_mod, T, E, k, R, sizes):
    rng = np.random.default_rng(T * 11 + E)
    topk = _random_topk(rng, T, E, k)
    sb = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    ep = oracle_mod.ep_layout(topk, E, R, sb)
    one = oracle_mod.layout(topk, E, R)
    for key in ("slot", "expert_offsets", "rank_offsets"):
        assert np.array_equal(ep[key], one[key]), key


def test_ep_layout_workload_invariants(oracle_mod):
    d = inputs.make("olmoe")
    wl = d["workload"]
    G = wl.R
    sb = (np.arange(G + 1) * wl.T) // G
    ep = oracle_mod.ep_layout(d["topk_idx"], wl.E, wl.R, sb)
    s = ep["slot"].ravel()
    assert np.array_equal(np.sort(s), np.arange(wl.T * wl.k))
    # every row lies in its expert's segment, and rank r's rows are those of its experts
    e = d["topk_idx"].ravel()
    assert np.all((s >= ep["expert_offsets"][e]) & (s < ep["expert_offsets"][e + 1]))


def test_ep_layout_refusals(oracle_mod):
    topk = np.array([[0, 1], [2, 3]], np.int32)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.ep_layout(topk, 4, 2, np.array([0, 1], np.int64))       # shards end early
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.ep_layout(topk, 4, 2, np.array([0, 2, 1, 2], np.int64))  # decreasing
