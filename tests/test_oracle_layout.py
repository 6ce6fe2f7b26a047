"""Pins for the oracle's layout (CPU only).

The oracle assigns receive rows with one cursor per expert walked in token
order.  These tests check it against an independent formulation (sort all
(expert, token, column) triples and read off positions), against the
invariants a segment-descriptor layout must satisfy (counts sum to T*k, the
slot map is a bijection onto the receive buffer, rows of one expert are in
token order and inside that expert's segment), and against brute-force node
staging maps.  Reading: receive buffer is expert-major, ascending token index
inside an expert (FUSCO article, section "FUSCO 的核心创新", gives the
descriptor idea but not its contents).
"""
import itertools

import numpy as np
import pytest

from combine_moe_layout_06_b200 import inputs


def _brute_layout(topk, E, R, N):
    T, k = topk.shape
    triples = sorted((int(topk[t, j]), t, j) for t in range(T) for j in range(k))
    slot = np.full((T, k), -1, np.int64)
    for pos, (_, t, j) in enumerate(triples):
        slot[t, j] = pos
    counts = np.bincount(topk.ravel(), minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    # ranks from the ceil/floor rule, written from base/remainder
    base, rem = E // R, E % R
    sizes = [base + (1 if r < rem else 0) for r in range(R)]
    first = np.concatenate([[0], np.cumsum(sizes)])
    rank_offsets = offsets[first]
    rank_of = np.repeat(np.arange(R), sizes)
    node_of = rank_of // (R // N)
    node_slot = np.full((T, N), -1, np.int64)
    node_counts = np.zeros(N, np.int64)
    node_src = []
    for n in range(N):
        toks = [t for t in range(T) if any(node_of[topk[t, j]] == n for j in range(k))]
        for i, t in enumerate(toks):
            node_slot[t, n] = i
        node_counts[n] = len(toks)
        node_src += toks                     # staging rows of node n, in token order
    node_offsets = np.concatenate([[0], np.cumsum(node_counts)])
    return dict(slot=slot, expert_counts=counts, expert_offsets=offsets,
                rank_offsets=rank_offsets, node_slot=node_slot,
                node_counts=node_counts, node_offsets=node_offsets,
                node_src=np.array(node_src, np.int64))


def _random_topk(rng, T, E, k):
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32).reshape(T, k)


CASES = [
    # T, E, k, R, N
    (1, 1, 1, 1, 1),
    (5, 4, 2, 2, 1),
    (7, 8, 3, 4, 2),
    (33, 13, 4, 5, 1),
    (40, 16, 8, 8, 4),
    (64, 60, 4, 7, 7),
    (19, 9, 9, 3, 3),
    (0, 6, 2, 3, 1),
]


@pytest.mark.parametrize("T,E,k,R,N", CASES)
def test_layout_matches_brute_force(oracle_mod, T, E, k, R, N):
    rng = np.random.default_rng(T * 131 + E)
    topk = _random_topk(rng, T, E, k) if T else np.zeros((0, k), np.int32)
    got = oracle_mod.layout(topk, E, R, N, nodes=True)
    ref = _brute_layout(topk, E, R, N)
    for key in ref:
        assert np.array_equal(np.asarray(got[key], np.int64), ref[key]), key


@pytest.mark.parametrize("name", ["tiny"])
def test_layout_invariants_workload(oracle_mod, name):
    d = inputs.make(name)
    wl = d["workload"]
    topk = d["topk_idx"]
    lay = oracle_mod.layout(topk, wl.E, wl.R, wl.N, nodes=True)
    _check_invariants(topk, lay, wl.E, wl.R, wl.N)
    ref = _brute_layout(topk, wl.E, wl.R, wl.N)
    assert np.array_equal(lay["slot"], ref["slot"])


def _check_invariants(topk, lay, E, R, N):
    T, k = topk.shape
    slot = lay["slot"]
    counts = lay["expert_counts"]
    offs = lay["expert_offsets"]
    assert counts.sum() == T * k
    assert offs[0] == 0 and offs[-1] == T * k
    assert np.array_equal(np.diff(offs), counts)
    flat = np.sort(slot.ravel())
    assert np.array_equal(flat, np.arange(T * k)), "bijection onto [0, T*k)"
    e = topk.ravel()
    s = slot.ravel()
    assert np.all(s >= offs[e]) and np.all(s < offs[e + 1]), "slot inside its segment"
    t_of = np.repeat(np.arange(T), k)
    for ex in range(E):
        m = e == ex
        order = np.argsort(s[m])
        assert np.all(np.diff(t_of[m][order]) > 0), "token order inside an expert"
    # node staging: each token at most once per node, U = distinct (t, node)
    ns = lay["node_slot"]
    for n in range(N):
        col = ns[:, n]
        used = col[col >= 0]
        assert np.array_equal(np.sort(used), np.arange(used.size))
        assert np.all(np.diff(used) > 0)
    assert lay["node_offsets"][-1] == int((ns >= 0).sum())


@pytest.mark.parametrize("name", ["olmoe", "qwen3", "dsv3", "longctx"])
def test_layout_invariants_full_workloads(oracle_mod, name):
    d = inputs.make(name)
    wl = d["workload"]
    topk = d["topk_idx"]
    lay = oracle_mod.layout(topk, wl.E, wl.R, wl.N, nodes=True)
    T, k = topk.shape
    slot = lay["slot"].ravel()
    assert np.array_equal(np.bincount(slot, minlength=T * k), np.ones(T * k, np.int64))
    assert np.array_equal(lay["expert_counts"], np.bincount(topk.ravel(), minlength=wl.E))
    # rows of an expert: sorted by slot means sorted by token
    e = topk.ravel()
    t_of = np.repeat(np.arange(T), k)
    key = np.lexsort((t_of, e))          # expert-major, token order
    assert np.array_equal(slot[key], np.arange(T * k))
    if wl.N > 1:
        per_node = wl.E // wl.N
        touched = np.zeros((T, wl.N), bool)
        np.put_along_axis(touched, topk // per_node, True, axis=1)
        assert np.array_equal(lay["node_slot"] >= 0, touched)
        assert np.array_equal(lay["node_counts"], touched.sum(0))


def test_layout_refusals(oracle_mod):
    topk = np.array([[0, 1], [2, 3]], np.int32)
    with pytest.raises(oracle_mod.OracleError) as ei:
        oracle_mod.layout(np.array([[0, 4]], np.int32), 4, 2)
    assert ei.value.code == oracle_mod.EXPERT_OOB
    with pytest.raises(oracle_mod.OracleError) as ei:
        oracle_mod.layout(np.array([[-1, 2]], np.int32), 4, 2)
    assert ei.value.code == oracle_mod.EXPERT_OOB
    with pytest.raises(oracle_mod.OracleError) as ei:
        oracle_mod.layout(np.array([[1, 1]], np.int32), 4, 2)
    assert ei.value.code == oracle_mod.DUP_EXPERT
    # out-of-range wins over a repeat
    with pytest.raises(oracle_mod.OracleError) as ei:
        oracle_mod.layout(np.array([[1, 1], [0, 9]], np.int32), 4, 2)
    assert ei.value.code == oracle_mod.EXPERT_OOB
    with pytest.raises(oracle_mod.OracleError) as ei:
        oracle_mod.layout(topk, 4, 5)
    assert ei.value.code == oracle_mod.EMPTY_RANK
    with pytest.raises(oracle_mod.OracleError) as ei:
        oracle_mod.layout(topk, 4, 4, 3, nodes=True)
    assert ei.value.code == oracle_mod.BAD_NODES
    with pytest.raises(oracle_mod.OracleError) as ei:
        oracle_mod.layout(np.zeros((1, 5), np.int32), 4, 2)
    assert ei.value.code == oracle_mod.INVALID_ARG


def test_exhaustive_tiny(oracle_mod):
    """Every 2-token routing over 4 experts with k=2 (all ordered pairs)."""
    pairs = [p for p in itertools.permutations(range(4), 2)]
    for a in pairs:
        for b in pairs:
            topk = np.array([a, b], np.int32)
            got = oracle_mod.layout(topk, 4, 2, 2, nodes=True)
            ref = _brute_layout(topk, 4, 2, 2)
            for key in ("slot", "expert_offsets", "rank_offsets", "node_slot", "node_src"):
                assert np.array_equal(np.asarray(got[key], np.int64), ref[key])
