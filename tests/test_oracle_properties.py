"""Property-based pins for the oracle (CPU only, hypothesis): random small
configurations, including non-divisible partitions, k = E, empty rows of
experts and uneven source shards, each checked against an independent
formulation written here (sorted tuples for the layouts, set arithmetic for
the node staging, a bound on an fp64 sum for the combine)."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from combine_moe_layout_06_b200 import inputs

SETTINGS = settings(max_examples=60, deadline=None,
                    suppress_health_check=[HealthCheck.function_scoped_fixture])


@st.composite
def problems(draw):
    E = draw(st.integers(1, 12))
    k = draw(st.integers(1, E))
    R = draw(st.integers(1, E))
    N = draw(st.sampled_from([n for n in range(1, R + 1) if R % n == 0]))
    T = draw(st.integers(0, 30))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    rng = np.random.default_rng(seed)
    topk = (np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
            if T else np.zeros((0, k), np.int32))
    return T, E, k, R, N, topk, seed


def _rank_sizes(E, R):
    base, rem = divmod(E, R)
    return [base + (1 if r < rem else 0) for r in range(R)]


@SETTINGS
@given(problems())
def test_layout_is_sorted_tuples(oracle_mod, p):
    T, E, k, R, N, topk, _ = p
    lay = oracle_mod.layout(topk, E, R, N, nodes=True)
    order = sorted((int(topk[t, j]), t, j) for t in range(T) for j in range(k))
    want = np.full((T, k), -1, np.int64)
    for pos, (_, t, j) in enumerate(order):
        want[t, j] = pos
    assert np.array_equal(lay["slot"].astype(np.int64), want)
    first = np.concatenate([[0], np.cumsum(_rank_sizes(E, R))])
    assert np.array_equal(lay["rank_offsets"], lay["expert_offsets"][first])
    # node staging: one row per (token, node touched), node-major, token order
    node_of = np.repeat(np.arange(R), _rank_sizes(E, R)) // (R // N)
    src = [t for n in range(N) for t in range(T) if any(node_of[e] == n for e in topk[t])]
    assert np.array_equal(lay["node_src"], np.array(src, np.int64))


@SETTINGS
@given(problems(), st.integers(1, 4))
def test_sharded_layout_is_sorted_tuples(oracle_mod, p, G):
    T, E, k, R, N, topk, seed = p
    cuts = np.sort(np.random.default_rng(seed).integers(0, T + 1, G - 1))
    sb = np.concatenate([[0], cuts, [T]]).astype(np.int64)
    ep = oracle_mod.ep_layout(topk, E, R, sb)
    src = np.searchsorted(sb, np.arange(T), side="right") - 1
    order = sorted((int(topk[t, j]), int(src[t]), t, j) for t in range(T) for j in range(k))
    want = np.full((T, k), -1, np.int64)
    for pos, (_, _, t, j) in enumerate(order):
        want[t, j] = pos
    assert np.array_equal(ep["slot"].astype(np.int64), want)


@SETTINGS
@given(problems(), st.integers(1, 24))
def test_two_level_and_combine(oracle_mod, p, H):
    T, E, k, R, N, topk, seed = p
    x = inputs.random_bf16((T, H), seed=seed % 1000)
    lay = oracle_mod.layout(topk, E, R, N, nodes=True)
    flat = oracle_mod.dispatch_flat(x, lay["slot"])
    _, two = oracle_mod.dispatch_two_level(x, lay, R, N)
    assert np.array_equal(two, flat)
    w = np.random.default_rng(seed).random((T, k)).astype(np.float32)
    y = oracle_mod.combine(flat, w, lay["slot"])
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    yf = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # every row of token t is x[t]: y = bf16(x * sum of the weights), within
    # the fp32 FMA chain and one bf16 rounding
    exact = xf * w.astype(np.float64).sum(axis=1, keepdims=True)
    bound = 2.0 ** -8 * np.abs(exact) + (k + 1) * 2.0 ** -24 * np.abs(xf) * w.sum(1, keepdims=True) + 1e-40
    assert np.all(np.abs(yf - exact) <= bound)
