"""Pins for the oracle's dispatch, two-level dispatch, combine and bf16
conversion (CPU only).

Dispatch is pinned by the property that defines it (every destination row is
a bit copy of its token's row), two-level dispatch by equality with flat
dispatch plus the node-dedup count (FUSCO article, section
"负载均衡与跨节点去重": one copy per node touched), combine by closed forms
(k = 1 with weight 1 is the identity; an identity expert with weights summing
to one returns x), by an fp64 sum inside the fp32/bf16 rounding bound, and
the bf16 rounding by torch's CPU conversion (a library routine).
"""
import numpy as np
import pytest
import torch

from combine_moe_layout_06_b200 import inputs


def _bits_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------------------ bf16

def test_bf16_rne_matches_torch(oracle_mod):
    rng = np.random.default_rng(3)
    vals = np.concatenate([
        rng.standard_normal(200000).astype(np.float32),
        (rng.standard_normal(20000) * 1e30).astype(np.float32),
        (rng.standard_normal(20000) * 1e-38).astype(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, -3.3895314e38,
                  1e-45, -1e-45, 1.0, -1.0], np.float32),
    ])
    # exact ties: upper half odd/even with dropped bits exactly 0x8000
    hi = rng.integers(0, 0x7F7F, 5000).astype(np.uint32)
    ties = ((hi << 16) | 0x8000).view(np.float32)
    near = ((hi << 16) | 0x7FFF).view(np.float32)
    above = ((hi << 16) | 0x8001).view(np.float32)
    vals = np.concatenate([vals, ties, near, above])
    got = oracle_mod.f32_to_bf16(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_nan_and_widening(oracle_mod):
    nan_bits = np.array([0x7FC00000, 0xFFC00000, 0x7F800001, 0x7FA00000], np.uint32)
    out = oracle_mod.f32_to_bf16(nan_bits.view(np.float32))
    back = oracle_mod.bf16_to_f32(out)
    assert np.all(np.isnan(back))
    assert np.array_equal(out >> 15, (nan_bits >> 31).astype(np.uint16)), "sign kept"
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    wide = oracle_mod.bf16_to_f32(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    finite = ~np.isnan(ref)
    assert np.array_equal(wide[finite].view(np.uint32), ref[finite].view(np.uint32))


# ------------------------------------------------------------------ dispatch

def _case(T, H, E, k, R, N, seed):
    d = inputs.make_random(T, H, E, k, seed)
    return d["x"], d["topk_idx"], d["topk_w"]


CASES = [(1, 8, 4, 1, 1, 1), (7, 64, 8, 3, 4, 2), (33, 136, 13, 4, 5, 5),
         (100, 16, 32, 8, 8, 4), (65, 9, 16, 16, 4, 2)]


@pytest.mark.parametrize("T,H,E,k,R,N", CASES)
def test_dispatch_rows_are_copies(oracle_mod, T, H, E, k, R, N):
    x, topk, _ = _case(T, H, E, k, R, N, seed=T + H)
    lay = oracle_mod.layout(topk, E, R, N, nodes=True)
    recv = oracle_mod.dispatch_flat(x, lay["slot"])
    for t in range(T):
        for j in range(k):
            assert np.array_equal(recv[lay["slot"][t, j]], x[t])
    # every row written exactly once: rows grouped by expert hold their tokens
    rows_expert = np.repeat(np.arange(E), lay["expert_counts"])
    assert np.array_equal(np.sort(topk.ravel()), rows_expert)


@pytest.mark.parametrize("T,H,E,k,R,N", CASES)
def test_two_level_equals_flat_and_dedups(oracle_mod, T, H, E, k, R, N):
    x, topk, _ = _case(T, H, E, k, R, N, seed=3 * T + H)
    lay = oracle_mod.layout(topk, E, R, N, nodes=True)
    flat = oracle_mod.dispatch_flat(x, lay["slot"])
    staging, recv = oracle_mod.dispatch_two_level(x, lay, R, N)
    assert np.array_equal(recv, flat)
    first = oracle_mod.partition(E, R)
    node_of = np.repeat(np.arange(R), np.diff(first)) // (R // N)
    pairs = {(t, int(node_of[e])) for t in range(T) for e in topk[t]}
    assert staging.shape[0] == len(pairs), "one staging row per (token, node)"
    for n in range(N):
        lo, hi = lay["node_offsets"][n], lay["node_offsets"][n + 1]
        toks = sorted(t for (t, m) in pairs if m == n)
        assert hi - lo == len(toks)
        for i, t in enumerate(toks):
            assert np.array_equal(staging[lo + i], x[t])


# ------------------------------------------------------------------ combine

def test_combine_k1_unit_weight_is_identity(oracle_mod):
    x, topk, _ = _case(50, 40, 6, 1, 3, 1, seed=11)
    lay = oracle_mod.layout(topk, 6, 3)
    recv = oracle_mod.dispatch_flat(x, lay["slot"])
    y = oracle_mod.combine(recv, np.ones((50, 1), np.float32), lay["slot"])
    assert np.array_equal(y, x)


@pytest.mark.parametrize("T,H,E,k,R,N", CASES)
def test_round_trip_identity_expert(oracle_mod, T, H, E, k, R, N):
    x, topk, w = _case(T, H, E, k, R, N, seed=5 * T + H)   # renormalised
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)
    lay = oracle_mod.layout(topk, E, R, N)
    recv = oracle_mod.dispatch_flat(x, lay["slot"])
    y = _bits_to_f64(oracle_mod.combine(recv, w, lay["slot"]))
    xf = _bits_to_f64(x)
    assert np.all(np.abs(y - xf) <= 1e-3 + 1e-2 * np.abs(xf))


def _bound(terms):
    """fp32 FMA chain then one bf16 rounding: |err| <= 2^-8 |exact| +
    (1 + 2^-8) k 2^-24 sum|terms| (each FMA rounds once)."""
    exact = terms.sum(axis=-1)
    k = terms.shape[-1]
    return exact, 2.0 ** -8 * np.abs(exact) + (1 + 2.0 ** -8) * k * 2.0 ** -24 * np.abs(terms).sum(-1) + 1e-45


@pytest.mark.parametrize("T,H,E,k,R,N", CASES)
def test_combine_within_rounding_bound_of_fp64(oracle_mod, T, H, E, k, R, N):
    x, topk, w = _case(T, H, E, k, R, N, seed=7 * T + H)
    lay = oracle_mod.layout(topk, E, R, N)
    eo = inputs.random_bf16((T * k, H), seed=T * k + H)
    y = _bits_to_f64(oracle_mod.combine(eo, w, lay["slot"]))
    eof = _bits_to_f64(eo)
    terms = w.astype(np.float64)[:, None, :] * np.stack(
        [eof[lay["slot"][:, j]] for j in range(k)], axis=-1)     # [T, H, k]
    exact, bound = _bound(terms)
    assert np.all(np.abs(y - exact) <= bound)


def test_combine_per_expert_scale_closed_form(oracle_mod):
    """eo row of expert e holds bf16(x * (1 + e/64)); y must be
    sum_j w_j bf16(x (1 + e_j/64)) within the rounding bound, so a swap of two
    of a token's rows (identity expert cannot see it) would fail."""
    T, H, E, k, R = 64, 32, 16, 4, 4
    x, topk, w = _case(T, H, E, k, R, 1, seed=99)
    lay = oracle_mod.layout(topk, E, R)
    xf = _bits_to_f64(x)
    scaled = np.empty((T, k, H), np.float64)
    eo = np.zeros((T * k, H), np.uint16)
    for t in range(T):
        for j in range(k):
            e = topk[t, j]
            b = oracle_mod.f32_to_bf16((xf[t] * (1 + e / 64.0)).astype(np.float32))
            eo[lay["slot"][t, j]] = b
            scaled[t, j] = _bits_to_f64(b)
    y = _bits_to_f64(oracle_mod.combine(eo, w, lay["slot"]))
    terms = np.transpose(w.astype(np.float64)[:, :, None] * scaled, (0, 2, 1))
    exact, bound = _bound(terms)
    assert np.all(np.abs(y - exact) <= bound)
    # a variant with two weights swapped must be detectably different
    w_sw = w.copy()
    w_sw[:, [0, 1]] = w_sw[:, [1, 0]]
    y_sw = _bits_to_f64(oracle_mod.combine(eo, w_sw, lay["slot"]))
    assert np.any(np.abs(y_sw - exact) > bound)


def test_combine_tokens_subset_matches_full(oracle_mod):
    x, topk, w = _case(40, 24, 8, 3, 2, 1, seed=5)
    lay = oracle_mod.layout(topk, 8, 2)
    eo = inputs.random_bf16((120, 24), seed=2)
    full = oracle_mod.combine(eo, w, lay["slot"])
    toks = np.array([39, 0, 17, 17, 5])
    assert np.array_equal(oracle_mod.combine_tokens(eo, w, lay["slot"], toks), full[toks])


def test_combine_accumulation_order_is_column_order(oracle_mod):
    """fp32 is not associative: pick values where j order matters and check
    the oracle's result equals the left-to-right fp32 FMA chain."""
    big, small = np.float32(2.0 ** 8), np.float32(2.0 ** -9)
    eo_f = np.array([[big], [small], [-big]], np.float32)   # rows j = 0, 1, 2
    eo = oracle_mod.f32_to_bf16(eo_f)
    slot = np.array([[0, 1, 2]], np.int32)
    w = np.ones((1, 3), np.float32)
    y = _bits_to_f64(oracle_mod.combine(eo, w, slot))
    # ((0 + 256) + 2^-9) rounds to 256 in fp32? no: 256 + 2^-9 is exact in
    # fp32 (24-bit mantissa spans 2^8 .. 2^-15), then - 256 leaves 2^-9.
    assert y[0, 0] == 2.0 ** -9
    eo2 = oracle_mod.f32_to_bf16(np.array([[2.0 ** 20], [2.0 ** -9], [-(2.0 ** 20)]], np.float32))
    y2 = _bits_to_f64(oracle_mod.combine(eo2, w, slot))
    assert y2[0, 0] == 0.0, "2^20 + 2^-9 rounds back to 2^20 in fp32 before the subtraction"


# ------------------------------------------------------------ reduce-scatter order

@pytest.mark.parametrize("T,H,E,k,R,N", CASES)
def test_rank_partial_combine_within_rounding_bound(oracle_mod, T, H, E, k, R, N):
    """Per-rank fp32 partials added in rank order: within the bound of the
    fp64 sum (k FMAs plus R adds, one bf16 rounding)."""
    x, topk, w = _case(T, H, E, k, R, N, seed=11 * T + H)
    lay = oracle_mod.layout(topk, E, R, N)
    eo = inputs.random_bf16_bits((T * k, H), seed=T + 3 * H)
    y = _bits_to_f64(oracle_mod.combine_rank_partials(eo, w, lay["slot"], lay["rank_offsets"]))
    eof = _bits_to_f64(eo)
    terms = w.astype(np.float64)[:, None, :] * np.stack(
        [eof[lay["slot"][:, j]] for j in range(k)], axis=-1)
    exact = terms.sum(-1)
    bound = (2.0 ** -8 * np.abs(exact)
             + (1 + 2.0 ** -8) * (k + R) * 2.0 ** -24 * np.abs(terms).sum(-1) + 1e-45)
    assert np.all(np.abs(y - exact) <= bound)


def test_rank_partial_combine_single_rank_equals_column_order(oracle_mod):
    """With one rank the partial is the whole column-order sum (+0 + p = p)."""
    x, topk, w = _case(90, 48, 12, 3, 1, 1, seed=4)
    lay = oracle_mod.layout(topk, 12, 1)
    eo = inputs.random_bf16_bits((270, 48), seed=8)
    assert np.array_equal(oracle_mod.combine_rank_partials(eo, w, lay["slot"], lay["rank_offsets"]),
                          oracle_mod.combine(eo, w, lay["slot"]))


def test_rank_partial_combine_order_is_rank_order(oracle_mod):
    """Per-rank partials first, then their sum, not one column-order sum
    (fp32 addition is not associative): a token whose expert on rank 1
    carries -2^20 and whose experts on rank 0 carry 2^20 and 2^-9 gives 0
    (rank 0's partial 2^20 + 2^-9 rounds to 2^20 before the -2^20 is added),
    where the column-order sum gives 2^-9."""
    E, R = 4, 2                      # ranks own experts {0,1} and {2,3}
    topk = np.array([[2, 0, 1]], np.int32)
    lay = oracle_mod.layout(topk, E, R)
    vals = {0: 2.0 ** 20, 1: 2.0 ** -9, 2: -(2.0 ** 20)}
    eo = np.zeros((3, 1), np.uint16)
    for j, e in enumerate(topk[0]):
        eo[lay["slot"][0, j], 0] = oracle_mod.f32_to_bf16(np.float32(vals[int(e)])).item()
    w = np.ones((1, 3), np.float32)
    y_rs = _bits_to_f64(oracle_mod.combine_rank_partials(eo, w, lay["slot"], lay["rank_offsets"]))
    y_col = _bits_to_f64(oracle_mod.combine(eo, w, lay["slot"]))
    assert y_rs[0, 0] == 0.0          # (2^20 + 2^-9) - 2^20 in fp32 = 0
    assert y_col[0, 0] == 2.0 ** -9   # -2^20 + 2^20 + 2^-9 in column order


def test_rank_partial_combine_adds_ranks_first_to_last(oracle_mod):
    """Three ranks of one expert each, partials p0 = 1 + 2^-8 (weight 1 + 2^-8
    on 1.0), p1 = p2 = 2^-24.  In rank order each 2^-24 is half an fp32 ulp of
    the running total and rounds away (ties to even), leaving 1 + 2^-8, a bf16
    tie that rounds to 1.0 (0x3F80).  Last rank first would add 2^-24 + 2^-24
    = 2^-23 exactly, then 1 + 2^-8 + 2^-23, which rounds up to 0x3F81.  With
    two ranks the order could not show: a single add commutes."""
    E, R = 3, 3
    topk = np.array([[0, 1, 2]], np.int32)
    lay = oracle_mod.layout(topk, E, R)
    assert list(lay["rank_offsets"]) == [0, 1, 2, 3]
    vals = {0: 1.0, 1: 2.0 ** -24, 2: 2.0 ** -24}
    eo = np.zeros((3, 1), np.uint16)
    for j, e in enumerate(topk[0]):
        eo[lay["slot"][0, j], 0] = oracle_mod.f32_to_bf16(np.float32(vals[int(e)])).item()
    w = np.array([[1.0 + 2.0 ** -8, 1.0, 1.0]], np.float32)
    y = oracle_mod.combine_rank_partials(eo, w, lay["slot"], lay["rank_offsets"])
    assert y[0, 0] == 0x3F80
