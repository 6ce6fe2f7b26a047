"""GPU parity over a seeded random sweep of problem shapes and engine flags.

Each case draws T, H, E, k, R, N and a flag combination from a fixed seed,
runs layout, dispatch (flat or two-level, every engine) and combine through
the C ABI, and compares with the oracle: layout arrays, receive rows and
staging rows bit for bit, combine bit for bit (and within the combine
tolerance).  The shapes reach ragged tails (T not a multiple of a chunk),
rows of 2-, 4- and 16-byte vectors, k up to 32, more than one node and the
histogram paths of both the single-chunk and multi-chunk layouts.
"""
import numpy as np
import pytest

import moe_testlib as M
from combine_moe_layout_06_b200 import capi, inputs

pytestmark = pytest.mark.gpu

TWO = capi.MOE_FLAG_TWO_LEVEL
FLAG_CHOICES = [0, TWO, TWO | capi.MOE_FLAG_TWO_LEVEL_SPLIT, capi.MOE_FLAG_COPY_VECTOR,
                TWO | capi.MOE_FLAG_COPY_VECTOR, capi.MOE_FLAG_COPY_BULK,
                TWO | capi.MOE_FLAG_COPY_BULK, capi.MOE_FLAG_LAYOUT_CLUSTER,
                TWO | capi.MOE_FLAG_LAYOUT_CLUSTER]


def _cases(n=40, seed=20261202):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        E = int(rng.integers(1, 300))
        k = int(rng.integers(1, min(E, 32) + 1))
        R = int(rng.integers(1, min(E, 32) + 1))
        divisors = [d for d in range(1, R + 1) if R % d == 0 and d <= 32]
        N = int(rng.choice(divisors))
        T = int(rng.choice([int(rng.integers(0, 300)), int(rng.integers(300, 3000))]))
        H = int(rng.choice([int(rng.integers(1, 128)), int(rng.integers(1, 64)) * 2,
                            int(rng.integers(1, 128)) * 8]))
        flags = int(rng.choice(FLAG_CHOICES))
        out.append((i, T, H, E, k, R, N, flags))
    return out


@pytest.mark.parametrize("case", _cases(), ids=lambda c: f"c{c[0]}-T{c[1]}-H{c[2]}-E{c[3]}-k{c[4]}-R{c[5]}-N{c[6]}-f{c[7]}")
def test_random_shape_parity(oracle_mod, case):
    _, T, H, E, k, R, N, flags = case
    d = inputs.make_random(max(T, 1), H, E, k, seed=T * 7 + E * 3 + k)
    x, topk, w = d["x"][:T], d["topk_idx"][:T], d["topk_w"][:T]
    two = bool(flags & TWO)
    ref = oracle_mod.layout(topk, E, R, N, nodes=True)
    cfg = M.cfg_of(T, H, E, k, R, N, flags)
    lay, _ = M.gpu_layout(cfg, topk)
    want = ref if two else {k_: v for k_, v in ref.items() if not k_.startswith("node")}
    M.assert_layout_equal(lay.host(), want)
    if T == 0:
        assert capi.moe_get_error(lay.struct) == capi.MOE_OK
        return
    x_dev = M.to_dev(x)
    recv, staging = M.gpu_dispatch(cfg, lay, x_dev, fill=0x7F81)
    assert np.array_equal(M.bits(recv), oracle_mod.dispatch_flat(x, ref["slot"]))
    if two:
        staging_ref, _ = oracle_mod.dispatch_two_level(x, ref, R, N)
        U = int(ref["node_offsets"][-1])
        st = M.bits(staging)
        assert np.array_equal(st[:U], staging_ref)
        assert np.all(st[U:] == 0x7F81), "no stray staging writes"
    eo = inputs.random_bf16_bits((T * k, H), seed=T + H + k)
    y = M.bits(M.gpu_combine(cfg, lay, M.to_dev(eo), w))
    y_ref = oracle_mod.combine(eo, w, ref["slot"])
    M.assert_combine_close(y, y_ref)
    assert np.array_equal(y, y_ref)
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK
