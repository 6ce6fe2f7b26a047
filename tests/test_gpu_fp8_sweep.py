"""GPU parity of the fp8 two-level dispatch over a seeded random sweep of
shapes: T, H, E, k, R, N and the form (one kernel, or the split form with
MOE_FLAG_TWO_LEVEL_SPLIT) drawn from a fixed seed.  Hidden sizes span even
and odd numbers of 16-value groups (the one kernel's 32-byte and 16-byte
accesses), every launch shape of that kernel (up to 8192 values per row),
rows that are not a multiple of 16 values (the split form whatever the
flag), and N + k up to the one kernel's limit of 32.  Receive codes and
scales must equal the oracle's fp8 dispatch and the staging rows its
quantizer of the staged tokens, bit for bit, with no stray staging writes."""
import numpy as np
import pytest
import torch

import moe_testlib as M
from combine_moe_layout_06_b200 import capi, inputs

pytestmark = pytest.mark.gpu


def _cases(n=40, seed=20261203):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        R = int(rng.choice([2, 4, 6, 8, 12, 16]))
        divisors = [d for d in range(2, R + 1) if R % d == 0]
        N = int(rng.choice(divisors))
        E = int(rng.integers(R, 257))
        k = int(rng.integers(1, min(E, 32 - N) + 1))
        T = int(rng.choice([int(rng.integers(1, 200)), int(rng.integers(200, 1500))]))
        kind = int(rng.choice(3, p=[0.5, 0.4, 0.1]))
        if kind == 0:      # even group count: 32-byte accesses
            H = 32 * int(rng.integers(1, 257))
        elif kind == 1:    # odd group count: 16-byte accesses
            H = 16 * (2 * int(rng.integers(0, 256)) + 1)
        else:              # not a multiple of 16 values: the split form
            H = 8 * (2 * int(rng.integers(1, 200)) + 1)
        form = capi.MOE_FLAG_TWO_LEVEL_SPLIT if rng.random() < 0.2 else 0
        out.append((i, T, H, E, k, R, N, form))
    return out


@pytest.mark.parametrize("case", _cases(), ids=lambda c: f"c{c[0]}-T{c[1]}-H{c[2]}-E{c[3]}-k{c[4]}-R{c[5]}-N{c[6]}-f{c[7]}")
def test_fp8_two_level_random_shapes(oracle_mod, case):
    _, T, H, E, k, R, N, form = case
    d = inputs.make_random(T, H, E, k, seed=T * 5 + H + N)
    x, topk = d["x"], d["topk_idx"]
    ref = oracle_mod.layout(topk, E, R, N, nodes=True)
    cfg = M.cfg_of(T, H, E, k, R, N, capi.MOE_FLAG_TWO_LEVEL | form)
    lay, _ = M.gpu_layout(cfg, topk)
    rows = capi.moe_node_staging_rows(cfg)
    st_q = torch.full((rows, H), 0x55, dtype=torch.uint8, device="cuda")
    st_s = torch.zeros(rows, dtype=torch.float32, device="cuda")
    recv_q = torch.empty((T * k, H), dtype=torch.uint8, device="cuda")
    recv_s = torch.empty(T * k, dtype=torch.float32, device="cuda")
    capi.moe_dispatch_fp8_two_level(cfg, lay.struct, M.to_dev(x), st_q, st_s, recv_q, recv_s)
    assert capi.moe_get_error(lay.struct) == capi.MOE_OK
    rq, rs = oracle_mod.dispatch_fp8(x, ref["slot"])
    assert np.array_equal(recv_q.cpu().numpy(), rq)
    assert np.array_equal(recv_s.cpu().numpy(), rs)
    xq, xs = oracle_mod.quantize_rows_fp8(x)
    U = int(ref["node_offsets"][-1])
    st = st_q.cpu().numpy()
    assert np.array_equal(st[:U], xq[ref["node_src"]])
    assert np.array_equal(st_s.cpu().numpy()[:U], xs[ref["node_src"]])
    assert np.all(st[U:] == 0x55), "no stray staging writes"
