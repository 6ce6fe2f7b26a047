"""Host side of expert parallelism over sharded sources, on CPU (gloo, world
size 2 and 3): the count all-gather, in source-rank order, and the rows each
rank receives (the library's moe_ep_receive_rows), checked against the
oracle's sharded-source layout; and the set-up bench.py runs on every rank
of its multi-GPU step."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from combine_moe_layout_06_b200 import build
    build.build()


def _rank_main(rank, world, port, topk, sb, E, out):
    import datetime

    import torch
    import torch.distributed as dist

    from combine_moe_layout_06_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = topk[sb[rank]:sb[rank + 1]].ravel()
        counts = torch.from_numpy(np.bincount(mine, minlength=E).astype(np.int32))
        counts_all = ep.gather_counts(counts)
        out.put((rank, counts_all.numpy(), ep.receive_rows(counts_all.numpy(), world)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,sizes,E,k", [(2, [30, 11], 13, 4), (3, [0, 25, 8], 9, 3)])
def test_count_exchange_and_receive_rows_gloo(oracle_mod, world, sizes, E, k):
    rng = np.random.default_rng(world * 5 + E)
    T = sum(sizes)
    topk = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    sb = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    ref = oracle_mod.ep_layout(topk, E, world, sb)
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, topk, sb, E, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted((out.get(timeout=10) for _ in range(world)), key=lambda g: g[0])
    want_rows = np.diff(ref["rank_offsets"])
    for rank, counts_all, rows in got:
        assert np.array_equal(counts_all, ref["counts"]), "source-rank order on every rank"
        assert np.array_equal(rows, want_rows)


def test_receive_rows_partition():
    from combine_moe_layout_06_b200 import ep
    counts_all = np.array([[1, 2, 3, 4, 5, 6, 7], [7, 6, 5, 4, 3, 2, 1]])
    # 7 experts on 3 ranks: 3, 2, 2
    assert ep.receive_rows(counts_all, 3).tolist() == [24, 16, 16]


@pytest.mark.parametrize("G,E,R,k,seed", [(1, 8, 2, 2, 0), (3, 60, 7, 4, 1), (4, 256, 8, 8, 2),
                                          (2, 9, 9, 3, 3), (5, 37, 4, 5, 4)])
def test_receive_rows_against_oracle_sharded_layout(oracle_mod, G, E, R, k, seed):
    """moe_ep_receive_rows over every source's counts equals the row counts
    of the oracle's sharded-source layout (rank_offsets differences)."""
    from combine_moe_layout_06_b200 import capi
    rng = np.random.default_rng(seed)
    sizes = rng.integers(0, 50, size=G)
    T = int(sizes.sum())
    topk = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32).reshape(T, k)
    sb = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    ref = oracle_mod.ep_layout(topk, E, R, sb)
    counts_all = np.stack([np.bincount(topk[sb[g]:sb[g + 1]].ravel(), minlength=E)
                           for g in range(G)]).astype(np.int32)
    assert np.array_equal(counts_all, ref["counts"])
    assert capi.moe_ep_receive_rows(counts_all, R) == np.diff(ref["rank_offsets"]).tolist()


def test_receive_rows_refusals():
    from combine_moe_layout_06_b200 import capi
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_ep_receive_rows(np.zeros((2, 3), np.int32), 4)      # E < R
    assert ei.value.status == capi.MOE_ERR_EMPTY_RANK
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_ep_receive_rows(np.array([[1, -1, 2]], np.int32), 2)  # negative count
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_ep_receive_rows(np.zeros((1, 3), np.int32), 0)
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG


def _bench_plan_rank(rank, world, port, topk, sb, E, out):
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = topk[sb[rank]:sb[rank + 1]].ravel()
        local = torch.from_numpy(np.bincount(mine, minlength=E).astype(np.int32))
        buf = torch.zeros((world, E), dtype=torch.int32)
        counts_all, rows, cap = bench.ep_plan(local, world, out=buf)
        assert counts_all.data_ptr() == buf.data_ptr(), "gathered in place"
        out.put((rank, counts_all.numpy().copy(), list(rows), cap))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,sizes,E,k", [(2, [40, 17], 10, 3), (3, [5, 0, 31], 7, 2)])
def test_bench_expert_parallel_plan_gloo(oracle_mod, world, sizes, E, k):
    """The set-up bench.py's multi-GPU step runs on every rank (count
    all-gather, rows per expert rank, common capacity), as gloo ranks: every
    rank sees the same counts in source order, the oracle's row counts and
    their maximum."""
    rng = np.random.default_rng(world * 11 + E)
    T = sum(sizes)
    topk = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    sb = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    ref = oracle_mod.ep_layout(topk, E, world, sb)
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bench_plan_rank, args=(r, world, port, topk, sb, E, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted((out.get(timeout=10) for _ in range(world)), key=lambda g: g[0])
    want_rows = np.diff(ref["rank_offsets"]).tolist()
    for rank, counts_all, rows, cap in got:
        assert np.array_equal(counts_all, ref["counts"])
        assert rows == want_rows
        assert cap == max(max(want_rows), 1)
