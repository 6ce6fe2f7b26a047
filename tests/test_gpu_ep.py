"""GPU parity of expert parallelism over sharded sources against the
oracle's sharded-source layout, bit for bit.

Single process: G ranks emulated as G shards and G receive / expert-output
buffers on one GPU, each rank's kernels launched in turn on one stream (no
kernel waits on another).  Two processes: two ranks on one GPU with a gloo
group for the count exchange and the barriers, each writing into and
reading from the other's buffers through CUDA IPC mappings.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch

import moe_testlib as M
from combine_moe_layout_06_b200 import buffers, capi, inputs

pytestmark = pytest.mark.gpu

CANARY = 0x7F81


def _shards(T, G, sizes=None):
    if sizes is None:
        return (np.arange(G + 1, dtype=np.int64) * T) // G
    return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)


def _run_virtual(oracle_mod, x, topk, w, eo, E, R, sb, cap_extra=5, engine=0):
    T, k = topk.shape
    H = x.shape[1]
    G = sb.size - 1
    ref = oracle_mod.ep_layout(topk, E, R, sb)
    rows = np.diff(ref["rank_offsets"]).astype(np.int64)
    cap = int(rows.max()) + cap_extra
    M.ensure_lib()
    recv = [torch.full((cap + 3, H), CANARY, dtype=torch.int16, device="cuda").view(torch.bfloat16)
            for _ in range(R)]
    eo_bufs = []
    for r in range(R):
        b = torch.zeros((cap + 3, H), dtype=torch.bfloat16, device="cuda")
        lo, hi = int(ref["rank_offsets"][r]), int(ref["rank_offsets"][r + 1])
        n = min(hi - lo, cap + 3)
        if n > 0:
            b[:n] = buffers.bf16_from_bits(eo[lo:lo + n])
        eo_bufs.append(b)
    ranks = []
    for g in range(G):
        a, b = int(sb[g]), int(sb[g + 1])
        cfg = capi.config(b - a, H, E, k, R, 1, engine)
        lay = buffers.DeviceLayout(cfg)
        tk = torch.from_numpy(np.ascontiguousarray(topk[a:b])).cuda()
        capi.moe_layout(cfg, tk, lay.struct)
        ranks.append((cfg, lay, tk, a, b))
    counts_all = torch.stack([lay.expert_counts for _, lay, _, _, _ in ranks])
    i32 = dict(dtype=torch.int32, device="cuda")
    eps = []
    for g, (cfg, lay, tk, a, b) in enumerate(ranks):
        ep = (torch.zeros(E + 1, **i32), torch.zeros(R + 1, **i32), torch.zeros(max((b - a) * k, 1), **i32))
        st = capi.ep_layout_struct(*ep)
        capi.moe_ep_layout(cfg, g, G, tk, counts_all, lay.struct, st)
        eps.append((ep, st))
    for g, (cfg, lay, tk, a, b) in enumerate(ranks):
        capi.moe_ep_dispatch(cfg, lay.struct, eps[g][1], M.to_dev(x[a:b]), recv, cap)
    ys = []
    for g, (cfg, lay, tk, a, b) in enumerate(ranks):
        y = torch.empty((b - a, H), dtype=torch.bfloat16, device="cuda")
        capi.moe_ep_combine(cfg, lay.struct, eps[g][1], eo_bufs, cap,
                            torch.from_numpy(np.ascontiguousarray(w[a:b])).cuda(), y)
        ys.append(y)
    torch.cuda.synchronize()
    return ref, rows, cap, ranks, eps, recv, ys


def _check(oracle_mod, x, w, eo, ref, rows, ranks, eps, recv, ys):
    recv_ref = oracle_mod.dispatch_flat(x, ref["slot"])
    y_ref = oracle_mod.combine(eo, w, ref["slot"])
    for g, (cfg, lay, tk, a, b) in enumerate(ranks):
        (eo_off, r_off, slot), _ = eps[g]
        assert np.array_equal(eo_off.cpu().numpy(), ref["expert_offsets"])
        assert np.array_equal(r_off.cpu().numpy(), ref["rank_offsets"])
        assert np.array_equal(slot.cpu().numpy()[: (b - a) * cfg.top_k].reshape(b - a, cfg.top_k),
                              ref["slot"][a:b])
        assert np.array_equal(M.bits(ys[g]), y_ref[a:b]), f"combine of rank {g}"
        assert capi.moe_get_error(lay.struct) == capi.MOE_OK
    for r, buf in enumerate(recv):
        got = M.bits(buf)
        lo, hi = ref["rank_offsets"][r], ref["rank_offsets"][r + 1]
        assert np.array_equal(got[: hi - lo], recv_ref[lo:hi]), f"receive buffer of rank {r}"
        assert np.all(got[hi - lo:] == CANARY), "no stray writes"


@pytest.mark.parametrize("name,G", [("olmoe", 4), ("longctx", 7), ("qwen3", 8), ("tiny", 2)])
def test_ep_workloads_virtual_ranks(oracle_mod, name, G):
    d = inputs.make(name)
    wl = d["workload"]
    x, topk, w = d["x"], d["topk_idx"], d["topk_w"]
    eo = inputs.random_bf16_bits((wl.T * wl.k, wl.H), seed=wl.seed + 7)
    sb = _shards(wl.T, G)
    out = _run_virtual(oracle_mod, x, topk, w, eo, wl.E, G, sb)
    _check(oracle_mod, x, w, eo, *out[:2], *out[3:])
    # contiguous shards in rank order: the rows of the single-source layout
    one = oracle_mod.layout(topk, wl.E, G)
    assert np.array_equal(out[0]["slot"], one["slot"])


@pytest.mark.parametrize("sizes,E,k,R,H", [
    ([7, 0, 26], 13, 4, 3, 136),           # an empty shard, ragged rows (272 bytes)
    ([1, 1, 1, 1, 300], 32, 8, 5, 2048),
    ([50, 60], 9, 9, 2, 9),                # odd rows: 2-byte vectors, k = E
])
def test_ep_uneven_shards(oracle_mod, sizes, E, k, R, H):
    T = sum(sizes)
    d = inputs.make_random(T, H, E, k, seed=T + E)
    eo = inputs.random_bf16_bits((T * k, H), seed=3 * T)
    sb = _shards(T, len(sizes), sizes)
    out = _run_virtual(oracle_mod, d["x"], d["topk_idx"], d["topk_w"], eo, E, R, sb)
    _check(oracle_mod, d["x"], d["topk_w"], eo, *out[:2], *out[3:])


def test_ep_capacity_overflow_is_refused(oracle_mod):
    T, H, E, k, R = 64, 64, 8, 2, 2
    d = inputs.make_random(T, H, E, k, seed=4)
    eo = inputs.random_bf16_bits((T * k, H), seed=5)
    ref, rows, cap, ranks, eps, recv, ys = _run_virtual(
        oracle_mod, d["x"], d["topk_idx"], d["topk_w"], eo, E, R, _shards(T, 2), cap_extra=-10)
    for r, buf in enumerate(recv):
        got = M.bits(buf)
        assert np.all(got[cap:] == CANARY), "nothing written at or beyond the capacity"
    assert any(capi.moe_get_error(lay.struct) == capi.MOE_ERR_BAD_LAYOUT
               for _, lay, _, _, _ in ranks)


def test_ep_refusals():
    M.ensure_lib()
    cfg = capi.config(4, 16, 8, 2, 2, 2, capi.MOE_FLAG_TWO_LEVEL)
    lay = buffers.DeviceLayout(cfg)
    ep = capi.ep_layout_struct(torch.zeros(9, dtype=torch.int32, device="cuda"),
                               torch.zeros(3, dtype=torch.int32, device="cuda"),
                               torch.zeros(8, dtype=torch.int32, device="cuda"))
    x = torch.zeros((4, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_ep_dispatch(cfg, lay.struct, ep, x, [x, x], 8)
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG
    flat = capi.config(4, 16, 8, 2, 2)
    lay = buffers.DeviceLayout(flat)
    with pytest.raises(capi.MoeError) as ei:
        capi.moe_ep_layout(flat, 2, 2, x, x, lay.struct, ep)          # source rank out of range
    assert ei.value.status == capi.MOE_ERR_INVALID_ARG


# ---------------------------------------------------------------- two processes

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ep_rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    import oracle
    from combine_moe_layout_06_b200 import ep as epmod
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        torch.cuda.set_device(0)
        d = inputs.make("olmoe")
        wl = d["workload"]
        sb = _shards(wl.T, world)
        a, b = int(sb[rank]), int(sb[rank + 1])
        ref = oracle.ep_layout(d["topk_idx"], wl.E, world, sb)
        cfg = capi.config(b - a, wl.H, wl.E, wl.k, world)
        me = epmod.ExpertParallelRank(cfg, rank, world)
        rows = me.layout(torch.from_numpy(np.ascontiguousarray(d["topk_idx"][a:b])).cuda())
        cap = int(rows.max())
        recv = torch.full((cap, wl.H), CANARY, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        eo_all = inputs.random_bf16_bits((wl.T * wl.k, wl.H), seed=wl.seed + 7)
        lo, hi = ref["rank_offsets"][rank], ref["rank_offsets"][rank + 1]
        eo = torch.zeros((cap, wl.H), dtype=torch.bfloat16, device="cuda")
        eo[: hi - lo] = buffers.bf16_from_bits(eo_all[lo:hi])
        recv_peers = epmod.share_buffer(recv)
        eo_peers = epmod.share_buffer(eo)
        torch.cuda.synchronize()
        dist.barrier()
        me.dispatch(buffers.bf16_from_bits(d["x"][a:b]), [p for p, _ in recv_peers], cap)
        torch.cuda.synchronize()
        dist.barrier()
        recv_ref = oracle.dispatch_flat(d["x"], ref["slot"])
        ok_recv = bool(np.array_equal(buffers.bits_of(recv)[: hi - lo], recv_ref[lo:hi]))
        y = torch.empty((b - a, wl.H), dtype=torch.bfloat16, device="cuda")
        me.combine([p for p, _ in eo_peers], cap,
                   torch.from_numpy(np.ascontiguousarray(d["topk_w"][a:b])).cuda(), y)
        torch.cuda.synchronize()
        dist.barrier()
        y_ref = oracle.combine(eo_all, d["topk_w"], ref["slot"])[a:b]
        ok_y = bool(np.array_equal(buffers.bits_of(y), y_ref))
        err = capi.moe_get_error(me.local.struct)
        del recv_peers, eo_peers
        dist.barrier()
        out.put((rank, ok_recv, ok_y, err))
    finally:
        dist.destroy_process_group()


def test_ep_two_processes_ipc():
    import torch.multiprocessing as mp
    M.ensure_lib()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(240)
        if p.exitcode is None:
            p.kill()
        assert p.exitcode == 0
    got = sorted(out.get(timeout=10) for _ in range(2))
    for rank, ok_recv, ok_y, err in got:
        assert ok_recv, f"receive buffer of rank {rank}"
        assert ok_y, f"combine of rank {rank}"
        assert err == capi.MOE_OK


def test_bench_multi_process_step_as_one_rank():
    """bench.py's multi-process expert-parallel step (what `--gpus N` runs under
    torchrun), taken by a process group of one rank on this GPU: local layout,
    NCCL count all-gather, sharded-source layout, dispatch into and combine
    from the ranks' buffers, NCCL barriers between the phases.  It must run
    without a device error and report every routed row as received."""
    import json
    import subprocess
    import sys
    M.ensure_lib()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    T = 1024
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--ep-processes",
                          "--workload", "olmoe", "--tokens", str(T), "--steps", "4", "--warmup", "3",
                          "--e2e-steps", "2"], capture_output=True, text=True, timeout=600, cwd=root)
    assert res.returncode == 0, res.stderr[-3000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    wl = inputs.WORKLOADS["olmoe"]
    assert line["n_gpus"] == 1 and line["value"] > 0
    assert line["expert_parallel"]["receive_rows"] == [T * wl.k]
    assert line["e2e"]["h2d_bytes_per_step"] == T * wl.H * 2 + T * wl.k * 8
    assert line["replicas"]["value"] > 0


def test_enable_peer_access_refusals_and_pairs():
    """moe_enable_peer_access: a device paired with itself or an index
    beyond the visible devices is refused up front; where two GPUs are
    visible, enabling a pair twice is fine."""
    M.ensure_lib()
    n = torch.cuda.device_count()
    for dev, peer in ((0, 0), (0, n), (-1, 0)):
        with pytest.raises(capi.MoeError) as ei:
            capi.moe_enable_peer_access(dev, peer)
        assert ei.value.status == capi.MOE_ERR_INVALID_ARG
    if n >= 2 and torch.cuda.can_device_access_peer(0, 1):
        capi.moe_enable_peer_access(0, 1)
        capi.moe_enable_peer_access(0, 1)
    assert torch.cuda.current_device() == 0
