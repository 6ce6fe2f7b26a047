"""Expert parallelism over sharded sources: the host side of one rank.

With one rank per GPU, rank g routes only its own tokens and every rank's
receive buffer holds its own experts' rows ("[None][feat] support
non-divisible EP in MoE alltoall and slurm benchmark", TensorRT-LLM PR #13888:
the NVLinkOneSided dispatch writes straight into peer receive buffers).  The
one exchange on the data path is an all-gather of the per-expert counts;
dispatch and combine are this library's kernels writing to, and reading
from, the ranks' buffers through peer-mapped pointers.  This module holds
only plumbing: the count exchange and receive sizes (torch.distributed), and
the mapping of every rank's buffer into this process (CUDA IPC handles of
torch storages).  Every step on the data runs in libmoe_layout.so.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import buffers, capi


def gather_counts(local_counts: torch.Tensor, group=None, out: torch.Tensor | None = None
                  ) -> torch.Tensor:
    """All-gather of every rank's int32 [E] expert counts -> [G, E], source
    rank order, written into `out` when given.  The tensors live where the
    group's backend wants them (CPU for gloo, the GPU for NCCL)."""
    world = dist.get_world_size(group)
    E = local_counts.numel()
    if out is None:
        out = torch.empty((world, E), dtype=local_counts.dtype, device=local_counts.device)
    dist.all_gather_into_tensor(out.view(-1), local_counts.contiguous(), group=group)
    return out


def receive_rows(counts_all, num_ranks: int) -> np.ndarray:
    """Rows each expert rank receives, from the gathered counts [G, E]
    (moe_ep_receive_rows() of the library: the ceil/floor partition's
    experts of each rank, summed over all sources)."""
    return np.array(capi.moe_ep_receive_rows(np.asarray(counts_all), num_ranks), np.int64)


def share_buffer(t: torch.Tensor, group=None) -> list:
    """Device addresses of every rank's `t` (same shape on every rank), as
    usable from this process's kernels: this rank's own address, and the
    peers' through CUDA IPC mappings of their storages.  A peer on another
    GPU is opened in that GPU's context, so peer access from this rank's GPU
    to it is enabled too (moe_enable_peer_access); a pair of GPUs that cannot
    reach each other raises here, before any kernel touches peer memory.
    The returned list keeps the mapped storages alive (second element of each
    pair)."""
    storage = t.untyped_storage()
    handle = storage._share_cuda_()
    offset = t.storage_offset() * t.element_size()
    handles = [None] * dist.get_world_size(group)
    dist.all_gather_object(handles, (handle, offset), group=group)
    me = dist.get_rank(group)
    mine = t.device.index
    out = []
    for r, (h, off) in enumerate(handles):
        if r == me:
            out.append((t.data_ptr(), t))
        else:
            peer_dev = int(h[0])   # the device the peer's storage lives on
            if peer_dev != mine:
                capi.moe_enable_peer_access(mine, peer_dev)
            peer = torch.UntypedStorage._new_shared_cuda(*h)
            out.append((peer.data_ptr() + off, peer))
    return out


class ExpertParallelRank:
    """One rank's step: local layout, count exchange, sharded-source layout,
    dispatch into every rank's receive buffer, combine from every rank's
    expert outputs.  `cfg` describes this rank's shard (num_tokens = its
    tokens, num_ranks = the number of ranks, flat)."""

    def __init__(self, cfg: capi.MoeConfig, rank: int, world: int, device="cuda", group=None):
        self.cfg, self.rank, self.world, self.group = cfg, rank, world, group
        self.local = buffers.DeviceLayout(cfg, device)
        i32 = dict(dtype=torch.int32, device=device)
        self.expert_offsets = torch.zeros(cfg.num_experts + 1, **i32)
        self.rank_offsets = torch.zeros(cfg.num_ranks + 1, **i32)
        self.slot = torch.zeros(max(cfg.num_tokens * cfg.top_k, 1), **i32)
        self.ep = capi.ep_layout_struct(self.expert_offsets, self.rank_offsets, self.slot)
        self.counts_all = None

    def layout(self, topk: torch.Tensor, exchange_device="cpu") -> np.ndarray:
        """Local layout, count exchange, sharded-source layout.  Returns the
        rows every rank receives (host int64 [R])."""
        capi.moe_layout(self.cfg, topk, self.local.struct)
        counts = self.local.expert_counts.to(exchange_device)
        counts_all = gather_counts(counts, self.group)
        self.counts_all = counts_all.to(self.local.expert_counts.device)
        capi.moe_ep_layout(self.cfg, self.rank, self.world, topk, self.counts_all,
                           self.local.struct, self.ep)
        return receive_rows(counts_all.cpu().numpy(), self.cfg.num_ranks)

    def dispatch(self, x: torch.Tensor, recv_bufs, capacity_rows: int) -> None:
        capi.moe_ep_dispatch(self.cfg, self.local.struct, self.ep, x, recv_bufs, capacity_rows)

    def combine(self, expert_out_bufs, capacity_rows: int, w: torch.Tensor, y: torch.Tensor) -> None:
        capi.moe_ep_combine(self.cfg, self.local.struct, self.ep, expert_out_bufs, capacity_rows, w, y)
