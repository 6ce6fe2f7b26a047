"""Device buffers for one dispatch/combine problem, allocated with torch.

torch is used here for device memory only; all work on these buffers runs in
libmoe_layout.so through :mod:`combine_moe_layout_06_b200.capi`.
"""
from __future__ import annotations

import torch

from . import capi


class DeviceLayout:
    """The moe_layout_t arrays of one configuration, plus its workspace.

    ``node_src`` (two-level only): also allocate the staging-row -> token map,
    which makes the second dispatch phase divide its work by staging rows."""

    def __init__(self, cfg: capi.MoeConfig, device="cuda", node_src: bool = True):
        T, k, E, R, N = cfg.num_tokens, cfg.top_k, cfg.num_experts, cfg.num_ranks, cfg.num_nodes
        i32 = dict(dtype=torch.int32, device=device)
        self.cfg = cfg
        self.expert_counts = torch.zeros(E, **i32)
        self.expert_offsets = torch.zeros(E + 1, **i32)
        self.rank_offsets = torch.zeros(R + 1, **i32)
        self.slot = torch.zeros(T * k, **i32)
        self.error_word = torch.zeros(1, **i32)
        ws = capi.moe_layout_workspace_bytes(cfg)
        # zeroed once: a counter of moe_layout_dispatch's kernels lives in it
        # and must start at zero
        self.workspace = torch.zeros(ws, dtype=torch.uint8, device=device)
        self.two_level = bool(cfg.flags & capi.MOE_FLAG_TWO_LEVEL)
        if self.two_level:
            self.node_counts = torch.zeros(N, **i32)
            self.node_offsets = torch.zeros(N + 1, **i32)
            self.node_slot = torch.zeros(T * N, **i32)
            self.node_src = (torch.full((max(capi.moe_node_staging_rows(cfg), 1),), -1, **i32)
                             if node_src else None)
        else:
            self.node_counts = self.node_offsets = self.node_slot = self.node_src = None
        self.struct = capi.layout_struct(
            self.expert_counts, self.expert_offsets, self.rank_offsets, self.slot,
            self.error_word, self.workspace, self.node_counts, self.node_offsets, self.node_slot,
            self.node_src)

    def host(self) -> dict:
        """Copy of the arrays on the host (numpy), shaped like the oracle's."""
        cfg = self.cfg
        out = {
            "expert_counts": self.expert_counts.cpu().numpy(),
            "expert_offsets": self.expert_offsets.cpu().numpy(),
            "rank_offsets": self.rank_offsets.cpu().numpy(),
            "slot": self.slot.cpu().numpy().reshape(cfg.num_tokens, cfg.top_k),
        }
        if self.two_level:
            out["node_counts"] = self.node_counts.cpu().numpy()
            out["node_offsets"] = self.node_offsets.cpu().numpy()
            out["node_slot"] = self.node_slot.cpu().numpy().reshape(cfg.num_tokens, cfg.num_nodes)
            if self.node_src is not None:
                U = int(out["node_offsets"][cfg.num_nodes])
                out["node_src"] = self.node_src[:U].cpu().numpy()
        return out


def bf16_empty(rows: int, hidden: int, device="cuda") -> torch.Tensor:
    return torch.empty((rows, hidden), dtype=torch.bfloat16, device=device)


def bf16_from_bits(bits, device="cuda") -> torch.Tensor:
    """numpy uint16 bf16 bit patterns -> bf16 tensor on device."""
    import numpy as np
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def bits_of(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host)."""
    import numpy as np
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
