"""Data-parallel sharding of one logical MoE batch over torch.distributed ranks.

Each rank holds a contiguous slice of the batch (slices in rank order).  The
capacity cut and the load-balance statistics are those of the whole batch: the
per-expert counts and probability sums of every slice are all-gathered (the
exchange that data-parallel MoE training does before its load-balance loss,
"Hand-building a LLaMA4-MoE" (dpshk.com/news/5809432) §3.1), and the second
phase on each rank keeps only the capacity left after the lower ranks'
assignments.  The one collective is an all-gather (NCCL over NVLink on GPUs)
of each slice's statistics, packed in one buffer: E fp64 probability sums, E
int32 counts and the int32 number of real (unmasked) tokens.  The computation
before and after runs in libmoe's kernels (moe_dp_route, moe_dp_finish).
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist

from . import (MoEConfig, Workspace, allocate_outputs, moe_dp_finish, moe_dp_max_rows, moe_dp_route,
               moe_dp_workspace_size)


def gather_rank_order(t: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """[world, *t.shape] with rank r's tensor in row r (through host memory
    when the backend cannot gather device tensors)."""
    staged = t.is_cuda and dist.get_backend(group) != "nccl"
    src = t.cpu() if staged else t.contiguous()
    parts = [torch.empty_like(src) for _ in range(world)]
    dist.all_gather(parts, src, group=group)
    out = torch.stack(parts)
    return out.to(t.device) if staged else out


class SliceStats:
    """One slice's routing statistics in a single device buffer, so that one
    all-gather carries them: E fp64 probability sums, then E int32 expert
    counts and the int32 number of real tokens.  `psum`, `counts` and `real`
    are views into the buffer that the route call fills."""

    def __init__(self, E: int, device):
        self.E = E
        nbytes = (8 * E + 4 * (E + 1) + 7) // 8 * 8  # rows of the gathered buffer stay 8-byte multiples
        self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.psum = self.buf[:8 * E].view(torch.float64)
        ints = self.buf[8 * E:8 * E + 4 * (E + 1)].view(torch.int32)
        self.counts, self.real = ints[:E], ints[E:]

    @staticmethod
    def unpack(allb: torch.Tensor, E: int) -> tuple:
        """(all_counts [world, E] int32, all_psum [world, E] fp64, all_real [world] int32)
        from the gathered buffers [world, nbytes]."""
        psum = allb[:, :8 * E].clone().view(torch.float64)
        ints = allb[:, 8 * E:8 * E + 4 * (E + 1)].clone().view(torch.int32)
        return ints[:, :E].contiguous(), psum, ints[:, E].contiguous()

    def gather(self, world: int, group=None) -> tuple:
        """The unpacked statistics of every rank, in rank order."""
        return SliceStats.unpack(gather_rank_order(self.buf, world, group), self.E)


class DataParallelMoE:
    """One rank's share of a data-parallel MoE layer forward.

    `route(x, logits_in, token_mask)` and `finish(x, all_counts, all_psum,
    all_real)` default to the library's two phases; tests of the orchestration
    on CPU ranks may substitute stand-ins with the same signatures.  A route
    stand-in fills local_counts, local_psum and local_real."""

    def __init__(self, cfg_local: MoEConfig, weights: dict, group=None, device="cuda",
                 route: Optional[Callable] = None, finish: Optional[Callable] = None, T_global: Optional[int] = None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.cfg = cfg_local
        self.weights = weights
        if T_global is None:
            t = torch.tensor([cfg_local.T], dtype=torch.int64, device=device)
            dist.all_reduce(t, group=self.group)
            T_global = int(t.item())
        self.T_global = T_global
        self._route = route or self._lib_route
        self._finish = finish or self._lib_finish
        self.device = device
        if route is None or finish is None:
            self.outputs = allocate_outputs(cfg_local, device)
            rows = max(moe_dp_max_rows(cfg_local, T_global), 1)
            self.outputs["src_assign"] = torch.empty(rows, dtype=torch.int32, device=device)
            self.ws = Workspace(cfg_local, device, nbytes=moe_dp_workspace_size(cfg_local, T_global))
        self.stats = SliceStats(cfg_local.E, device)
        self.local_counts, self.local_psum, self.local_real = self.stats.counts, self.stats.psum, self.stats.real

    def _lib_route(self, x, logits_in, token_mask):
        moe_dp_route(self.cfg, self.T_global, self.weights, x, self.outputs, self.local_counts, self.local_psum,
                     self.ws, logits_in, token_mask=token_mask, local_real=self.local_real)

    def _lib_finish(self, x, all_counts, all_psum, all_real):
        moe_dp_finish(self.cfg, self.T_global, all_counts, all_psum, self.world, self.rank, self.weights, x,
                      self.outputs, self.ws, all_real=all_real)
        return self.outputs

    def forward(self, x_local: torch.Tensor, logits_in: Optional[torch.Tensor] = None,
                token_mask: Optional[torch.Tensor] = None) -> dict:
        """token_mask ([T_local] uint8, 0 = padding) as in moe_forward; f and p
        then divide by the whole batch's real tokens."""
        self._route(x_local, logits_in, token_mask)
        all_counts, all_psum, all_real = self.stats.gather(self.world, self.group)
        return self._finish(x_local, all_counts, all_psum, all_real)
