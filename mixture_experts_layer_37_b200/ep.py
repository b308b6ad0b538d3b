"""Expert parallelism over torch.distributed ranks.

Each rank holds a contiguous slice of one logical batch and a contiguous block
of E/world experts; tokens travel to the ranks of their experts and the expert
outputs travel back ("Hand-building a LLaMA4-MoE" (dpshk.com/news/5809432)
§2.5; "MoE: gating, experts, load balancing, capacity factor"
(dpshk.com/news/6005940) §4.1).  Capacity, drops and statistics are those of
the whole batch, so the result equals one single-device forward.

The two all-to-alls are not separate collectives: libmoe's dispatch kernel
stores every kept token row straight into the receive buffer of the rank that
holds its expert, and its combine kernel loads the expert rows straight from
the owners' output buffers, over NVLink peer mappings of the other ranks'
buffers (CUDA IPC, exchanged once at construction).  The collectives left are
one all-gather of each slice's statistics (E probability sums, E counts and
the real-token count, packed in one buffer: the one data-parallel MoE needs as
well) and two barriers: the owners' GEMMs must not start before every rank's rows have
landed, and the combine must not read before every owner's GEMMs are done.  Every rank takes the same steps, even
when it sends or receives no rows ("Hand-building a LLaMA4-MoE" §4.3: a rank
that skips a collective deadlocks the group).
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import (MoEConfig, Workspace, allocate_outputs, moe_ep_combine, moe_ep_dispatch, moe_ep_expert_ffn,
               moe_ep_recv_rows, moe_ep_route, moe_ep_workspace_size, moe_ipc_close, moe_ipc_export, moe_ipc_open)
from .dp import SliceStats


class ExpertParallelMoE:
    """One rank's share of an expert-parallel MoE layer forward.

    ``weights`` holds the router (and the shared experts, if any) and this
    rank's E/world routed experts (``local_expert_weights`` slices a full set).
    ``peers`` = (x_recv list, y_recv list), every rank's receive buffers as
    this process sees them, replaces the IPC exchange; ``phases`` replaces the
    library's four calls: route(x, logits_in, token_mask) (fills local_counts,
    local_psum, local_real), dispatch(x, all_counts, all_psum, all_real),
    ffn(x), combine() -> outputs.  Both exist for tests of the orchestration
    on CPU ranks."""

    def __init__(self, cfg_local: MoEConfig, weights: dict, T_global: Optional[int] = None, group=None,
                 device="cuda", peers: Optional[tuple] = None, phases: Optional[dict] = None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.cfg = cfg_local
        self.weights = weights
        self.device = device
        if T_global is None:
            t = torch.tensor([cfg_local.T], dtype=torch.int64,
                             device=device if dist.get_backend(group) == "nccl" else "cpu")
            dist.all_reduce(t, group=self.group)
            T_global = int(t.item())
        self.T_global = T_global
        self.E_local = cfg_local.E // self.world
        self.stats = SliceStats(cfg_local.E, device)
        self.local_counts, self.local_psum, self.local_real = self.stats.counts, self.stats.psum, self.stats.real
        self._opened = []
        self._flag = None
        ph = phases or {}
        self._route = ph.get("route", self._lib_route)
        self._dispatch = ph.get("dispatch", self._lib_dispatch)
        self._ffn = ph.get("ffn", self._lib_ffn)
        self._combine = ph.get("combine", self._lib_combine)
        if phases is None:
            rows = max(moe_ep_recv_rows(cfg_local, T_global, self.world), 1)
            self.recv_rows = rows
            # x_recv and y_recv in one allocation: one IPC record per rank
            self._recv = torch.empty((2, rows, cfg_local.d), dtype=cfg_local.torch_dtype, device=device)
            self.x_recv, self.y_recv = self._recv[0], self._recv[1]
            self.recv_offsets = torch.zeros(self.E_local + 1, dtype=torch.int32, device=device)
            self.outputs = allocate_outputs(cfg_local, device)
            self.ws = Workspace(cfg_local, device, nbytes=moe_ep_workspace_size(cfg_local, T_global, self.world))
        if peers is not None:
            self.x_peers, self.y_peers = list(peers[0]), list(peers[1])
        elif phases is None:
            self.x_peers, self.y_peers = self._exchange_buffers()

    # -------------------------------------------------------------- plumbing
    def _exchange_buffers(self):
        """Every rank's receive buffers as device pointers in this process."""
        rec = moe_ipc_export(self._recv)
        recs = [None] * self.world
        dist.all_gather_object(recs, rec, group=self.group)
        xs, ys = [], []
        row_bytes = self.x_recv.stride(0) * self.x_recv.element_size()
        for r, rr in enumerate(recs):
            if r == self.rank:
                base = self._recv.data_ptr()
            else:
                base = moe_ipc_open(rr)
                self._opened.append((base, rr))
            xs.append(base)
            ys.append(base + self.recv_rows * row_bytes)
        return xs, ys

    def _barrier(self):
        """Orders this rank's next launch after every rank's launches so far."""
        if dist.get_backend(self.group) == "nccl":
            if self._flag is None:
                self._flag = torch.zeros(1, dtype=torch.int32, device=self.device)
            dist.all_reduce(self._flag, group=self.group)  # on the stream: later kernels wait for it
        else:
            if torch.cuda.is_available() and str(self.device).startswith("cuda"):
                torch.cuda.current_stream().synchronize()
            dist.barrier(group=self.group)

    # -------------------------------------------------------------- library phases
    def _lib_route(self, x, logits_in, token_mask):
        moe_ep_route(self.cfg, self.T_global, self.world, self.weights, x, self.outputs, self.local_counts,
                     self.local_psum, self.ws, logits_in, token_mask=token_mask, local_real=self.local_real)

    def _lib_dispatch(self, x, all_counts, all_psum, all_real):
        moe_ep_dispatch(self.cfg, self.T_global, all_counts, all_psum, self.world, self.rank, x, self.x_peers,
                        self.outputs, self.recv_offsets, self.ws, all_real=all_real)

    def _lib_ffn(self, x):
        moe_ep_expert_ffn(self.cfg, self.T_global, self.world, self.weights, x, self.x_recv, self.recv_offsets,
                          self.y_recv, self.ws)

    def _lib_combine(self):
        moe_ep_combine(self.cfg, self.T_global, self.world, self.y_peers, self.outputs, self.ws)
        return self.outputs

    # -------------------------------------------------------------- forward
    def forward(self, x_local: torch.Tensor, logits_in: Optional[torch.Tensor] = None,
                token_mask: Optional[torch.Tensor] = None, events: Optional[list] = None) -> dict:
        """token_mask ([T_local] uint8, 0 = padding) as in moe_forward.
        events: 6 CUDA events recorded on the current stream at the phase
        boundaries (start, after the dispatch, after the first barrier, after
        the expert FFNs, after the second barrier, after the combine)."""
        mark = (lambda i: events[i].record()) if events is not None else (lambda i: None)
        mark(0)
        self._route(x_local, logits_in, token_mask)
        all_counts, all_psum, all_real = self.stats.gather(self.world, self.group)
        self._dispatch(x_local, all_counts, all_psum, all_real)
        mark(1)
        self._barrier()
        mark(2)
        self._ffn(x_local)
        mark(3)
        self._barrier()
        mark(4)
        out = self._combine()
        mark(5)
        return out

    def close(self) -> None:
        """Unmaps the peers' buffers once no rank can still read or write them."""
        self._barrier()
        if torch.cuda.is_available() and str(self.device).startswith("cuda"):
            torch.cuda.current_stream().synchronize()
        for ptr, rec in self._opened:
            moe_ipc_close(ptr, rec)
        self._opened = []
        dist.barrier(group=self.group)  # peers keep their allocations until every mapping is gone
