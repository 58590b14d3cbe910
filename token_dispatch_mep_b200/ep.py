"""The exchange between expert-parallel ranks, one process per GPU.

MoonEP runs one EP rank per GPU: each holds S tokens, every rank receives
exactly S*K token slots in fixed buffers, and replica gradients go back to
the home ranks (MoonEP release page, "How MoonEP works"; "Why this matters to
engineers": static buffer shapes, tokens written straight into their
expert-ordered position).  This module is the host side of that exchange on
top of the rank-addressed kernels of libmep:

* every rank's receive buffer, expert-output buffer and segment-gradient
  buffer is mapped into every other rank's address space once (CUDA IPC
  handles exchanged through the process group), and the R addresses of each
  kind go into a device pointer array;
* the plan: each rank counts its own pairs per expert, one all-gather of those
  R x E histograms follows, and every rank computes the identical tables and
  its own pairs' slots on its own GPU (the ids themselves never leave their
  rank);
* dispatch: each rank writes its own tokens' rows straight into the owning
  ranks' receive buffers (one kernel, peer stores);
* combine: each rank reads its tokens' K expert-output rows straight from
  the ranks that computed them (one kernel, peer loads);
* backward: each home rank sums its experts' segment gradients straight from
  the ranks that hold them (one kernel, peer loads).

Ordering between ranks, before a phase that reads or writes another rank's
memory and again before that memory is reused, takes one of two forms:

* ``sync="host"`` (the default): the rank's stream is synchronised and the
  process group's barrier is passed; no kernel waits on another rank's kernel.
* ``sync="device"``: one mep_rank_barrier kernel on the rank's stream -- every
  rank stores the crossing's epoch into its word of every rank's flag array
  (mapped like the buffers) and waits, bounded by the library's wait limit,
  for all R words of its own; the host never blocks between phases.  Its
  kernels wait on the other ranks' kernels, so each rank must run on a GPU of
  its own.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import (SCHEDULES, IpcHandle, Plan, Shape, mep_combine_ranked_tokens,
               mep_dispatch_ranked_tokens, mep_ipc_close, mep_ipc_export, mep_ipc_open,
               mep_plan_rank, mep_rank_barrier, mep_rank_histogram, mep_read_status,
               mep_reduce_replica_grads_ranked, mep_status_string, pointer_table)

__all__ = ["ExchangeGroup", "gather_counts", "gather_router_ids", "local_segments",
           "max_local_segments"]


def _all_gather(t: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's ``t`` stacked rank by rank (NCCL on the device, any other
    backend through host memory); the result is on ``t``'s device."""
    world = dist.get_world_size(group)
    src = t.contiguous()
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world * src.shape[0],) + tuple(src.shape[1:]), dtype=src.dtype,
                          device=src.device)
        dist.all_gather_into_tensor(out, src, group=group)
        return out
    host = src.cpu()
    parts = [torch.empty_like(host) for _ in range(world)]
    dist.all_gather(parts, host, group=group)
    return torch.cat(parts).to(src.device)


def gather_counts(counts_local: torch.Tensor, group=None) -> torch.Tensor:
    """The plan's one exchange: every rank's per-expert histogram (int32
    ``[E]``) gathered into ``[R, E]``, row r from rank r."""
    if counts_local.dtype != torch.int32 or counts_local.dim() != 1:
        raise TypeError("counts_local must be an int32 [E] tensor")
    return _all_gather(counts_local.view(1, -1), group)


def gather_router_ids(idx_local: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' top-K expert ids ``[R*S, K]`` in global token order (rank r's
    S rows at r*S), from each rank's own ``[S, K]`` int32 ids.  Not used by
    the exchange (the plan needs only the histograms, ``gather_counts``); the
    tests use it to compute the whole-range plan as a reference."""
    if idx_local.dtype != torch.int32 or idx_local.dim() != 2:
        raise TypeError("idx_local must be an int32 [S, K] tensor")
    return _all_gather(idx_local, group)


def max_local_segments(shape: Shape) -> int:
    """Most segments one rank can hold: one per expert at most (in both plans
    an expert has at most one segment per rank), and at most one per slot."""
    return min(shape.E, shape.SK)


def local_segments(plan_host: dict, rank: int) -> list:
    """Rank ``rank``'s segments in slot order as (segment index, expert,
    first local slot, slot count): row j of the rank's expert-output and
    gradient buffers belongs to the j-th of them."""
    ptr, idx, seg = plan_host["rank_seg_ptr"], plan_host["rank_seg_idx"], plan_host["seg"]
    out = []
    for j in range(int(ptr[rank]), int(ptr[rank + 1])):
        s = int(idx[j])
        e, r, start, count = (int(v) for v in seg[s])
        if r != rank:
            raise RuntimeError(f"segment {s} is listed for rank {rank} but belongs to rank {r}")
        out.append((s, e, start, count))
    return out


@dataclass
class _Mapped:
    handle: IpcHandle
    ptr: int


class ExchangeGroup:
    """One EP rank's buffers, the peer mappings and the exchange steps.

    ``shape.R`` must equal the group's size; rank r of the group is EP rank r
    and holds global tokens [r*S, (r+1)*S).  Buffers (this rank's, mapped by
    every peer):

    * ``recv``  bf16 [S*K, H]: dispatch destination, this rank's slots.
    * ``y``     bf16 [S*K, H]: expert outputs of those slots, written by the
      caller's expert compute before ``combine``.
    * ``grads`` fp32 [min(E, S*K), P]: row j = weight gradient of this
      rank's j-th segment (``local_segments``), written before ``reduce``.
    * ``home``  fp32 [E/R, P]: this rank's home experts' summed gradients.
    """

    def __init__(self, shape, H: int, P: int = 0, group=None, device=None,
                 schedule: str = "contiguous", B: int = 0, sync: str = "host"):
        self.shape = shape if isinstance(shape, Shape) else Shape(*shape)
        s = self.shape
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if self.world != s.R:
            raise ValueError(f"group has {self.world} ranks, the shape {s.R}")
        if schedule not in SCHEDULES:
            raise ValueError(f"unknown schedule {schedule!r}")
        if schedule == "capped" and B < 1:
            raise ValueError("the capped schedule needs B >= 1")
        if sync not in ("host", "device"):
            raise ValueError(f"unknown sync {sync!r}")
        self.schedule = schedule
        self.sync = sync
        self.epoch = 0            # device barrier crossings so far
        self.B = int(B)
        self.gathered_bytes = 0   # bytes the last plan exchanged (R x E int32)
        self.H, self.P = int(H), int(P)
        self.device = torch.device(device) if device is not None else \
            torch.device("cuda", torch.cuda.current_device())
        bf = dict(dtype=torch.bfloat16, device=self.device)
        self.recv = torch.zeros((s.SK, self.H), **bf)
        self.y = torch.zeros((s.SK, self.H), **bf)
        f32 = dict(dtype=torch.float32, device=self.device)
        self.grads = torch.zeros((max(1, max_local_segments(s)), max(1, self.P)), **f32)
        self.home = torch.zeros((s.E // s.R, max(1, self.P)), **f32)
        self.plan = Plan(s, self.device)
        self._mapped: list[_Mapped] = []
        self.recv_table = self._share(self.recv)
        self.y_table = self._share(self.y)
        self.grad_table = self._share(self.grads)
        if sync == "device":
            # word r of every rank's array: rank r's last crossing
            self.flags = torch.zeros(s.R, dtype=torch.int32, device=self.device)
            self.flag_table = self._share(self.flags)

    # ------------------------------------------------------------ mapping
    def _share(self, t: torch.Tensor) -> torch.Tensor:
        """Exchange ``t``'s IPC description with every rank and map the
        peers' buffers; returns the device array of the R addresses."""
        mine = bytes(mep_ipc_export(t))
        allh = [None] * self.world
        dist.all_gather_object(allh, mine, group=self.group)
        ptrs = []
        for r, hb in enumerate(allh):
            if r == self.rank:
                ptrs.append(t.data_ptr())
                continue
            h = IpcHandle.from_buffer_copy(hb)
            p = mep_ipc_open(h, self.device)
            self._mapped.append(_Mapped(h, p))
            ptrs.append(p)
        return pointer_table(ptrs, self.device)

    def barrier(self):
        """Every rank's work so far done before anything later on this rank's
        stream: a host barrier, or the device barrier (sync="device"), whose
        errors land in the plan's status word (``check``)."""
        if self.sync == "device":
            self.epoch += 1
            mep_rank_barrier(self.flag_table, self.flags, self.rank, self.epoch,
                             self.plan.status_tensor)
            return
        self.host_barrier()

    def host_barrier(self):
        """This rank's GPU work done, then every rank at the same point."""
        if self.device.type == "cuda":
            torch.cuda.current_stream(self.device).synchronize()
        dist.barrier(group=self.group)

    def check(self):
        st = mep_read_status(self.plan)
        if st != 0:
            raise RuntimeError(f"rank {self.rank}: device status {mep_status_string(st)}")

    # ------------------------------------------------------------ steps
    @property
    def token_begin(self) -> int:
        return self.rank * self.shape.S

    def make_plan(self, idx_local: torch.Tensor) -> Plan:
        """Count this rank's pairs per expert, gather every rank's histogram
        and compute the plan's tables (identical on every rank) and this
        rank's own pairs' slots."""
        idx = idx_local.to(self.device).contiguous()
        counts = mep_rank_histogram(self.shape, idx, plan=self.plan)
        all_counts = gather_counts(counts, self.group)
        self.gathered_bytes = all_counts.numel() * all_counts.element_size()
        self.max_rank_replicas = mep_plan_rank(self.shape, self.schedule, self.rank, idx,
                                               all_counts, self.plan, B=self.B)
        return self.plan

    def dispatch(self, x_local: torch.Tensor) -> torch.Tensor:
        """Send this rank's S token rows to their slots on every rank; returns
        this rank's receive buffer once every rank's rows have arrived."""
        self.barrier()      # every rank is done with its receive buffer
        mep_dispatch_ranked_tokens(self.shape, self.H, self.plan, self.token_begin, x_local,
                                   self.recv_table, token_count=self.shape.S)
        self.barrier()      # every rank's rows have landed
        return self.recv

    def combine(self, topk_w_local: torch.Tensor, out_local: torch.Tensor) -> torch.Tensor:
        """Weighted sum of this rank's tokens' K expert-output rows, read
        from the ranks that hold them (``y`` of every rank must be written)."""
        self.barrier()      # every rank's expert outputs are written
        mep_combine_ranked_tokens(self.shape, self.H, self.plan, self.token_begin, self.y_table,
                                  topk_w_local, out_local, token_count=self.shape.S)
        self.barrier()      # no rank still reads this rank's y
        return out_local

    def reduce(self) -> torch.Tensor:
        """Sum this rank's home experts' segment gradients from every rank
        that holds a segment of them (``grads`` of every rank written)."""
        if self.P == 0:
            return self.home
        self.barrier()      # every rank's segment gradients are written
        mep_reduce_replica_grads_ranked(self.shape, self.plan, self.P, self.rank,
                                        self.grad_table, self.grads.shape[0], self.home)
        self.barrier()      # no rank still reads this rank's grads
        return self.home

    def close(self):
        """Unmap the peers' buffers (after every rank's last exchange)."""
        self.host_barrier()
        for m in self._mapped:
            mep_ipc_close(m.handle, m.ptr, self.device)
        self._mapped.clear()
        dist.barrier(group=self.group)
