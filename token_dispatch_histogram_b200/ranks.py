"""Rank-local form of the path: one rank of R, one process per GPU.

The one-buffer path (EpLayer) holds all R ranks as partitions of one static
buffer.  Here each rank holds only its own tokens and its own S*K-row receive
buffer, and rows move through a device table of the R ranks' buffer addresses
(this GPU's buffer and the peers' buffers mapped into this process, e.g. by
symmetric memory or CUDA IPC).  The MoonEP page ("Online planning, zero copy
και στατικά σχήματα") has tokens written straight into their final
expert-grouped rows on the remote ranks; the UltraEP page ("その仕組みは高速な
エキスパート複製に依存する") plans from the exact source-rank x expert load
matrix.  One step on rank r:

  count()           local histogram -> counts_row (ep_route_stats on S tokens)
  gather            all ranks' rows -> counts [R, E] (the one collective)
  plan_and_layout() ep_plan_from_counts + ep_layout_rank, or the quota-driven
                    ep_quota_plan_from_counts + ep_quota_layout_rank (no further exchange)
  dispatch()        ep_dispatch_peer: rows into the receiving ranks' buffers
  combine()         ep_combine_peer: expert rows back from those buffers
  grad_reduce()     ep_replica_grad_reduce_peer: replica gradients home

Every device step is one of libep.so's kernels; this module only allocates
and sequences.  gather_counts is the collective, through torch.distributed.

RankLocalJob runs the R ranks over the processes of a torch.distributed group,
R / world ranks per process (one process per GPU; world = R is one rank per
GPU), with the peer tables built from CUDA IPC handles exchanged over the
group (ep_ipc_export / ep_ipc_open) and a host fence between the ranks'
dispatch and their combine.
"""
import numpy as np
import torch
import torch.distributed as dist

from . import (EP_IPC_HANDLE_BYTES, ep_combine_peer, ep_dispatch_peer, ep_ipc_close, ep_ipc_export, ep_ipc_open,
               ep_layout_rank, ep_plan_from_counts, ep_plan_layout, ep_quota_counts_workspace_size,
               ep_quota_layout_rank, ep_quota_plan_from_counts, ep_quota_plan_layout,
               ep_quota_replica_grad_reduce_peer, ep_replica_grad_reduce_peer, ep_route_stats, ep_status_read,
               ep_workspace_size)


def _on_backend(t, group=None):
    """`t` on the device the group's backend exchanges: CPU for gloo, this
    process's current GPU for NCCL."""
    backend = dist.get_backend(group)
    if backend == "gloo":
        return t.cpu()
    if backend == "nccl" and not t.is_cuda:
        return t.to(torch.device("cuda", torch.cuda.current_device()))
    return t


def all_gather_rows(rows, group=None):
    """Concatenate every process's [n, ...] block (the same n everywhere) in
    process order, on every process; returned on rows' device."""
    world = dist.get_world_size(group)
    mine = _on_backend(rows.contiguous(), group)
    parts = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(parts, mine, group=group)
    return torch.cat(parts).to(rows.device)  # back where the caller's rows live


def gather_counts(counts_row, counts, group=None):
    """All-gather every rank's [E] expert counts into counts [R, E], row r =
    rank r's, on every rank (NCCL on GPUs, gloo on CPU)."""
    R = dist.get_world_size(group)
    if counts.shape != (R, counts_row.numel()):
        raise ValueError(f"counts must be [{R}, {counts_row.numel()}]")
    if dist.get_backend(group) == "gloo" and counts.is_cuda:
        counts.copy_(all_gather_rows(counts_row.view(1, -1), group))
        return counts
    parts = list(counts.unbind(0))
    dist.all_gather(parts, counts_row.contiguous(), group=group)
    return counts


def pack_export(rank, handle, offset, pid):
    """One exchanged record: [rank, offset, pid] int64 then the handle bytes."""
    head = np.array([rank, offset, pid], dtype=np.int64).view(np.uint8)
    return np.concatenate([head, np.frombuffer(handle, dtype=np.uint8)])


def unpack_export(rec):
    rec = np.ascontiguousarray(rec, dtype=np.uint8)
    rank, offset, pid = (int(v) for v in rec[:24].view(np.int64))
    return rank, offset, pid, bytes(rec[24:24 + EP_IPC_HANDLE_BYTES])


RECORD_BYTES = 24 + EP_IPC_HANDLE_BYTES


def exchange_addresses(local, R, group=None, exporter=None, opener=None):
    """Addresses of all R ranks' buffers in this process.

    local: {rank: tensor} for the ranks this process holds (every process
    holds the same number).  Each process exports its buffers (CUDA IPC
    handles), the records are all-gathered over the group, and the other
    processes' buffers are opened here.  Returns (addrs [R] ints, opened
    bases to close).  exporter/opener stand in for ep_ipc_export/ep_ipc_open
    (tests of the exchange without a GPU)."""
    import os
    exporter = exporter or ep_ipc_export
    opener = opener or ep_ipc_open
    pid = os.getpid()
    recs = []
    for r in sorted(local):
        h, off = exporter(local[r])
        recs.append(pack_export(r, h, off, pid))
    mine = torch.from_numpy(np.stack(recs))
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    every = all_gather_rows(mine, group).numpy() if world > 1 else mine.numpy()
    addrs = [0] * R
    opened = []
    seen = set()
    for rec in every:
        r, off, owner, h = unpack_export(rec)
        if not 0 <= r < R or r in seen:
            raise ValueError(f"rank {r} exported twice or out of range")
        seen.add(r)
        if owner == pid and r in local:
            addrs[r] = int(local[r].data_ptr())
        else:
            base, ptr = opener(h, off)
            opened.append(base)
            addrs[r] = int(ptr)
    if len(seen) != R:
        raise ValueError(f"{R - len(seen)} ranks exported no buffer")
    return addrs, opened


class RankLocalJob:
    """The rank-local form over the processes of a torch.distributed group
    (or this process alone): R ranks, R / world of them in each process
    (ranks [p*n, (p+1)*n) in process p), one EpRank each, on this process's
    GPU.  open_peers() must run once (collectively) before dispatch;
    close() (collectively) before the buffers are freed.

    One step: route() (counts of every local rank, one all-gather of the
    [n, E] blocks, plan and layout per rank), dispatch(), fence() (every
    rank's rows are written before any rank reads them: a stream
    synchronisation and a barrier), combine(), and with gradients
    grad_reduce() after a fence of its own."""

    def __init__(self, R, S, K, E, H, group=None, device="cuda", grad_n=0, grad_dtype=torch.float32):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.me = dist.get_rank(group) if dist.is_initialized() else 0
        if R % self.world:
            raise ValueError(f"R={R} ranks do not divide over {self.world} processes")
        self.R, self.S, self.K, self.E, self.H = R, S, K, E, H
        self.n = R // self.world
        self.device = torch.device(device)
        first = self.me * self.n
        self.ranks = [EpRank(first + i, R, S, K, E, H, device=self.device, grad_n=grad_n, grad_dtype=grad_dtype)
                      for i in range(self.n)]
        self.counts = torch.zeros((R, E), dtype=torch.int32, device=self.device)
        self._opened = []

    def open_peers(self):
        """Peer tables of all R ranks' receive buffers (and replica gradient
        buffers) in this process: own buffers by address, the other
        processes' through their IPC handles."""
        addrs, opened = exchange_addresses({rk.rank: rk.buf for rk in self.ranks}, self.R, self.group)
        self._opened += opened
        peers = torch.tensor(addrs, dtype=torch.int64, device=self.device)
        for rk in self.ranks:
            rk.set_peers(peers)
        if self.ranks[0].grad_n:
            gaddrs, gopened = exchange_addresses({rk.rank: rk.g_rep for rk in self.ranks}, self.R, self.group)
            self._opened += gopened
            gpeers = torch.tensor(gaddrs, dtype=torch.int64, device=self.device)
            for rk in self.ranks:
                rk.set_grad_peers(gpeers)

    def route(self, stream=None):
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(st):  # the row copies in order with the kernels
            for rk in self.ranks:
                rk.count(st)
            rows = torch.stack([rk.counts_row for rk in self.ranks])
            if self.world > 1:
                rows = all_gather_rows(rows, self.group)
            self.counts.copy_(rows)
            for rk in self.ranks:
                rk.counts.copy_(self.counts)
                rk.plan_and_layout(st)

    def dispatch(self, stream=None):
        for rk in self.ranks:
            rk.dispatch(stream)

    def combine(self, stream=None):
        for rk in self.ranks:
            rk.combine(stream)

    def grad_reduce(self, clear=False, stream=None):
        for rk in self.ranks:
            rk.grad_reduce(clear, stream)

    def fence(self):
        """Every process's queued work done, then a barrier: rows another
        process wrote into this one's buffers (or will read) are in place."""
        torch.cuda.synchronize(self.device)
        if self.world > 1:
            dist.barrier(group=self.group)

    def status(self, stream=None):
        st = 0
        for rk in self.ranks:
            st |= rk.status(stream)
        return st

    def close(self):
        """Unmap the other processes' buffers (after a fence, so no process
        still reads or writes them)."""
        self.fence()
        for base in self._opened:
            ep_ipc_close(base)
        self._opened = []
        if self.world > 1:
            dist.barrier(group=self.group)


class EpRank:
    """Static buffers of one rank of R: S tokens of top-K routing, H hidden.

    planner "exact": the exact-S*K replica plan (every rank receives S*K rows);
    "quota": the quota-driven plan with at most B replicas per rank (rank r
    receives rank_load[r] <= tau* rows).  buf is this rank's receive buffer of
    buf_rows rows (default S*K; a quota plan needs tau*, and rows past the
    buffer are skipped and flagged), expert-grouped: home experts in id order,
    then received replicas in match order.  peers must be set to the R ranks'
    buffers (set_peers) before dispatch/combine.  With grad_n > 0, g_home holds
    this rank's E/R home experts' gradients [E/R, grad_n] fp32 and g_rep the
    gradients of the replicas it receives [rep_rows, grad_n], row j = its j-th
    received replica (default E - E/R rows, enough for any plan; grad_peers:
    the R ranks' g_rep, set_grad_peers)."""

    def __init__(self, rank, R, S, K, E, H, device="cuda", grad_n=0, grad_dtype=torch.float32, rep_rows=None,
                 planner="exact", B=0, buf_rows=None):
        if E % R:
            raise ValueError("E must be a multiple of R")
        if planner not in ("exact", "quota"):
            raise ValueError(planner)
        self.rank, self.R, self.S, self.K, self.E, self.H = rank, R, S, K, E, H
        self.planner, self.B = planner, B
        self.device = torch.device(device)
        dev = self.device
        i32 = dict(dtype=torch.int32, device=dev)
        self.SK = S * K
        self.buf_rows = self.SK if buf_rows is None else buf_rows
        self.topk_local = torch.zeros((S, K), **i32)
        self.w_local = torch.zeros((S, K), dtype=torch.float32, device=dev)
        self.x_local = torch.zeros((S, H), dtype=torch.bfloat16, device=dev)
        self.out_local = torch.zeros((S, H), dtype=torch.bfloat16, device=dev)
        self.buf = torch.zeros((self.buf_rows, H), dtype=torch.bfloat16, device=dev)
        self.counts_row = torch.zeros(E, **i32)
        self.counts = torch.zeros((R, E), **i32)
        self.loads = torch.zeros(E, **i32)
        self.max_vio_local = torch.zeros(1, dtype=torch.float64, device=dev)
        if planner == "exact":
            self.plan_layout = ep_plan_layout(E, R)
            self.rank_first = None
        else:
            self.plan_layout = ep_quota_plan_layout(E, R)
            self.ws_q = torch.zeros(ep_quota_counts_workspace_size(E, R), dtype=torch.uint8, device=dev)
        self.plan = torch.zeros(self.plan_layout["words"], **i32)
        if planner == "quota":  # a view of the plan: each rank's first global row
            off = self.plan_layout["rank_off"]
            self.rank_first = self.plan[off:off + R]
        self.pos_local = torch.zeros(self.SK, **i32)
        self.ws = torch.zeros(ep_workspace_size(S, K, E), dtype=torch.uint8, device=dev)
        self.dev_status = torch.zeros(1, **i32)
        self.grad_n = grad_n
        if grad_n:
            self.g_home = torch.zeros((E // R, grad_n), dtype=torch.float32, device=dev)
            # a rank receives at most E - E/R replicas (one per chunk of another rank's expert)
            self.rep_rows = max(1, E - E // R) if rep_rows is None else rep_rows
            self.g_rep = torch.zeros((self.rep_rows, grad_n), dtype=grad_dtype, device=dev)
        self.peers = None
        self.grad_peers = None

    def set_peers(self, peers):
        """peers: device int64 [R] table of the R ranks' buf addresses."""
        if peers.numel() != self.R or peers.dtype != torch.int64:
            raise ValueError("peers must be an int64 table of R addresses")
        self.peers = peers

    def set_grad_peers(self, grad_peers):
        """grad_peers: device int64 [R] table of the R ranks' g_rep addresses."""
        if grad_peers.numel() != self.R or grad_peers.dtype != torch.int64:
            raise ValueError("grad_peers must be an int64 table of R addresses")
        self.grad_peers = grad_peers

    def count(self, stream=None):
        ep_route_stats(self.topk_local, self.E, self.counts_row, self.max_vio_local, self.ws, self.dev_status, stream)

    def plan_and_layout(self, stream=None):
        if self.planner == "exact":
            ep_plan_from_counts(self.counts, self.S, self.K, self.plan, self.loads, self.dev_status, stream)
            ep_layout_rank(self.topk_local, self.rank, self.counts, self.plan, self.ws, self.pos_local, None,
                           self.dev_status, stream)
        else:
            ep_quota_plan_from_counts(self.counts, self.S, self.K, self.B, self.loads, self.plan, self.ws_q,
                                      self.dev_status, stream)
            ep_quota_layout_rank(self.topk_local, self.rank, self.counts, self.plan, self.ws, self.pos_local,
                                 self.dev_status, stream)

    def route(self, group=None, stream=None):
        """count -> all-gather of the counts (torch.distributed) -> plan and layout."""
        self.count(stream)
        gather_counts(self.counts_row, self.counts, group)
        self.plan_and_layout(stream)

    def dispatch(self, stream=None):
        ep_dispatch_peer(self.x_local, self.K, self.pos_local, self.peers, self.buf_rows, self.R * self.SK,
                         self.rank_first, self.dev_status, stream)

    def combine(self, stream=None):
        ep_combine_peer(self.peers, self.buf_rows, self.R * self.SK, self.w_local, self.pos_local, self.out_local,
                        None, self.rank_first, self.dev_status, stream)

    def grad_reduce(self, clear=False, stream=None):
        fn = ep_replica_grad_reduce_peer if self.planner == "exact" else ep_quota_replica_grad_reduce_peer
        fn(self.g_home, self.grad_peers, self.rep_rows, self.g_rep.dtype, self.E, self.rank, self.plan, clear,
           self.dev_status, stream)

    def status(self, stream=None):
        return ep_status_read(self.dev_status, stream)
