"""Expert parallelism, one rank per GPU: buffers and the host-side plumbing
around the library's moonep_ep_* calls.

A step on rank r ("The Busiest Rank Sets Your Step Time", section
"Installation and integration": eight ranks over NVLink, the weight tensor
mapped from each home rank):

    moonep_ep_count      histogram of the rank's own ids -> counts [N + 1]
    gather_counts        all-gather -> counts_all [R][N + 1] on every rank
      (or both in one launch: moonep_ep_count_exchange stores the rank's
      counts into row r of every rank's counts_all through a peer table;
      then a barrier)
    moonep_ep_plan       every rank derives the same tables from counts_all
    moonep_ep_prefetch   slot weights read from the home ranks
    moonep_ep_dispatch   rows written into the destination ranks' buffers
    (expert computation; a barrier so every rank's rows have landed)
    moonep_ep_combine    rows read back from the ranks that computed them
  training, backward:
    moonep_ep_combine_backward  grad of the dispatched rows written on the ranks
                         that hold them (and the router weights' grad)
    (expert backward; a barrier)
    moonep_ep_dispatch_backward grad of the hidden states read back
    moonep_ep_reduce_grad replica gradients read (and cleared) on the receivers

The data path runs in the library's kernels; this module only allocates,
builds the peer-pointer tables and moves the counts between ranks.  Peers are
reached through their buffers' device addresses as this GPU sees them: CUDA
IPC mappings for one process per GPU (`map_peers`, whose PeerTable keeps the
mappings alive), or plain local addresses when all ranks share one device
(`Emulation`, used by the tests on one GPU).  The kernels never wait for another rank: the caller orders the
ranks between calls (stream order on one device; collectives or barriers
across processes).
"""
from __future__ import annotations

import numpy as np

from . import moonep as mp


def _torch():
    import torch
    return torch


def peer_table(tensors, device):
    """Device int64 array of the tensors' data pointers (a peer table).  The
    table holds plain addresses: the caller keeps the tensors referenced for
    as long as it is used (see PeerTable)."""
    torch = _torch()
    return torch.tensor([int(t.data_ptr()) for t in tensors], dtype=torch.int64, device=device)


class PeerTable:
    """A peer table together with the tensors it points into.  Keeping this
    object keeps the tensors, and so the memory the kernels reach through the
    table, alive: a tensor mapped from another process (exchange_buffers)
    unmaps that process's memory when it is freed, after which a kernel given
    the bare address would fault.  Pass the object itself wherever a peer
    table is expected."""

    def __init__(self, tensors, device):
        self.tensors = list(tensors)
        self.table = peer_table(self.tensors, device)

    def data_ptr(self):
        return self.table.data_ptr()


def _table(t):
    return t.table if isinstance(t, PeerTable) else t


class RankBuffers:
    """Buffers of one expert-parallel rank.  cfg: dict(R, L, S, K, H, B, C,
    C_max).  w_elems / g_elems: weight and gradient elements per expert (0 =
    no prefetch / reduce buffers).  bf16 tensors are held as int16 (same
    bits)."""

    def __init__(self, cfg, rank, device="cuda", w_elems=0, g_elems=0, poison=False):
        torch = _torch()
        self.cfg, self.rank, self.device = dict(cfg), int(rank), device
        R, L, S, K, H, B, Cm = (cfg[n] for n in ("R", "L", "S", "K", "H", "B", "C_max"))
        self.N = R * L
        dev = torch.device(device)
        fill = -1 if poison else 0
        self.ws = torch.zeros(mp.moonep_ep_workspace_bytes(cfg) // 4, dtype=torch.int32, device=dev)
        self.counts = torch.zeros(self.N + 1, dtype=torch.int32, device=dev)
        self.counts_all = torch.zeros((R, self.N + 1), dtype=torch.int32, device=dev)
        self.ids = torch.zeros(max(S * K, 1), dtype=torch.int32, device=dev)
        self.w = torch.zeros(max(S * K, 1), dtype=torch.float32, device=dev)
        self.x = torch.zeros((max(S, 1), H), dtype=torch.int16, device=dev)
        self.recv = torch.full((max(Cm, 1), H), fill, dtype=torch.int16, device=dev)
        self.dest = torch.full((max(S * K, 1),), -7, dtype=torch.int32, device=dev)
        self.out = torch.full((max(S, 1), H), fill, dtype=torch.int16, device=dev)
        self.w_elems, self.g_elems = int(w_elems), int(g_elems)
        if self.w_elems:
            self.w_home = torch.zeros((L, self.w_elems), dtype=torch.int16, device=dev)
            self.w_slot = torch.full((max(B, 1), self.w_elems), fill, dtype=torch.int16, device=dev)
        if self.g_elems:
            self.g_home = torch.zeros((L, self.g_elems), dtype=torch.float32, device=dev)
            self.g_rep = torch.zeros((max(B, 1), self.g_elems), dtype=torch.float32, device=dev)

    def set_routing(self, topk_idx, topk_w):
        """This rank's router output: [S, K] ids and weights."""
        torch = _torch()
        n = self.cfg["S"] * self.cfg["K"]
        if n:
            self.ids[:n].copy_(torch.from_numpy(np.ascontiguousarray(topk_idx, np.int32).reshape(-1)))
            self.w[:n].copy_(torch.from_numpy(np.ascontiguousarray(topk_w, np.float32).reshape(-1)))

    # one rank's calls (peer tables built by the caller)
    def count(self, stream=None, counts_all_peers=None):
        """The rank's counts; with counts_all_peers (every rank's counts_all)
        also stored into row `rank` of each of them."""
        if counts_all_peers is None:
            mp.moonep_ep_count(self.cfg, self.rank, self.ids, self.ws, self.counts, stream)
        else:
            mp.moonep_ep_count_exchange(self.cfg, self.rank, self.ids, self.ws, self.counts,
                                        _table(counts_all_peers), stream)

    def plan(self, flags=0, stream=None):
        mp.moonep_ep_plan(self.cfg, flags, self.rank, self.counts_all, self.ws, stream)

    # peer tables: a PeerTable, or a device int64 tensor of addresses whose
    # memory the caller keeps alive
    def dispatch(self, recv_peers, stream=None):
        mp.moonep_ep_dispatch(self.cfg, self.rank, self.ws, self.x, self.ids, _table(recv_peers), self.dest, stream)

    def combine(self, y_peers, stream=None):
        mp.moonep_ep_combine(self.cfg, self.rank, self.ws, _table(y_peers), self.dest, self.w, self.out, stream)

    def combine_backward(self, grad_out, y_peers, grad_y_peers, grad_w=None, stream=None):
        """grad_out [S][H] bf16 (int16) of this rank; grad_w [S][K] fp32 or None."""
        mp.moonep_ep_combine_backward(self.cfg, self.rank, self.ws, grad_out, _table(y_peers), self.dest, self.w,
                                      _table(grad_y_peers), grad_w, stream)

    def dispatch_backward(self, grad_recv_peers, grad_x, stream=None):
        """grad_x [S][H] bf16 (int16) of this rank, from every rank's grad_recv."""
        mp.moonep_ep_dispatch_backward(self.cfg, self.rank, self.ws, _table(grad_recv_peers), self.dest, grad_x,
                                       stream)

    def prefetch(self, w_home_peers, stream=None):
        mp.moonep_ep_prefetch(self.cfg, self.rank, self.ws, _table(w_home_peers), self.w_slot, self.w_elems,
                              stream)

    def reduce_grad(self, g_rep_peers, stream=None):
        mp.moonep_ep_reduce_grad(self.cfg, self.rank, self.ws, self.g_home, _table(g_rep_peers), self.g_elems,
                                 stream)

    def read_plan(self, tables=True):
        return mp.moonep_plan_read(self.cfg, self.ws, tables=tables)


# ---------------------------------------------------------------------------
# across processes (one rank per GPU)
# ---------------------------------------------------------------------------

def gather_counts(counts, counts_all, group=None):
    """All-gather of every rank's counts [N + 1] into counts_all [R][N + 1]
    (row q = rank q's).  counts and counts_all live on the backend's device
    (CUDA for NCCL, CPU for gloo)."""
    import torch.distributed as dist
    dist.all_gather_into_tensor(counts_all.view(-1), counts.view(-1), group=group)
    return counts_all


def check_same_config(cfg, group=None):
    """Every rank must plan the same configuration; raises ValueError (on
    every rank) if they differ."""
    import torch.distributed as dist
    mine = tuple(int(cfg[n]) for n in ("R", "L", "S", "K", "H", "B", "C", "C_max"))
    got = [None] * dist.get_world_size(group)
    dist.all_gather_object(got, mine, group=group)
    if any(g != mine for g in got):
        raise ValueError("ranks disagree on the configuration: %s" % (got,))
    if len(got) != mine[0]:
        raise ValueError("R=%d ranks configured, %d processes in the group" % (mine[0], len(got)))


def exchange_buffers(tensor, group=None):
    """Maps every rank's `tensor` into this process: returns a list of R
    tensors, entry q aliasing rank q's buffer (this rank's own tensor at its
    own index).  Uses CUDA IPC handles sent over the process group; every
    rank's tensor must be a whole CUDA tensor of the same shape and dtype.
    A mapped tensor unmaps the peer's memory when it is freed: keep the list
    (or the PeerTable of map_peers) for as long as kernels use the
    addresses."""
    import torch.distributed as dist
    from torch.multiprocessing.reductions import reduce_tensor
    me = dist.get_rank(group)
    fn, args = reduce_tensor(tensor)
    got = [None] * dist.get_world_size(group)
    dist.all_gather_object(got, (fn, args), group=group)
    out = []
    for q, (f, a) in enumerate(got):
        out.append(tensor if q == me else f(*a))
    return out


def map_peers(tensor, device, group=None):
    """exchange_buffers and the device table of the mapped addresses, kept
    together (a PeerTable)."""
    return PeerTable(exchange_buffers(tensor, group), device)


# ---------------------------------------------------------------------------
# R ranks on one device
# ---------------------------------------------------------------------------

class Emulation:
    """R expert-parallel ranks on one device, each with its own buffers: the
    ranks' kernels run one after another on one stream (no kernel waits for
    another), the peer tables hold local addresses and the count all-gather
    is a copy.  The data each kernel reads and writes, and every index it
    computes, are those of one rank per GPU."""

    def __init__(self, cfg, device="cuda", w_elems=0, g_elems=0, poison=False):
        torch = _torch()
        self.cfg = dict(cfg)
        self.R = cfg["R"]
        self.ranks = [RankBuffers(cfg, r, device, w_elems, g_elems, poison) for r in range(self.R)]
        self.recv_peers = peer_table([rb.recv for rb in self.ranks], device)
        self.counts_all_peers = peer_table([rb.counts_all for rb in self.ranks], device)
        if w_elems:
            self.w_home_peers = peer_table([rb.w_home for rb in self.ranks], device)
        if g_elems:
            self.g_rep_peers = peer_table([rb.g_rep for rb in self.ranks], device)
        self.torch = torch

    def set_routing(self, topk_idx, topk_w):
        """Global router output [R, S, K]: rank r gets row r."""
        for r, rb in enumerate(self.ranks):
            rb.set_routing(np.asarray(topk_idx)[r], np.asarray(topk_w)[r])

    def plan(self, flags=0, stream=None, exchange=False):
        """Every rank's count, the exchange of the counts (a copy, or with
        exchange=True the ranks' own stores into every counts_all), then every
        rank's plan."""
        if exchange:
            for rb in self.ranks:
                rb.count(stream, self.counts_all_peers)
        else:
            for rb in self.ranks:
                rb.count(stream)
            allc = self.torch.stack([rb.counts for rb in self.ranks])
            for rb in self.ranks:
                rb.counts_all.copy_(allc)
        for rb in self.ranks:
            rb.plan(flags, stream)

    def dispatch(self, stream=None):
        for rb in self.ranks:
            rb.dispatch(self.recv_peers, stream)

    def combine(self, y_peers=None, stream=None):
        yp = self.recv_peers if y_peers is None else y_peers
        for rb in self.ranks:
            rb.combine(yp, stream)

    def combine_backward(self, grad_out, grad_y_peers, grad_w=None, y_peers=None, stream=None):
        """grad_out, grad_w: per-rank lists ([S][H] bf16, [S][K] fp32 or
        None); grad_y_peers: peer table of the ranks' grad_y buffers."""
        yp = self.recv_peers if y_peers is None else y_peers
        for r, rb in enumerate(self.ranks):
            rb.combine_backward(grad_out[r], yp, grad_y_peers, None if grad_w is None else grad_w[r], stream)

    def dispatch_backward(self, grad_recv_peers, grad_x, stream=None):
        """grad_x: per-rank list of [S][H] bf16 outputs."""
        for r, rb in enumerate(self.ranks):
            rb.dispatch_backward(grad_recv_peers, grad_x[r], stream)

    def prefetch(self, stream=None):
        for rb in self.ranks:
            rb.prefetch(self.w_home_peers, stream)

    def reduce_grad(self, stream=None):
        for rb in self.ranks:
            rb.reduce_grad(self.g_rep_peers, stream)
