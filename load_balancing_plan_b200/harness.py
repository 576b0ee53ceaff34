"""Device-side harness around the C ABI: allocates the caller-owned buffers
with torch, uploads seeded inputs, runs the calls of the step and reads
results back.  Used by the GPU tests, the smoke check and the benchmark.

The stand-in expert here (y = bf16(float(recv) * scale[expert of row])) is
harness, not product: the pages' group GEMM is out of scope and a
per-expert scale takes its place so that combine has something to gather.
"""
from __future__ import annotations

import numpy as np

from . import inputs
from . import moonep as mp


def _torch():
    import torch
    return torch


def as_i16(a: np.ndarray):
    """uint16 bf16 bit patterns -> torch int16 tensor (same bits)."""
    torch = _torch()
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16))


def to_u16(t) -> np.ndarray:
    return t.detach().cpu().contiguous().view(_torch().int16).numpy().view(np.uint16)


class Problem:
    """Buffers of one MoE layer on one device.

    cfg: dict(R, L, S, K, H, B, C, C_max).  w_elems / g_elems: weight and
    gradient elements per expert (0 = no prefetch / reduce buffers)."""

    def __init__(self, cfg, device="cuda", w_elems=0, g_elems=0, poison=False):
        torch = _torch()
        self.cfg = dict(cfg)
        self.device = device
        R, L, S, K, H, B, Cm = (cfg[n] for n in ("R", "L", "S", "K", "H", "B", "C_max"))
        self.N, self.T = R * L, R * S
        dev = torch.device(device)
        ws_words = mp.moonep_plan_workspace_bytes(cfg) // 4
        self.ws = torch.zeros(ws_words, dtype=torch.int32, device=dev)
        self.ids = torch.zeros(max(self.T * K, 1), dtype=torch.int32, device=dev)
        self.w = torch.zeros(max(self.T * K, 1), dtype=torch.float32, device=dev)
        self.x = torch.zeros((max(self.T, 1), H), dtype=torch.int16, device=dev)
        self.recv = torch.empty((max(R * Cm, 1), H), dtype=torch.int16, device=dev)
        self.dest = torch.empty(max(self.T * K, 1), dtype=torch.int32, device=dev)
        self.out = torch.empty((max(self.T, 1), H), dtype=torch.int16, device=dev)
        fill = -1 if poison else 0
        self.recv.fill_(fill)
        self.out.fill_(fill)
        self.dest.fill_(-7)
        self.w_elems, self.g_elems = int(w_elems), int(g_elems)
        if self.w_elems:
            self.w_home = torch.empty((self.N, self.w_elems), dtype=torch.int16, device=dev)
            self.w_slot = torch.full((max(R * B, 1), self.w_elems), fill, dtype=torch.int16, device=dev)
        if self.g_elems:
            self.g_home = torch.empty((self.N, self.g_elems), dtype=torch.float32, device=dev)
            self.g_rep = torch.zeros((max(R * B, 1), self.g_elems), dtype=torch.float32, device=dev)

    # ---------------------------------------------------------------- inputs
    def set_routing(self, topk_idx: np.ndarray, topk_w: np.ndarray):
        torch = _torch()
        n = self.T * self.cfg["K"]
        if n:
            self.ids[:n].copy_(torch.from_numpy(np.ascontiguousarray(topk_idx, np.int32).reshape(-1)))
            self.w[:n].copy_(torch.from_numpy(np.ascontiguousarray(topk_w, np.float32).reshape(-1)))

    def fill_x(self, seed: int):
        inputs.cb_fill_torch(self.x.view(_torch().bfloat16), seed, inputs.STREAM_X)

    def fill_weights(self, seed: int):
        torch = _torch()
        if self.w_elems:
            inputs.cb_fill_torch(self.w_home.view(torch.bfloat16), seed, inputs.STREAM_W)
        if self.g_elems:
            inputs.cb_fill_torch(self.g_home, seed, inputs.STREAM_G_HOME)

    def fill_g_rep(self, seed: int):
        if self.g_elems:
            inputs.cb_fill_torch(self.g_rep, seed, inputs.STREAM_G_REP)

    # ----------------------------------------------------------------- calls
    def plan(self, stream=None, flags=0):
        if flags:
            mp.moonep_plan_ex(self.cfg, flags, self.ids, self.ws, stream)
        else:
            mp.moonep_plan(self.cfg, self.ids, self.ws, stream)

    def dispatch(self, stream=None):
        mp.moonep_dispatch(self.cfg, self.ws, self.x, self.ids, self.recv, self.dest, stream)

    def combine(self, y=None, stream=None):
        mp.moonep_combine(self.cfg, self.ws, self.recv if y is None else y, self.dest, self.w, self.out, stream)

    def prefetch(self, stream=None):
        mp.moonep_prefetch(self.cfg, self.ws, self.w_home, self.w_slot, self.w_elems, stream)

    def reduce_grad(self, stream=None):
        mp.moonep_reduce_grad(self.cfg, self.ws, self.g_home, self.g_rep, self.g_elems, stream)

    def read_plan(self, tables=True):
        return mp.moonep_plan_read(self.cfg, self.ws, tables=tables)

    # ------------------------------------------------------- stand-in expert
    def row_expert(self, pl=None):
        """Expert of every receive row (-1 = unused), from the plan's segment
        tables."""
        torch = _torch()
        if pl is None:
            pl = self.read_plan()
        c = self.cfg
        R, L, B, Cm = c["R"], c["L"], c["B"], c["C_max"]
        SEG = 2 * L + B
        m = np.full(R * Cm, -1, np.int64)
        so = pl["seg_off"].reshape(R, SEG)
        sl = pl["seg_len"].reshape(R, SEG)
        se = pl["slot_expert"].reshape(R, B) if B else np.zeros((R, 0), np.int64)
        for r in range(R):
            for s in range(SEG):
                if sl[r, s] == 0:
                    continue
                e = r * L + s if s < L else (se[r, s - L] if s < L + B else r * L + (s - L - B))
                m[r * Cm + so[r, s]: r * Cm + so[r, s] + sl[r, s]] = e
        # pieces without a slot (remote weights) are in the piece tables only
        for q in range(pl["n_replicas"]):
            if pl["rep_slot"][q] < 0:
                lo = pl["rep_recv"][q] * Cm + pl["rep_off"][q]
                m[lo: lo + pl["rep_cnt"][q]] = pl["rep_expert"][q]
        return torch.from_numpy(m).to(self.device)

    def expert_scale(self, scale: np.ndarray, row_expert=None):
        """y = bf16(float(recv) * scale[expert(row)]), one fp32 multiply per
        element, rows without an expert left as they are."""
        torch = _torch()
        if row_expert is None:
            row_expert = self.row_expert()
        s = torch.from_numpy(np.asarray(scale, np.float32)).to(self.device)
        used = row_expert >= 0
        y = self.recv.clone()
        rows = used.nonzero().flatten()
        if rows.numel():
            xr = self.recv[rows].view(torch.bfloat16).float()
            yr = (xr * s[row_expert[rows]][:, None]).to(torch.bfloat16)
            y[rows] = yr.view(torch.int16)
        return y

    def expert_scale_inplace(self, scale: np.ndarray, row_expert=None, chunk_rows: int = 1 << 16):
        """The same stand-in expert applied to recv in place, a chunk of rows
        at a time (for full-size buffers, where a copy of recv would not
        fit): recv[row] = bf16(float(recv[row]) * scale[expert(row)]) for every
        row with an expert."""
        torch = _torch()
        if row_expert is None:
            row_expert = self.row_expert()
        s = torch.from_numpy(np.asarray(scale, np.float32)).to(self.device)
        nrows = self.recv.shape[0]
        for r0 in range(0, nrows, chunk_rows):
            re = row_expert[r0:r0 + chunk_rows]
            rows = (re >= 0).nonzero().flatten()
            if rows.numel() == 0:
                continue
            blk = self.recv[r0:r0 + chunk_rows]
            xr = blk[rows].view(torch.bfloat16).float()
            blk[rows] = (xr * s[re[rows]][:, None]).to(torch.bfloat16).view(torch.int16)
            del xr
        return self.recv
