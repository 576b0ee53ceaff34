"""CPU oracle for the MoonEP hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package.  The product library never calls it, and it shares no
code with the CUDA path: the arithmetic lives in ``moonep_oracle.c`` (plain
single-threaded C) and this module only marshals numpy arrays into it.

Each function follows a step of the method as stated in the pages (cited in
the C file):
  plan          -- validate, histogram, keep/spill, spill planner, layout, dest
  plan_unitwise -- an independent row-at-a-time simulator of the same rule
  dispatch      -- recv[dest[g]] = x[token(g)]
  expert_scale  -- stand-in expert y = bf16(float(recv) * scale[e])
  combine       -- out = bf16(fma chain over k of w * y[dest])
  prefetch      -- w_slot[r][b] = w_home[slot_expert[r][b]]
  reduce_grad   -- g_home[e] += replicas in receiver order; zero the replicas
  combine_backward  -- grad_y[dest] = bf16(w * grad_out); grad_w = <grad_out, y[dest]> (fp64)
  dispatch_backward -- grad_x[t] = bf16(fp32 sum over k of grad_recv[dest[t,k]])
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moonep_oracle.c")
_LIB = os.path.join(_HERE, "libmoonep_oracle.so")

ST_EXPERT_ID = 0x1
ST_CAPACITY = 0x2
ST_FALLBACK = 0x100


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no OpenMP, no intrinsics)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("R", "L", "S", "K", "H", "B", "C", "C_max")]


_P = ctypes.POINTER(ctypes.c_int32)
_PLAN_FIELDS = ["cnt", "keep", "spill", "home_off", "fb_cnt", "fb_off",
                "load", "deficit", "fill", "slots_used",
                "slot_expert", "slot_cnt", "slot_off", "slot_first_j",
                "rep_ptr", "rep_expert", "rep_recv", "rep_slot", "rep_first_j", "rep_cnt",
                "rep_off", "recv_ptr", "seg_off", "seg_len", "alloc", "dest"]


class _Plan(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_int32) for n in ("status", "fallback_rows", "n_replicas",
                                               "migrated_rows")]
                + [(n, _P) for n in _PLAN_FIELDS])


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        vp = ctypes.c_void_p
        lib.or_plan_ex.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, vp, ctypes.POINTER(_Plan)]
        lib.or_plan_ex.restype = ctypes.c_int
        lib.or_plan_unitwise_ex.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, vp, vp, vp, vp, vp, vp, vp]
        lib.or_plan_unitwise_ex.restype = ctypes.c_int
        lib.or_dispatch.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp, ctypes.c_int64]
        lib.or_copy_out.argtypes = [ctypes.POINTER(_Cfg), vp, vp, ctypes.c_int, vp, vp, vp, vp, vp, vp]
        lib.or_copy_out.restype = ctypes.c_int64
        lib.or_expert_scale.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp, vp, vp, vp, ctypes.c_int,
                                        vp, vp, vp, vp, vp]
        lib.or_combine.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp, vp, vp, ctypes.c_int64]
        lib.or_prefetch.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp, ctypes.c_int64]
        lib.or_reduce_grad.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp, vp, vp, ctypes.c_int64]
        lib.or_combine_backward.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp, vp, vp, vp, ctypes.c_int64]
        lib.or_dispatch_backward.argtypes = [ctypes.POINTER(_Cfg), vp, vp, vp, vp, ctypes.c_int64]
        lib.or_f32_to_bf16_export.argtypes = [ctypes.c_float]
        lib.or_f32_to_bf16_export.restype = ctypes.c_uint16
        lib.or_bf16_to_f32_export.argtypes = [ctypes.c_uint16]
        lib.or_bf16_to_f32_export.restype = ctypes.c_float
        _lib = lib
    return _lib


def _cfg(cfg: dict) -> _Cfg:
    return _Cfg(*(int(cfg[n]) for n in ("R", "L", "S", "K", "H", "B", "C", "C_max")))


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


MODE_HEADROOM, MODE_REMOTE, MODE_ONE_GROUP = 0, 1, 2


def plan(cfg: dict, topk_idx: np.ndarray, mode: int = MODE_HEADROOM) -> dict:
    """Run the plan on int32 topk_idx [R, S, K]; returns every table plus the
    header counts as a dict of numpy arrays / ints.  mode 1: remote weights
    (pieces beyond a receiver's B slots read their expert remotely); mode 2:
    a receiver takes replicas of one home group only."""
    lib = _load()
    R, L, S, K, B = (int(cfg[n]) for n in "RLSKB")
    N = R * L
    P = N + R
    ids = np.ascontiguousarray(topk_idx, dtype=np.int32).reshape(-1)
    assert ids.size == R * S * K
    sizes = dict(cnt=N, keep=N, spill=N, home_off=N, fb_cnt=N, fb_off=N,
                 load=R, deficit=R, fill=R, slots_used=R,
                 slot_expert=R * B, slot_cnt=R * B, slot_off=R * B, slot_first_j=R * B,
                 rep_ptr=N + 1, rep_expert=P, rep_recv=P, rep_slot=P, rep_first_j=P, rep_cnt=P,
                 rep_off=P, recv_ptr=R + 1,
                 seg_off=R * (2 * L + B), seg_len=R * (2 * L + B), alloc=N * R,
                 dest=R * S * K)
    arrs = {k: np.zeros(max(v, 1), np.int32) for k, v in sizes.items()}
    p = _Plan(0, 0, 0, 0, *(arrs[k].ctypes.data_as(_P) for k in _PLAN_FIELDS))
    c = _cfg(cfg)
    lib.or_plan_ex(ctypes.byref(c), int(mode), _ptr(ids), ctypes.byref(p))
    out = {k: arrs[k][:sizes[k]] for k in _PLAN_FIELDS}
    npc = p.n_replicas
    for k in ("rep_expert", "rep_recv", "rep_slot", "rep_first_j", "rep_cnt", "rep_off"):
        out[k] = out[k][:npc]
    out["alloc"] = out["alloc"].reshape(N, R)
    out["dest"] = out["dest"].reshape(R, S, K)
    out.update(status=p.status, fallback_rows=p.fallback_rows, n_replicas=p.n_replicas,
               migrated_rows=p.migrated_rows)
    return out


def plan_unitwise(cfg: dict, topk_idx: np.ndarray, mode: int = MODE_HEADROOM) -> dict:
    lib = _load()
    R, L, S, K, B = (int(cfg[n]) for n in "RLSKB")
    N = R * L
    ids = np.ascontiguousarray(topk_idx, dtype=np.int32).reshape(-1)
    alloc = np.zeros(max(N * R, 1), np.int32)
    se = np.zeros(max(R * B, 1), np.int32)
    sc = np.zeros(max(R * B, 1), np.int32)
    fb = np.zeros(max(N, 1), np.int32)
    dest = np.zeros(max(ids.size, 1), np.int32)
    st = np.zeros(1, np.int32)
    lib.or_plan_unitwise_ex(ctypes.byref(_cfg(cfg)), int(mode), _ptr(ids), _ptr(alloc), _ptr(se),
                            _ptr(sc), _ptr(fb), _ptr(dest), _ptr(st))
    return dict(alloc=alloc[:N * R].reshape(N, R), slot_expert=se[:R * B], slot_cnt=sc[:R * B],
                fb_cnt=fb[:N], dest=dest[:ids.size].reshape(R, S, K), status=int(st[0]))


def dispatch(cfg: dict, dest: np.ndarray, x: np.ndarray, recv: np.ndarray, n_tokens=None):
    """x: uint16 bf16 bits [T, H]; recv: uint16 [R*C_max, H] (written in place)."""
    lib = _load()
    T = int(cfg["R"]) * int(cfg["S"])
    n = T if n_tokens is None else int(n_tokens)
    d = np.ascontiguousarray(dest, dtype=np.int32)
    assert x.dtype == np.uint16 and recv.dtype == np.uint16
    lib.or_dispatch(ctypes.byref(_cfg(cfg)), _ptr(d), _ptr(x), _ptr(recv), n)
    return recv


def copy_out(cfg: dict, pl: dict, recv: np.ndarray, out: np.ndarray) -> int:
    """Copy the rows the plan uses from recv to out (both uint16 [R*C_max, H]);
    returns the number of rows copied."""
    lib = _load()
    assert recv.dtype == np.uint16 and out.dtype == np.uint16
    n = int(pl["n_replicas"])
    reps = [np.ascontiguousarray(pl[k][:n], dtype=np.int32) if n else np.zeros(1, np.int32)
            for k in ("rep_recv", "rep_slot", "rep_off", "rep_cnt")]
    return int(lib.or_copy_out(ctypes.byref(_cfg(cfg)), _ptr(np.ascontiguousarray(pl["seg_off"], np.int32)),
                               _ptr(np.ascontiguousarray(pl["seg_len"], np.int32)), n,
                               *(_ptr(a) for a in reps), _ptr(recv), _ptr(out)))


def expert_scale(cfg: dict, pl: dict, recv: np.ndarray, scale: np.ndarray, y: np.ndarray):
    lib = _load()
    n = int(pl["n_replicas"])
    reps = [np.ascontiguousarray(pl[k][:n], dtype=np.int32) if n else np.zeros(1, np.int32)
            for k in ("rep_expert", "rep_recv", "rep_slot", "rep_off", "rep_cnt")]
    lib.or_expert_scale(ctypes.byref(_cfg(cfg)), _ptr(np.ascontiguousarray(pl["seg_off"])),
                        _ptr(np.ascontiguousarray(pl["seg_len"])),
                        _ptr(np.ascontiguousarray(pl["slot_expert"])), _ptr(recv),
                        _ptr(np.ascontiguousarray(scale, dtype=np.float32)), _ptr(y), n,
                        *(_ptr(a) for a in reps))
    return y


def combine(cfg: dict, dest: np.ndarray, y: np.ndarray, w: np.ndarray, n_tokens=None):
    """Returns (out uint16 bf16 bits [n, H], acc fp32 [n, H])."""
    lib = _load()
    T = int(cfg["R"]) * int(cfg["S"])
    n = T if n_tokens is None else int(n_tokens)
    H = int(cfg["H"])
    out = np.zeros((max(n, 1), H), np.uint16)
    acc = np.zeros((max(n, 1), H), np.float32)
    lib.or_combine(ctypes.byref(_cfg(cfg)), _ptr(np.ascontiguousarray(dest, dtype=np.int32)),
                   _ptr(y), _ptr(np.ascontiguousarray(w, dtype=np.float32)), _ptr(out),
                   _ptr(acc), n)
    return out[:n], acc[:n]


def prefetch(cfg: dict, slot_expert: np.ndarray, w_home: np.ndarray, w_slot: np.ndarray,
             elems: int):
    lib = _load()
    lib.or_prefetch(ctypes.byref(_cfg(cfg)), _ptr(np.ascontiguousarray(slot_expert, np.int32)),
                    _ptr(w_home), _ptr(w_slot), int(elems))
    return w_slot


def reduce_grad(cfg: dict, pl: dict, g_home: np.ndarray, g_rep: np.ndarray, elems: int):
    lib = _load()
    rp = np.ascontiguousarray(pl["rep_ptr"], np.int32)
    rr = np.ascontiguousarray(pl["rep_recv"], np.int32)
    rs = np.ascontiguousarray(pl["rep_slot"], np.int32)
    if rr.size == 0:
        rr = np.zeros(1, np.int32)
        rs = np.zeros(1, np.int32)
    lib.or_reduce_grad(ctypes.byref(_cfg(cfg)), _ptr(rp), _ptr(rr), _ptr(rs), _ptr(g_home),
                       _ptr(g_rep), int(elems))
    return g_home, g_rep


def combine_backward(cfg: dict, dest: np.ndarray, grad_out: np.ndarray, y: np.ndarray, w: np.ndarray,
                     grad_y: np.ndarray, n_tokens=None, with_grad_w=True):
    """grad_out: uint16 bf16 [n, H]; y, grad_y: uint16 [R*C_max, H] (grad_y
    written in place at the dispatched rows).  Returns grad_w fp64 [n, K]."""
    lib = _load()
    T = int(cfg["R"]) * int(cfg["S"])
    n = T if n_tokens is None else int(n_tokens)
    K = int(cfg["K"])
    gw = np.zeros((max(n, 1), K), np.float64)
    lib.or_combine_backward(ctypes.byref(_cfg(cfg)), _ptr(np.ascontiguousarray(dest, dtype=np.int32)),
                            _ptr(grad_out), _ptr(y), _ptr(np.ascontiguousarray(w, dtype=np.float32)),
                            _ptr(grad_y), _ptr(gw) if with_grad_w else None, n)
    return gw[:n]


def dispatch_backward(cfg: dict, dest: np.ndarray, grad_recv: np.ndarray, n_tokens=None):
    """Returns (grad_x uint16 bf16 [n, H], acc fp32 [n, H])."""
    lib = _load()
    T = int(cfg["R"]) * int(cfg["S"])
    n = T if n_tokens is None else int(n_tokens)
    H = int(cfg["H"])
    gx = np.zeros((max(n, 1), H), np.uint16)
    acc = np.zeros((max(n, 1), H), np.float32)
    lib.or_dispatch_backward(ctypes.byref(_cfg(cfg)), _ptr(np.ascontiguousarray(dest, dtype=np.int32)),
                             _ptr(grad_recv), _ptr(gx), _ptr(acc), n)
    return gx[:n], acc[:n]


def f32_to_bf16(f: float) -> int:
    return int(_load().or_f32_to_bf16_export(float(f)))


def bf16_to_f32(u: int) -> float:
    return float(_load().or_bf16_to_f32_export(int(u)))
