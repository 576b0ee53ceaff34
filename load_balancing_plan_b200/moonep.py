"""Python binding of the MoonEP C ABI (include/moonep.h), by ctypes.

Argument marshalling only: every function below passes raw device pointers,
sizes and the CUDA stream to the function of the same name in libmoonep.so;
every step of the path runs in the library's sm_100a kernels.  Tensors may be
torch tensors (their data_ptr() is passed) or plain integer addresses.  The
library must be built (``python -m load_balancing_plan_b200.build``); there
is no fallback implementation, and importing this module fails loudly when
the library is missing.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOONEP_LIBRARY may point at another build of the same library (development
# builds with different tuning constants); the default is the in-tree build.
LIB_PATH = os.environ.get("MOONEP_LIBRARY") or os.path.join(_PKG, "libmoonep.so")

OK, ERR_ARG, ERR_CUDA, ERR_DEVICE = 0, 1, 2, 3
ST_EXPERT_ID, ST_CAPACITY, ST_TIMEOUT, ST_DEST, ST_CFG = 0x1, 0x2, 0x4, 0x8, 0x10
ST_ERROR_MASK, ST_FALLBACK = 0xFF, 0x100
WS_HEADER_WORDS = 64
PLAN_REMOTE_WEIGHTS = 0x1
PLAN_ONE_GROUP = 0x2


class MoonepError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("moonep error %d: %s" % (code, msg))
        self.code = code


class Cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("R", "L", "S", "K", "H", "B", "C", "C_max")]


class PlanInfo(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("status", "fallback_rows", "n_replicas", "migrated_rows")]


LAYOUT_FIELDS = ["words", "n_ranges", "max_pieces", "cnt", "keep", "spill", "home_off", "fb_cnt",
                 "fb_off", "load", "deficit", "fill", "slots_used", "slot_expert", "slot_cnt",
                 "slot_off", "slot_first_j", "rep_ptr", "rep_expert", "rep_recv", "rep_slot",
                 "rep_first_j", "rep_cnt", "rx_expert", "route_ptr", "route_end", "route_base",
                 "seg_off", "seg_len", "alloc", "tables_end", "base", "rep_off", "recv_ptr",
                 "slot_piece", "n_blocks", "blk"]


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in LAYOUT_FIELDS]


class RankBytes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("dispatch_bytes", "prefetch_bytes", "reduce_bytes")]


if not os.path.exists(LIB_PATH):
    raise ImportError("libmoonep.so is not built (%s); run python -m load_balancing_plan_b200.build"
                      % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i64 = ctypes.c_void_p, ctypes.c_int64
_CP = ctypes.POINTER(Cfg)
_sig = {
    "moonep_ws_layout": ([_CP, ctypes.POINTER(WsLayout)], ctypes.c_int),
    "moonep_plan_workspace_bytes": ([_CP], ctypes.c_size_t),
    "moonep_rank_bytes": ([_CP, _i64, ctypes.POINTER(RankBytes)], ctypes.c_int),
    "moonep_plan": ([_CP, _vp, _vp, _vp], ctypes.c_int),
    "moonep_plan_ex": ([_CP, ctypes.c_int32, _vp, _vp, _vp], ctypes.c_int),
    "moonep_dispatch": ([_CP, _vp, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moonep_combine": ([_CP, _vp, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moonep_prefetch": ([_CP, _vp, _vp, _vp, _i64, _vp], ctypes.c_int),
    "moonep_reduce_grad": ([_CP, _vp, _vp, _vp, _i64, _vp], ctypes.c_int),
    "moonep_plan_read": ([_CP, _vp, ctypes.POINTER(PlanInfo), _vp, _vp], ctypes.c_int),
    "moonep_plan_noalloc": ([_CP, _vp, _vp, _vp], ctypes.c_int),
    "moonep_combine_backward": ([_CP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moonep_dispatch_backward": ([_CP, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moonep_copy_out": ([_CP, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moonep_view_generation": ([_vp], _i64),
    "moonep_ep_ws_layout": ([_CP, ctypes.POINTER(WsLayout)], ctypes.c_int),
    "moonep_ep_workspace_bytes": ([_CP], ctypes.c_size_t),
    "moonep_ep_count": ([_CP, ctypes.c_int32, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moonep_ep_count_exchange": ([_CP, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moonep_ep_plan": ([_CP, ctypes.c_int32, ctypes.c_int32, _vp, _vp, _vp], ctypes.c_int),
    "moonep_ep_dispatch": ([_CP, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moonep_ep_combine": ([_CP, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moonep_ep_combine_backward": ([_CP, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moonep_ep_dispatch_backward": ([_CP, ctypes.c_int32, _vp, _vp, _vp, _vp, _vp], ctypes.c_int),
    "moonep_ep_prefetch": ([_CP, ctypes.c_int32, _vp, _vp, _vp, _i64, _vp], ctypes.c_int),
    "moonep_ep_reduce_grad": ([_CP, ctypes.c_int32, _vp, _vp, _vp, _i64, _vp], ctypes.c_int),
    "moonep_set_wait_limit": ([_i64], ctypes.c_int),
    "moonep_num_ranges": ([_i64, _i64], _i64),
    "moonep_last_error": ([], ctypes.c_char_p),
    "moonep_version": ([], ctypes.c_char_p),
}
for _name, (_args, _res) in _sig.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res

EXPORTS = tuple(_sig)


def cfg_of(d) -> Cfg:
    if isinstance(d, Cfg):
        return d
    return Cfg(*(int(d[n]) for n in ("R", "L", "S", "K", "H", "B", "C", "C_max")))


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    raise TypeError("cannot pass %r as a pointer" % type(t))


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc):
    if rc != OK:
        raise MoonepError(rc, last_error())
    return rc


def last_error() -> str:
    return _lib.moonep_last_error().decode()


def version() -> str:
    return _lib.moonep_version().decode()


def moonep_ws_layout(cfg) -> dict:
    out = WsLayout()
    _check(_lib.moonep_ws_layout(ctypes.byref(cfg_of(cfg)), ctypes.byref(out)))
    return {n: getattr(out, n) for n in LAYOUT_FIELDS}


def moonep_plan_workspace_bytes(cfg) -> int:
    n = _lib.moonep_plan_workspace_bytes(ctypes.byref(cfg_of(cfg)))
    if n == 0:
        raise MoonepError(ERR_ARG, last_error())
    return int(n)


def moonep_rank_bytes(cfg, elems_per_expert) -> dict:
    out = RankBytes()
    _check(_lib.moonep_rank_bytes(ctypes.byref(cfg_of(cfg)), int(elems_per_expert), ctypes.byref(out)))
    return dict(dispatch_bytes=out.dispatch_bytes, prefetch_bytes=out.prefetch_bytes,
                reduce_bytes=out.reduce_bytes)


def moonep_num_ranges(T, N) -> int:
    return int(_lib.moonep_num_ranges(int(T), int(N)))


def moonep_set_wait_limit(polls) -> None:
    _check(_lib.moonep_set_wait_limit(int(polls)))


def moonep_plan(cfg, topk_idx, ws, stream=None) -> None:
    _check(_lib.moonep_plan(ctypes.byref(cfg_of(cfg)), _p(topk_idx), _p(ws), _stream(stream)))


def moonep_plan_ex(cfg, flags, topk_idx, ws, stream=None) -> None:
    _check(_lib.moonep_plan_ex(ctypes.byref(cfg_of(cfg)), int(flags), _p(topk_idx), _p(ws), _stream(stream)))


def moonep_plan_noalloc(cfg, topk_idx, tables_out, stream=None) -> None:
    """moonep_plan without a caller workspace: the library's static device
    workspace is used and the header + tables are copied to tables_out
    (at least layout["tables_end"] int32 words).  The copy is tables only:
    moonep_dispatch refuses it as a workspace.  A tensor smaller than the
    copy is refused here (the C function sees only its address)."""
    if hasattr(tables_out, "numel") and hasattr(tables_out, "element_size"):
        need = 4 * moonep_ws_layout(cfg)["tables_end"]
        have = int(tables_out.numel()) * int(tables_out.element_size())
        if have < need:
            raise MoonepError(ERR_ARG, "moonep_plan_noalloc: tables_out holds %d bytes, the plan tables need %d"
                              % (have, need))
    _check(_lib.moonep_plan_noalloc(ctypes.byref(cfg_of(cfg)), _p(topk_idx), _p(tables_out),
                                    _stream(stream)))


def moonep_dispatch(cfg, ws, x, topk_idx, recv, dest, stream=None) -> None:
    _check(_lib.moonep_dispatch(ctypes.byref(cfg_of(cfg)), _p(ws), _p(x), _p(topk_idx), _p(recv),
                                _p(dest), _stream(stream)))


def moonep_copy_out(cfg, ws, recv, out, stream=None) -> None:
    _check(_lib.moonep_copy_out(ctypes.byref(cfg_of(cfg)), _p(ws), _p(recv), _p(out), _stream(stream)))


def moonep_view_generation(ws) -> int:
    return int(_lib.moonep_view_generation(_p(ws)))


def moonep_combine(cfg, ws, y, dest, topk_w, out, stream=None) -> None:
    _check(_lib.moonep_combine(ctypes.byref(cfg_of(cfg)), _p(ws), _p(y), _p(dest), _p(topk_w),
                               _p(out), _stream(stream)))


def moonep_combine_backward(cfg, ws, grad_out, y, dest, topk_w, grad_y, grad_w=None, stream=None) -> None:
    _check(_lib.moonep_combine_backward(ctypes.byref(cfg_of(cfg)), _p(ws), _p(grad_out), _p(y), _p(dest),
                                        _p(topk_w), _p(grad_y), _p(grad_w), _stream(stream)))


def moonep_dispatch_backward(cfg, ws, grad_recv, dest, grad_x, stream=None) -> None:
    _check(_lib.moonep_dispatch_backward(ctypes.byref(cfg_of(cfg)), _p(ws), _p(grad_recv), _p(dest),
                                         _p(grad_x), _stream(stream)))


def moonep_prefetch(cfg, ws, w_home, w_slot, elems_per_expert, stream=None) -> None:
    _check(_lib.moonep_prefetch(ctypes.byref(cfg_of(cfg)), _p(ws), _p(w_home), _p(w_slot),
                                int(elems_per_expert), _stream(stream)))


def moonep_reduce_grad(cfg, ws, g_home, g_rep, elems_per_expert, stream=None) -> None:
    _check(_lib.moonep_reduce_grad(ctypes.byref(cfg_of(cfg)), _p(ws), _p(g_home), _p(g_rep),
                                   int(elems_per_expert), _stream(stream)))


# ---------------------------------------------------------------- expert parallelism
# one rank's calls; peer tables are device arrays of R pointers (int64)

def moonep_ep_ws_layout(cfg) -> dict:
    out = WsLayout()
    _check(_lib.moonep_ep_ws_layout(ctypes.byref(cfg_of(cfg)), ctypes.byref(out)))
    return {n: getattr(out, n) for n in LAYOUT_FIELDS}


def moonep_ep_workspace_bytes(cfg) -> int:
    n = _lib.moonep_ep_workspace_bytes(ctypes.byref(cfg_of(cfg)))
    if n == 0:
        raise MoonepError(ERR_ARG, last_error())
    return int(n)


def moonep_ep_count(cfg, rank, topk_idx, ws, counts, stream=None) -> None:
    _check(_lib.moonep_ep_count(ctypes.byref(cfg_of(cfg)), int(rank), _p(topk_idx), _p(ws), _p(counts),
                                _stream(stream)))


def moonep_ep_count_exchange(cfg, rank, topk_idx, ws, counts, counts_all_peers, stream=None) -> None:
    _check(_lib.moonep_ep_count_exchange(ctypes.byref(cfg_of(cfg)), int(rank), _p(topk_idx), _p(ws), _p(counts),
                                         _p(counts_all_peers), _stream(stream)))


def moonep_ep_plan(cfg, flags, rank, counts_all, ws, stream=None) -> None:
    _check(_lib.moonep_ep_plan(ctypes.byref(cfg_of(cfg)), int(flags), int(rank), _p(counts_all), _p(ws),
                               _stream(stream)))


def moonep_ep_dispatch(cfg, rank, ws, x, topk_idx, recv_peers, dest, stream=None) -> None:
    _check(_lib.moonep_ep_dispatch(ctypes.byref(cfg_of(cfg)), int(rank), _p(ws), _p(x), _p(topk_idx),
                                   _p(recv_peers), _p(dest), _stream(stream)))


def moonep_ep_combine(cfg, rank, ws, y_peers, dest, topk_w, out, stream=None) -> None:
    _check(_lib.moonep_ep_combine(ctypes.byref(cfg_of(cfg)), int(rank), _p(ws), _p(y_peers), _p(dest),
                                  _p(topk_w), _p(out), _stream(stream)))


def moonep_ep_combine_backward(cfg, rank, ws, grad_out, y_peers, dest, topk_w, grad_y_peers, grad_w=None,
                               stream=None) -> None:
    _check(_lib.moonep_ep_combine_backward(ctypes.byref(cfg_of(cfg)), int(rank), _p(ws), _p(grad_out), _p(y_peers),
                                           _p(dest), _p(topk_w), _p(grad_y_peers), _p(grad_w), _stream(stream)))


def moonep_ep_dispatch_backward(cfg, rank, ws, grad_recv_peers, dest, grad_x, stream=None) -> None:
    _check(_lib.moonep_ep_dispatch_backward(ctypes.byref(cfg_of(cfg)), int(rank), _p(ws), _p(grad_recv_peers),
                                            _p(dest), _p(grad_x), _stream(stream)))


def moonep_ep_prefetch(cfg, rank, ws, w_home_peers, w_slot, elems_per_expert, stream=None) -> None:
    _check(_lib.moonep_ep_prefetch(ctypes.byref(cfg_of(cfg)), int(rank), _p(ws), _p(w_home_peers), _p(w_slot),
                                   int(elems_per_expert), _stream(stream)))


def moonep_ep_reduce_grad(cfg, rank, ws, g_home, g_rep_peers, elems_per_expert, stream=None) -> None:
    _check(_lib.moonep_ep_reduce_grad(ctypes.byref(cfg_of(cfg)), int(rank), _p(ws), _p(g_home), _p(g_rep_peers),
                                      int(elems_per_expert), _stream(stream)))


def moonep_plan_read(cfg, ws, tables=False, stream=None):
    """Header counts (and, with tables=True, every table as numpy arrays keyed
    by the layout names, reshaped like the header documents them)."""
    info = PlanInfo()
    lay = moonep_ws_layout(cfg)
    host = None
    if tables:
        host = np.zeros(lay["tables_end"] - lay["cnt"], np.int32)
    _check(_lib.moonep_plan_read(ctypes.byref(cfg_of(cfg)), _p(ws), ctypes.byref(info),
                                 None if host is None else host.ctypes.data, _stream(stream)))
    out = dict(status=info.status, fallback_rows=info.fallback_rows, n_replicas=info.n_replicas,
               migrated_rows=info.migrated_rows)
    if tables:
        c = cfg_of(cfg)
        R, L, B = c.R, c.L, c.B
        N = R * L
        P = info.n_replicas
        sizes = dict(cnt=N, keep=N, spill=N, home_off=N, fb_cnt=N, fb_off=N, load=R, deficit=R,
                     fill=R, slots_used=R, slot_expert=R * B, slot_cnt=R * B, slot_off=R * B,
                     slot_first_j=R * B, rep_ptr=N + 1, rep_expert=P, rep_recv=P, rep_slot=P,
                     rep_first_j=P, rep_cnt=P, rep_off=P, recv_ptr=R + 1, slot_piece=R * B,
                     rx_expert=N, route_ptr=N + 1,
                     route_end=2 * N + P, route_base=2 * N + P, seg_off=R * (2 * L + B),
                     seg_len=R * (2 * L + B), alloc=N * R)
        for k, n in sizes.items():
            o = lay[k] - lay["cnt"]
            out[k] = host[o:o + n].copy()
        out["alloc"] = out["alloc"].reshape(N, R)
    return out
