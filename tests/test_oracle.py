"""Pins for the CPU oracle, against what the pages and the mathematics fix:
brute-force enumeration against an independent row-at-a-time simulator,
invariants, closed forms, special cases that reduce to a library sort, the
pages' printed numbers, and error bounds for the float steps."""
import itertools

import numpy as np
import pytest

from tests import planchecks as pc
from load_balancing_plan_b200 import inputs


def _cfg(R, L, S, K, H, B, C_max=None):
    C = S * K
    return dict(R=R, L=L, S=S, K=K, H=H, B=B, C=C, C_max=C if C_max is None else C_max)


def _compare_unitwise(oracle, cfg, ids):
    pl = oracle.plan(cfg, ids)
    un = oracle.plan_unitwise(cfg, ids)
    assert pl["status"] == un["status"]
    if pl["status"] & oracle.ST_CAPACITY:
        return pl
    assert np.array_equal(pl["dest"], un["dest"])
    assert np.array_equal(pl["alloc"], un["alloc"])
    assert np.array_equal(pl["slot_expert"], un["slot_expert"])
    assert np.array_equal(pl["slot_cnt"], un["slot_cnt"])
    assert np.array_equal(pl["fb_cnt"], un["fb_cnt"])
    pc.check_plan(cfg, ids, pl)
    return pl


def _enumerate(oracle, R, L, S, K, B, C_max_mult=None, distinct=True):
    N = R * L
    T = R * S
    C = S * K
    cfg = _cfg(R, L, S, K, 8, B, None if C_max_mult is None else C * C_max_mult)
    if distinct:
        choices = list(itertools.permutations(range(N), K))
    else:
        choices = list(itertools.product(range(N), repeat=K))
    n_fb = n_full = 0
    for combo in itertools.product(range(len(choices)), repeat=T):
        ids = np.array([choices[c] for c in combo], np.int32).reshape(R, S, K)
        pl = _compare_unitwise(oracle, cfg, ids)
        n_full += 1
        n_fb += pl["fallback_rows"] > 0
    return n_full, n_fb


@pytest.mark.parametrize("R,L,S,K,B,mult,expect", [
    (2, 2, 2, 2, 2, None, 20736),   # 12^4 inputs, distinct K
    (3, 1, 2, 1, 1, None, 729),
    (2, 2, 3, 1, 2, None, 4096),
    (2, 2, 3, 1, 0, 2, 4096),       # no slots at all: every overflow row falls back
])
def test_bruteforce_matches_unitwise(oracle_lib, R, L, S, K, B, mult, expect):
    n, _ = _enumerate(oracle_lib, R, L, S, K, B, mult)
    assert n == expect


def test_bruteforce_slot_limited(oracle_lib):
    # R=4, L=1, S=2, K=1, B=1: 65536 inputs; contains inputs where a receiver
    # would need more than B slots, so the headroom fallback is exercised
    n, n_fb = _enumerate(oracle_lib, 4, 1, 2, 1, 1, 4)
    assert n == 4 ** 8
    assert n_fb > 0


def test_known_gap_example(oracle_lib):
    # ranks 0-2 each one row over capacity in their second expert, rank 3 with
    # a deficit of 3: it would need 3 slots but has B = 2, so one row falls back
    R, L, S, K, B = 4, 2, 2, 2, 2
    cfg = _cfg(R, L, S, K, 8, B, 8)
    cnt = np.array([2, 3, 2, 3, 2, 3, 1, 0])
    ids = pc.ids_from_counts(cnt, R, S, K)
    pl = _compare_unitwise(oracle_lib, cfg, ids)
    assert pl["fallback_rows"] == 1
    assert pl["slots_used"].tolist() == [0, 0, 0, 2]
    assert pl["status"] & oracle_lib.ST_FALLBACK


def test_capacity_error(oracle_lib):
    R, L, S, K, B = 4, 2, 2, 2, 0
    cfg = _cfg(R, L, S, K, 8, B)                 # no headroom, no slots
    ids = pc.ids_from_counts(np.array([4, 4, 2, 2, 2, 2, 0, 0]), R, S, K)
    pl = oracle_lib.plan(cfg, ids)
    assert pl["status"] & oracle_lib.ST_CAPACITY


def test_bad_expert_id(oracle_lib):
    cfg = _cfg(2, 2, 2, 1, 8, 1)
    ids = np.array([0, 1, 4, 2], np.int32).reshape(2, 2, 1)
    assert oracle_lib.plan(cfg, ids)["status"] & oracle_lib.ST_EXPERT_ID
    ids = np.array([0, -1, 3, 2], np.int32).reshape(2, 2, 1)
    assert oracle_lib.plan(cfg, ids)["status"] & oracle_lib.ST_EXPERT_ID


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("B", [0, 1, 2, 4])
def test_random_histograms(oracle_lib, seed, B):
    # the plan tables depend only on the histogram; drive the planner from
    # random skewed histograms realised with distinct experts per token
    rng = np.random.default_rng(seed)
    R, L, S, K = 8, 4, 64, 4
    cnt = pc.random_counts(rng, R * L, R * S, K, skew=1.0 + seed)
    ids = pc.ids_from_counts(cnt, R, S, K)
    cfg = _cfg(R, L, S, K, 8, B, R * S * K)
    _compare_unitwise(oracle_lib, cfg, ids)


@pytest.mark.parametrize("seed", range(5))
def test_spec_workloads_small(oracle_lib, seed):
    # tiny workload of the library (R=4, L=4, S=64, K=2, B=4), bias scale 1
    w = inputs.WORKLOADS["tiny"]
    r = inputs.routing(w.R, w.L, w.S, w.K, seed, alpha=1.0)
    pl = _compare_unitwise(oracle_lib, w.cfg(), r.topk_idx)
    assert pl["fallback_rows"] == 0


def test_balanced_is_counting_sort(oracle_lib):
    # maxvio = 0: no rank overflows, so each home rank's rows are a stable
    # counting sort of its copies by expert
    R, L, S, K = 4, 4, 64, 2
    r = inputs.routing(R, L, S, K, 0, balanced=True)
    cfg = _cfg(R, L, S, K, 8, 4)
    pl = oracle_lib.plan(cfg, r.topk_idx)
    assert pl["migrated_rows"] == 0 and pl["n_replicas"] == 0
    ids = r.topk_idx.reshape(-1).astype(np.int64)
    g = np.arange(ids.size)
    expect = np.empty(ids.size, np.int64)
    for h in range(R):
        sel = g[ids // L == h]
        order = sel[np.argsort(ids[sel], kind="stable")]
        expect[order] = h * cfg["C_max"] + np.arange(order.size)
    assert np.array_equal(pl["dest"].reshape(-1), expect)


def test_single_rank_is_stable_sort(oracle_lib):
    # R = 1, K = 1: dest is the position in a stable sort by expert id
    rng = np.random.default_rng(3)
    S, L = 500, 7
    ids = rng.integers(0, L, S).astype(np.int32).reshape(1, S, 1)
    cfg = _cfg(1, L, S, 1, 8, 2)
    pl = oracle_lib.plan(cfg, ids)
    perm = np.argsort(ids.reshape(-1), kind="stable")
    inv = np.empty(S, np.int64)
    inv[perm] = np.arange(S)
    assert np.array_equal(pl["dest"].reshape(-1), inv)


def test_empty_input(oracle_lib):
    cfg = _cfg(4, 2, 0, 2, 8, 2)
    ids = np.zeros((4, 0, 2), np.int32)
    pl = oracle_lib.plan(cfg, ids)
    assert pl["status"] == 0 and pl["n_replicas"] == 0
    assert pl["alloc"].sum() == 0


# ---------------------------------------------------------------------------
# The pages' printed numbers
# ---------------------------------------------------------------------------

def _read_planning_table():
    import os
    rows = []
    with open(os.path.join(os.path.dirname(__file__), "golden", "planning_table.txt")) as f:
        for line in f:
            if line.startswith("#") or "=" in line or not line.strip():
                continue
            rows.append([float(x) for x in line.split()])
    return np.array(rows)


def test_planning_table_arithmetic():
    # the page's own columns agree: peak/mean = peak / (S*K), and the tokens
    # that must leave the hottest rank bound the migrated share from below
    t = _read_planning_table()
    cap, total = 16384, 8 * 16384
    assert np.allclose(t[:, 3], t[:, 1] / cap, atol=6e-4)
    assert np.all(t[:, 5] / 100 + 1e-4 >= (t[:, 1] - cap) / total)
    assert np.all(t[:, 4] == 1.0)


@pytest.mark.parametrize("sigma", [0.0, 0.5, 1.0, 2.0, 5.0])
def test_planning_table_setup_balances(oracle_lib, sigma):
    # the page's setup (256 experts, 8 ranks, S=2048, K=8) with B = E/R = 32:
    # every rank receives exactly 16384 rows at every skew (the page's
    # MoonEP peak/mean column is 1.000000 throughout)
    R, L, S, K = 8, 32, 2048, 8
    if sigma == 0.0:
        r = inputs.routing(R, L, S, K, 0, balanced=True)
    else:
        r = inputs.lognormal_routing(R, L, S, K, 0, sigma)
    cfg = _cfg(R, L, S, K, 8, 32)
    pl = oracle_lib.plan(cfg, r.topk_idx)
    info = pc.check_plan(cfg, r.topk_idx, pl)
    assert pl["fallback_rows"] == 0
    assert np.all(info["rows"] == 16384)
    peak = pl["load"].max()
    assert pl["migrated_rows"] >= peak - 16384


# ---------------------------------------------------------------------------
# Float steps
# ---------------------------------------------------------------------------

def test_bf16_rounding_matches_torch(oracle_lib):
    import torch
    rng = np.random.default_rng(0)
    f = np.concatenate([
        rng.standard_normal(4000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),    # subnormals
        np.array([0.0, -0.0, np.inf, -np.inf, 1.0, 3.0e38, -3.4e38], np.float32),
        # exact ties between two bf16 values, both parities
        (np.arange(0, 200, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
    ]).astype(np.float32)
    ours = np.array([oracle_lib.f32_to_bf16(v) for v in f], np.uint16)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    nan = oracle_lib.f32_to_bf16(float("nan"))
    assert (nan & 0x7F80) == 0x7F80 and (nan & 0x7F)
    assert oracle_lib.bf16_to_f32(0x3F80) == 1.0


def _tiny_e2e(oracle, seed, K=2, scale=None):
    w = inputs.WORKLOADS["tiny"]
    cfg = dict(w.cfg(), K=K, C=w.S * K, C_max=2 * w.S * K)
    r = inputs.routing(w.R, w.L, w.S, K, seed, alpha=1.0)
    pl = oracle.plan(cfg, r.topk_idx)
    assert not (pl["status"] & (oracle.ST_CAPACITY | oracle.ST_EXPERT_ID))
    T, H = w.T, w.H
    x = inputs.cb_bf16_np(seed, inputs.STREAM_X, np.arange(T * H)).reshape(T, H)
    recv = np.zeros((w.R * cfg["C_max"], H), np.uint16)
    oracle.dispatch(cfg, pl["dest"], x, recv)
    return cfg, r, pl, x, recv


@pytest.mark.parametrize("seed", range(3))
def test_dispatch_places_rows(oracle_lib, seed):
    cfg, r, pl, x, recv = _tiny_e2e(oracle_lib, seed)
    d = pl["dest"].reshape(-1)
    tok = np.repeat(np.arange(x.shape[0]), cfg["K"])
    assert np.array_equal(recv[d], x[tok])
    used = np.zeros(recv.shape[0], bool)
    used[d] = True
    assert np.all(recv[~used] == 0)    # rows outside the plan untouched


@pytest.mark.parametrize("seed", range(3))
def test_expert_and_combine_against_fp64(oracle_lib, seed):
    import torch
    cfg, r, pl, x, recv = _tiny_e2e(oracle_lib, seed)
    N = cfg["R"] * cfg["L"]
    scale = inputs.expert_scales(N, seed)
    y = np.zeros_like(recv)
    oracle_lib.expert_scale(cfg, pl, recv, scale, y)
    # stand-in expert: one fp32 multiply rounded to bf16 (torch as the check)
    rexp = pc.row_expert_map(cfg, pl)
    used = rexp >= 0
    xf = torch.from_numpy(inputs.bf16_bits_to_f32_np(recv[used]))
    sf = torch.from_numpy(scale[rexp[used]])[:, None]
    ref = (xf * sf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(y[used], ref)
    # combine against the plain definition out = sum_k w_k y_k in fp64
    out, acc = oracle_lib.combine(cfg, pl["dest"], y, r.topk_w)
    K = cfg["K"]
    d = pl["dest"].reshape(-1, K)
    yv = inputs.bf16_bits_to_f32_np(y).astype(np.float64)
    terms = r.topk_w.reshape(-1, K, 1).astype(np.float64) * yv[d]
    exact = terms.sum(1)
    bound = K * 2.0 ** -24 * np.abs(terms).sum(1)
    assert np.all(np.abs(acc - exact) <= bound + 1e-30)
    outf = inputs.bf16_bits_to_f32_np(out)
    assert np.all(np.abs(outf - acc) <= 2.0 ** -8 * np.abs(acc))
    nz = exact != 0
    assert np.max(np.abs(outf[nz] - exact[nz]) / np.abs(exact[nz])) <= 4e-3


@pytest.mark.parametrize("K", [2, 4])
def test_combine_mean_of_copies_is_exact(oracle_lib, K):
    # weights 1/K (a power of two), identity expert: the mean of K copies of
    # the same row is that row, bit for bit
    cfg, r, pl, x, recv = _tiny_e2e(oracle_lib, 1, K=K)
    w = np.full(r.topk_w.shape, 1.0 / K, np.float32)
    out, _ = oracle_lib.combine(cfg, pl["dest"], recv, w)
    assert np.array_equal(out, x)


def test_combine_detects_planted_mistakes(oracle_lib):
    # the fp64 check above fails for a dropped term or a wrong index
    cfg, r, pl, x, recv = _tiny_e2e(oracle_lib, 2)
    K = cfg["K"]
    out, acc = oracle_lib.combine(cfg, pl["dest"], recv, r.topk_w)
    d = pl["dest"].reshape(-1, K)
    yv = inputs.bf16_bits_to_f32_np(recv).astype(np.float64)
    w = r.topk_w.reshape(-1, K, 1).astype(np.float64)
    exact = (w * yv[d]).sum(1)
    dropped = (w[:, :1] * yv[d[:, :1]]).sum(1)
    assert np.max(np.abs(dropped - exact)) > 1e-2
    swapped = (w * yv[np.roll(d, 1, axis=0)]).sum(1)
    assert np.max(np.abs(swapped - exact)) > 1e-2


def test_prefetch_and_reduce_grad(oracle_lib):
    w = inputs.WORKLOADS["tiny"]
    cfg = w.cfg()
    r = inputs.routing(w.R, w.L, w.S, w.K, 0, alpha=1.0)
    pl = oracle_lib.plan(cfg, r.topk_idx)
    N, R, B = w.N, w.R, w.B
    assert pl["n_replicas"] > 0
    # prefetch: slots hold copies of their experts; empty slots untouched
    E = 64
    w_home = inputs.cb_bf16_np(0, inputs.STREAM_W, np.arange(N * E)).reshape(N, E)
    w_slot = np.full((R * B, E), 0xFFFF, np.uint16)
    oracle_lib.prefetch(cfg, pl["slot_expert"], w_home, w_slot, E)
    se = pl["slot_expert"]
    assert np.array_equal(w_slot[se >= 0], w_home[se[se >= 0]])
    assert np.all(w_slot[se < 0] == 0xFFFF)
    # reduce_grad: fp32 sum in receiver order, within the recursive-summation
    # bound of the exact sum; used slots zeroed; other slots and experts kept
    g_home = inputs.cb_f32_np(0, inputs.STREAM_G_HOME, np.arange(N * E)).reshape(N, E)
    g_rep = inputs.cb_f32_np(0, inputs.STREAM_G_REP, np.arange(R * B * E)).reshape(R * B, E)
    h0, r0 = g_home.copy(), g_rep.copy()
    oracle_lib.reduce_grad(cfg, pl, g_home, g_rep, E)
    slot_of = pl["rep_recv"] * B + pl["rep_slot"]
    for e in range(N):
        q = slot_of[pl["rep_ptr"][e]:pl["rep_ptr"][e + 1]]
        terms = np.concatenate([h0[e:e + 1], r0[q]]).astype(np.float64)
        exact = terms.sum(0)
        bound = len(q) * 2.0 ** -24 * np.abs(terms).sum(0)
        assert np.all(np.abs(g_home[e] - exact) <= bound)
        if len(q) == 0:
            assert np.array_equal(g_home[e], h0[e])
    used = np.zeros(R * B, bool)
    used[slot_of] = True
    assert np.all(g_rep[used] == 0)
    assert np.array_equal(g_rep[~used], r0[~used])


# ---------------------------------------------------------------------------
# The input generator (shared by both sides, holds none of the method)
# ---------------------------------------------------------------------------

def test_counter_generator_host_device_forms_agree():
    import torch
    idx = np.arange(5000)
    a = inputs.cb_f32_np(3, inputs.STREAM_X, idx)
    t = torch.empty(5000, dtype=torch.float32)
    inputs.cb_fill_torch(t, 3, inputs.STREAM_X, chunk=1234)
    assert np.array_equal(a, t.numpy())
    tb = torch.empty(5000, dtype=torch.bfloat16)
    inputs.cb_fill_torch(tb, 3, inputs.STREAM_X)
    assert np.array_equal(inputs.cb_bf16_np(3, inputs.STREAM_X, idx),
                          tb.view(torch.int16).numpy().view(np.uint16))
    assert abs(a.mean()) < 0.05 and abs(a.std() - 1.0) < 0.05


@pytest.mark.parametrize("target", [1.0, 2.0, 4.0])
def test_routing_hits_maxvio(target):
    r = inputs.routing(8, 8, 512, 8, 0, maxvio=target)
    assert abs(r.maxvio - target) <= 0.05 * target
    ids = r.topk_idx.reshape(-1, 8)
    assert all(len(set(row)) == 8 for row in ids[:500].tolist())
    assert np.allclose(r.topk_w.reshape(-1, 8).sum(1), 1.0, atol=1e-6)
    assert np.all(np.diff(r.topk_w.reshape(-1, 8), axis=1) <= 0)


# ---------------------------------------------------------------------------
# Remote-weights mode: overflow beyond a receiver's slots is still placed on
# it and reads its weights from the home rank, so no row falls back
# ---------------------------------------------------------------------------

def _compare_unitwise_remote(oracle, cfg, ids):
    pl = oracle.plan(cfg, ids, mode=oracle.MODE_REMOTE)
    un = oracle.plan_unitwise(cfg, ids, mode=oracle.MODE_REMOTE)
    assert pl["status"] == un["status"] == 0
    for k in ("dest", "alloc", "slot_expert", "slot_cnt", "fb_cnt"):
        assert np.array_equal(pl[k], un[k]), k
    info = pc.check_plan(cfg, ids, pl)
    assert pl["fallback_rows"] == 0
    assert np.all(info["rows"] == cfg["C"])            # the hard invariant, for any B
    n = pl["n_replicas"]
    # the first B pieces of a receiver have slots, the rest are remote
    for r in range(cfg["R"]):
        q = np.nonzero(pl["rep_recv"][:n] == r)[0]
        slots = pl["rep_slot"][q]
        assert np.array_equal(slots, np.where(np.arange(len(q)) < cfg["B"], np.arange(len(q)), -1))
        assert np.array_equal(q, np.arange(pl["recv_ptr"][r], pl["recv_ptr"][r + 1]))
    return pl


@pytest.mark.parametrize("R,L,S,K,B", [(2, 2, 2, 2, 1), (3, 1, 2, 1, 0), (4, 1, 2, 1, 1), (2, 2, 3, 1, 0)])
def test_bruteforce_remote_mode(oracle_lib, R, L, S, K, B):
    N, T = R * L, R * S
    cfg = _cfg(R, L, S, K, 8, B)
    choices = list(itertools.permutations(range(N), K))
    n = 0
    for combo in itertools.product(range(len(choices)), repeat=T):
        ids = np.array([choices[c] for c in combo], np.int32).reshape(R, S, K)
        _compare_unitwise_remote(oracle_lib, cfg, ids)
        n += 1
    assert n == len(choices) ** T


def test_remote_mode_closes_the_known_gap(oracle_lib):
    R, L, S, K, B = 4, 2, 2, 2, 2
    cfg = _cfg(R, L, S, K, 8, B)                       # no headroom needed
    ids = pc.ids_from_counts(np.array([2, 3, 2, 3, 2, 3, 1, 0]), R, S, K)
    pl = _compare_unitwise_remote(oracle_lib, cfg, ids)
    assert pl["slots_used"].tolist() == [0, 0, 0, 2]
    assert (pl["rep_slot"] < 0).sum() == 1              # the third piece on rank 3 is remote


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("B", [0, 1, 2])
def test_remote_mode_random_histograms(oracle_lib, seed, B):
    rng = np.random.default_rng(seed)
    R, L, S, K = 8, 4, 64, 4
    cnt = pc.random_counts(rng, R * L, R * S, K, skew=1.0 + seed)
    ids = pc.ids_from_counts(cnt, R, S, K)
    cfg = _cfg(R, L, S, K, 8, B)
    pl = _compare_unitwise_remote(oracle_lib, cfg, ids)
    # with slots for every piece the two modes agree
    if B >= R * L:
        assert np.array_equal(pl["dest"], oracle_lib.plan(cfg, ids)["dest"])


def test_remote_mode_equals_headroom_mode_when_slots_suffice(oracle_lib):
    for seed in range(5):
        w = inputs.WORKLOADS["tiny"]
        r = inputs.routing(w.R, w.L, w.S, w.K, seed, alpha=1.0)
        a = oracle_lib.plan(w.cfg(), r.topk_idx)
        b = oracle_lib.plan(w.cfg(), r.topk_idx, mode=oracle_lib.MODE_REMOTE)
        if a["fallback_rows"] == 0:
            assert np.array_equal(a["dest"], b["dest"]) and np.array_equal(a["alloc"], b["alloc"])


def test_remote_mode_inference_workload(oracle_lib):
    # the inference workload (B = 4): seed 1 falls back 887 rows under the
    # headroom rule; with remote weights every rank holds exactly S*K rows
    w = inputs.WORKLOADS["inference"]
    r = inputs.routing(w.R, w.L, w.S, w.K, 1, maxvio=4.0)
    cfg = dict(w.cfg(), C_max=w.C)
    pl = oracle_lib.plan(cfg, r.topk_idx, mode=oracle_lib.MODE_REMOTE)
    info = pc.check_plan(cfg, r.topk_idx, pl)
    assert pl["fallback_rows"] == 0 and np.all(info["rows"] == w.C)
    assert (pl["rep_slot"] < 0).sum() > 0


def test_remote_pieces_carry_no_replica_gradient(oracle_lib):
    # remote pieces have no slot, so reduce_grad adds slotted pieces only and
    # leaves every other slot as it was
    R, L, S, K, B = 4, 2, 2, 2, 2
    cfg = _cfg(R, L, S, K, 8, B)
    ids = pc.ids_from_counts(np.array([2, 3, 2, 3, 2, 3, 1, 0]), R, S, K)
    pl = oracle_lib.plan(cfg, ids, mode=oracle_lib.MODE_REMOTE)
    E = 16
    gh = inputs.cb_f32_np(1, inputs.STREAM_G_HOME, np.arange(R * L * E)).reshape(R * L, E)
    gr = inputs.cb_f32_np(1, inputs.STREAM_G_REP, np.arange(R * B * E)).reshape(R * B, E)
    h0, r0 = gh.copy(), gr.copy()
    oracle_lib.reduce_grad(cfg, pl, gh, gr, E)
    slotted = pl["rep_slot"] >= 0
    slots = pl["rep_recv"][slotted] * B + pl["rep_slot"][slotted]
    for e in range(R * L):
        q = [pl["rep_recv"][i] * B + pl["rep_slot"][i] for i in range(pl["rep_ptr"][e], pl["rep_ptr"][e + 1])
             if pl["rep_slot"][i] >= 0]
        want = h0[e].astype(np.float64) + r0[q].astype(np.float64).sum(0)
        assert np.allclose(gh[e], want, rtol=0, atol=4 * 2.0 ** -24 * (np.abs(h0[e]) + np.abs(r0[q]).sum(0)))
    used = np.zeros(R * B, bool)
    used[slots] = True
    assert np.all(gr[used] == 0) and np.array_equal(gr[~used], r0[~used])


# ---------------------------------------------------------------------------
# copy-out (zero_copy = false): the rows in use, and only those
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode_name,seed", [("MODE_HEADROOM", 0), ("MODE_HEADROOM", 3), ("MODE_REMOTE", 1),
                                            ("MODE_ONE_GROUP", 2)])
def test_copy_out_copies_exactly_the_rows_in_use(oracle_lib, mode_name, seed):
    # against the row -> expert map built from the plan's segment and piece
    # tables with numpy: rows with an expert are copied, the rest untouched
    R, L, S, K, H, B = 6, 3, 40, 4, 24, 2
    cfg = _cfg(R, L, S, K, H, B, C_max=2 * S * K)
    rng = np.random.default_rng(seed)
    cnt = pc.random_counts(rng, R * L, R * S, K, skew=1.5)
    ids = pc.ids_from_counts(cnt, R, S, K)
    pl = oracle_lib.plan(cfg, ids, mode=getattr(oracle_lib, mode_name))
    assert pl["status"] & 0xFF == 0
    rows = R * cfg["C_max"]
    recv = inputs.cb_bf16_np(seed, inputs.STREAM_X, np.arange(rows * H)).reshape(rows, H)
    out = np.full((rows, H), 0xBEEF, np.uint16)
    n = oracle_lib.copy_out(cfg, pl, recv, out)
    used = pc.row_expert_map(cfg, pl) >= 0
    assert n == used.sum() == R * S * K
    assert np.array_equal(out[used], recv[used])
    assert np.all(out[~used] == 0xBEEF)


def test_plan_invariants_detect_planted_mistakes(oracle_lib):
    # the invariant checker used on every plan must reject plausible mistakes:
    # two copies of different experts swapped, a copy sent to a row outside
    # its expert's segments, a capacity overrun, receivers out of order
    R, L, S, K, B = 4, 2, 16, 2, 4
    cfg = _cfg(R, L, S, K, 8, B, C_max=2 * S * K)
    cnt = np.array([40, 14, 26, 12, 12, 8, 8, 8])
    ids = pc.ids_from_counts(cnt, R, S, K)
    pl = oracle_lib.plan(cfg, ids)
    pc.check_plan(cfg, ids, pl)
    assert pl["n_replicas"] >= 2

    def rejects(mutate):
        bad = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in pl.items()}
        mutate(bad)
        with pytest.raises(AssertionError):
            pc.check_plan(cfg, ids, bad)

    flat = ids.reshape(-1)
    a = int(np.nonzero(flat == 0)[0][0])
    b = int(np.nonzero(flat == 3)[0][0])

    def swap(p):
        d = p["dest"].reshape(-1)
        d[a], d[b] = d[b], d[a]
    rejects(swap)

    def stray(p):
        d = p["dest"].reshape(-1)
        d[a] = (d[a] + cfg["C"]) % (R * cfg["C_max"])
    rejects(stray)

    def overrun(p):
        al = p["alloc"].reshape(R * L, R)
        al[0, 0] += 1
        al[0, 1] -= 1
    rejects(overrun)

    rp = pl["rep_ptr"]
    split = [e for e in range(R * L) if rp[e + 1] - rp[e] >= 2]
    assert split                      # an expert spread over two receivers

    def reorder(p):
        e = split[0]
        lo, hi = p["rep_ptr"][e], p["rep_ptr"][e + 1]
        p["rep_recv"][lo:hi] = p["rep_recv"][lo:hi][::-1].copy()
    rejects(reorder)


@pytest.mark.parametrize("seed", [0, 3])
def test_sampled_weighted_combine_matches_the_whole_problem(oracle_lib, seed):
    # the full-size GPU tests check combine on sampled tokens through a mini
    # problem built from just those tokens' rows; on the tiny workload, which
    # the oracle runs whole (plan, dispatch, stand-in expert, combine), the
    # mini problem gives the same bf16 outputs and fp32 sums for the sample
    from tests import sampled
    oracle = oracle_lib
    wl = inputs.WORKLOADS["tiny"]
    cfg = wl.cfg()
    r = inputs.routing(wl.R, wl.L, wl.S, wl.K, seed, alpha=1.0)
    opl = oracle.plan(cfg, r.topk_idx)
    assert opl["n_replicas"] > 0                        # replica rows are in the sample's reach
    x = inputs.cb_bf16_np(seed, inputs.STREAM_X, np.arange(wl.T * wl.H)).reshape(wl.T, wl.H)
    recv = np.zeros((wl.R * cfg["C_max"], wl.H), np.uint16)
    oracle.dispatch(cfg, opl["dest"], x, recv)
    y = recv.copy()
    oracle.expert_scale(cfg, opl, recv, inputs.expert_scales(wl.N, seed), y)
    out, acc = oracle.combine(cfg, opl["dest"], y, r.topk_w)
    ts = np.sort(np.random.default_rng(seed).choice(wl.T, 48, replace=False))
    out_s, acc_s = sampled.sampled_weighted_combine(oracle, r, seed, ts, wl.N, wl.K, wl.H)
    assert np.array_equal(out_s, out[ts])
    assert np.array_equal(acc_s.view(np.uint32), acc[ts].view(np.uint32))
