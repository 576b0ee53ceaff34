"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle
on the same seeded inputs.  Plan tables, destinations, dispatched rows,
prefetched weights and reduced gradients must be bit-exact; combine must be
bit-exact against the oracle's bf16 output (same fma order) and within 4e-3
relative of its fp32 sum.  Small cases are compared in full; the full-size
workloads in the launch configuration the benchmark times are compared in
full for every table and destination and on sampled rows and elements."""
import numpy as np
import pytest

import oracle
from load_balancing_plan_b200 import inputs
from tests import planchecks as pc
from tests import sampled

pytestmark = pytest.mark.gpu

PLAN_TABLES = ["cnt", "keep", "spill", "home_off", "fb_cnt", "fb_off", "load", "deficit", "fill",
               "slots_used", "slot_expert", "slot_cnt", "slot_off", "slot_first_j", "rep_ptr",
               "rep_expert", "rep_recv", "rep_slot", "rep_first_j", "rep_cnt", "rep_off", "recv_ptr",
               "seg_off", "seg_len", "alloc"]
COUNTS = ["fallback_rows", "n_replicas", "migrated_rows"]


@pytest.fixture(scope="module")
def env():
    import torch
    from load_balancing_plan_b200 import build
    build.build()
    oracle.build()
    from load_balancing_plan_b200 import harness
    from load_balancing_plan_b200 import moonep as mp
    assert torch.cuda.is_available()
    yield torch, mp, harness
    torch.cuda.empty_cache()


def cfg_of(R, L, S, K, H, B, headroom=0.0):
    C = S * K
    return dict(R=R, L=L, S=S, K=K, H=H, B=B, C=C, C_max=int(np.floor((1 + headroom) * C)))


def compare_plan(gpl, opl):
    assert gpl["status"] == opl["status"], (hex(gpl["status"]), hex(opl["status"]))
    if opl["status"] & (oracle.ST_CAPACITY | oracle.ST_EXPERT_ID):
        return
    for k in COUNTS:
        assert gpl[k] == opl[k], k
    for k in PLAN_TABLES:
        a, b = np.asarray(gpl[k]), np.asarray(opl[k])
        assert a.shape == b.shape, (k, a.shape, b.shape)
        assert np.array_equal(a, b), k


def x_host(seed, T, H):
    return inputs.cb_bf16_np(seed, inputs.STREAM_X, np.arange(T * H, dtype=np.int64)).reshape(T, H)


def run_full_compare(env, cfg, ids, w, seed=0, w_elems=64, g_elems=64, scale_seed=0, remote=False,
                     one_group=False):
    """Every step on a small problem, compared element by element."""
    torch, mp, harness = env
    R, L, S, K, H, B, Cm = (cfg[n] for n in ("R", "L", "S", "K", "H", "B", "C_max"))
    N, T = R * L, R * S
    prob = harness.Problem(cfg, poison=True, w_elems=w_elems, g_elems=g_elems)
    prob.set_routing(ids, w)
    prob.fill_x(seed)
    prob.fill_weights(seed)
    prob.fill_g_rep(seed)
    prob.plan(flags=mp.PLAN_REMOTE_WEIGHTS if remote else mp.PLAN_ONE_GROUP if one_group else 0)
    gpl = prob.read_plan()
    mode = oracle.MODE_REMOTE if remote else oracle.MODE_ONE_GROUP if one_group else oracle.MODE_HEADROOM
    opl = oracle.plan(cfg, ids, mode=mode)
    compare_plan(gpl, opl)
    failed = bool(opl["status"] & (oracle.ST_CAPACITY | oracle.ST_EXPERT_ID))
    if not failed:
        pc.check_plan(cfg, ids, gpl | {"dest": opl["dest"]})

    prob.dispatch()
    torch.cuda.synchronize()
    recv_g = harness.to_u16(prob.recv)
    dest_g = prob.dest[:T * K].cpu().numpy()
    if failed:
        # a failed plan: dispatch and copy-out write nothing
        assert np.all(recv_g == 0xFFFF)
        assert np.all(dest_g == -7)
        out_c = torch.full_like(prob.recv, 0x1357)
        mp.moonep_copy_out(cfg, prob.ws, prob.recv, out_c)
        torch.cuda.synchronize()
        assert np.all(harness.to_u16(out_c) == 0x1357)
        return prob, gpl, opl
    assert np.array_equal(dest_g, opl["dest"].reshape(-1))
    xh = x_host(seed, T, H)
    assert np.array_equal(harness.to_u16(prob.x[:T]), xh)
    recv_o = np.full((R * Cm, H), 0xFFFF, np.uint16)
    oracle.dispatch(cfg, opl["dest"], xh, recv_o)
    assert np.array_equal(recv_g, recv_o)

    # zero_copy = false: the rows in use copied out, the rest untouched
    out_c = torch.full_like(prob.recv, 0x1357)
    mp.moonep_copy_out(cfg, prob.ws, prob.recv, out_c)
    torch.cuda.synchronize()
    out_co = np.full((R * Cm, H), 0x1357, np.uint16)
    assert oracle.copy_out(cfg, opl, recv_o, out_co) == T * K
    assert np.array_equal(harness.to_u16(out_c), out_co)

    # stand-in expert, then combine, against the oracle's chain
    scale = inputs.expert_scales(N, scale_seed)
    y_g = prob.expert_scale(scale)
    y_o = recv_o.copy()
    oracle.expert_scale(cfg, opl, recv_o, scale, y_o)
    assert np.array_equal(harness.to_u16(y_g), y_o)
    prob.combine(y_g)
    torch.cuda.synchronize()
    out_g = harness.to_u16(prob.out[:T])
    out_o, acc_o = oracle.combine(cfg, opl["dest"], y_o, w)
    assert np.array_equal(out_g, out_o)
    og = inputs.bf16_bits_to_f32_np(out_g).astype(np.float64)
    nz = acc_o != 0
    assert np.all(og[~nz] == 0)
    if nz.any():
        assert np.max(np.abs(og[nz] - acc_o[nz]) / np.abs(acc_o[nz])) <= 4e-3

    # prefetch and reduce_grad
    if w_elems:
        w_home = harness.to_u16(prob.w_home)
        ws_o = np.full((max(R * B, 1), w_elems), 0xFFFF, np.uint16)
        oracle.prefetch(cfg, opl["slot_expert"], w_home, ws_o, w_elems)
        prob.prefetch()
        torch.cuda.synchronize()
        assert np.array_equal(harness.to_u16(prob.w_slot), ws_o)
    if g_elems:
        gh = prob.g_home.cpu().numpy().copy()
        gr = prob.g_rep.cpu().numpy().copy()
        prob.reduce_grad()
        torch.cuda.synchronize()
        oracle.reduce_grad(cfg, opl, gh, gr, g_elems)
        gh_g, gr_g = prob.g_home.cpu().numpy(), prob.g_rep.cpu().numpy()
        assert np.array_equal(gh_g.view(np.uint32), gh.view(np.uint32))
        assert np.array_equal(gr_g.view(np.uint32), gr.view(np.uint32))
    return prob, gpl, opl


# ---------------------------------------------------------------------------
# small problems, compared in full
# ---------------------------------------------------------------------------

def test_device_generator_matches_host(env):
    torch, mp, harness = env
    t = torch.empty(1 << 20, dtype=torch.bfloat16, device="cuda")
    inputs.cb_fill_torch(t, 5, inputs.STREAM_X, offset=12345)
    h = inputs.cb_bf16_np(5, inputs.STREAM_X, np.arange(12345, 12345 + (1 << 20)))
    assert np.array_equal(t.view(torch.int16).cpu().numpy().view(np.uint16), h)
    f = torch.empty(1 << 20, dtype=torch.float32, device="cuda")
    inputs.cb_fill_torch(f, 6, inputs.STREAM_G_REP)
    assert np.array_equal(f.cpu().numpy(), inputs.cb_f32_np(6, inputs.STREAM_G_REP, np.arange(1 << 20)))


@pytest.mark.parametrize("seed", range(5))
def test_tiny_workload(env, seed):
    w = inputs.WORKLOADS["tiny"]
    r = inputs.routing(w.R, w.L, w.S, w.K, seed, alpha=1.0)
    run_full_compare(env, w.cfg(), r.topk_idx, r.topk_w, seed=seed, w_elems=2 * 128 * 256 // 64,
                     g_elems=128 * 256 // 32)


def test_tiny_reduce_grad_full_size_grads(env):
    # tiny workload with the stated gradient size H*I = 128*256 per replica
    w = inputs.WORKLOADS["tiny"]
    r = inputs.routing(w.R, w.L, w.S, w.K, 1, alpha=1.0)
    run_full_compare(env, w.cfg(), r.topk_idx, r.topk_w, seed=1, w_elems=2 * 128 * 256,
                     g_elems=128 * 256)


@pytest.mark.parametrize("case", [
    # R, L, S, K, H, B, headroom, routing
    (4, 4, 64, 2, 128, 4, 0.0, "balanced"),
    (1, 7, 500, 1, 8, 2, 0.0, "uniform"),              # single rank: stable sort
    (3, 5, 333, 3, 296, 2, 1.0, "skew"),                # ragged sizes, headroom
    (4, 4, 100, 2, 64, 0, 3.0, "skew"),                 # no slots: all overflow falls back
    (16, 24, 64, 8, 64, 4, 0.25, "skew4"),              # inference-style slot limit
    (8, 8, 40, 64, 16, 8, 0.0, "skew"),                 # K at its maximum
    (2, 2, 300, 2, 20008, 2, 1.0, "skew"),              # rows split in several pieces
    (64, 64, 32, 8, 32, 8, 0.0, "skew"),                # N at its maximum
    (5, 3, 1000, 4, 40, 3, 1.0, "skew"),                # T > ranges: several tokens per range
    (2, 2, 4, 2, 1 << 20, 2, 1.0, "skew"),              # H at its maximum (2 MB rows)
    (2, 4, 64, 2, 16, 1024, 1.0, "skew"),               # B at its maximum
    (64, 2, 8, 2, 16, 1024, 1.0, "skew"),               # R * B at its maximum (65536 slots)
    (1, 3, 1, 2, 16, 1, 0.0, "uniform"),                # one token (T = 1): range and token of each id
    (2, 3, 1, 1, 16, 1, 1.0, "uniform"),                # one token per rank, K = 1
])
def test_edge_cases(env, case):
    R, L, S, K, H, B, hr, kind = case
    cfg = cfg_of(R, L, S, K, H, B, hr)
    rng = np.random.default_rng(R * 1000 + S)
    if kind == "balanced":
        r = inputs.routing(R, L, S, K, 0, balanced=True)
        ids, w = r.topk_idx, r.topk_w
    elif kind == "uniform":
        ids = rng.integers(0, R * L, (R, S, K)).astype(np.int32)
        w = rng.random((R, S, K)).astype(np.float32)
    else:
        target = 4.0 if kind == "skew4" else None
        r = inputs.routing(R, L, S, K, 0, alpha=1.0 if target is None else None, maxvio=target)
        ids, w = r.topk_idx, r.topk_w
    run_full_compare(env, cfg, ids, w, w_elems=64, g_elems=64)


@pytest.mark.parametrize("seed", range(4))
def test_random_histograms(env, seed):
    rng = np.random.default_rng(seed)
    R, L, S, K, B = 8, 4, 64, 4, 1 + seed
    cnt = pc.random_counts(rng, R * L, R * S, K, skew=1.0 + seed)
    ids = pc.ids_from_counts(cnt, R, S, K)
    # shuffle tokens so the copies of an expert spread over the token ranges
    flat = ids.reshape(R * S, K)[rng.permutation(R * S)]
    ids = np.ascontiguousarray(flat.reshape(R, S, K))
    w = rng.random((R, S, K)).astype(np.float32)
    run_full_compare(env, cfg_of(R, L, S, K, 64, B, 3.0), ids, w)


def test_empty_input(env):
    torch, mp, harness = env
    cfg = cfg_of(4, 2, 0, 2, 64, 2)
    ids = np.zeros((4, 0, 2), np.int32)
    prob = harness.Problem(cfg, w_elems=64, g_elems=64)
    prob.plan()
    prob.dispatch()
    prob.combine()
    prob.prefetch()
    prob.reduce_grad()
    gpl = prob.read_plan()
    compare_plan(gpl, oracle.plan(cfg, ids))


def test_capacity_error_writes_nothing(env):
    R, L, S, K, B = 4, 2, 2, 2, 0
    cfg = cfg_of(R, L, S, K, 16, B)
    ids = pc.ids_from_counts(np.array([4, 4, 2, 2, 2, 2, 0, 0]), R, S, K)
    w = np.full((R, S, K), 0.5, np.float32)
    prob, gpl, opl = run_full_compare(env, cfg, ids, w)
    assert gpl["status"] & oracle.ST_CAPACITY


def test_bad_expert_id_writes_nothing(env):
    torch, mp, harness = env
    cfg = cfg_of(2, 2, 4, 2, 16, 2)
    ids = np.array([0, 1, 2, 3, 0, 4, 1, 2, 3, 0, 1, 2, 0, 1, 2, 3], np.int32).reshape(2, 4, 2)
    w = np.full((2, 4, 2), 0.5, np.float32)
    prob, gpl, opl = run_full_compare(env, cfg, ids, w)
    assert gpl["status"] & mp.ST_EXPERT_ID
    g_home0, g_rep0 = prob.g_home.clone(), prob.g_rep.clone()
    prob.combine()
    prob.prefetch()
    prob.reduce_grad()
    torch.cuda.synchronize()
    assert np.all(harness.to_u16(prob.out) == 0xFFFF)
    assert np.all(harness.to_u16(prob.w_slot) == 0xFFFF)
    assert torch.equal(prob.g_rep, g_rep0) and torch.equal(prob.g_home, g_home0)


def test_workspace_of_other_cfg_is_refused(env):
    torch, mp, harness = env
    cfg = cfg_of(4, 4, 64, 2, 128, 4)
    r = inputs.routing(4, 4, 64, 2, 0, alpha=1.0)
    prob = harness.Problem(cfg, poison=True)
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.plan()
    other = dict(cfg, B=3)      # same workspace size class, different cfg
    assert mp.moonep_plan_workspace_bytes(other) <= prob.ws.numel() * 4
    mp.moonep_dispatch(other, prob.ws, prob.x, prob.ids, prob.recv, prob.dest)
    info = mp.moonep_plan_read(cfg, prob.ws)
    assert info["status"] & mp.ST_CFG
    assert np.all(harness.to_u16(prob.recv) == 0xFFFF)


def test_replan_on_same_workspace(env):
    torch, mp, harness = env
    cfg = cfg_of(4, 4, 64, 2, 128, 4)
    prob = harness.Problem(cfg)
    for seed in range(3):
        r = inputs.routing(4, 4, 64, 2, seed, alpha=1.0 + seed)
        prob.set_routing(r.topk_idx, r.topk_w)
        prob.plan()
        compare_plan(prob.read_plan(), oracle.plan(cfg, r.topk_idx))


def test_plan_wait_timeout_sets_status(env):
    # a wait limit of zero makes the plan's grid barrier give up; the status
    # says so, later calls write nothing, and the next plan is clean again
    torch, mp, harness = env
    cfg = cfg_of(4, 4, 64, 2, 128, 4)
    r = inputs.routing(4, 4, 64, 2, 0, alpha=1.0)
    prob = harness.Problem(cfg, poison=True)
    prob.set_routing(r.topk_idx, r.topk_w)
    try:
        mp.moonep_set_wait_limit(0)
        prob.plan()
        info = prob.read_plan(tables=False)
    finally:
        mp.moonep_set_wait_limit(1 << 22)
    assert info["status"] & mp.ST_TIMEOUT
    prob.dispatch()
    torch.cuda.synchronize()
    assert np.all(harness.to_u16(prob.recv) == 0xFFFF)
    prob.plan()
    compare_plan(prob.read_plan(), oracle.plan(cfg, r.topk_idx))


def test_dispatch_wait_timeout_is_reported_or_complete(env):
    torch, mp, harness = env
    cfg = cfg_of(8, 4, 512, 4, 4096, 4, headroom=1.0)
    r = inputs.routing(8, 4, 512, 4, 0, alpha=1.0)
    assert oracle.plan(cfg, r.topk_idx)["status"] & 0xFF == 0
    prob = harness.Problem(cfg)
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.fill_x(0)
    prob.plan()
    try:
        mp.moonep_set_wait_limit(0)
        prob.dispatch()
        info = prob.read_plan(tables=False)
    finally:
        mp.moonep_set_wait_limit(1 << 22)
    opl = oracle.plan(cfg, r.topk_idx)
    if not info["status"] & mp.ST_TIMEOUT:
        assert np.array_equal(prob.dest.cpu().numpy(), opl["dest"].reshape(-1))
    # the context stays usable
    prob.plan()
    prob.dispatch()
    torch.cuda.synchronize()
    assert prob.read_plan(tables=False)["status"] & mp.ST_ERROR_MASK == 0
    assert np.array_equal(prob.dest.cpu().numpy(), opl["dest"].reshape(-1))


@pytest.mark.parametrize("kernel", ["prefetch", "combine", "combine_backward", "copy_out"])
def test_pipeline_wait_timeout_is_reported_and_recoverable(env, kernel):
    # every TMA pipeline gives up after wait_limit polls (0 here): it either
    # finishes anyway or records MOONEP_ST_TIMEOUT and returns; the context
    # stays usable and the next plan clears the status
    torch, mp, harness = env
    cfg = cfg_of(8, 4, 512, 4, 4096, 4, headroom=1.0)
    r = inputs.routing(8, 4, 512, 4, 0, alpha=1.0)
    E = 64 * 1024
    prob = harness.Problem(cfg, w_elems=E)
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.fill_x(0)
    prob.fill_weights(0)

    def run():
        if kernel == "prefetch":
            prob.prefetch()
            return prob.w_slot
        if kernel == "combine":
            prob.combine()
            return prob.out
        if kernel == "combine_backward":
            gy = torch.zeros_like(prob.recv)
            gw = torch.zeros(prob.T * cfg["K"], dtype=torch.float32, device="cuda")
            mp.moonep_combine_backward(cfg, prob.ws, prob.x, prob.recv, prob.dest, prob.w, gy, gw)
            return gy
        out = torch.full_like(prob.recv, 0x1357)
        mp.moonep_copy_out(cfg, prob.ws, prob.recv, out)
        return out

    prob.plan()
    prob.dispatch()
    torch.cuda.synchronize()
    try:
        mp.moonep_set_wait_limit(0)
        got = run().clone()
        torch.cuda.synchronize()
        status = prob.read_plan(tables=False)["status"]
    finally:
        mp.moonep_set_wait_limit(1 << 22)
    assert status & mp.ST_ERROR_MASK & ~mp.ST_TIMEOUT == 0
    prob.plan()
    prob.dispatch()
    ref = run().clone()
    torch.cuda.synchronize()
    assert prob.read_plan(tables=False)["status"] & mp.ST_ERROR_MASK == 0
    if not status & mp.ST_TIMEOUT:
        assert torch.equal(got, ref)


# ---------------------------------------------------------------------------
# full-size workloads (the benchmark's launch configuration), sampled
# ---------------------------------------------------------------------------

def check_weighted_combine(torch, harness, prob, route, seed, n_tok=384, rng_seed=5):
    """Combine after the stand-in expert, on sampled tokens of a full-size
    problem whose prob.out holds the GPU combine of prob.recv after
    expert_scale_inplace: bit-exact against the oracle's bf16 output on those
    tokens (sampled.sampled_weighted_combine) and within 4e-3 of its fp32
    sum."""
    c = prob.cfg
    K, H, N, T = c["K"], c["H"], prob.N, prob.T
    rng = np.random.default_rng(rng_seed)
    ts = np.sort(rng.choice(T, n_tok, replace=False))
    out_o, acc_o = sampled.sampled_weighted_combine(oracle, route, seed, ts, N, K, H)
    out_g = harness.to_u16(prob.out[torch.from_numpy(ts).cuda()])
    assert np.array_equal(out_g, out_o)
    got = inputs.bf16_bits_to_f32_np(out_g)
    nz = acc_o != 0
    assert np.all(got[~nz] == 0)
    assert np.max(np.abs(got[nz] - acc_o[nz]) / np.abs(acc_o[nz])) <= 4e-3


# (workload, target maxvio, seed); inference seed 1 needs the headroom
FULL = [("mid", 2.0, 0), ("skew", 0.0, 0), ("skew", 8.0, 0), ("inference", 4.0, 0),
        ("inference", 4.0, 1), ("training", 8.0, 0)]


@pytest.mark.parametrize("name,maxvio,seed", FULL)
def test_full_size(env, name, maxvio, seed):
    torch, mp, harness = env
    wl = inputs.WORKLOADS[name]
    cfg = wl.cfg()
    R, L, S, K, H, B, Cm = (cfg[n] for n in ("R", "L", "S", "K", "H", "B", "C_max"))
    N, T = wl.N, wl.T
    r = inputs.routing(R, L, S, K, seed, maxvio=maxvio)
    assert maxvio == 0.0 or abs(r.maxvio - maxvio) <= 0.05 * maxvio
    w_elems = wl.w_elems if name in ("mid", "training") else 0
    g_elems = wl.g_elems if name in ("mid", "training") else 0
    prob = harness.Problem(cfg, poison=True, w_elems=w_elems, g_elems=g_elems)
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.fill_x(seed)
    prob.fill_weights(seed)
    prob.fill_g_rep(seed)
    prob.plan()
    if w_elems:
        prob.prefetch()
    prob.dispatch()
    prob.combine()
    torch.cuda.synchronize()
    gpl = prob.read_plan()
    opl = oracle.plan(cfg, r.topk_idx)
    compare_plan(gpl, opl)
    if name != "inference":
        assert gpl["fallback_rows"] == 0
    assert bool(gpl["status"] & mp.ST_FALLBACK) == (gpl["fallback_rows"] > 0)
    if gpl["fallback_rows"] == 0:
        assert np.all(gpl["alloc"].sum(0) == cfg["C"])        # exactly S*K rows per rank
    else:
        assert np.all(gpl["alloc"].sum(0) <= Cm)
    if name == "inference" and seed == 1:
        assert gpl["fallback_rows"] > 0                         # the headroom path is exercised
    dest = prob.dest[:T * K].cpu().numpy()
    assert np.array_equal(dest, opl["dest"].reshape(-1))

    rng = np.random.default_rng(1)
    # dispatched rows: sampled copies, against the generator by index
    gs = rng.choice(T * K, 2048, replace=False)
    rows = harness.to_u16(prob.recv[torch.from_numpy(dest[gs]).long().cuda()])
    tok = gs // K
    want = inputs.cb_bf16_np(seed, inputs.STREAM_X, (tok[:, None] * H + np.arange(H)[None, :]))
    assert np.array_equal(rows, want)
    # rows outside every segment stay untouched
    used = np.zeros(R * Cm, bool)
    used[dest] = True
    free = np.nonzero(~used)[0]
    if free.size:
        pick = rng.choice(free, min(256, free.size), replace=False)
        assert np.all(harness.to_u16(prob.recv[torch.from_numpy(pick).cuda()]) == 0xFFFF)
    # combine with the identity expert: out[t] from K copies of x[t]
    ts = rng.choice(T, 256, replace=False)
    xs = inputs.cb_bf16_np(seed, inputs.STREAM_X, ts[:, None] * H + np.arange(H)[None, :])
    mini = dict(R=1, L=1, S=len(ts), K=K, H=H, B=0, C=len(ts) * K, C_max=len(ts) * K)
    y_mini = np.repeat(xs, K, axis=0)
    d_mini = np.arange(len(ts) * K, dtype=np.int32).reshape(1, len(ts), K)
    w_mini = r.topk_w.reshape(T, K)[ts]
    out_o, acc_o = oracle.combine(mini, d_mini, y_mini, w_mini)
    out_g = harness.to_u16(prob.out[torch.from_numpy(ts).cuda()])
    assert np.array_equal(out_g, out_o)
    # combine after the stand-in expert (scales != 1, replica rows scaled by
    # their expert's scale), sampled tokens against the oracle
    prob.expert_scale_inplace(inputs.expert_scales(N, seed), prob.row_expert(gpl))
    prob.combine()
    torch.cuda.synchronize()
    check_weighted_combine(torch, harness, prob, r, seed)
    # prefetch: every used slot, sampled elements
    if w_elems:
        idx = np.sort(rng.choice(w_elems, 4096, replace=False))
        it = torch.from_numpy(idx).cuda()
        for slot in np.nonzero(gpl["slot_expert"] >= 0)[0]:
            e = int(gpl["slot_expert"][slot])
            got = harness.to_u16(prob.w_slot[int(slot)][it])
            assert np.array_equal(got, inputs.cb_bf16_np(seed, inputs.STREAM_W, e * w_elems + idx))
        for slot in np.nonzero(gpl["slot_expert"] < 0)[0][:4]:
            assert np.all(harness.to_u16(prob.w_slot[int(slot)][it]) == 0xFFFF)
    # reduce_grad: sampled columns, against the oracle on those columns
    if g_elems:
        prob.reduce_grad()
        torch.cuda.synchronize()
        idx = np.sort(rng.choice(g_elems, 2048, replace=False))
        it = torch.from_numpy(idx).cuda()
        gh = inputs.cb_f32_np(seed, inputs.STREAM_G_HOME,
                              np.arange(N)[:, None] * g_elems + idx[None, :]).astype(np.float32)
        gr = inputs.cb_f32_np(seed, inputs.STREAM_G_REP,
                              np.arange(R * B)[:, None] * g_elems + idx[None, :]).astype(np.float32)
        gh = np.ascontiguousarray(gh)
        gr = np.ascontiguousarray(gr)
        oracle.reduce_grad(cfg, opl, gh, gr, len(idx))
        got_h = prob.g_home[:, it].cpu().numpy()
        got_r = prob.g_rep[:, it].cpu().numpy()
        assert np.array_equal(got_h.view(np.uint32), gh.view(np.uint32))
        assert np.array_equal(got_r.view(np.uint32), gr.view(np.uint32))
        rel = np.abs(got_h - gh) / np.maximum(np.abs(gh), 1e-30)
        assert rel.max() <= 1e-6
    del prob
    torch.cuda.empty_cache()


@pytest.mark.parametrize("maxvio", [0.0, 1.0, 2.0, 4.0, 8.0])
@pytest.mark.parametrize("seed", [1, 2, 3, 4])
def test_skew_sweep_plans(env, maxvio, seed):
    # plan tables and destinations of the skew-sweep workload for every seed
    torch, mp, harness = env
    wl = inputs.WORKLOADS["skew"]
    cfg = wl.cfg()
    r = inputs.routing(wl.R, wl.L, wl.S, wl.K, seed, maxvio=maxvio)
    prob = harness.Problem(dict(cfg, H=8))   # H does not enter the plan or dest
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.plan()
    prob.dispatch()
    torch.cuda.synchronize()
    cfg8 = dict(cfg, H=8)
    opl = oracle.plan(cfg8, r.topk_idx)
    compare_plan(prob.read_plan(), opl)
    assert np.array_equal(prob.dest.cpu().numpy(), opl["dest"].reshape(-1))
    assert opl["fallback_rows"] == 0


def test_reduce_grad_twice_after_one_plan(env):
    # the work counter reduce_grad hands units out with resets itself: a second
    # call after the same plan (new replica gradients) is exact again
    torch, mp, harness = env
    w = inputs.WORKLOADS["tiny"]
    cfg = w.cfg()
    r = inputs.routing(w.R, w.L, w.S, w.K, 2, alpha=1.0)
    E = 128 * 256
    prob = harness.Problem(cfg, g_elems=E)
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.fill_weights(2)
    prob.plan()
    opl = oracle.plan(cfg, r.topk_idx)
    for seed in (2, 3):
        prob.fill_g_rep(seed)
        gh = prob.g_home.cpu().numpy().copy()
        gr = prob.g_rep.cpu().numpy().copy()
        prob.reduce_grad()
        torch.cuda.synchronize()
        oracle.reduce_grad(cfg, opl, gh, gr, E)
        assert np.array_equal(prob.g_home.cpu().numpy().view(np.uint32), gh.view(np.uint32))
        assert np.array_equal(prob.g_rep.cpu().numpy().view(np.uint32), gr.view(np.uint32))


# ---------------------------------------------------------------------------
# remote-weights plan mode (the pages' inference fallback)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("case", [
    # R, L, S, K, H, B
    (4, 2, 2, 2, 16, 2),        # the known gap: a third piece on rank 3 is remote
    (16, 24, 64, 8, 64, 4),     # inference-style slot limit
    (8, 4, 64, 4, 64, 0),       # no slots at all: every piece remote
    (4, 4, 64, 2, 128, 4),
    (64, 64, 32, 8, 32, 1),     # N at its maximum, one slot
])
def test_remote_weights_mode(env, case):
    R, L, S, K, H, B = case
    cfg = cfg_of(R, L, S, K, H, B)                       # C_max = C: no headroom needed
    if (R, L) == (4, 2):
        ids = pc.ids_from_counts(np.array([2, 3, 2, 3, 2, 3, 1, 0]), R, S, K)
        w = np.full((R, S, K), 0.5, np.float32)
    else:
        r = inputs.routing(R, L, S, K, 1, maxvio=4.0 if R * L > 64 else None, alpha=None if R * L > 64 else 1.0)
        ids, w = r.topk_idx, r.topk_w
    prob, gpl, opl = run_full_compare(env, cfg, ids, w, remote=True)
    assert gpl["fallback_rows"] == 0
    assert np.all(gpl["alloc"].sum(0) == cfg["C"])
    if B == 0 and gpl["n_replicas"]:
        assert np.all(gpl["rep_slot"] == -1)


def test_remote_weights_inference_workload(env):
    # the inference workload at seed 1 falls back 887 rows under the headroom
    # rule; with remote weights and C_max = C every rank holds exactly S*K rows
    torch, mp, harness = env
    wl = inputs.WORKLOADS["inference"]
    cfg = dict(wl.cfg(), C_max=wl.C)
    r = inputs.routing(wl.R, wl.L, wl.S, wl.K, 1, maxvio=4.0)
    prob = harness.Problem(cfg, poison=True)
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.fill_x(1)
    prob.plan(flags=mp.PLAN_REMOTE_WEIGHTS)
    prob.dispatch()
    prob.combine()
    torch.cuda.synchronize()
    gpl = prob.read_plan()
    opl = oracle.plan(cfg, r.topk_idx, mode=oracle.MODE_REMOTE)
    compare_plan(gpl, opl)
    assert gpl["fallback_rows"] == 0 and (gpl["rep_slot"] < 0).sum() > 0
    dest = prob.dest.cpu().numpy()
    assert np.array_equal(dest, opl["dest"].reshape(-1))
    gs = np.random.default_rng(0).choice(wl.T * wl.K, 1024, replace=False)
    rows = harness.to_u16(prob.recv[torch.from_numpy(dest[gs]).long().cuda()])
    want = inputs.cb_bf16_np(1, inputs.STREAM_X, (gs // wl.K)[:, None] * wl.H + np.arange(wl.H)[None, :])
    assert np.array_equal(rows, want)
    # with C_max = C and no fallback every receive row is used
    assert not np.any(np.all(harness.to_u16(prob.recv[::97]) == 0xFFFF, axis=1))
    # combine of the dispatched rows themselves (identity expert), sampled
    # tokens against the oracle; then after the stand-in expert, whose rows of
    # pieces without a slot (remote weights) also take their expert's scale
    ts = np.sort(np.random.default_rng(3).choice(wl.T, 256, replace=False))
    xs = inputs.cb_bf16_np(1, inputs.STREAM_X, ts[:, None] * wl.H + np.arange(wl.H)[None, :])
    mini = dict(R=1, L=1, S=len(ts), K=wl.K, H=wl.H, B=0, C=len(ts) * wl.K, C_max=len(ts) * wl.K)
    d_mini = np.arange(len(ts) * wl.K, dtype=np.int32).reshape(1, len(ts), wl.K)
    out_o, _ = oracle.combine(mini, d_mini, np.repeat(xs, wl.K, axis=0), r.topk_w.reshape(wl.T, wl.K)[ts])
    assert np.array_equal(harness.to_u16(prob.out[torch.from_numpy(ts).cuda()]), out_o)
    prob.expert_scale_inplace(inputs.expert_scales(wl.N, 1), prob.row_expert(gpl))
    prob.combine()
    torch.cuda.synchronize()
    check_weighted_combine(torch, harness, prob, r, 1)


# ---------------------------------------------------------------------------
# several layers through one set of buffers
# ---------------------------------------------------------------------------

def test_layers_share_buffers(env):
    # a model runs its MoE layers one after another through the same per-rank
    # buffers (workspace, receive rows, replica weight slots, replica
    # gradients); the slots a layer fills differ from the last layer's, and
    # the plan mode may change between layers.  Every layer matches the
    # oracle run on the oracle's own carried-over buffers.
    torch, mp, harness = env
    cfg = cfg_of(8, 6, 96, 4, 64, 3, headroom=0.25)
    R, L, S, K, H, B, Cm = (cfg[n] for n in ("R", "L", "S", "K", "H", "B", "C_max"))
    N, T, E = R * L, R * S, 512
    prob = harness.Problem(cfg, poison=True, w_elems=E, g_elems=E)
    recv_o = np.full((R * Cm, H), 0xFFFF, np.uint16)
    wslot_o = np.full((R * B, E), 0xFFFF, np.uint16)
    layers = [(11, 1.5, False), (12, 6.0, True), (13, 3.0, False), (14, 0.0, False)]
    seen_slots = []
    for layer, (seed, maxvio, remote) in enumerate(layers):
        r = inputs.routing(R, L, S, K, seed, maxvio=maxvio)
        prob.set_routing(r.topk_idx, r.topk_w)
        prob.fill_x(seed)
        prob.fill_weights(seed)
        prob.fill_g_rep(seed)
        mode = oracle.MODE_REMOTE if remote else oracle.MODE_HEADROOM
        prob.plan(flags=mp.PLAN_REMOTE_WEIGHTS if remote else 0)
        opl = oracle.plan(cfg, r.topk_idx, mode=mode)
        assert opl["status"] & 0xFF == 0
        compare_plan(prob.read_plan(), opl)
        seen_slots.append(tuple(opl["slot_expert"].tolist()))
        # forward: prefetch, dispatch, stand-in expert, combine
        prob.prefetch()
        prob.dispatch()
        torch.cuda.synchronize()
        oracle.prefetch(cfg, opl["slot_expert"], harness.to_u16(prob.w_home), wslot_o, E)
        assert np.array_equal(harness.to_u16(prob.w_slot), wslot_o), layer
        oracle.dispatch(cfg, opl["dest"], x_host(seed, T, H), recv_o)
        assert np.array_equal(harness.to_u16(prob.recv), recv_o), layer
        scale = inputs.expert_scales(N, seed)
        y_g = prob.expert_scale(scale)
        y_o = recv_o.copy()
        oracle.expert_scale(cfg, opl, recv_o, scale, y_o)
        prob.combine(y_g)
        torch.cuda.synchronize()
        out_o, _ = oracle.combine(cfg, opl["dest"], y_o, r.topk_w)
        assert np.array_equal(harness.to_u16(prob.out[:T]), out_o), layer
        # backward: replica gradients back to their home experts
        gh = prob.g_home.cpu().numpy().copy()
        gr = prob.g_rep.cpu().numpy().copy()
        prob.reduce_grad()
        torch.cuda.synchronize()
        oracle.reduce_grad(cfg, opl, gh, gr, E)
        assert np.array_equal(prob.g_home.cpu().numpy().view(np.uint32), gh.view(np.uint32)), layer
        assert np.array_equal(prob.g_rep.cpu().numpy().view(np.uint32), gr.view(np.uint32)), layer
    # the layers really used different slot assignments
    assert len(set(seen_slots)) == len(layers)


# ---------------------------------------------------------------------------
# one-home-group plan mode (the pages' planner variant)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("case", [
    # R, L, S, K, H, B, headroom
    (3, 1, 2, 1, 16, 2, 1.0),       # two senders, one receiver: a row falls back
    (8, 4, 64, 4, 64, 4, 1.0),      # B = E/R
    (8, 8, 128, 8, 64, 2, 1.0),     # fewer slots than L: both limits bind
    (16, 24, 64, 8, 32, 24, 1.0),   # many groups, long spill stream
    (16, 48, 64, 8, 32, 48, 1.0),   # 768 experts: the whole CTA plans
])
def test_one_group_mode(env, case):
    R, L, S, K, H, B, hr = case
    cfg = cfg_of(R, L, S, K, H, B, headroom=hr)
    for seed in range(3):
        r = inputs.routing(R, L, S, K, seed, maxvio=min(4.0, R - 1.0))
        prob, gpl, opl = run_full_compare(env, cfg, r.topk_idx, r.topk_w, seed=seed, one_group=True)
        n = opl["n_replicas"]
        groups = [set((opl["rep_expert"][:n][opl["rep_recv"][:n] == q] // L).tolist()) for q in range(R)]
        assert all(len(g) <= 1 for g in groups)


def test_one_group_worked_example(env):
    # experts 0 and 1 three rows each, expert 2 none (R=3, L=1, C=2): the
    # receiver takes expert 0's spilled row; expert 1's stays on rank 1 at row C
    torch, mp, harness = env
    cfg = cfg_of(3, 1, 2, 1, 16, 2, headroom=1.0)
    ids = pc.ids_from_counts(np.array([3, 3, 0]), 3, 2, 1)
    w = np.ones((3, 2, 1), np.float32)
    prob, gpl, opl = run_full_compare(env, cfg, ids, w, one_group=True)
    assert prob.dest[:6].cpu().tolist() == [0, 1, 8, 4, 5, 6]
    assert gpl["fallback_rows"] == 1


def test_one_group_mid_workload(env):
    # the mid workload's routing under the one-group rule: the plan, every
    # destination and sampled rows against the oracle
    torch, mp, harness = env
    wl = inputs.WORKLOADS["mid"]
    cfg = dict(wl.cfg(), C_max=2 * wl.C)
    r = inputs.routing(wl.R, wl.L, wl.S, wl.K, 1, maxvio=wl.maxvio[0])
    prob = harness.Problem(cfg)
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.fill_x(1)
    prob.plan(flags=mp.PLAN_ONE_GROUP)
    prob.dispatch()
    torch.cuda.synchronize()
    opl = oracle.plan(cfg, r.topk_idx, mode=oracle.MODE_ONE_GROUP)
    compare_plan(prob.read_plan(), opl)
    assert opl["fallback_rows"] > 0
    dest = prob.dest[:wl.T * wl.K].cpu().numpy()
    assert np.array_equal(dest, opl["dest"].reshape(-1))
    rng = np.random.default_rng(3)
    g = np.sort(rng.choice(wl.T * wl.K, 256, replace=False))
    t = g // wl.K
    xs = inputs.cb_bf16_np(1, inputs.STREAM_X, t[:, None] * wl.H + np.arange(wl.H)[None, :])
    got = harness.to_u16(prob.recv[torch.from_numpy(dest[g]).long().cuda()])
    assert np.array_equal(got, xs)


def test_plan_flags_exclude_each_other(env):
    torch, mp, harness = env
    w = inputs.WORKLOADS["tiny"]
    prob = harness.Problem(w.cfg())
    with pytest.raises(mp.MoonepError) as ei:
        prob.plan(flags=mp.PLAN_REMOTE_WEIGHTS | mp.PLAN_ONE_GROUP)
    assert ei.value.code == mp.ERR_ARG


# ---------------------------------------------------------------------------
# zero_copy = false and the lifetime of zero-copy views
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name,mode", [("mid", 0), ("inference", 0), ("inference", 2)])
def test_copy_out_full_size(env, name, mode):
    # every row the plan uses is copied, no other row is written (a property
    # that holds at any size, checked on the device over all rows)
    torch, mp, harness = env
    wl = inputs.WORKLOADS[name]
    cfg = dict(wl.cfg(), C_max=2 * wl.C) if mode == 2 else wl.cfg()
    r = inputs.routing(wl.R, wl.L, wl.S, wl.K, 1, maxvio=wl.maxvio[0])
    prob = harness.Problem(cfg)
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.fill_x(1)
    prob.plan(flags=mp.PLAN_ONE_GROUP if mode == 2 else 0)
    prob.dispatch()
    out = torch.full_like(prob.recv, 0x1357)
    mp.moonep_copy_out(cfg, prob.ws, prob.recv, out)
    torch.cuda.synchronize()
    assert mp.moonep_plan_read(cfg, prob.ws)["status"] & mp.ST_ERROR_MASK == 0
    used = prob.row_expert() >= 0
    assert int(used.sum()) == wl.T * wl.K
    assert torch.equal(out[used], prob.recv[used])
    assert bool((out[~used] == 0x1357).all())
    del out


def test_views_go_stale_after_the_next_dispatch(env):
    torch, mp, harness = env
    from load_balancing_plan_b200 import views
    w = inputs.WORKLOADS["tiny"]
    cfg = w.cfg()
    r = inputs.routing(w.R, w.L, w.S, w.K, 0, alpha=1.0)
    prob = harness.Problem(cfg)
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.fill_x(0)
    prob.plan()
    prob.dispatch()
    used1 = (prob.row_expert() >= 0).view(w.R, w.C_max)[1]
    v = views.RecvView(cfg, prob.ws, prob.recv, rank=1)
    first = v.tensor.clone()
    kept = v.copy()                       # zero_copy = false
    assert v.valid()
    assert torch.equal(kept[used1], first[used1])
    # a second step writes other rows into the same buffer
    r2 = inputs.routing(w.R, w.L, w.S, w.K, 5, alpha=1.0)
    prob.set_routing(r2.topk_idx, r2.topk_w)
    prob.fill_x(5)
    prob.plan()
    prob.dispatch()
    torch.cuda.synchronize()
    assert not v.valid()
    with pytest.raises(views.StaleViewError):
        v.tensor
    with pytest.raises(views.StaleViewError):
        v.copy()
    # the buffer now holds the second step's rows; the copy taken before
    # still holds the first step's
    assert not torch.equal(prob.recv.view(w.R, w.C_max, w.H)[1][used1], first[used1])
    assert torch.equal(kept[used1], first[used1])
    # combine moves the generation too
    v2 = views.RecvView(cfg, prob.ws, prob.recv)
    prob.combine()
    assert not v2.valid()
