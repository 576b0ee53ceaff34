"""GPU parity of the expert-parallel calls (one rank per GPU), with the R
ranks emulated on one device: each rank has its own workspace and buffers,
peers are reached through peer-pointer tables, and the count all-gather is a
copy (load_balancing_plan_b200.ep.Emulation).  Every rank's plan tables must
equal the oracle's plan of the concatenated ids; each rank's destinations,
receive rows, combined outputs, prefetched slots, reduced gradients and the
backward pair's grad_y and grad_x must equal the oracle's (bit-exact; combine
also within 4e-3 of the oracle's fp32 sum; grad_w within its fp32 dot-product
bound).  The kernels of different ranks never wait for one another, so running
them one after another on one GPU computes exactly what one GPU per rank
would."""
import numpy as np
import pytest

import oracle
from load_balancing_plan_b200 import inputs
from tests import planchecks as pc

pytestmark = pytest.mark.gpu

PLAN_TABLES = ["cnt", "keep", "spill", "home_off", "fb_cnt", "fb_off", "load", "deficit", "fill",
               "slots_used", "slot_expert", "slot_cnt", "slot_off", "slot_first_j", "rep_ptr",
               "rep_expert", "rep_recv", "rep_slot", "rep_first_j", "rep_cnt", "rep_off", "recv_ptr",
               "seg_off", "seg_len", "alloc"]


@pytest.fixture(scope="module")
def env():
    import torch
    from load_balancing_plan_b200 import build
    build.build()
    oracle.build()
    from load_balancing_plan_b200 import ep, harness
    from load_balancing_plan_b200 import moonep as mp
    assert torch.cuda.is_available()
    yield torch, mp, ep, harness
    torch.cuda.empty_cache()


def cfg_of(R, L, S, K, H, B, headroom=0.0):
    C = S * K
    return dict(R=R, L=L, S=S, K=K, H=H, B=B, C=C, C_max=int(np.floor((1 + headroom) * C)))


def scale_rows(torch, harness, rb, row_expert, scale):
    """The stand-in expert on one rank's receive rows (in place)."""
    s = torch.from_numpy(np.asarray(scale, np.float32)).to(rb.recv.device)
    re = torch.from_numpy(row_expert).to(rb.recv.device)
    rows = (re >= 0).nonzero().flatten()
    if rows.numel():
        xr = rb.recv[rows].view(torch.bfloat16).float()
        rb.recv[rows] = (xr * s[re[rows]][:, None]).to(torch.bfloat16).view(torch.int16)


def run_ep_compare(env, cfg, ids, w, seed=0, E=256, mode=0, exchange=False):
    torch, mp, ep, harness = env
    R, L, S, K, H, B, Cm = (cfg[n] for n in ("R", "L", "S", "K", "H", "B", "C_max"))
    N, T = R * L, R * S
    em = ep.Emulation(cfg, w_elems=E, g_elems=E, poison=True)
    em.set_routing(ids, w)
    x = inputs.cb_bf16_np(seed, inputs.STREAM_X, np.arange(T * H)).reshape(R, S, H)
    wh = inputs.cb_bf16_np(seed, inputs.STREAM_W, np.arange(N * E)).reshape(R, L, E)
    gh = inputs.cb_f32_np(seed, inputs.STREAM_G_HOME, np.arange(N * E)).reshape(R, L, E)
    gr = inputs.cb_f32_np(seed, inputs.STREAM_G_REP, np.arange(R * B * E)).reshape(R, B, E)
    for r, rb in enumerate(em.ranks):
        rb.x[:S].copy_(torch.from_numpy(x[r].view(np.int16)))
        rb.w_home.copy_(torch.from_numpy(wh[r].view(np.int16)))
        rb.g_home.copy_(torch.from_numpy(np.ascontiguousarray(gh[r])))
        if B:
            rb.g_rep.copy_(torch.from_numpy(np.ascontiguousarray(gr[r])))
    flags = {0: 0, oracle.MODE_REMOTE: mp.PLAN_REMOTE_WEIGHTS, oracle.MODE_ONE_GROUP: mp.PLAN_ONE_GROUP}[mode]
    if exchange:
        # the ranks' counts_all start as garbage: only the ranks' own stores fill them
        for rb in em.ranks:
            rb.counts_all.fill_(-5)
    em.plan(flags, exchange=exchange)
    em.prefetch()
    em.dispatch()
    torch.cuda.synchronize()
    opl = oracle.plan(cfg, ids, mode=mode)
    if opl["status"] & (oracle.ST_CAPACITY | oracle.ST_EXPERT_ID):
        # a failed plan: every rank reports it and no rank writes anything
        for rb in em.ranks:
            assert rb.read_plan(tables=False)["status"] == opl["status"]
            assert bool((rb.recv == -1).all()) and bool((rb.dest == -7).all())
            assert bool((rb.w_slot == -1).all())
        return em, opl
    for r, rb in enumerate(em.ranks):
        gpl = rb.read_plan()
        assert gpl["status"] == opl["status"], (r, hex(gpl["status"]), hex(opl["status"]))
        for k in ("fallback_rows", "n_replicas", "migrated_rows"):
            assert gpl[k] == opl[k], (r, k)
        for k in PLAN_TABLES:
            assert np.array_equal(np.asarray(gpl[k]), np.asarray(opl[k])), (r, k)
    # destinations and receive rows, rank by rank
    recv_o = np.full((R * Cm, H), 0xFFFF, np.uint16)
    oracle.dispatch(cfg, opl["dest"], x.reshape(T, H), recv_o)
    for r, rb in enumerate(em.ranks):
        assert np.array_equal(rb.dest[:S * K].cpu().numpy(), opl["dest"][r].reshape(-1)), r
        assert np.array_equal(harness.to_u16(rb.recv), recv_o[r * Cm:(r + 1) * Cm]), r
    # prefetch: every rank's slots
    ws_o = np.full((R * B, E), 0xFFFF, np.uint16)
    oracle.prefetch(cfg, opl["slot_expert"], wh.reshape(N, E), ws_o, E)
    for r, rb in enumerate(em.ranks):
        if B:
            assert np.array_equal(harness.to_u16(rb.w_slot), ws_o[r * B:(r + 1) * B]), r
    # stand-in expert on every rank's rows, then combine
    scale = inputs.expert_scales(N, seed)
    row_e = pc.row_expert_map(cfg, opl)
    for r, rb in enumerate(em.ranks):
        scale_rows(torch, harness, rb, row_e[r * Cm:(r + 1) * Cm], scale)
    em.combine()
    torch.cuda.synchronize()
    y_o = recv_o.copy()
    oracle.expert_scale(cfg, opl, recv_o, scale, y_o)
    out_o, acc_o = oracle.combine(cfg, opl["dest"], y_o, w)
    for r, rb in enumerate(em.ranks):
        got = harness.to_u16(rb.out[:S])
        assert np.array_equal(got, out_o[r * S:(r + 1) * S]), r
        a = acc_o[r * S:(r + 1) * S]
        g = inputs.bf16_bits_to_f32_np(got)
        nz = a != 0
        assert np.all(g[~nz] == 0)
        if nz.any():
            assert np.max(np.abs(g[nz] - a[nz]) / np.abs(a[nz])) <= 4e-3
    ep_backward_compare(env, em, cfg, opl, y_o, w, seed)
    # reduce_grad: each home rank's gradients, every receiver's cleared slots
    em.reduce_grad()
    torch.cuda.synchronize()
    gh_o = np.ascontiguousarray(gh.reshape(N, E))
    gr_o = np.ascontiguousarray(gr.reshape(R * B, E)) if B else np.zeros((1, E), np.float32)
    oracle.reduce_grad(cfg, opl, gh_o, gr_o, E)
    for r, rb in enumerate(em.ranks):
        assert np.array_equal(rb.g_home.cpu().numpy().view(np.uint32), gh_o[r * L:(r + 1) * L].view(np.uint32)), r
        if B:
            assert np.array_equal(rb.g_rep.cpu().numpy().view(np.uint32), gr_o[r * B:(r + 1) * B].view(np.uint32)), r
    return em, opl


def ep_backward_compare(env, em, cfg, opl, y_o, w, seed):
    """The training backward pair, rank by rank: combine_backward writes
    grad_y into the ranks that hold the rows (and grad_w from y read on
    them); dispatch_backward then reads that grad_y back.  grad_y and grad_x
    bit-exact to the oracle; grad_w within the fp32 bound of its H-term dot
    product, |err| <= H * 2^-24 * sum |grad_out * y|."""
    torch, mp, ep, harness = env
    R, S, K, H, Cm = (cfg[n] for n in ("R", "S", "K", "H", "C_max"))
    T = R * S
    G = inputs.cb_bf16_np(seed + 7, inputs.STREAM_Y, np.arange(T * H)).reshape(T, H)
    g_d = [harness.as_i16(G[r * S:(r + 1) * S]).to(rb.recv.device) for r, rb in enumerate(em.ranks)]
    grad_y = [torch.full((max(Cm, 1), H), -1, dtype=torch.int16, device=rb.recv.device) for rb in em.ranks]
    grad_w = [torch.full((max(S * K, 1),), float("nan"), dtype=torch.float32, device=rb.recv.device)
              for rb in em.ranks]
    grad_x = [torch.full((max(S, 1), H), -1, dtype=torch.int16, device=rb.recv.device) for rb in em.ranks]
    gy_peers = ep.peer_table(grad_y, em.ranks[0].recv.device)
    for r, rb in enumerate(em.ranks):
        rb.combine_backward(g_d[r], em.recv_peers, gy_peers, grad_w[r])
    for r, rb in enumerate(em.ranks):
        rb.dispatch_backward(gy_peers, grad_x[r])
    torch.cuda.synchronize()
    for rb in em.ranks:
        assert rb.read_plan(tables=False)["status"] & mp.ST_ERROR_MASK == 0
    gy_o = np.full((R * Cm, H), 0xFFFF, np.uint16)
    gw_o = oracle.combine_backward(cfg, opl["dest"], G, y_o, w, gy_o)
    gx_o, _ = oracle.dispatch_backward(cfg, opl["dest"], gy_o)
    d = np.asarray(opl["dest"]).reshape(-1, K)
    f64 = lambda u: inputs.bf16_bits_to_f32_np(u).astype(np.float64)
    mag = np.einsum("th,tkh->tk", np.abs(f64(G)), np.abs(f64(y_o)[d]))
    for r in range(R):
        assert np.array_equal(harness.to_u16(grad_y[r][:Cm]), gy_o[r * Cm:(r + 1) * Cm]), r
        got = grad_w[r][:S * K].cpu().numpy().reshape(S, K).astype(np.float64)
        assert np.all(np.abs(got - gw_o[r * S:(r + 1) * S]) <= H * 2.0 ** -24 * mag[r * S:(r + 1) * S] + 1e-30), r
        assert np.array_equal(harness.to_u16(grad_x[r][:S]), gx_o[r * S:(r + 1) * S]), r


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("exchange", [False, True])
def test_ep_tiny_workload(env, seed, exchange):
    # exchange: each rank's counting launch stores its counts into every
    # rank's counts_all (moonep_ep_count_exchange) instead of an all-gather
    wl = inputs.WORKLOADS["tiny"]
    r = inputs.routing(wl.R, wl.L, wl.S, wl.K, seed, alpha=1.0)
    em, opl = run_ep_compare(env, wl.cfg(), r.topk_idx, r.topk_w, seed=seed, exchange=exchange)
    assert opl["n_replicas"] > 0
    if exchange:
        N = wl.R * wl.L
        for q, rb in enumerate(em.ranks):
            ca = rb.counts_all.cpu().numpy()
            for rr in range(wl.R):
                assert np.array_equal(ca[rr, :N], np.bincount(r.topk_idx[rr].reshape(-1), minlength=N)), (q, rr)
            assert not ca[:, N].any()


@pytest.mark.parametrize("case", [
    # R, L, S, K, H, B, headroom, mode
    (8, 4, 300, 4, 64, 4, 0.0, 0),            # ragged token ranges, every rank a sender or receiver
    (4, 2, 2, 2, 16, 2, 0.5, 0),              # fallback rows in the headroom
    (16, 24, 64, 8, 64, 4, 0.0, 1),           # remote weights (pieces without a slot)
    (8, 6, 96, 4, 64, 3, 2.0, 2),             # one home group per receiver
    (8, 6, 96, 4, 64, 3, 1.0, 2),             # the same with too little headroom: every rank refuses
    (2, 64, 1500, 8, 128, 64, 0.0, 0),        # few ranks, many experts
    (64, 2, 16, 2, 32, 2, 0.5, 0),            # R at its maximum
])
def test_ep_small_cases(env, case):
    R, L, S, K, H, B, headroom, mode = case
    exchange = R in (4, 64)  # the fallback case and the one with R at its maximum: counts exchanged in the launch
    cfg = cfg_of(R, L, S, K, H, B, headroom)
    if (R, L) == (4, 2):
        ids = pc.ids_from_counts(np.array([2, 3, 2, 3, 2, 3, 1, 0]), R, S, K)
        w = np.full((R, S, K), 0.5, np.float32)
    else:
        rt = inputs.routing(R, L, S, K, 3, alpha=1.5)
        ids, w = rt.topk_idx, rt.topk_w
    em, opl = run_ep_compare(env, cfg, ids, w, seed=1, mode=mode, exchange=exchange)
    if (R, L) == (4, 2):
        assert opl["fallback_rows"] > 0
    if mode == oracle.MODE_ONE_GROUP:
        assert bool(opl["status"] & oracle.ST_CAPACITY) == (headroom < 2.0)


def test_ep_mid_workload_plan_and_rows(env):
    # the mid workload split over 8 ranks, the counts exchanged in the
    # counting launches: every rank's tables and destinations in full, and
    # sampled dispatched rows and combined tokens
    torch, mp, ep, harness = env
    wl = inputs.WORKLOADS["mid"]
    cfg = wl.cfg()
    R, S, K, H, Cm = wl.R, wl.S, wl.K, wl.H, cfg["C_max"]
    r = inputs.routing(wl.R, wl.L, wl.S, wl.K, 0, maxvio=2.0)
    em = ep.Emulation(cfg, poison=True)
    em.set_routing(r.topk_idx, r.topk_w)
    for q, rb in enumerate(em.ranks):
        inputs.cb_fill_torch(rb.x.view(torch.bfloat16), 0, inputs.STREAM_X, offset=q * S * H)
    em.plan(exchange=True)
    em.dispatch()
    em.combine()
    torch.cuda.synchronize()
    opl = oracle.plan(cfg, r.topk_idx)
    rng = np.random.default_rng(0)
    for q, rb in enumerate(em.ranks):
        gpl = rb.read_plan()
        assert gpl["status"] == opl["status"]
        for k in PLAN_TABLES:
            assert np.array_equal(np.asarray(gpl[k]), np.asarray(opl[k])), (q, k)
        dest = rb.dest[:S * K].cpu().numpy()
        assert np.array_equal(dest, opl["dest"][q].reshape(-1)), q
        # sampled copies of this rank's tokens, found in their destination rank's buffer
        gs = rng.choice(S * K, 128, replace=False)
        for g in gs:
            d = int(dest[g])
            row = harness.to_u16(em.ranks[d // Cm].recv[d % Cm])
            t = q * S + g // K
            assert np.array_equal(row, inputs.cb_bf16_np(0, inputs.STREAM_X, t * H + np.arange(H)))
        # combine with the identity expert: out[t] from K copies of x[t]
        ts = rng.choice(S, 32, replace=False)
        xs = inputs.cb_bf16_np(0, inputs.STREAM_X, (q * S + ts)[:, None] * H + np.arange(H)[None, :])
        mini = dict(R=1, L=1, S=len(ts), K=K, H=H, B=0, C=len(ts) * K, C_max=len(ts) * K)
        d_mini = np.arange(len(ts) * K, dtype=np.int32).reshape(1, len(ts), K)
        out_o, _ = oracle.combine(mini, d_mini, np.repeat(xs, K, axis=0), r.topk_w[q][ts])
        assert np.array_equal(harness.to_u16(rb.out[torch.from_numpy(ts).cuda()]), out_o), q


@pytest.mark.parametrize("exchange", [False, True])
def test_ep_bad_id_on_one_rank_stops_every_rank(env, exchange):
    torch, mp, ep, harness = env
    wl = inputs.WORKLOADS["tiny"]
    cfg = wl.cfg()
    r = inputs.routing(wl.R, wl.L, wl.S, wl.K, 0, alpha=1.0)
    ids = r.topk_idx.copy()
    ids[2, 5, 1] = wl.N + 3            # one bad id, on rank 2
    em = ep.Emulation(cfg, poison=True)
    em.set_routing(ids, r.topk_w)
    em.plan(exchange=exchange)
    em.dispatch()
    torch.cuda.synchronize()
    for rb in em.ranks:
        assert rb.read_plan(tables=False)["status"] & mp.ST_EXPERT_ID
        assert bool((rb.recv == -1).all()) and bool((rb.dest == -7).all())


def test_ep_and_single_gpu_workspaces_do_not_mix(env):
    # a single-GPU plan's workspace is refused by the expert-parallel
    # dispatch, and a rank's workspace by the single-GPU dispatch (and by
    # another rank's dispatch): MOONEP_ST_CFG, nothing written
    torch, mp, ep, harness = env
    wl = inputs.WORKLOADS["tiny"]
    cfg = wl.cfg()
    r = inputs.routing(wl.R, wl.L, wl.S, wl.K, 0, alpha=1.0)
    em = ep.Emulation(cfg, poison=True)
    em.set_routing(r.topk_idx, r.topk_w)
    em.plan()
    prob = harness.Problem(cfg, poison=True)
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.plan()
    rb0, rb1 = em.ranks[0], em.ranks[1]
    # single-GPU dispatch with rank 0's workspace
    mp.moonep_dispatch(cfg, rb0.ws, prob.x, prob.ids, prob.recv, prob.dest)
    # rank 1's dispatch with rank 0's workspace
    mp.moonep_ep_dispatch(cfg, 1, rb0.ws, rb1.x, rb1.ids, em.recv_peers, rb1.dest)
    torch.cuda.synchronize()
    assert rb0.read_plan(tables=False)["status"] & mp.ST_CFG
    assert bool((prob.recv == -1).all()) and bool((rb1.dest == -7).all())
    # the expert-parallel dispatch with the single-GPU workspace
    mp.moonep_ep_dispatch(cfg, 0, prob.ws, rb0.x, rb0.ids, em.recv_peers, rb0.dest)
    torch.cuda.synchronize()
    assert prob.read_plan(tables=False)["status"] & mp.ST_CFG
    assert bool((rb0.dest == -7).all())
    for rb in em.ranks:
        assert bool((rb.recv == -1).all())


@pytest.mark.parametrize("case", [
    # R, L, S, K, H, B, headroom
    (4, 3, 50, 1, 24, 2, 1.0),       # K = 1, H not a multiple of 64
    (8, 2, 40, 2, 64, 0, 6.0),       # no prefetch slots: every spill falls back
    (3, 5, 7, 3, 16, 5, 1.0),        # ranges of a token or two, odd R
    (8, 8, 40, 64, 16, 8, 0.0),      # K at its maximum: a second id per producer lane
    (2, 2, 300, 2, 20008, 2, 1.0),   # long rows: several chunks per token in the gathers
])
def test_ep_edge_cases(env, case):
    R, L, S, K, H, B, headroom = case
    cfg = cfg_of(R, L, S, K, H, B, headroom=headroom)
    rt = inputs.routing(R, L, S, K, 2, alpha=1.5)
    em, opl = run_ep_compare(env, cfg, rt.topk_idx, rt.topk_w, seed=2)
    assert opl["status"] & oracle.ST_CAPACITY == 0
    if B == 0:
        assert opl["n_replicas"] == 0 and opl["fallback_rows"] > 0


@pytest.mark.parametrize("exchange", [False, True])
def test_ep_empty_ranks(env, exchange):
    # S = 0: nothing to count, plan or move; every call returns without error
    # (with the exchange, each rank still stores its zero row everywhere)
    torch, mp, ep, harness = env
    cfg = cfg_of(4, 2, 0, 2, 16, 2)
    em = ep.Emulation(cfg, w_elems=64, g_elems=64)
    if exchange:
        for rb in em.ranks:
            rb.counts_all.fill_(-5)
    em.plan(exchange=exchange)
    em.prefetch()
    em.dispatch()
    em.combine()
    em.reduce_grad()
    torch.cuda.synchronize()
    for rb in em.ranks:
        info = rb.read_plan(tables=False)
        assert info["status"] & mp.ST_ERROR_MASK == 0
        assert info["n_replicas"] == 0 and info["fallback_rows"] == 0
        assert not rb.counts_all.cpu().numpy().any()


@pytest.mark.parametrize("kernel", ["dispatch", "combine", "combine_backward", "prefetch"])
def test_ep_wait_timeout_is_reported_and_recoverable(env, kernel):
    # the expert-parallel forms give up after wait_limit polls (0 here) like
    # the single-GPU ones: each rank either finishes or records
    # MOONEP_ST_TIMEOUT in its own workspace and returns; the next plan
    # clears the status and the step then matches the oracle
    torch, mp, ep, harness = env
    cfg = cfg_of(4, 4, 512, 4, 4096, 4, headroom=1.0)
    R, S, K, H, Cm = 4, 512, 4, 4096, cfg["C_max"]
    r = inputs.routing(4, 4, 512, 4, 0, alpha=1.0)
    E = 64 * 1024
    em = ep.Emulation(cfg, w_elems=E, poison=True)
    em.set_routing(r.topk_idx, r.topk_w)
    for q, rb in enumerate(em.ranks):
        inputs.cb_fill_torch(rb.x.view(torch.bfloat16), 0, inputs.STREAM_X, offset=q * S * H)
        inputs.cb_fill_torch(rb.w_home.view(torch.bfloat16), 0, inputs.STREAM_W, offset=q * 4 * E)
    grad_y = [torch.zeros_like(rb.recv) for rb in em.ranks]
    gy_peers = ep.PeerTable(grad_y, "cuda")

    def run():
        if kernel == "dispatch":
            em.dispatch()
            return [rb.dest.clone() for rb in em.ranks] + [rb.recv.clone() for rb in em.ranks]
        if kernel == "combine":
            em.combine()
            return [rb.out.clone() for rb in em.ranks]
        if kernel == "combine_backward":
            em.combine_backward([rb.x for rb in em.ranks], gy_peers)
            return [g.clone() for g in grad_y]
        em.prefetch()
        return [rb.w_slot.clone() for rb in em.ranks]

    em.plan()
    if kernel != "dispatch":
        em.dispatch()
    torch.cuda.synchronize()
    try:
        mp.moonep_set_wait_limit(0)
        got = run()
        torch.cuda.synchronize()
        status = [rb.read_plan(tables=False)["status"] for rb in em.ranks]
    finally:
        mp.moonep_set_wait_limit(1 << 22)
    for st in status:
        assert st & mp.ST_ERROR_MASK & ~mp.ST_TIMEOUT == 0
    em.plan()
    em.dispatch()
    ref = run()
    torch.cuda.synchronize()
    for rb in em.ranks:
        assert rb.read_plan(tables=False)["status"] & mp.ST_ERROR_MASK == 0
    if not any(st & mp.ST_TIMEOUT for st in status):
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    # after recovery the step matches the oracle
    opl = oracle.plan(cfg, r.topk_idx)
    for q, rb in enumerate(em.ranks):
        assert np.array_equal(rb.dest[:S * K].cpu().numpy(), opl["dest"][q].reshape(-1)), q
