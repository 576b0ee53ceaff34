"""moonep_plan_noalloc: the planning step for callers that cannot allocate
device memory (for example a plug-in that a host framework hands tensors to
but no allocator, or code whose device memory belongs to a pooled allocator
that must not see extra cudaMalloc calls).  Its workspace is a static array
inside the library; the caller passes only the router ids and a buffer for
the plan tables.  These tests call it through the C ABI and check that two
calls in a row give the same plan as moonep_plan with a caller-allocated
workspace (integer tables: bit for bit), and that a configuration too large
for the static workspace is refused with a clear error.

This file is collected last on purpose: a failure here comes after every
other test has run."""
import numpy as np
import pytest

from load_balancing_plan_b200 import inputs

TABLES = ["cnt", "keep", "spill", "home_off", "fb_cnt", "fb_off", "load", "deficit", "fill",
          "slots_used", "slot_expert", "slot_cnt", "slot_off", "slot_first_j", "rep_ptr",
          "rep_expert", "rep_recv", "rep_slot", "rep_first_j", "rep_cnt", "rx_expert",
          "route_ptr", "route_end", "route_base", "seg_off", "seg_len", "alloc"]


@pytest.fixture(scope="module")
def mp():
    from load_balancing_plan_b200 import build
    build.build()
    from load_balancing_plan_b200 import moonep
    return moonep


def test_refuses_configuration_above_static_workspace(mp):
    # 4096 experts over 64 ranks with many tokens needs far more than 2 MiB
    cfg = dict(R=64, L=64, S=1024, K=8, H=64, B=8, C=8192, C_max=8192)
    assert mp.moonep_plan_workspace_bytes(cfg) > (2 << 20)
    with pytest.raises(mp.MoonepError) as ei:
        mp.moonep_plan_noalloc(cfg, 256, 256, stream=0)
    assert ei.value.code == mp.ERR_ARG
    assert "static workspace" in mp.last_error()


@pytest.mark.parametrize("name", ["mid", "skew", "inference", "training"])
def test_refuses_the_larger_workloads(mp, name):
    # of the library's workloads only tiny (28 KB) and profile (0.55 MiB) fit
    # the 2 MiB static workspace; mid already needs 2.07 MiB
    cfg = inputs.WORKLOADS[name].cfg()
    assert mp.moonep_plan_workspace_bytes(cfg) > (2 << 20)
    with pytest.raises(mp.MoonepError) as ei:
        mp.moonep_plan_noalloc(cfg, 256, 256, stream=0)
    assert ei.value.code == mp.ERR_ARG
    assert "static workspace" in mp.last_error()


@pytest.mark.parametrize("name", ["tiny", "profile"])
def test_small_workloads_fit(mp, name):
    assert mp.moonep_plan_workspace_bytes(inputs.WORKLOADS[name].cfg()) <= (2 << 20)


def test_binding_refuses_a_short_output_tensor(mp):
    # the C function sees only an address; the binding checks the tensor's
    # size before any GPU work (a CPU tensor is enough to show the refusal)
    import torch
    cfg = inputs.WORKLOADS["tiny"].cfg()
    need = mp.moonep_ws_layout(cfg)["tables_end"]
    short = torch.zeros(need - 1, dtype=torch.int32)
    with pytest.raises(mp.MoonepError) as ei:
        mp.moonep_plan_noalloc(cfg, 256, short, stream=0)
    assert ei.value.code == mp.ERR_ARG
    assert "tables_out holds" in str(ei.value)


def _plan_both(mp, torch, cfg, route):
    dev = torch.device("cuda")
    ids = torch.from_numpy(route.topk_idx.reshape(-1).copy()).to(dev)
    lay = mp.moonep_ws_layout(cfg)
    ws = torch.zeros(lay["words"], dtype=torch.int32, device=dev)
    mp.moonep_plan(cfg, ids, ws)
    ref = mp.moonep_plan_read(cfg, ws, tables=True)
    out = torch.full((lay["tables_end"],), -9, dtype=torch.int32, device=dev)
    mp.moonep_plan_noalloc(cfg, ids, out)
    got = mp.moonep_plan_read(cfg, out, tables=True)
    return ref, got


def _same(ref, got):
    for k in ("status", "fallback_rows", "n_replicas", "migrated_rows"):
        assert got[k] == ref[k], k
    for k in TABLES:
        n = len(ref[k]) if k != "rx_expert" else len(set(np.asarray(ref["rep_expert"]).tolist()))
        if k in ("route_end", "route_base"):
            n = 2 * (len(ref["cnt"])) + ref["n_replicas"]
        a = np.asarray(got[k]).reshape(-1)[:n]
        b = np.asarray(ref[k]).reshape(-1)[:n]
        assert np.array_equal(a, b), k


@pytest.mark.gpu
def test_two_calls_in_a_row_match_moonep_plan(mp):
    import torch
    assert torch.cuda.is_available()
    # two consecutive calls on the shared static workspace, different router
    # outputs and a different configuration the second time, so a stale value
    # left by the first call would show
    wl = inputs.WORKLOADS["profile"]
    r1 = inputs.routing(wl.R, wl.L, wl.S, wl.K, 0, maxvio=2.0)
    ref1, got1 = _plan_both(mp, torch, wl.cfg(), r1)
    t = inputs.WORKLOADS["tiny"]
    r2 = inputs.routing(t.R, t.L, t.S, t.K, 3, alpha=1.0)
    ref2, got2 = _plan_both(mp, torch, t.cfg(), r2)
    torch.cuda.synchronize()
    assert ref1["n_replicas"] > 0 and ref2["n_replicas"] > 0
    _same(ref1, got1)
    _same(ref2, got2)


@pytest.mark.gpu
def test_tables_only_copy_is_refused_by_dispatch_and_accepted_by_prefetch(mp):
    """The copy holds no dispatch scratch: moonep_dispatch given it as a
    workspace sets MOONEP_ST_CFG and writes nothing.  prefetch reads only the
    tables and gives the same slots as with the full workspace.  The copy is
    allocated with the full workspace size, so even a dispatch that ignored the
    mark would read inside the buffer."""
    import torch
    from load_balancing_plan_b200 import harness
    dev = torch.device("cuda")
    wl = inputs.WORKLOADS["tiny"]
    cfg = wl.cfg()
    r = inputs.routing(wl.R, wl.L, wl.S, wl.K, 1, alpha=1.0)
    E = 1024
    full = harness.Problem(cfg, poison=True, w_elems=E)
    full.set_routing(r.topk_idx, r.topk_w)
    full.fill_x(0)
    full.fill_weights(0)
    full.plan()
    full.prefetch()
    lay = mp.moonep_ws_layout(cfg)
    copy = torch.full((lay["words"],), 7, dtype=torch.int32, device=dev)
    mp.moonep_plan_noalloc(cfg, full.ids, copy)
    torch.cuda.synchronize()
    assert int(copy[18]) == 0x5A5A5A5A
    assert int(full.ws[18]) == 0
    info = mp.moonep_plan_read(cfg, copy)
    assert info["status"] & mp.ST_ERROR_MASK == 0 and info["n_replicas"] > 0

    # dispatch on the copy: refused on the device, nothing written
    recv = torch.full_like(full.recv, -1)
    dest = torch.full_like(full.dest, -7)
    mp.moonep_dispatch(cfg, copy, full.x, full.ids, recv, dest)
    torch.cuda.synchronize()
    info = mp.moonep_plan_read(cfg, copy)
    assert info["status"] & mp.ST_CFG
    assert bool((recv == -1).all()) and bool((dest == -7).all())

    # prefetch with a fresh copy: same slots as with the full workspace
    copy2 = torch.empty(lay["tables_end"], dtype=torch.int32, device=dev)
    mp.moonep_plan_noalloc(cfg, full.ids, copy2)
    w_slot = torch.full_like(full.w_slot, -1)
    mp.moonep_prefetch(cfg, copy2, full.w_home, w_slot, E)
    torch.cuda.synchronize()
    assert mp.moonep_plan_read(cfg, copy2)["status"] & mp.ST_ERROR_MASK == 0
    assert torch.equal(w_slot, full.w_slot)
