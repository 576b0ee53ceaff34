"""The expert-parallel step as separate processes, one per rank: each process
owns its buffers, maps the other ranks' buffers through CUDA IPC
(ep.map_peers), gets every rank's counts (an all-gather over the process
group, or each rank's counting launch storing its counts into every rank's
mapped counts_all) and orders the ranks between calls with barriers, as one
process per GPU does.  Here both processes share one GPU (the kernels of
different ranks never wait for one another, so running them in two contexts
on one device computes what two devices would; only NVLink is missing).  The
process group is gloo, so the all-gathered counts travel through host
memory.  Each rank checks its own destinations,
receive rows, combined outputs, prefetched slots, backward gradients and
reduced gradients against the oracle, bit for bit (grad_w within its fp32
bound)."""
import socket

import numpy as np
import pytest
import torch.multiprocessing as tmp

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q, case):
    import datetime
    import os
    import torch
    import torch.distributed as dist
    import oracle
    from load_balancing_plan_b200 import ep, harness, inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=90))
    errors = []
    try:
        torch.cuda.set_device(0)
        dev = torch.device("cuda", 0)
        L, S, K, H, B, hr, seed, exchange = case
        R = world
        C = S * K
        cfg = dict(R=R, L=L, S=S, K=K, H=H, B=B, C=C, C_max=int(np.floor((1 + hr) * C)))
        N, T, Cm, E = R * L, R * S, cfg["C_max"], 64
        ep.check_same_config(cfg)
        rt = inputs.routing(R, L, S, K, seed, alpha=1.5)
        rb = ep.RankBuffers(cfg, rank, dev, w_elems=E, g_elems=E, poison=True)
        rb.set_routing(rt.topk_idx[rank], rt.topk_w[rank])
        x = inputs.cb_bf16_np(seed, inputs.STREAM_X, np.arange(T * H)).reshape(R, S, H)
        wh = inputs.cb_bf16_np(seed, inputs.STREAM_W, np.arange(N * E)).reshape(R, L, E)
        gh = inputs.cb_f32_np(seed, inputs.STREAM_G_HOME, np.arange(N * E)).reshape(R, L, E)
        gr = inputs.cb_f32_np(seed, inputs.STREAM_G_REP, np.arange(R * B * E)).reshape(R, B, E)
        rb.x[:S].copy_(torch.from_numpy(x[rank].view(np.int16)))
        rb.w_home.copy_(torch.from_numpy(wh[rank].view(np.int16)))
        rb.g_home.copy_(torch.from_numpy(np.ascontiguousarray(gh[rank])))
        if B:
            rb.g_rep.copy_(torch.from_numpy(np.ascontiguousarray(gr[rank])))
        grad_y = torch.full((max(Cm, 1), H), -1, dtype=torch.int16, device=dev)
        grad_w = torch.full((max(S * K, 1),), float("nan"), dtype=torch.float32, device=dev)
        grad_x = torch.full((max(S, 1), H), -1, dtype=torch.int16, device=dev)
        G = inputs.cb_bf16_np(seed + 7, inputs.STREAM_Y, np.arange(T * H)).reshape(T, H)
        g_out = harness.as_i16(G[rank * S:(rank + 1) * S]).to(dev)
        torch.cuda.synchronize()

        def between():
            torch.cuda.synchronize()
            dist.barrier()

        # peers: every rank's buffers mapped into this process (the PeerTable
        # objects keep the mappings alive)
        recv_peers = ep.map_peers(rb.recv, dev)
        w_home_peers = ep.map_peers(rb.w_home, dev)
        g_rep_peers = ep.map_peers(rb.g_rep, dev)
        grad_y_peers = ep.map_peers(grad_y, dev)
        counts_all_peers = ep.map_peers(rb.counts_all, dev)

        if exchange:
            # each rank's counting launch stores its counts into every rank's
            # counts_all; the barrier then stands in for the all-gather
            rb.counts_all.fill_(-5)
            between()
            rb.count(counts_all_peers=counts_all_peers)
            between()
        else:
            rb.count()
            counts_all = torch.zeros((R, N + 1), dtype=torch.int32)
            ep.gather_counts(rb.counts.cpu(), counts_all)
            rb.counts_all.copy_(counts_all)
        rb.plan()
        rb.prefetch(w_home_peers)
        rb.dispatch(recv_peers)
        between()
        # the expert: identity (the expert outputs are the dispatched rows)
        rb.combine(recv_peers)
        rb.combine_backward(g_out, recv_peers, grad_y_peers, grad_w)
        between()
        rb.dispatch_backward(grad_y_peers, grad_x)
        rb.reduce_grad(g_rep_peers)
        between()

        opl = oracle.plan(cfg, rt.topk_idx)
        info = rb.read_plan(tables=False)
        if info["status"] != opl["status"]:
            errors.append("status %x != %x" % (info["status"], opl["status"]))
        recv_o = np.full((R * Cm, H), 0xFFFF, np.uint16)
        oracle.dispatch(cfg, opl["dest"], x.reshape(T, H), recv_o)
        if not np.array_equal(rb.dest[:S * K].cpu().numpy(), opl["dest"][rank].reshape(-1)):
            errors.append("dest")
        if not np.array_equal(harness.to_u16(rb.recv), recv_o[rank * Cm:(rank + 1) * Cm]):
            errors.append("recv")
        out_o, _ = oracle.combine(cfg, opl["dest"], recv_o, rt.topk_w)
        if not np.array_equal(harness.to_u16(rb.out[:S]), out_o[rank * S:(rank + 1) * S]):
            errors.append("combine")
        ws_o = np.full((R * B, E), 0xFFFF, np.uint16)
        oracle.prefetch(cfg, opl["slot_expert"], wh.reshape(N, E), ws_o, E)
        if B and not np.array_equal(harness.to_u16(rb.w_slot), ws_o[rank * B:(rank + 1) * B]):
            errors.append("prefetch")
        gy_o = np.full((R * Cm, H), 0xFFFF, np.uint16)
        gw_o = oracle.combine_backward(cfg, opl["dest"], G, recv_o, rt.topk_w, gy_o)
        if not np.array_equal(harness.to_u16(grad_y[:Cm]), gy_o[rank * Cm:(rank + 1) * Cm]):
            errors.append("combine_backward grad_y")
        d = np.asarray(opl["dest"]).reshape(-1, K)
        f64 = lambda u: inputs.bf16_bits_to_f32_np(u).astype(np.float64)
        mag = np.einsum("th,tkh->tk", np.abs(f64(G)), np.abs(f64(recv_o)[d]))[rank * S:(rank + 1) * S]
        got = grad_w[:S * K].cpu().numpy().reshape(S, K).astype(np.float64)
        if not np.all(np.abs(got - gw_o[rank * S:(rank + 1) * S]) <= H * 2.0 ** -24 * mag + 1e-30):
            errors.append("combine_backward grad_w")
        gx_o, _ = oracle.dispatch_backward(cfg, opl["dest"], gy_o)
        if not np.array_equal(harness.to_u16(grad_x[:S]), gx_o[rank * S:(rank + 1) * S]):
            errors.append("dispatch_backward")
        gh_o = np.ascontiguousarray(gh.reshape(N, E))
        gr_o = np.ascontiguousarray(gr.reshape(R * B, E)) if B else np.zeros((1, E), np.float32)
        oracle.reduce_grad(cfg, opl, gh_o, gr_o, E)
        if not np.array_equal(rb.g_home.cpu().numpy().view(np.uint32), gh_o[rank * L:(rank + 1) * L].view(np.uint32)):
            errors.append("reduce_grad home")
        if B and not np.array_equal(rb.g_rep.cpu().numpy().view(np.uint32),
                                    gr_o[rank * B:(rank + 1) * B].view(np.uint32)):
            errors.append("reduce_grad slots")
        q.put((rank, errors, int(opl["n_replicas"]), int(opl["fallback_rows"])))
        # keep every mapping alive until all ranks have checked
        dist.barrier()
    except Exception as e:  # report, then leave the group
        q.put((rank, ["exception: %r" % (e,)], -1, -1))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [
    # L, S, K, H, B, headroom, seed, counts exchanged in the counting launch
    (4, 64, 2, 64, 2, 0.5, 3, False),
    (8, 300, 4, 136, 3, 1.0, 1, True),
])
def test_two_processes_on_cuda_ipc(case):
    import oracle
    from load_balancing_plan_b200 import build
    build.build()
    oracle.build()
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q, case)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted((q.get(timeout=240) for _ in range(2)), key=lambda t: t[0])
    finally:
        for p in procs:
            p.join(120)
            if p.exitcode is None:
                p.kill()
    for rank, errors, n_rep, fb in res:
        assert errors == [], (rank, errors)
    assert res[0][2] > 0  # the skew made replicas, so rows crossed between the processes
    for p in procs:
        assert p.exitcode == 0
