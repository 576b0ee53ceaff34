"""The host side of expert parallelism on CPU, as two gloo ranks: the
all-gather that gives every rank every rank's counts, and the check that the
ranks plan the same configuration.  (The counts here are histograms of each
rank's own router ids plus its status word, as moonep_ep_count leaves them.)
The device side of the same path is covered on the GPU by test_gpu_ep."""
import socket

import numpy as np
import torch.multiprocessing as tmp

from load_balancing_plan_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, cfg_of_rank):
    import datetime
    import os
    import torch
    import torch.distributed as dist
    from load_balancing_plan_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = inputs.WORKLOADS["tiny"]
        cfg = dict(wl.cfg(), R=world, L=wl.L * wl.R // world)
        N = cfg["R"] * cfg["L"]
        r = inputs.routing(cfg["R"], cfg["L"], cfg["S"], cfg["K"], 5, alpha=1.0)
        mine = np.bincount(r.topk_idx[rank].reshape(-1), minlength=N).astype(np.int32)
        status = 0x1 if rank == 1 else 0
        counts = torch.from_numpy(np.concatenate([mine, [status]]).astype(np.int32))
        counts_all = torch.zeros((world, N + 1), dtype=torch.int32)
        ep.gather_counts(counts, counts_all)
        err = None
        try:
            ep.check_same_config(cfg_of_rank(cfg, rank))
        except ValueError as e:
            err = str(e)
        q.put((rank, counts_all.numpy().copy(), r.topk_idx, err))
    finally:
        dist.destroy_process_group()


def _same(cfg, rank):
    return cfg


def _differ(cfg, rank):
    return dict(cfg, B=cfg["B"] + rank)


def _run(cfg_of_rank):
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, cfg_of_rank)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(2)), key=lambda t: t[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    return res


def test_two_ranks_gather_each_others_counts():
    res = _run(_same)
    (_, ca0, ids, err0), (_, ca1, _, err1) = res
    N = ca0.shape[1] - 1
    assert err0 is None and err1 is None
    # both ranks hold the same [R][N + 1] table: row q = rank q's histogram
    # and status; the column sums are the histogram of all ids
    assert np.array_equal(ca0, ca1)
    for q in range(2):
        assert np.array_equal(ca0[q, :N], np.bincount(ids[q].reshape(-1), minlength=N))
    assert list(ca0[:, N]) == [0, 0x1]
    assert np.array_equal(ca0[:, :N].sum(0), np.bincount(ids.reshape(-1), minlength=N))


def test_ranks_with_different_configurations_both_refuse():
    res = _run(_differ)
    for _, _, _, err in res:
        assert err is not None and "disagree" in err


def test_peer_table_keeps_its_tensors():
    # the table holds plain addresses; the PeerTable object holds the tensors
    # behind them, so they live as long as the table is in use
    import gc
    import weakref
    import torch
    from load_balancing_plan_b200 import ep
    ts = [torch.zeros(4, dtype=torch.int32) for _ in range(3)]
    refs = [weakref.ref(t) for t in ts]
    pt = ep.PeerTable(ts, "cpu")
    assert pt.table.tolist() == [t.data_ptr() for t in ts]
    assert pt.data_ptr() == pt.table.data_ptr()
    assert ep._table(pt) is pt.table and ep._table(pt.table) is pt.table
    del ts
    gc.collect()
    assert all(r() is not None for r in refs)
    del pt
    gc.collect()
    assert all(r() is None for r in refs)
