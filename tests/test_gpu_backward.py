"""GPU parity of the backward pair against the oracle: combine_backward's
grad_y bit for bit (one fp32 multiply rounded to bf16, as in the oracle) and
grad_w within the worst-case bound of any fp32 summation order of H products
(|err| <= H * 2^-24 * sum |products|) around the oracle's fp64 sum;
dispatch_backward bit for bit (fp32 adds in k order, one rounding)."""
import numpy as np
import pytest

import oracle
from load_balancing_plan_b200 import inputs

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


@pytest.fixture(scope="module")
def env():
    import torch
    from load_balancing_plan_b200 import build
    build.build()
    oracle.build()
    from load_balancing_plan_b200 import harness
    from load_balancing_plan_b200 import moonep as mp
    yield torch, mp, harness
    torch.cuda.empty_cache()


def f64(u16):
    return inputs.bf16_bits_to_f32_np(u16).astype(np.float64)


def _case(env, cfg, ids, w, seed, with_w=True):
    torch, mp, harness = env
    R, K, H, Cm = cfg["R"], cfg["K"], cfg["H"], cfg["C_max"]
    T = R * cfg["S"]
    prob = harness.Problem(cfg, poison=True)
    prob.set_routing(ids, w)
    prob.fill_x(seed)
    prob.plan()
    prob.dispatch()
    opl = oracle.plan(cfg, ids)
    assert opl["status"] & 0xFF == 0
    rows = R * Cm
    Y = inputs.cb_bf16_np(seed, inputs.STREAM_Y, np.arange(rows * H)).reshape(rows, H)
    G = inputs.cb_bf16_np(seed + 7, inputs.STREAM_Y, np.arange(T * H)).reshape(T, H)
    dev = "cuda"
    y_d = harness.as_i16(Y).to(dev)
    g_d = harness.as_i16(G).to(dev)
    grad_y = torch.full((rows, H), -1, dtype=torch.int16, device=dev)
    grad_w = torch.full((T * K,), float("nan"), dtype=torch.float32, device=dev) if with_w else None
    mp.moonep_combine_backward(cfg, prob.ws, g_d, y_d if with_w else None, prob.dest, prob.w, grad_y, grad_w)
    grad_x = torch.full((T, H), -1, dtype=torch.int16, device=dev)
    mp.moonep_dispatch_backward(cfg, prob.ws, y_d, prob.dest, grad_x)
    torch.cuda.synchronize()
    assert mp.moonep_plan_read(cfg, prob.ws)["status"] & mp.ST_ERROR_MASK == 0
    # oracle
    gy_o = np.full((rows, H), 0xFFFF, np.uint16)
    gw_o = oracle.combine_backward(cfg, opl["dest"], G, Y, w, gy_o, with_grad_w=with_w)
    assert np.array_equal(harness.to_u16(grad_y), gy_o)
    if with_w:
        d = opl["dest"].reshape(-1, K)
        mag = np.einsum("th,tkh->tk", np.abs(f64(G)), np.abs(f64(Y)[d]))
        got = grad_w.cpu().numpy().reshape(-1, K).astype(np.float64)
        assert np.all(np.abs(got - gw_o) <= H * U * mag + 1e-30)
    gx_o, acc_o = oracle.dispatch_backward(cfg, opl["dest"], Y)
    assert np.array_equal(harness.to_u16(grad_x), gx_o)
    return prob


@pytest.mark.parametrize("seed", range(3))
def test_tiny(env, seed):
    w = inputs.WORKLOADS["tiny"]
    r = inputs.routing(w.R, w.L, w.S, w.K, seed, alpha=1.0)
    _case(env, w.cfg(), r.topk_idx, r.topk_w, seed)


@pytest.mark.parametrize("case", [
    (3, 5, 333, 3, 296, 2, 1.0),
    (8, 8, 40, 64, 16, 8, 0.0),      # K at its maximum: several k batches
    (2, 2, 300, 2, 20008, 2, 1.0),   # long rows
    (1, 7, 500, 1, 8, 2, 0.0),
    (2, 2, 4, 2, 1 << 20, 2, 1.0),   # H at its maximum (2 MB rows)
])
def test_edge_cases(env, case):
    R, L, S, K, H, B, hr = case
    C = S * K
    cfg = dict(R=R, L=L, S=S, K=K, H=H, B=B, C=C, C_max=int(np.floor((1 + hr) * C)))
    r = inputs.routing(R, L, S, K, 0, alpha=1.0)
    _case(env, cfg, r.topk_idx, r.topk_w, 1)


def test_without_router_weight_gradient(env):
    w = inputs.WORKLOADS["tiny"]
    r = inputs.routing(w.R, w.L, w.S, w.K, 3, alpha=1.0)
    _case(env, w.cfg(), r.topk_idx, r.topk_w, 3, with_w=False)


def test_full_size_sampled(env):
    # the mid workload: every grad_y row of sampled tokens, their grad_w and
    # grad_x, against the oracle computed token by token
    torch, mp, harness = env
    wl = inputs.WORKLOADS["mid"]
    cfg = wl.cfg()
    R, K, H, Cm, T = wl.R, wl.K, wl.H, wl.C_max, wl.T
    r = inputs.routing(wl.R, wl.L, wl.S, wl.K, 0, maxvio=2.0)
    prob = harness.Problem(cfg)
    prob.set_routing(r.topk_idx, r.topk_w)
    prob.plan()
    prob.dispatch()
    y_d = torch.empty((R * Cm, H), dtype=torch.int16, device="cuda")
    inputs.cb_fill_torch(y_d.view(torch.bfloat16), 0, inputs.STREAM_Y)
    g_d = torch.empty((T, H), dtype=torch.int16, device="cuda")
    inputs.cb_fill_torch(g_d.view(torch.bfloat16), 7, inputs.STREAM_Y)
    grad_y = torch.zeros((R * Cm, H), dtype=torch.int16, device="cuda")
    grad_w = torch.zeros((T * K,), dtype=torch.float32, device="cuda")
    grad_x = torch.zeros((T, H), dtype=torch.int16, device="cuda")
    mp.moonep_combine_backward(cfg, prob.ws, g_d, y_d, prob.dest, prob.w, grad_y, grad_w)
    mp.moonep_dispatch_backward(cfg, prob.ws, y_d, prob.dest, grad_x)
    torch.cuda.synchronize()
    dest = prob.dest.cpu().numpy().reshape(T, K)
    rng = np.random.default_rng(5)
    ts = np.sort(rng.choice(T, 128, replace=False))
    n = len(ts)
    G = inputs.cb_bf16_np(7, inputs.STREAM_Y, ts[:, None] * H + np.arange(H)[None, :])
    d = dest[ts]
    Ys = inputs.cb_bf16_np(0, inputs.STREAM_Y, d.reshape(-1)[:, None] * H + np.arange(H)[None, :])
    mini = dict(R=1, L=1, S=n, K=K, H=H, B=0, C=n * K, C_max=n * K)
    d_mini = np.arange(n * K, dtype=np.int32).reshape(1, n, K)
    w_mini = np.ascontiguousarray(r.topk_w.reshape(T, K)[ts])
    gy_o = np.zeros((n * K, H), np.uint16)
    gw_o = oracle.combine_backward(mini, d_mini, G, Ys, w_mini, gy_o)
    got_rows = harness.to_u16(grad_y[torch.from_numpy(d.reshape(-1)).long().cuda()])
    assert np.array_equal(got_rows, gy_o)
    mag = np.einsum("th,tkh->tk", np.abs(f64(G)), np.abs(f64(Ys)).reshape(n, K, H))
    got_w = grad_w.cpu().numpy().reshape(T, K)[ts].astype(np.float64)
    assert np.all(np.abs(got_w - gw_o) <= H * U * mag + 1e-30)
    gx_o, _ = oracle.dispatch_backward(mini, d_mini, Ys)
    assert np.array_equal(harness.to_u16(grad_x[torch.from_numpy(ts).cuda()]), gx_o)
