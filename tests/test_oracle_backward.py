"""Pins for the oracle's backward steps against the mathematics: dispatch and
combine are linear maps, so their backward steps are their adjoints (inner
product identities), the router-weight gradient is the derivative of the
forward combine (finite differences of the oracle's own forward), and
K = 1 with unit weights reduces both to exact copies."""
import numpy as np
import pytest

from load_balancing_plan_b200 import inputs

U = 2.0 ** -24


def _setup(oracle, seed, K=2, R=4, L=4, S=64, H=128, B=4):
    C = S * K
    cfg = dict(R=R, L=L, S=S, K=K, H=H, B=B, C=C, C_max=2 * C)
    r = inputs.routing(R, L, S, K, seed, alpha=1.0)
    pl = oracle.plan(cfg, r.topk_idx)
    assert pl["status"] & 0xFF == 0
    T = R * S
    x = inputs.cb_bf16_np(seed, inputs.STREAM_X, np.arange(T * H)).reshape(T, H)
    g_rows = inputs.cb_bf16_np(seed, inputs.STREAM_Y, np.arange(R * cfg["C_max"] * H)).reshape(-1, H)
    g_out = inputs.cb_bf16_np(seed + 1, inputs.STREAM_Y, np.arange(T * H)).reshape(T, H)
    return cfg, r, pl, x, g_rows, g_out


def f64(u16):
    return inputs.bf16_bits_to_f32_np(u16).astype(np.float64)


@pytest.mark.parametrize("seed", range(3))
def test_dispatch_backward_is_the_adjoint_of_dispatch(oracle_lib, seed):
    cfg, r, pl, x, G, _ = _setup(oracle_lib, seed)
    K = cfg["K"]
    recv = np.zeros_like(G)
    oracle_lib.dispatch(cfg, pl["dest"], x, recv)
    gx, acc = oracle_lib.dispatch_backward(cfg, pl["dest"], G)
    d = pl["dest"].reshape(-1, K)
    used = np.zeros(G.shape[0], bool)
    used[d.reshape(-1)] = True
    lhs = np.sum(f64(recv)[used] * f64(G)[used])              # <dispatch(x), G>
    rhs = np.sum(f64(x) * acc.astype(np.float64))             # <x, dispatch_bwd(G)>
    bound = np.sum(np.abs(f64(x)) * (K * U) * np.abs(f64(G)[d]).sum(1))
    assert abs(lhs - rhs) <= bound + 1e-9
    # the fp32 sum against the exact sum, and the bf16 rounding of it
    exact = f64(G)[d].sum(1)
    assert np.all(np.abs(acc - exact) <= K * U * np.abs(f64(G)[d]).sum(1) + 1e-30)
    assert np.all(np.abs(f64(gx) - acc) <= 2.0 ** -8 * np.abs(acc))


def test_dispatch_backward_detects_a_dropped_term(oracle_lib):
    cfg, r, pl, x, G, _ = _setup(oracle_lib, 0)
    K = cfg["K"]
    gx, acc = oracle_lib.dispatch_backward(cfg, pl["dest"], G)
    d = pl["dest"].reshape(-1, K)
    dropped = f64(G)[d[:, :1]].sum(1)
    assert np.max(np.abs(dropped - acc)) > 1e-2


@pytest.mark.parametrize("seed", range(3))
def test_combine_backward_grad_y_is_the_adjoint_in_y(oracle_lib, seed):
    cfg, r, pl, x, Y, g = _setup(oracle_lib, seed)
    K = cfg["K"]
    grad_y = np.full_like(Y, 0xFFFF)
    gw = oracle_lib.combine_backward(cfg, pl["dest"], g, Y, r.topk_w, grad_y)
    d = pl["dest"].reshape(-1, K)
    w = r.topk_w.reshape(-1, K).astype(np.float64)
    # grad_y rows are w * grad_out, rounded once to bf16
    want = w[:, :, None] * f64(g)[:, None, :]
    got = f64(grad_y)[d]
    assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want))
    used = np.zeros(Y.shape[0], bool)
    used[d.reshape(-1)] = True
    assert np.all(grad_y[~used] == 0xFFFF)                     # nothing written elsewhere
    # adjoint: <combine(y), g> == <y, grad_y> in exact arithmetic
    out, acc = oracle_lib.combine(cfg, pl["dest"], Y, r.topk_w)
    lhs = np.sum(acc.astype(np.float64) * f64(g))
    rhs = np.sum(f64(Y)[d] * want)
    terms = np.abs(w[:, :, None] * f64(Y)[d]).sum(1)
    assert abs(lhs - rhs) <= np.sum(np.abs(f64(g)) * K * U * terms) + 1e-9


@pytest.mark.parametrize("seed", range(2))
def test_combine_backward_grad_w_matches_finite_differences(oracle_lib, seed):
    # combine is linear in w: the change of the oracle's forward fp32 sum under
    # a perturbation of one weight, projected on grad_out, is grad_w
    cfg, r, pl, x, Y, g = _setup(oracle_lib, seed)
    K = cfg["K"]
    grad_y = np.zeros_like(Y)
    gw = oracle_lib.combine_backward(cfg, pl["dest"], g, Y, r.topk_w, grad_y)
    _, acc0 = oracle_lib.combine(cfg, pl["dest"], Y, r.topk_w)
    rng = np.random.default_rng(seed)
    d = pl["dest"].reshape(-1, K)
    for t, k in zip(rng.integers(0, d.shape[0], 12), rng.integers(0, K, 12)):
        w2 = r.topk_w.copy().reshape(-1, K)
        w2[t, k] = np.float32(w2[t, k] + np.float32(0.25))
        dw = float(w2[t, k]) - float(r.topk_w.reshape(-1, K)[t, k])
        _, acc1 = oracle_lib.combine(cfg, pl["dest"], Y, w2.reshape(r.topk_w.shape))
        fd = np.sum(f64(g)[t] * (acc1[t].astype(np.float64) - acc0[t].astype(np.float64))) / dw
        scale = np.sum(np.abs(f64(g)[t] * f64(Y)[d[t, k]])) + 1.0
        assert abs(fd - gw[t, k]) <= 1e-4 * scale
        # and the plain definition
        assert gw[t, k] == pytest.approx(np.dot(f64(g)[t], f64(Y)[d[t, k]]), rel=1e-12, abs=1e-12)


def test_single_choice_unit_weight_is_a_copy(oracle_lib):
    # K = 1 and weight 1: both backward steps are exact copies
    cfg, r, pl, x, Y, g = _setup(oracle_lib, 4, K=1)
    w = np.ones_like(r.topk_w)
    d = pl["dest"].reshape(-1)
    grad_y = np.zeros_like(Y)
    oracle_lib.combine_backward(cfg, pl["dest"], g, Y, w, grad_y, with_grad_w=False)
    assert np.array_equal(grad_y[d], g)
    gx, _ = oracle_lib.dispatch_backward(cfg, pl["dest"], Y)
    assert np.array_equal(gx, Y[d])
