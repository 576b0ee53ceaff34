"""Pins for the oracle's one-home-group plan mode ("The Busiest Rank Sets Your
Step Time", section "Installation and integration", the paragraph on B after
the weight-tensor figure: a rank duplicates experts of at most one remote home
group, so B = E/R slots always suffice).  The mode is the headroom rule with
one more condition on a receiver: once it holds a piece of an expert of home
group h it takes rows of group h only.

Pinned by brute force against the independent row-at-a-time simulator, by a
worked example done by hand, by the special case where one home group spills
(the condition never binds, so the plan is the headroom rule's), and by the
property the passage gives it (with B >= E/R the slot count never binds)."""
import itertools

import numpy as np
import pytest

from tests import planchecks as pc
from load_balancing_plan_b200 import inputs


def _cfg(R, L, S, K, B, C_max=None):
    C = S * K
    return dict(R=R, L=L, S=S, K=K, H=8, B=B, C=C, C_max=C if C_max is None else C_max)


def _groups_per_receiver(cfg, pl):
    n = pl["n_replicas"]
    L = cfg["L"]
    out = []
    for r in range(cfg["R"]):
        q = np.nonzero(pl["rep_recv"][:n] == r)[0]
        out.append(set((pl["rep_expert"][q] // L).tolist()))
    return out


def _compare(oracle, cfg, ids):
    pl = oracle.plan(cfg, ids, mode=oracle.MODE_ONE_GROUP)
    un = oracle.plan_unitwise(cfg, ids, mode=oracle.MODE_ONE_GROUP)
    assert pl["status"] == un["status"]
    if pl["status"] & oracle.ST_CAPACITY:
        return pl
    for k in ("dest", "alloc", "slot_expert", "slot_cnt", "fb_cnt"):
        assert np.array_equal(pl[k], un[k]), k
    info = pc.check_plan(cfg, ids, pl)
    groups = _groups_per_receiver(cfg, pl)
    assert all(len(g) <= 1 for g in groups), groups
    # a receiver never takes from its own group (it spills nothing)
    assert all(r not in g for r, g in enumerate(groups))
    # rows a receiver could not take are exactly the rows that fell back
    unfilled = np.maximum(cfg["C"] - info["rows"], 0).sum()
    assert unfilled == pl["fallback_rows"]
    return pl


@pytest.mark.parametrize("R,L,S,K,B", [
    (3, 1, 2, 1, 1),     # 729 inputs: two senders, one receiver is the smallest conflict
    (3, 2, 2, 1, 2),     # 46656 inputs
    (2, 2, 2, 2, 2),     # two ranks: one sender at most, the condition never binds
    (4, 1, 2, 1, 1),     # 65536 inputs
])
def test_bruteforce_matches_unitwise(oracle_lib, R, L, S, K, B):
    N, T = R * L, R * S
    cfg = _cfg(R, L, S, K, B, C_max=R * S * K)
    choices = list(itertools.permutations(range(N), K))
    n = nfb = 0
    for combo in itertools.product(range(len(choices)), repeat=T):
        ids = np.array([choices[c] for c in combo], np.int32).reshape(R, S, K)
        pl = _compare(oracle_lib, cfg, ids)
        n += 1
        nfb += pl["fallback_rows"] > 0
    assert n == len(choices) ** T
    if R >= 3:
        assert nfb > 0        # the condition binds somewhere


def test_worked_example_two_senders_one_receiver(oracle_lib):
    # R=3, L=1, S=2, K=1, so C=2.  Experts 0 and 1 take 3 rows each, expert 2
    # none: ranks 0 and 1 are one row over, rank 2 is two rows short.  The
    # headroom rule gives rank 2 one row of each; one group per receiver lets
    # rank 2 take expert 0's row only, and expert 1's last row stays on rank 1
    # in its headroom (row C).
    cfg = _cfg(3, 1, 2, 1, 2, C_max=4)
    ids = pc.ids_from_counts(np.array([3, 3, 0]), 3, 2, 1)
    base = oracle_lib.plan(cfg, ids)
    assert base["fallback_rows"] == 0
    assert base["alloc"].reshape(3, 3).tolist() == [[2, 0, 1], [0, 2, 1], [0, 0, 0]]
    pl = _compare(oracle_lib, cfg, ids)
    assert pl["alloc"].reshape(3, 3).tolist() == [[2, 0, 1], [0, 3, 0], [0, 0, 0]]
    assert pl["fallback_rows"] == 1 and pl["fb_cnt"].tolist() == [0, 1, 0]
    assert pl["slot_expert"].reshape(3, 2).tolist() == [[-1, -1], [-1, -1], [0, -1]]
    assert pl["migrated_rows"] == 1
    # token order: expert 0 holds global tokens 0..2, expert 1 tokens 3..5;
    # expert 0's third copy is rank 2's first row, expert 1's third copy is
    # rank 1's row C = 2
    assert pl["dest"].reshape(-1).tolist() == [0, 1, 2 * 4 + 0, 4 + 0, 4 + 1, 4 + 2]


@pytest.mark.parametrize("seed", range(6))
def test_one_spilling_group_is_the_headroom_rule(oracle_lib, seed):
    # all overflow from one home rank: every receiver's pieces are of that
    # group whatever the rule, so the plan is the headroom rule's
    rng = np.random.default_rng(seed)
    R, L, S, K, B = 8, 4, 64, 4, 4
    C, T, N = S * K, R * S, R * L
    hot = int(rng.integers(R))
    cnt = np.zeros(N, np.int64)
    # the hot rank takes between C and 2C rows, the rest spread evenly below C
    hot_rows = int(rng.integers(C + 1, 2 * C))
    share = np.full(L, hot_rows // L)
    share[: hot_rows % L] += 1
    cnt[hot * L:(hot + 1) * L] = share
    rest = T * K - hot_rows
    others = [h for h in range(R) if h != hot]
    per = np.full(len(others) * L, rest // (len(others) * L))
    per[: rest % (len(others) * L)] += 1
    for i, h in enumerate(others):
        cnt[h * L:(h + 1) * L] = per[i * L:(i + 1) * L]
    assert cnt.sum() == T * K and cnt.max() <= T
    assert all(cnt[h * L:(h + 1) * L].sum() <= C for h in others)
    ids = pc.ids_from_counts(cnt, R, S, K)
    cfg = _cfg(R, L, S, K, B, C_max=2 * C)
    a = oracle_lib.plan(cfg, ids)
    b = _compare(oracle_lib, cfg, ids)
    for k in ("dest", "alloc", "slot_expert", "fb_cnt"):
        assert np.array_equal(a[k], b[k]), k


@pytest.mark.parametrize("seed", range(8))
def test_slots_never_bind_with_b_equal_e_over_r(oracle_lib, seed):
    # the passage's reason for B = E/R: a receiver holds pieces of at most L
    # experts, so L slots give the same plan as unlimited slots
    rng = np.random.default_rng(100 + seed)
    R, L, S, K = 8, 4, 64, 4
    cnt = pc.random_counts(rng, R * L, R * S, K, skew=0.7 + 0.5 * seed)
    ids = pc.ids_from_counts(cnt, R, S, K)
    Cm = R * S * K
    pl = _compare(oracle_lib, _cfg(R, L, S, K, L, C_max=Cm), ids)
    wide = _compare(oracle_lib, _cfg(R, L, S, K, R * L, C_max=Cm), ids)
    assert np.array_equal(pl["dest"], wide["dest"])
    assert np.array_equal(pl["alloc"], wide["alloc"])
    assert pl["slots_used"].max() <= L


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("B", [1, 2, 4])
def test_random_histograms(oracle_lib, seed, B):
    rng = np.random.default_rng(seed)
    R, L, S, K = 8, 4, 64, 4
    cnt = pc.random_counts(rng, R * L, R * S, K, skew=1.0 + seed)
    ids = pc.ids_from_counts(cnt, R, S, K)
    _compare(oracle_lib, _cfg(R, L, S, K, B, C_max=R * S * K), ids)


def test_workload_routing(oracle_lib):
    # the tiny and mid workloads' routings at maxvio 2
    for name in ("tiny", "mid"):
        w = inputs.WORKLOADS[name]
        if w.T * w.K > 1 << 18:
            continue
        r = inputs.routing(w.R, w.L, w.S, w.K, 0, maxvio=2.0)
        cfg = dict(w.cfg(), C_max=2 * w.C)
        _compare(oracle_lib, cfg, r.topk_idx)
