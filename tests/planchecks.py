"""Invariant checks on a plan, written from the method's statement with numpy
only (no oracle code, no library code).

A plan is a dict with the tables named in the library header: cnt, keep,
spill, home_off, fb_cnt, fb_off, load, deficit, fill, slots_used,
slot_expert, slot_cnt, slot_off, slot_first_j, rep_ptr, rep_recv, rep_slot,
rep_first_j, rep_cnt, seg_off, seg_len, alloc [N, R], dest [R, S, K] and the
counts status, fallback_rows, n_replicas, migrated_rows.
"""
import numpy as np


def row_expert_map(cfg, pl):
    """Expert of every row of the [R, C_max] receive buffer (-1 = no row)."""
    R, L, B, Cm = cfg["R"], cfg["L"], cfg["B"], cfg["C_max"]
    SEG = 2 * L + B
    m = np.full(R * Cm, -1, np.int64)
    so = np.asarray(pl["seg_off"]).reshape(R, SEG)
    sl = np.asarray(pl["seg_len"]).reshape(R, SEG)
    se = np.asarray(pl["slot_expert"]).reshape(R, B) if B > 0 else np.zeros((R, 0), np.int64)
    for r in range(R):
        for s in range(SEG):
            if sl[r, s] == 0:
                continue
            if s < L:
                e = r * L + s
            elif s < L + B:
                e = se[r, s - L]
            else:
                e = r * L + (s - L - B)
            lo = r * Cm + so[r, s]
            assert np.all(m[lo:lo + sl[r, s]] == -1), "overlapping segments"
            m[lo:lo + sl[r, s]] = e
    # remote pieces (no slot) are described by the piece tables only
    n = int(pl.get("n_replicas", 0))
    if n and "rep_off" in pl:
        for q in range(n):
            if int(pl["rep_slot"][q]) < 0:
                lo = int(pl["rep_recv"][q]) * Cm + int(pl["rep_off"][q])
                cnt = int(pl["rep_cnt"][q])
                assert np.all(m[lo:lo + cnt] == -1), "overlapping segments"
                m[lo:lo + cnt] = int(pl["rep_expert"][q])
    return m


def check_plan(cfg, ids, pl):
    """Assert every invariant the method states or implies.  Returns a dict of
    derived facts (per-rank rows, spilled chunk count, receivers)."""
    R, L, S, K, B, C, Cm = (cfg[n] for n in ("R", "L", "S", "K", "B", "C", "C_max"))
    N = R * L
    ids = np.asarray(ids).reshape(-1).astype(np.int64)
    cnt = np.bincount(ids, minlength=N) if ids.size else np.zeros(N, np.int64)
    assert np.array_equal(np.asarray(pl["cnt"]), cnt), "histogram"
    load = cnt.reshape(R, L).sum(1)
    assert np.array_equal(np.asarray(pl["load"]), load)
    alloc = np.asarray(pl["alloc"]).reshape(N, R)
    # every routed copy is placed exactly once
    assert np.array_equal(alloc.sum(1), cnt), "sum_r alloc[e][r] == cnt[e]"
    rows = alloc.sum(0)
    fb = int(pl["fallback_rows"])
    assert fb == int(np.asarray(pl["fb_cnt"]).sum())
    if fb == 0:
        # the hard invariant: every rank holds exactly S*K rows
        assert np.all(rows == C), "rows per rank == S*K"
    assert np.all(rows <= Cm)
    # replica slots per rank never exceed B
    su = np.asarray(pl["slots_used"])
    assert np.all(su <= B) and np.all(su >= 0)
    if "rep_slot" in pl:
        nrep = int(pl["n_replicas"])
        slotted = np.asarray(pl["rep_slot"])[:nrep] >= 0
        assert np.array_equal(np.bincount(np.asarray(pl["rep_recv"])[:nrep][slotted], minlength=R), su)
    if B > 0:
        assert np.array_equal((np.asarray(pl["slot_expert"]).reshape(R, B) >= 0).sum(1), su)
    # closed form: migrated rows = total home overflow - fallback
    over = np.maximum(load - C, 0).sum()
    assert int(pl["migrated_rows"]) == int(over) - fb
    # at most one slot per (expert, receiver) pair; a rank that spills never receives
    nrep = int(pl["n_replicas"])
    rr = np.asarray(pl["rep_recv"])[:nrep]
    rp = np.asarray(pl["rep_ptr"])
    for e in range(N):
        recv = rr[rp[e]:rp[e + 1]]
        assert len(set(recv.tolist())) == len(recv)
        assert np.all(np.diff(recv) > 0), "receivers ascend within an expert"
        assert not np.any(load[recv] > C)
    spilled_chunks = int((np.maximum(cnt - np.asarray(pl["keep"]), 0) > 0).sum())
    receivers = int((load < C).sum())
    if fb == 0 and spilled_chunks > 0:
        assert nrep <= spilled_chunks + receivers - 1
    # destinations: injective, inside the expert's own segments, stable in g
    dest = np.asarray(pl["dest"]).reshape(-1).astype(np.int64)
    assert dest.size == ids.size
    if dest.size:
        assert dest.min() >= 0 and dest.max() < R * Cm
        assert np.unique(dest).size == dest.size, "dest injective"
        rexp = row_expert_map(cfg, pl)
        assert np.array_equal(rexp[dest], ids), "row belongs to the routed expert"
        # rows used == segment rows: total segment length equals the copies
        assert int((rexp >= 0).sum()) == dest.size
        # local and slot segments inside [0, C); fallback segments inside [C, C_max)
        r_of = dest // Cm
        row = dest % Cm
        home = ids // L
        assert np.all(row[r_of != home] < C)
        # stable: copies of an expert numbered in ascending g fill rows in order
        # within each segment (same rank, contiguous rows)
        order = np.lexsort((np.arange(ids.size), ids))
        e_sorted, d_sorted = ids[order], dest[order]
        same = (e_sorted[1:] == e_sorted[:-1]) & (d_sorted[1:] // Cm == d_sorted[:-1] // Cm)
        step = d_sorted[1:] - d_sorted[:-1]
        # consecutive copies on the same rank either continue a segment (+1)
        # or jump forward to a later segment of the same expert (fallback)
        assert np.all(step[same] >= 1)
    return dict(rows=rows, spilled_chunks=spilled_chunks, receivers=receivers)


def ids_from_counts(cnt, R, S, K):
    """A routing with distinct experts per token realising the histogram cnt
    (requires sum(cnt) == R*S*K and cnt[e] <= R*S): the sorted multiset laid
    out column-major over tokens."""
    T = R * S
    cnt = np.asarray(cnt, np.int64)
    assert cnt.sum() == T * K and np.all(cnt <= T)
    flat = np.repeat(np.arange(cnt.size), cnt)
    ids = flat.reshape(K, T).T
    return np.ascontiguousarray(ids.reshape(R, S, K).astype(np.int32))


def random_counts(rng, N, T, K, skew):
    """Random histogram with sum T*K and every entry <= T."""
    total = T * K
    w = rng.pareto(skew, N) + 1e-3 if skew > 0 else np.ones(N)
    c = np.floor(w / w.sum() * total).astype(np.int64)
    c = np.minimum(c, T)
    rem = total - c.sum()
    while rem > 0:
        room = np.nonzero(c < T)[0]
        pick = rng.choice(room, size=min(rem, room.size), replace=False)
        c[pick] += 1
        rem = total - c.sum()
    return c
