"""Pins for two arithmetic shortcuts the plan kernel takes, checked here as
plain-Python models on the CPU (the GPU parity tests check the kernel's
tables against the oracle):

- the receiver walk for all receivers at once: receiver r starts at
  min(D_r, total) (D_r: the deficits of the taking receivers before it) and
  takes min(d_r, total - start); when no receiver's chunk limit is below that
  take, these are exactly the one-after-another walk's starts and takes (and
  chunk ranges), and when some limit is below it the check says so;
- the multiply-high division: floor(n / d) = (n * m) >> 64 with
  m = floor((2^64 - 1) / d) + 1, for 32-bit n and d >= 2.
"""
import bisect
import random


def first_above(a, v):
    """First index m with a[m] > v (a strictly increasing), or len(a)."""
    return bisect.bisect_right(a, v)


def walk_one_by_one(defs, ce, ch, L, B, remote, one_group):
    """The receiver walk as the pages' rule states it, receiver after
    receiver: returns (start, take, first chunk, pieces) per receiver."""
    M = len(ce)
    total = ce[-1] if M else 0
    pos, out = 0, []
    for d in defs:
        if d > 0 and pos < total and (remote or B > 0):
            i0 = first_above(ce, pos)
            i1 = M - 1 if remote else min(i0 + B - 1, M - 1)
            if one_group:
                h = ch[i0] // L
                i1 = min(i1, first_above(ch, (h + 1) * L - 1) - 1)
            take = min(d, ce[i1] - pos)
            il = first_above(ce, pos + take - 1)
            out.append((pos, take, i0, il - i0 + 1))
            pos += take
        else:
            out.append((pos, 0, None, 0))
    return out


def walk_all_at_once(defs, ce, ch, L, B, remote, one_group):
    """The kernel's shortcut: every receiver from prefix sums, then the check.
    Returns (ok, [(start, take, first chunk, pieces)])."""
    M = len(ce)
    total = ce[-1] if M else 0
    a = [max(d, 0) if (remote or B > 0) else 0 for d in defs]
    out, ok, run = [], True, 0
    for r, ar in enumerate(a):
        st = min(run, total)
        run += ar
        tk = min(ar, total - st)
        if tk > 0:
            i0 = first_above(ce, st)
            i1 = M - 1 if remote else min(i0 + B - 1, M - 1)
            if one_group:
                i1 = min(i1, first_above(ch, (ch[i0] // L + 1) * L - 1) - 1)
            if ce[i1] - st < tk:
                ok = False
            out.append((st, tk, i0, first_above(ce, st + tk - 1) - i0 + 1))
        else:
            out.append((st, 0, None, 0))
    return ok, out


def random_case(rng):
    R = rng.randint(1, 10)
    L = rng.randint(1, 6)
    B = rng.randint(0, 4)
    N = R * L
    # spilled experts in ascending order with positive spill; deficits of receivers
    spill = [rng.choice([0, 0, rng.randint(1, 9)]) for _ in range(N)]
    ch = [e for e in range(N) if spill[e] > 0]
    ce, acc = [], 0
    for e in ch:
        acc += spill[e]
        ce.append(acc)
    total = acc
    defs = [rng.choice([0, rng.randint(1, 12)]) for _ in range(R)]
    # the plan's invariant: the deficits add up to the spill
    diff = total - sum(defs)
    if diff > 0:
        defs[rng.randrange(R)] += diff
    elif diff < 0:
        for r in range(R):
            cut = min(defs[r], -diff)
            defs[r] -= cut
            diff += cut
    return defs, ce, ch, L, B


def test_all_at_once_walk_equals_the_walk_when_no_limit_binds():
    rng = random.Random(1)
    seen_ok = seen_limited = 0
    for _ in range(20000):
        defs, ce, ch, L, B = random_case(rng)
        for remote, one_group in ((False, False), (True, False), (False, True)):
            seq = walk_one_by_one(defs, ce, ch, L, B, remote, one_group)
            ok, par = walk_all_at_once(defs, ce, ch, L, B, remote, one_group)
            # the check passes exactly when no receiver's take was cut by a limit
            total = ce[-1] if ce else 0
            a = [d if (remote or B > 0) else 0 for d in defs]
            uncut = all(t == min(ar, max(0, total - p)) for (p, t, _, _), ar in zip(seq, a))
            assert ok == uncut
            if ok:
                seen_ok += 1
                for (ps, ts, cs, ns), (pp, tp, cp, np_) in zip(seq, par):
                    assert ts == tp and ns == np_
                    if ts:
                        assert ps == pp and cs == cp
            else:
                seen_limited += 1
    assert seen_ok > 1000 and seen_limited > 1000


def test_multiply_high_division_is_exact_for_32_bit_operands():
    rng = random.Random(2)

    def q(n, d):
        m = (2 ** 64 - 1) // d + 1
        return (n * m) >> 64

    cases = []
    for _ in range(100000):
        d = rng.choice([rng.randint(2, 64), rng.randint(2, 1 << 20), rng.randint(2, 2 ** 32 - 1)])
        n = rng.choice([rng.randint(0, 2 ** 32 - 1), (rng.randint(0, 2 ** 32 - 1) // d) * d,
                        (rng.randint(0, 2 ** 32 - 1) // d) * d - 1])
        cases.append((max(n, 0), d))
    for d in (2, 3, 7, 8, 127, 4096, 65535, 2 ** 31 - 1, 2 ** 31, 2 ** 32 - 1):
        for n in (0, 1, d - 1, d, d + 1, 2 ** 32 - 1, ((2 ** 32 - 1) // d) * d, ((2 ** 32 - 1) // d) * d - 1):
            if 0 <= n < 2 ** 32:
                cases.append((n, d))
    for n, d in cases:
        assert q(n, d) == n // d, (n, d)
