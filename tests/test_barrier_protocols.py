"""Barrier protocols of the three tensor-core kernels, model-checked on the CPU.

Each kernel role (TMA producer, MMA issuer, softmax warpgroup) is restated as
the sequence of mbarrier operations it performs -- waits on a phase parity,
thread arrivals, and asynchronous arrivals (a TMA copy completing, or
tcgen05.commit once the thread's MMAs are done) -- and random interleavings
are explored under mbarrier semantics: a barrier completes a phase when its
pending count reaches zero, and a wait for parity P succeeds while the
current phase's parity differs from P (so a barrier that completed two phases
before a waiter looked hides the one it waits for).  A schedule in which
every unfinished role waits is a deadlock.  The sequences mirror
csrc/fwd_kernel.cuh and csrc/bwd_kernels.cuh; a change to a kernel's barrier
use is a change here too.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.phase = 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier's count"
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def parity_done(self, parity):
        return (self.phase & 1) != parity


def explore(bars, roles, seed, max_steps=200000):
    """Run one random interleaving; return None, or the blocked ops on deadlock."""
    rng = random.Random(seed)
    B = {n: Bar(c) for n, c in bars.items()}
    cur = {}
    for n, g in roles.items():
        cur[n] = next(g, None)
    pending = []  # asynchronous arrivals not yet landed
    for _ in range(max_steps):
        ready = []
        for n, op in cur.items():
            if op is None:
                continue
            if op[0] == "wait" and not B[op[1]].parity_done(op[2]):
                continue
            if op[0] == "phase_ge" and B[op[1]].phase < op[2]:
                continue
            ready.append(n)
        if pending and (not ready or rng.random() < 0.4):
            B[pending.pop(rng.randrange(len(pending)))].arrive()
            continue
        if not ready:
            if all(op is None for op in cur.values()):
                return None
            return {n: op for n, op in cur.items() if op is not None}
        n = rng.choice(ready)
        op = cur[n]
        nxt = None
        if op[0] == "arrive":
            B[op[1]].arrive()
        elif op[0] == "async":
            pending.append(op[1])
        elif op[0] == "sync":  # named barrier: arrive, then wait for the phase to turn
            target = B[op[1]].phase + 1
            B[op[1]].arrive()
            nxt = ("phase_ge", op[1], target)
        cur[n] = nxt if nxt is not None else next(roles[n], None)
    raise AssertionError("schedule did not finish")


# --------------------------------------------------------------- forward
def fwd_protocol(items, SK, SV, NS=3, bias_ring=False, rng=None):
    bars = {"q_full": 1, "q_empty": 1, "acc_done": 1, "xchg": 2}
    for s in range(SK):
        bars[f"k_full{s}"] = 1
        bars[f"k_empty{s}"] = 1
    for s in range(SV):
        bars[f"v_full{s}"] = 1
        bars[f"v_empty{s}"] = 1
    for x in range(NS):
        bars[f"s_full{x}"] = 1
        bars[f"p_full{x}"] = 2
        bars[f"pv_done{x}"] = 1
    for x in range(2):
        bars[f"b_full{x}"] = 1
        bars[f"b_empty{x}"] = 2
    grow = rng or random.Random(0)

    def k_producer():
        c = 0
        for u, nt in enumerate(items):
            if u > 0:
                yield ("wait", "q_empty", (u - 1) & 1)
            yield ("async", "q_full")
            for _ in range(nt):
                yield ("wait", f"k_empty{c % SK}", ((c // SK) & 1) ^ 1)
                yield ("async", f"k_full{c % SK}")
                if bias_ring:
                    yield ("wait", f"b_empty{c & 1}", ((c >> 1) & 1) ^ 1)
                    yield ("async", f"b_full{c & 1}")
                c += 1

    def v_producer():
        for c in range(sum(items)):
            yield ("wait", f"v_empty{c % SV}", ((c // SV) & 1) ^ 1)
            yield ("async", f"v_full{c % SV}")

    def s_issuer():
        c = 0
        for u, nt in enumerate(items):
            yield ("wait", "q_full", u & 1)
            for _ in range(nt):
                yield ("wait", f"k_full{c % SK}", (c // SK) & 1)
                if c >= NS:
                    yield ("wait", f"pv_done{c % NS}", ((c // NS) - 1) & 1)
                yield ("async", f"s_full{c % NS}")
                yield ("async", f"k_empty{c % SK}")
                c += 1
            yield ("async", "q_empty")

    def pv_issuer():
        c = 0
        for nt in items:
            for _ in range(nt):
                yield ("wait", f"v_full{c % SV}", (c // SV) & 1)
                yield ("wait", f"p_full{c % NS}", (c // NS) & 1)
                yield ("async", f"pv_done{c % NS}")
                yield ("async", f"v_empty{c % SV}")
                c += 1
            yield ("async", "acc_done")

    def warpgroup():
        c = 0
        for u, nt in enumerate(items):
            for it in range(nt):
                yield ("wait", f"s_full{c % NS}", (c // NS) & 1)
                if bias_ring:
                    yield ("wait", f"b_full{c & 1}", (c >> 1) & 1)
                    yield ("arrive", f"b_empty{c & 1}")
                yield ("sync", "xchg")  # row-max exchange
                if it > 0 and grow.random() < 0.3:  # O rescale after P V of the last tile
                    yield ("wait", f"pv_done{(c - 1) % NS}", ((c - 1) // NS) & 1)
                yield ("arrive", f"p_full{c % NS}")
                c += 1
            yield ("sync", "xchg")  # row-sum exchange
            yield ("wait", "acc_done", u & 1)

    roles = {"kprod": k_producer(), "vprod": v_producer(), "s": s_issuer(), "pv": pv_issuer(),
             "wg0": warpgroup(), "wg1": warpgroup()}
    return bars, roles


# ------------------------------------------------------------------- dQ
def dq_protocol(items, SK, SV, bias_ring=False, ds_double=True, three_issuers=True):
    """three_issuers: dP and dQ MMAs issued by threads of their own (the
    kernel); else one thread issues dP(c + 1) and then dQ(c)."""
    bars = {"q_full": 1, "q_empty": 1, "o_full": 1, "o_empty": 1, "dp_full": 1, "dp_used": 2,
            "ds_full": 2, "ds_full0": 2, "ds_full1": 2, "acc_done": 1}
    for s in range(SK):
        bars[f"k_full{s}"] = 1
        bars[f"k_empty{s}"] = 2
    for s in range(SV):
        bars[f"v_full{s}"] = 1
        bars[f"v_empty{s}"] = 1
    for x in range(2):
        bars[f"s_full{x}"] = 1
        bars[f"dq_done{x}"] = 1
        bars[f"b_full{x}"] = 1
        bars[f"b_empty{x}"] = 2

    def ds(c):
        return (f"ds_full{c & 1}", (c >> 1) & 1) if ds_double else ("ds_full", c & 1)

    def producer():
        c = 0
        for u, nt in enumerate(items):
            if u > 0:
                yield ("wait", "q_empty", (u - 1) & 1)
            yield ("async", "q_full")
            if u > 0:
                yield ("wait", "o_empty", (u - 1) & 1)
            yield ("async", "o_full")
            for _ in range(nt):
                if bias_ring:  # the bias block goes ahead of K
                    yield ("wait", f"b_empty{c & 1}", ((c >> 1) & 1) ^ 1)
                    yield ("async", f"b_full{c & 1}")
                yield ("wait", f"k_empty{c % SK}", ((c // SK) & 1) ^ 1)
                yield ("async", f"k_full{c % SK}")
                yield ("wait", f"v_empty{c % SV}", ((c // SV) & 1) ^ 1)
                yield ("async", f"v_full{c % SV}")
                c += 1

    def s_issuer():
        c = 0
        for u, nt in enumerate(items):
            yield ("wait", "q_full", u & 1)
            for _ in range(nt):
                yield ("wait", f"k_full{c % SK}", (c // SK) & 1)
                if c >= 2:
                    yield ("wait", f"dq_done{c & 1}", ((c >> 1) - 1) & 1)
                yield ("async", f"s_full{c & 1}")
                yield ("async", f"k_empty{c % SK}")
                c += 1
            yield ("async", "q_empty")

    def dq_issuer():
        c = 0

        def dp(cc):
            yield ("wait", f"v_full{cc % SV}", (cc // SV) & 1)
            if cc > 0:
                yield ("wait", "dp_used", (cc - 1) & 1)
            yield ("async", "dp_full")
            yield ("async", f"v_empty{cc % SV}")

        for u, nt in enumerate(items):
            yield ("wait", "o_full", u & 1)
            yield from dp(c)
            for it in range(nt):
                if it + 1 < nt:
                    yield from dp(c + 1)
                yield ("wait", f"k_full{c % SK}", (c // SK) & 1)
                yield ("wait",) + ds(c)
                yield ("async", f"dq_done{c & 1}")
                yield ("async", f"k_empty{c % SK}")
                c += 1
            yield ("async", "o_empty")
            yield ("async", "acc_done")

    def dp_issuer():
        c = 0
        for u, nt in enumerate(items):
            yield ("wait", "o_full", u & 1)
            for _ in range(nt):
                yield ("wait", f"v_full{c % SV}", (c // SV) & 1)
                if c > 0:
                    yield ("wait", "dp_used", (c - 1) & 1)
                yield ("async", "dp_full")
                yield ("async", f"v_empty{c % SV}")
                c += 1
            yield ("async", "o_empty")

    def dq_only_issuer():
        c = 0
        for u, nt in enumerate(items):
            for _ in range(nt):
                yield ("wait", f"k_full{c % SK}", (c // SK) & 1)
                yield ("wait",) + ds(c)
                yield ("async", f"dq_done{c & 1}")
                yield ("async", f"k_empty{c % SK}")
                c += 1
            yield ("async", "acc_done")

    def warpgroup():
        c = 0
        for u, nt in enumerate(items):
            for _ in range(nt):
                yield ("wait", f"s_full{c & 1}", (c >> 1) & 1)
                if bias_ring:
                    yield ("wait", f"b_full{c & 1}", (c >> 1) & 1)
                    yield ("arrive", f"b_empty{c & 1}")
                yield ("wait", "dp_full", c & 1)
                yield ("arrive", "dp_used")
                yield ("arrive", ds(c)[0])
                c += 1
            yield ("wait", "acc_done", u & 1)

    if three_issuers:
        roles = {"prod": producer(), "s": s_issuer(), "dp": dp_issuer(), "dq": dq_only_issuer(),
                 "wg0": warpgroup(), "wg1": warpgroup()}
    else:
        roles = {"prod": producer(), "s": s_issuer(), "dq": dq_issuer(), "wg0": warpgroup(),
                 "wg1": warpgroup()}
    return bars, roles


# ---------------------------------------------------------------- dK / dV
def dkdv_protocol(total, SQ, SO, s_double=False, p_double=True, bias_ring=False):
    """s_double: S^T double-buffered (d = 64): S^T(i + 1) is issued before
    the wait for P^T(i); s_full, p_full and s_free then go by block parity
    (p_double=False models one P^T-ready barrier instead).  bias_ring: the
    dense bias staged by TMA in two slots, issued ahead of each block's Q,
    released by the warpgroups once P^T is formed."""
    bars = {"kv_full": 1, "dp_full": 1, "ds_full": 2, "dp_free": 1, "acc_done": 2}
    if bias_ring:
        for x in range(2):
            bars[f"b_full{x}"] = 1
            bars[f"b_empty{x}"] = 2
    nb = 2 if s_double else 1
    for x in range(nb):
        bars[f"s_full{x}"] = 1
        bars[f"p_full{x}"] = 2
        bars[f"s_free{x}"] = 1
    for s in range(SQ):
        bars[f"q_full{s}"] = 1
        bars[f"q_empty{s}"] = 2
    for s in range(SO):
        bars[f"o_full{s}"] = 1
        bars[f"o_empty{s}"] = 2
    for x in range(2):
        bars[f"vec_full{x}"] = 1
        bars[f"vec_empty{x}"] = 2

    def par(name, it):
        # (barrier, parity) of block it's phase
        if s_double and (p_double or name != "p_full"):
            return (f"{name}{it & 1}", (it >> 1) & 1)
        return (f"{name}0", it & 1)

    def producer():
        yield ("async", "kv_full")
        for it in range(total):
            if bias_ring:
                yield ("wait", f"b_empty{it & 1}", ((it >> 1) & 1) ^ 1)
                yield ("async", f"b_full{it & 1}")
            yield ("wait", f"q_empty{it % SQ}", ((it // SQ) & 1) ^ 1)
            yield ("async", f"q_full{it % SQ}")
            yield ("wait", f"o_empty{it % SO}", ((it // SO) & 1) ^ 1)
            yield ("async", f"o_full{it % SO}")
            yield ("wait", f"vec_empty{it & 1}", ((it >> 1) & 1) ^ 1)
            yield ("arrive", f"vec_full{it & 1}")

    def issue_s(it):
        yield ("wait", f"q_full{it % SQ}", (it // SQ) & 1)
        if it >= nb:
            yield ("wait",) + par("s_free", it - nb)
        yield ("async", par("s_full", it)[0])
        yield ("async", f"q_empty{it % SQ}")

    def chain_s():
        yield ("wait", "kv_full", 0)
        if s_double and total > 0:
            yield from issue_s(0)
        for it in range(total):
            if s_double:
                if it + 1 < total:
                    yield from issue_s(it + 1)
            else:
                yield from issue_s(it)
            yield ("wait", f"o_full{it % SO}", (it // SO) & 1)
            yield ("wait",) + par("p_full", it)
            yield ("async", par("s_free", it)[0])
            yield ("async", f"o_empty{it % SO}")
        yield ("async", "acc_done")

    def chain_dp():
        yield ("wait", "kv_full", 0)
        for it in range(total):
            yield ("wait", f"o_full{it % SO}", (it // SO) & 1)
            if it > 0:
                yield ("wait", "dp_free", (it - 1) & 1)
            yield ("async", "dp_full")
            yield ("async", f"o_empty{it % SO}")
            yield ("wait", f"q_full{it % SQ}", (it // SQ) & 1)
            yield ("wait", "ds_full", it & 1)
            yield ("async", "dp_free")
            yield ("async", f"q_empty{it % SQ}")
        yield ("async", "acc_done")

    def warpgroup():
        for it in range(total):
            yield ("wait", f"vec_full{it & 1}", (it >> 1) & 1)
            yield ("wait",) + par("s_full", it)
            if bias_ring:
                yield ("wait", f"b_full{it & 1}", (it >> 1) & 1)
                yield ("arrive", f"b_empty{it & 1}")
            yield ("arrive", par("p_full", it)[0])
            yield ("wait", "dp_full", it & 1)
            yield ("arrive", "ds_full")
            yield ("arrive", f"vec_empty{it & 1}")
        yield ("wait", "acc_done", 0)

    roles = {"prod": producer(), "s": chain_s(), "dp": chain_dp(), "wg0": warpgroup(),
             "wg1": warpgroup()}
    return bars, roles


ITEM_SETS = [[1], [3], [8, 8, 8, 8], [2, 1, 5, 3], [1, 1, 1, 1, 1]]
SEEDS = range(60)


@pytest.mark.parametrize("SK,SV,bias_ring", [(3, 2, False), (4, 4, False), (2, 2, True)])
def test_forward_protocol_has_no_deadlock(SK, SV, bias_ring):
    for items in ITEM_SETS:
        for seed in SEEDS:
            bars, roles = fwd_protocol(items, SK, SV, bias_ring=bias_ring, rng=random.Random(seed))
            blocked = explore(bars, roles, seed)
            assert blocked is None, (items, seed, blocked)


@pytest.mark.parametrize("SK,SV,bias_ring", [(3, 2, False), (4, 3, False), (2, 2, True)])
def test_dq_protocol_has_no_deadlock(SK, SV, bias_ring):
    for items in ITEM_SETS:
        for seed in SEEDS:
            for three in (True, False):
                bars, roles = dq_protocol(items, SK, SV, bias_ring=bias_ring, three_issuers=three)
                blocked = explore(bars, roles, seed)
                assert blocked is None, (items, seed, three, blocked)


def test_dq_protocol_with_one_ds_barrier_can_lose_a_wakeup():
    # The model catches the race the double-buffered dS barrier removes.
    found = False
    for seed in range(200):
        bars, roles = dq_protocol([8, 8, 8], 4, 3, ds_double=False, three_issuers=False)
        if explore(bars, roles, seed) is not None:
            found = True
            break
    assert found


def test_dkdv_double_s_with_one_p_barrier_can_lose_a_wakeup():
    # with S^T(i + 1) issued before the wait for P^T(i), the warpgroups can
    # publish P^T(i + 1) before the issuer looks for P^T(i): one barrier would
    # then have completed two phases
    found = False
    for seed in range(200):
        bars, roles = dkdv_protocol(40, 4, 4, s_double=True, p_double=False)
        if explore(bars, roles, seed) is not None:
            found = True
            break
    assert found


@pytest.mark.parametrize("SQ,SO,s_double,bias_ring",
                         [(3, 2, False, False), (2, 2, False, False), (4, 4, False, False),
                          (4, 4, True, False), (2, 2, True, False), (2, 2, True, True)])
def test_dkdv_protocol_has_no_deadlock(SQ, SO, s_double, bias_ring):
    for total in (1, 2, 3, 7, 40):
        for seed in SEEDS:
            bars, roles = dkdv_protocol(total, SQ, SO, s_double, bias_ring=bias_ring)
            blocked = explore(bars, roles, seed)
            assert blocked is None, (total, seed, blocked)
