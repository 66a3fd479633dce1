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


# ------------------------------------------------- fused backward (dK, dV, dQ)
def bwd_items(groups, ntk, G, causal):
    """Work items of the fused backward in ticket order: (group, key tile n,
    blocks), each block (query tile m, head) with its dQ turn index, first
    and last flags.  Within a group the key tiles come from the last to the
    first, and the dQ contributions to a query tile are added in that same
    (descending) order; an item walks its query tiles from the first of its
    band up, heads inner."""
    ntq = ntk
    items = []
    for grp in range(groups):
        for n in range(ntk - 1, -1, -1):
            mlo = n if causal else 0
            blocks = []
            for m in range(mlo, ntq):
                contrib = list(range(m, -1, -1)) if causal else list(range(ntk - 1, -1, -1))
                for h in range(G):
                    idx = contrib.index(n)
                    blocks.append(((grp, h, m), idx, idx == 0, idx == len(contrib) - 1))
            items.append(blocks)
    return items


def bwd_protocol(items, ctas, SQ, SO, dq_shared, reducers=2):
    """Barriers and roles of every CTA of the fused backward.  Besides
    mbarrier ops, roles yield ("ticket",) (the atomic work-item counter),
    ("publish", slot, t) / ("read", slot) (the item ring's slots), and
    ("turn_wait", key, v) / ("turn_set", key, v) (the dQ turn counters in
    global memory, one per (tile, reducer quarter))."""
    bars = {}
    roles = {}
    for c in range(ctas):
        def b(name, count):
            bars[f"{c}:{name}"] = count
        b("kv_full", 1)
        b("kv_empty", 2)
        for x in range(SQ):
            b(f"q_full{x}", 1)
            b(f"q_empty{x}", 2)
        for x in range(SO):
            b(f"o_full{x}", 1)
            b(f"o_empty{x}", 2)
        for x in range(2):
            b(f"vec_full{x}", 1)
            b(f"vec_empty{x}", 2)
            b(f"dq_full{x}", 1)
            b(f"dq_free{x}", reducers)
            b(f"item_full{x}", 1)
            b(f"item_empty{x}", 2 + 2 + reducers)
        for n_, k_ in (("s_full", 1), ("p_full", 2), ("s_free", 1), ("dp_full", 1),
                       ("ds_full", 2), ("ds_free", 1), ("acc_done", 2), ("acc_free", 2)):
            b(n_, k_)

        def B(name, c=c):
            return f"{c}:{name}"

        def consume(k, c=c, B=B):
            yield ("wait", B(f"item_full{k & 1}"), (k >> 1) & 1)
            t = yield ("read", (c, k & 1))
            yield ("arrive", B(f"item_empty{k & 1}"))
            return t

        def producer(c=c, B=B, consume=consume):
            k = u = i = 0
            while True:
                t = yield ("ticket",)
                yield ("wait", B(f"item_empty{k & 1}"), ((k >> 1) & 1) ^ 1)
                yield ("publish", (c, k & 1), t)
                yield ("arrive", B(f"item_full{k & 1}"))
                k += 1
                if t is None:
                    return
                nb = len(items[t])
                if nb == 0:
                    continue
                if u > 0:
                    yield ("wait", B("kv_empty"), (u - 1) & 1)
                yield ("async", B("kv_full"))
                for _ in range(nb):
                    yield ("wait", B(f"q_empty{i % SQ}"), ((i // SQ) & 1) ^ 1)
                    yield ("async", B(f"q_full{i % SQ}"))
                    yield ("wait", B(f"o_empty{i % SO}"), ((i // SO) & 1) ^ 1)
                    yield ("async", B(f"o_full{i % SO}"))
                    yield ("wait", B(f"vec_empty{i & 1}"), ((i >> 1) & 1) ^ 1)
                    yield ("arrive", B(f"vec_full{i & 1}"))
                    i += 1
                u += 1

        def issuer_s(c=c, B=B, consume=consume):
            k = u = i = 0
            while True:
                t = yield from consume(k)
                k += 1
                if t is None:
                    return
                nb = len(items[t])
                if nb == 0:
                    continue
                yield ("wait", B("kv_full"), u & 1)
                for blk in range(nb):
                    yield ("wait", B(f"q_full{i % SQ}"), (i // SQ) & 1)
                    if i > 0:
                        yield ("wait", B("s_free"), (i - 1) & 1)
                    yield ("async", B("s_full"))
                    yield ("async", B(f"q_empty{i % SQ}"))
                    yield ("wait", B(f"o_full{i % SO}"), (i // SO) & 1)
                    yield ("wait", B("p_full"), i & 1)
                    if blk == 0 and u > 0:
                        yield ("wait", B("acc_free"), (u - 1) & 1)
                    yield ("async", B("s_free"))
                    yield ("async", B(f"o_empty{i % SO}"))
                    i += 1
                yield ("async", B("acc_done"))
                yield ("async", B("kv_empty"))
                u += 1

        def issuer_dp(c=c, B=B, consume=consume):
            k = u = i = 0
            while True:
                t = yield from consume(k)
                k += 1
                if t is None:
                    return
                nb = len(items[t])
                if nb == 0:
                    continue
                yield ("wait", B("kv_full"), u & 1)
                for blk in range(nb):
                    yield ("wait", B(f"o_full{i % SO}"), (i // SO) & 1)
                    if dq_shared and i > 0:
                        yield ("wait", B(f"dq_free{(i - 1) & 1}"), ((i - 1) >> 1) & 1)
                    yield ("async", B("dp_full"))
                    yield ("async", B(f"o_empty{i % SO}"))
                    yield ("wait", B("ds_full"), i & 1)
                    yield ("wait", B(f"q_full{i % SQ}"), (i // SQ) & 1)
                    if not dq_shared and i >= 2:
                        yield ("wait", B(f"dq_free{i & 1}"), ((i >> 1) - 1) & 1)
                    yield ("async", B(f"dq_full{i & 1}"))
                    if blk == 0 and u > 0:
                        yield ("wait", B("acc_free"), (u - 1) & 1)
                    yield ("async", B("ds_free"))
                    yield ("async", B(f"q_empty{i % SQ}"))
                    i += 1
                yield ("async", B("acc_done"))
                yield ("async", B("kv_empty"))
                u += 1

        def compute(c=c, B=B, consume=consume):
            k = u = i = 0
            while True:
                t = yield from consume(k)
                k += 1
                if t is None:
                    return
                nb = len(items[t])
                for _ in range(nb):
                    yield ("wait", B(f"vec_full{i & 1}"), (i >> 1) & 1)
                    yield ("wait", B("s_full"), i & 1)
                    yield ("arrive", B("p_full"))
                    yield ("wait", B("dp_full"), i & 1)
                    if i > 0:
                        yield ("wait", B("ds_free"), (i - 1) & 1)
                    yield ("arrive", B("ds_full"))
                    yield ("arrive", B(f"vec_empty{i & 1}"))
                    i += 1
                if nb > 0:
                    yield ("wait", B("acc_done"), u & 1)
                    yield ("arrive", B("acc_free"))
                    u += 1

        def reducer(r, c=c, B=B, consume=consume):
            # the next block's turn is taken (and its sums fetched) before
            # this block's turn is passed on
            k = i = 0
            while True:
                t = yield from consume(k)
                k += 1
                if t is None:
                    return
                blocks = items[t]
                if blocks and not blocks[0][2]:
                    yield ("turn_wait", (blocks[0][0], r), blocks[0][1])
                for j, (tile, idx, first, last) in enumerate(blocks):
                    yield ("wait", B(f"dq_full{i & 1}"), (i >> 1) & 1)
                    yield ("arrive", B(f"dq_free{i & 1}"))
                    if j + 1 < len(blocks) and not blocks[j + 1][2]:
                        yield ("turn_wait", (blocks[j + 1][0], r), blocks[j + 1][1])
                    if not last:
                        yield ("turn_set", (tile, r), idx + 1)
                    i += 1

        roles[f"{c}:prod"] = producer()
        roles[f"{c}:s"] = issuer_s()
        roles[f"{c}:dp"] = issuer_dp()
        roles[f"{c}:wg0"] = compute()
        roles[f"{c}:wg1"] = compute()
        for r in range(reducers):
            roles[f"{c}:red{r}"] = reducer(r)
    return bars, roles


def explore_bwd(bars, roles, n_items, seed, max_steps=400000):
    """explore() plus the work-item counter, the item slots and the turn
    counters; returns None, or the blocked ops on deadlock."""
    rng = random.Random(seed)
    Bs = {n: Bar(c) for n, c in bars.items()}
    slots, turns = {}, {}
    ticket = [0]
    cur = {n: next(g) for n, g in roles.items()}
    pending = []

    def ready(op):
        if op is None:
            return False
        if op[0] == "wait":
            return Bs[op[1]].parity_done(op[2])
        if op[0] == "turn_wait":
            return turns.get(op[1], 0) == op[2]
        return True

    for _ in range(max_steps):
        rd = [n for n, op in cur.items() if ready(op)]
        if pending and (not rd or rng.random() < 0.4):
            Bs[pending.pop(rng.randrange(len(pending)))].arrive()
            continue
        if not rd:
            if all(op is None for op in cur.values()):
                return None
            return {n: op for n, op in cur.items() if op is not None}
        n = rng.choice(rd)
        op = cur[n]
        send = None
        if op[0] == "arrive":
            Bs[op[1]].arrive()
        elif op[0] == "async":
            pending.append(op[1])
        elif op[0] == "ticket":
            send = ticket[0] if ticket[0] < n_items else None
            ticket[0] += 1
        elif op[0] == "publish":
            slots[op[1]] = op[2]
        elif op[0] == "read":
            send = slots[op[1]]
        elif op[0] == "turn_set":
            assert turns.get(op[1], 0) == op[2] - 1, "turn passed out of order"
            turns[op[1]] = op[2]
        try:
            cur[n] = roles[n].send(send) if send is not None or op[0] in ("ticket", "read") \
                else next(roles[n])
        except StopIteration:
            cur[n] = None
    raise AssertionError("schedule did not finish")


ITEM_SETS = [[1], [3], [8, 8, 8, 8], [2, 1, 5, 3], [1, 1, 1, 1, 1]]
SEEDS = range(60)


@pytest.mark.parametrize("SK,SV,bias_ring", [(3, 2, False), (4, 4, False), (2, 2, True)])
def test_forward_protocol_has_no_deadlock(SK, SV, bias_ring):
    for items in ITEM_SETS:
        for seed in SEEDS:
            bars, roles = fwd_protocol(items, SK, SV, bias_ring=bias_ring, rng=random.Random(seed))
            blocked = explore(bars, roles, seed)
            assert blocked is None, (items, seed, blocked)


@pytest.mark.parametrize("SQ,SO,dq_shared", [(2, 2, True), (2, 1, True), (4, 4, False)])
@pytest.mark.parametrize("causal", [True, False])
def test_fused_backward_protocol_has_no_deadlock(SQ, SO, dq_shared, causal):
    # Several CTAs take work items from the ticket counter in random order and
    # wait on each other's dQ turns; every interleaving must finish.
    for groups, ntk, G, ctas in ((1, 1, 1, 1), (2, 3, 2, 2), (1, 4, 1, 3), (3, 2, 2, 2)):
        items = bwd_items(groups, ntk, G, causal)
        for seed in range(25):
            bars, roles = bwd_protocol(items, ctas, SQ, SO, dq_shared)
            blocked = explore_bwd(bars, roles, len(items), seed)
            assert blocked is None, (groups, ntk, G, ctas, seed, blocked)


def test_fused_backward_turns_follow_key_tile_order():
    # The dQ contributions to every (query tile, quarter) come in the order
    # the key tiles are handed out: turn indices consecutive from 0.
    items = bwd_items(2, 4, 2, True)
    seen = {}
    for blocks in items:
        for tile, idx, first, last in blocks:
            seen.setdefault(tile, []).append((idx, first, last))
    for tile, lst in seen.items():
        idxs = sorted(x[0] for x in lst)
        assert idxs == list(range(len(lst)))
        assert [x[1] for x in sorted(lst)][0] and [x[2] for x in sorted(lst)][-1]


def test_fused_backward_model_catches_a_wrong_turn_order():
    # Planting the contribution order opposite to the ticket order in the
    # model makes the waits cycle: the explorer reports the deadlock.
    items = bwd_items(1, 3, 1, True)
    rev = []
    for blocks in items:
        nb = []
        for tile, idx, first, last in blocks:
            n_contrib = tile[2] + 1
            j = n_contrib - 1 - idx
            nb.append((tile, j, j == 0, j == n_contrib - 1))
        rev.append(nb)
    found = False
    for seed in range(40):
        bars, roles = bwd_protocol(rev, 1, 2, 2, True)
        if explore_bwd(bars, roles, len(rev), seed) is not None:
            found = True
            break
    assert found
