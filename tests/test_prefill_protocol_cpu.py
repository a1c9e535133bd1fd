"""A model of the persistent prefill kernel's synchronisation (pa_prefill_tc_kernel in
csrc/pa_prefill.cu), run on the CPU.

The kernel's warps meet only through mbarriers: a producer warp (work items, Q rows, K
and V tiles by TMA), one issuing thread (tcgen05 products, which the tensor core runs in
issue order, each committed to a barrier), and the softmax warps of two groups. Here each
of them is a coroutine that takes the same steps on the same barriers (a barrier is a
count of arrivals plus a transaction count, and completes a phase when both reach zero);
copies land and the tensor core runs at random points, and the coroutines are scheduled
in a random order. Every read of a buffer (the Q buffer, a K or V slot, a group's S/P
columns and its O) checks that it sees the version it should, and a run that stops making
progress is a deadlock. The items cover what the kernel sees: items with no rows, groups
without rows, groups with equal tile counts (two q heads of one kv head) and the second
group needing one tile more (256 rows of one head).

A mistake planted in the model (the issuing thread returning a K slot once one group's S
has read it) has to be caught, as a stale read or a run that stops, so that the checks are
known to bite.
"""
import random

import pytest


class Bar:
    """An mbarrier: `count` arrivals and the expected transaction bytes complete a phase."""

    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0

    def _check(self):
        assert self.pending >= 0, "arrival underflow"
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self):
        self.pending -= 1
        self._check()

    def expect_tx_arrive(self, n):
        self.tx += n
        self.pending -= 1
        self._check()

    def complete_tx(self, n):
        self.tx -= n
        self._check()

    def done(self, parity):
        return (self.phase & 1) != parity


def run(seed, NK=3, NV=2, NG=2, NW=4, early_k_release=False, max_steps=400_000):
    rng = random.Random(seed)
    items = []
    for _ in range(rng.randint(1, 12)):
        r = rng.random()
        if r < 0.12:
            items.append((0, 0))                      # no query rows in this item
        elif r < 0.55:
            g = rng.randint(1, 6)
            items.append((g, g))                      # two heads over the same rows
        else:
            g0 = rng.randint(1, 6)
            items.append((g0, 0 if rng.random() < 0.2 else g0 + 1))  # 256 rows of one head
    k_full = [Bar(1) for _ in range(NK)]
    k_empty = [Bar(1) for _ in range(NK)]
    v_full = [Bar(1) for _ in range(NV)]
    v_empty = [Bar(1) for _ in range(NV)]
    q_full, q_free = Bar(1), Bar(1)
    item_full = [Bar(1), Bar(1)]
    item_free = [Bar(1 + NW * NG), Bar(1 + NW * NG)]
    s_full = [Bar(1) for _ in range(NG)]
    p_full = [Bar(NW) for _ in range(NG)]
    pv_done = [Bar(1) for _ in range(NG)]
    o_free = [Bar(NW) for _ in range(NG)]
    slots = [None, None]
    kslot, vslot, qbuf = [None] * NK, [None] * NV, [None]
    S, P, O = [None] * NG, [None] * NG, [None] * NG
    inflight, tc_q, work = [], [], [0]

    def producer():
        kt = vt = nq = it = 0
        while True:
            k = work[0]
            work[0] += 1
            valid = k < len(items)
            gt = items[k] if valid else (0, 0)
            ntiles = max(gt)
            slot = it & 1
            if it >= 2:
                while not item_free[slot].done(((it >> 1) - 1) & 1):
                    yield
            slots[slot] = (valid, k, gt, ntiles)
            item_full[slot].arrive()
            yield
            if not valid:
                return
            if ntiles == 0:
                it += 1
                continue
            if nq > 0:
                while not q_free.done((nq - 1) & 1):
                    yield
            q_full.expect_tx_arrive(1)
            inflight.append((q_full, ("q", k)))
            nq += 1
            ik = iv = 0
            while ik < ntiles or iv < ntiles:
                if ik < ntiles and (kt < NK or k_empty[kt % NK].done(((kt // NK) & 1) ^ 1)):
                    k_full[kt % NK].expect_tx_arrive(1)
                    inflight.append((k_full[kt % NK], ("k", kt % NK, (k, ik))))
                    kt += 1
                    ik += 1
                if iv < ik and (vt < NV or v_empty[vt % NV].done(((vt // NV) & 1) ^ 1)):
                    v_full[vt % NV].expect_tx_arrive(1)
                    inflight.append((v_full[vt % NV], ("v", vt % NV, (k, iv))))
                    vt += 1
                    iv += 1
                yield
            it += 1

    def tensor_core():
        while True:
            if tc_q:
                op = tc_q.pop(0)
                if op[0] == "S":
                    _, g, item, j, ks = op
                    assert qbuf[0] == item, f"S read Q of item {qbuf[0]} for item {item}"
                    assert kslot[ks] == (item, j), f"S read K {kslot[ks]} for {(item, j)}"
                    assert P[g] is None or P[g][2], "S overwrote a P not yet read"
                    S[g], P[g] = (item, j), None
                elif op[0] == "PV":
                    _, g, item, j, vs, first = op
                    assert P[g] is not None and P[g][:2] == (item, j) and not P[g][2], \
                        f"P V read P {P[g]} for {(item, j)}"
                    assert vslot[vs] == (item, j), f"P V read V {vslot[vs]} for {(item, j)}"
                    if first:
                        assert O[g] is None or O[g][2], f"P V overwrote O {O[g]} before it was read"
                        O[g] = [item, 1, False]
                    else:
                        assert O[g][0] == item and O[g][1] == j, f"O {O[g]} at P V {(item, j)}"
                        O[g][1] += 1
                    P[g] = (item, j, True)
                else:  # a commit: arrives once the products issued before it have finished
                    op[1]()
            yield

    def issuer():
        ts, tp = [0] * NG, [0] * NG
        krel = vrel = kb = nq = it = 0
        while True:
            slot = it & 1
            while not item_full[slot].done((it >> 1) & 1):
                yield
            valid, k, gt, ntiles = slots[slot]
            item_free[slot].arrive()
            if not valid:
                return
            if ntiles == 0:
                it += 1
                continue
            while not q_full.done(nq & 1):
                yield
            ns, npv = [0] * NG, [0] * NG
            rk = rv = 0
            q_released = False
            while True:
                for g in range(NG):
                    jp, gv = npv[g], kb + npv[g]
                    if (jp < ns[g] and p_full[g].done(tp[g] & 1)
                            and v_full[gv % NV].done((gv // NV) & 1)
                            and (jp > 0 or nq == 0 or o_free[g].done((nq - 1) & 1))):
                        tc_q.append(("PV", g, k, jp, gv % NV, jp == 0))
                        tc_q.append(("commit", pv_done[g].arrive))
                        npv[g] += 1
                        tp[g] += 1
                    js, gk = ns[g], kb + ns[g]
                    if js < gt[g] and npv[g] >= js and k_full[gk % NK].done((gk // NK) & 1):
                        tc_q.append(("S", g, k, js, gk % NK))
                        tc_q.append(("commit", s_full[g].arrive))
                        ns[g] += 1
                        ts[g] += 1
                if not q_released and all(ns[g] == gt[g] for g in range(NG)):
                    tc_q.append(("commit", q_free.arrive))
                    q_released = True
                if early_k_release:   # the planted mistake: one group's S is enough
                    readers = lambda r: ns[0] > r or gt[0] <= r
                else:
                    readers = lambda r: all(not (r < gt[g] and ns[g] <= r) for g in range(NG))
                while rk < ntiles and readers(rk):
                    tc_q.append(("commit", k_empty[krel % NK].arrive))
                    krel += 1
                    rk += 1
                while rv < ntiles and all(not (rv < gt[g] and npv[g] <= rv) for g in range(NG)):
                    tc_q.append(("commit", v_empty[vrel % NV].arrive))
                    vrel += 1
                    rv += 1
                if all(npv[g] >= gt[g] for g in range(NG)) and rv == ntiles:
                    break
                yield
            kb += ntiles
            nq += 1
            it += 1

    def softmax(g, w):
        tg = vg = it = 0
        while True:
            slot = it & 1
            while not item_full[slot].done((it >> 1) & 1):
                yield
            valid, k, gt, ntiles = slots[slot]
            item_free[slot].arrive()
            if not valid:
                return
            if ntiles == 0:
                it += 1
                continue
            for j in range(gt[g]):
                while not s_full[g].done((tg + j) & 1):
                    yield
                assert S[g] == (k, j), f"softmax read S {S[g]} for {(k, j)}"
                yield
                if w == 0:
                    P[g] = (k, j, False)       # every warp writes its rows; warp 0 stands for all
                if rng.random() < 0.3:         # zeroing V rows outside the keys
                    gv = vg + j
                    while not v_full[gv % NV].done((gv // NV) & 1):
                        yield
                    assert vslot[gv % NV] == (k, j), "zeroed rows of the wrong V tile"
                p_full[g].arrive()
                yield
            if gt[g] > 0:
                while not pv_done[g].done((tg + gt[g] - 1) & 1):
                    yield
                assert O[g][0] == k and O[g][1] == gt[g], f"epilogue read O {O[g]} for item {k}"
                yield
            o_free[g].arrive()
            if w == 0 and gt[g] > 0:
                O[g][2] = True
            tg += gt[g]
            vg += ntiles
            it += 1

    tasks = [producer(), issuer()] + [softmax(g, w) for g in range(NG) for w in range(NW)]
    tc = tensor_core()
    alive = list(range(len(tasks)))
    steps = 0
    while alive:
        steps += 1
        if steps > max_steps:
            raise RuntimeError(f"no progress (deadlock), seed {seed}, items {items}")
        if inflight and rng.random() < 0.4:
            bar, act = inflight.pop(rng.randrange(len(inflight)))
            if act[0] == "q":
                qbuf[0] = act[1]
            elif act[0] == "k":
                kslot[act[1]] = act[2]
            else:
                vslot[act[1]] = act[2]
            bar.complete_tx(1)
        if rng.random() < 0.5:
            next(tc)
        t = rng.choice(alive)
        try:
            next(tasks[t])
        except StopIteration:
            alive.remove(t)
    while tc_q:
        next(tc)
    return steps


@pytest.mark.parametrize("rings", [(3, 2), (6, 4)], ids=["head_dim128", "head_dim64"])
def test_protocol_holds(rings):
    nk, nv = rings
    for seed in range(150):
        run(seed, NK=nk, NV=nv)


def test_a_planted_early_k_release_is_caught():
    for seed in range(150):
        try:
            run(seed, early_k_release=True)
        except (AssertionError, RuntimeError):  # a stale read, or no progress
            return
    pytest.fail("the early K release went unnoticed")
