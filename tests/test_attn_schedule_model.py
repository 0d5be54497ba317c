"""A host model of the persistent attention kernel's barrier protocol (attn_tc2.cu), run under
random interleavings of its roles (no GPU).

Roles, as in the kernel:
* the producer: publishes units in two shared slots, loads each unit's Q, and streams its K and
  V tiles through a ring of NSLOT slots (K0, K1, V0, K2, V1, ...; the ring runs on across units);
* the two MMA issuers (one per 128-row sub-tile): per ring item, S = Q K^T for a K tile its
  sub-tile attends, O += P V for a V tile, committed in two halves;
* the two softmax groups: per tile, read S (then S is free), store P in two halves, each after
  the matching half of the previous P V; per unit, read O after the unit's last product.
* the tensor pipe: executes the issuers' products and commits in issue order, asynchronously.

Every wait in the kernel is on an mbarrier phase by its parity. The model records, for each
wait, how many phases of that barrier had completed; a wait may only see the phase it asks
for or the one before it (two phases ahead would alias the parity). The model checks that,
that every role finishes (no deadlock), and the kernel's hazards: S overwritten only after it
was read, P only after the products reading it, O only after the previous unit's epilogue read
it, Q only after the unit's last S completed.
"""
import random

import pytest

NSLOT = 3


def frame_needed(fk, fa, fb, w, r):
    i0 = (fa - fk + r - 1) // r if fa > fk else 0
    return i0 < w and fk + r * i0 <= fb


def unit_walk(l0, rows, N, w, r):
    """Sub-tile masks of the tiles of one unit (256 rows), frame by frame, 128 keys a tile."""
    fa0, fb0 = l0 // N, (min(l0 + 128, rows) - 1) // N
    valid1 = l0 + 128 < rows
    fa1 = (l0 + 128) // N if valid1 else fa0
    fb1 = (min(l0 + 256, rows) - 1) // N if valid1 else fa1
    tiles = []
    for f in range(max(0, fa0 - r * (w - 1)), (fb1 if valid1 else fb0) + 1):
        m = (1 if frame_needed(f, fa0, fb0, w, r) else 0) | \
            (2 if valid1 and frame_needed(f, fa1, fb1, w, r) else 0)
        tiles += [m] * ((N + 127) // 128) if m else []
    return tiles


class Bar:
    """An mbarrier: phases complete after `count` arrivals each."""

    def __init__(self, name, count):
        self.name, self.count, self.arrived, self.done = name, count, 0, 0

    def arrive(self):
        self.arrived += 1
        if self.arrived == self.count:
            self.arrived, self.done = 0, self.done + 1

    def ready(self, phase):
        # a parity wait on `phase` must never find the barrier two phases ahead
        assert self.done <= phase + 1, f"{self.name}: phase {phase} waited, {self.done} completed"
        return self.done > phase


def simulate(units, seed, NSLOT=NSLOT):
    rnd = random.Random(seed)
    U = len(units)
    items = []                                  # (unit, kind, tile) in ring order
    for u, tiles in enumerate(units):
        T = len(tiles)
        if T:
            items.append((u, "K", 0))
        for j in range(T):
            if j + 1 < T:
                items.append((u, "K", j + 1))
            items.append((u, "V", j))
    B = lambda n, c=1: Bar(n, c)
    full = [B(f"full{i}") for i in range(NSLOT)]
    empty = [B(f"empty{i}", 2) for i in range(NSLOT)]
    qfull, qfree = B("qfull"), B("qfree", 2)
    ufull, uempty = [B("ufull0"), B("ufull1")], [B("uempty0", 4), B("uempty1", 4)]
    sfull, sfree = [B("sfull0"), B("sfull1")], [B("sfree0"), B("sfree1")]
    pfull, pva, pvdone = [B("pfull0"), B("pfull1")], [B("pva0"), B("pva1")], [B("pvdone0"), B("pvdone1")]
    odone, ofree = [B("odone0"), B("odone1")], [B("ofree0"), B("ofree1")]
    slot_unit = [None, None]
    pipe = []                                   # the tensor pipe's queue, in issue order
    # hazard state: S buffer read count, P halves, O owner, Q owner
    s_written = [0, 0]; s_read = [0, 0]
    p_written = [[0, 0], [0, 0]]; p_read = [[0, 0], [0, 0]]
    o_unit = [None, None]; o_read_done = [-1, -1]
    q_unit = [None]
    slot_item = [None] * NSLOT                  # the ring item each slot holds

    def producer():
        it = nq = 0
        for i in range(U + 1):
            s = i & 1
            if i >= 2:
                while not uempty[s].ready((i - 2) >> 1):
                    yield
            slot_unit[s] = i if i < U else -1
            ufull[s].arrive()
            if i == U:
                return
            if i >= 1:
                while not qfree.ready(i - 1):
                    yield
            q_unit[0] = i
            qfull.arrive()
            nq += 1
            for (u, kind, j) in items:
                if u != i:
                    continue
                sl = it % NSLOT
                if it >= NSLOT:
                    while not empty[sl].ready(it // NSLOT - 1):
                        yield
                slot_item[sl] = it
                full[sl].arrive()
                it += 1
                yield

    def issuer(q):
        it = ns = npv = 0
        want = 1 << q
        for i in range(U + 1):
            s = i & 1
            while not ufull[s].ready(i >> 1):
                yield
            un = slot_unit[s]
            uempty[s].arrive()
            if un < 0:
                return
            while not qfull.ready(i):
                yield
            npv0 = npv
            tiles = units[un]
            mine = [it2 for it2, (u, kind, j) in enumerate(items) if u == un]
            last_k = max((k for k in mine if items[k][1] == "K"), default=None)
            for ii in mine:
                u, kind, j = items[ii]
                sl = it % NSLOT
                while not full[sl].ready(it // NSLOT):
                    yield
                if tiles[j] & want:
                    if kind == "K":
                        if ns > 0:
                            while not sfree[q].ready(ns - 1):
                                yield
                        pipe.append(("S", q, ns, un, ii))
                        pipe.append(("commit", sfull[q]))
                        pipe.append(("commit", empty[sl]))
                        ns += 1
                    else:
                        while not pfull[q].ready(npv):
                            yield
                        if npv == npv0 and i >= 1:
                            while not ofree[q].ready(i - 1):
                                yield
                        pipe.append(("PV", q, npv, 0, un, npv > npv0, ii))
                        pipe.append(("commit", pva[q]))
                        pipe.append(("PV", q, npv, 1, un, True, ii))
                        pipe.append(("commit", pvdone[q]))
                        pipe.append(("commit", empty[sl]))
                        npv += 1
                else:
                    empty[sl].arrive()                  # a tile this sub-tile skips
                if ii == last_k:
                    pipe.append(("commit", qfree))
                it += 1
                yield
            if npv == npv0 and i >= 1:
                while not ofree[q].ready(i - 1):
                    yield
            pipe.append(("commit", odone[q]))

    def softmax(q):
        k = 0
        for i in range(U + 1):
            s = i & 1
            while not ufull[s].ready(i >> 1):
                yield
            un = slot_unit[s]
            uempty[s].arrive()
            if un < 0:
                return
            k0 = k
            for m in units[un]:
                if not (m & (1 << q)):
                    continue
                while not sfull[q].ready(k):
                    yield
                assert s_written[q] == k + 1
                s_read[q] = k + 1
                sfree[q].arrive()
                yield
                if k >= 1:
                    while not pva[q].ready(k - 1):
                        yield
                assert p_read[q][0] >= k, "P half 0 overwritten before its product read it"
                p_written[q][0] = k + 1
                yield
                if k >= 1:
                    while not pvdone[q].ready(k - 1):
                        yield
                assert p_read[q][1] >= k, "P half 1 overwritten before its product read it"
                p_written[q][1] = k + 1
                pfull[q].arrive()
                k += 1
                yield
            while not odone[q].ready(i):
                yield
            if k > k0:
                assert o_unit[q] == un
            o_read_done[q] = i
            ofree[q].arrive()

    def tensor_pipe():
        while True:
            if pipe and rnd.random() < 0.7:
                op = pipe.pop(0)
                if op[0] in ("S", "PV"):
                    assert slot_item[op[-1] % NSLOT] == op[-1], "ring slot reloaded before its product"
                if op[0] == "S":
                    _, q, n, un, _ii = op
                    assert s_read[q] == n, "S overwritten before the softmax read it"
                    assert q_unit[0] == un, "Q reloaded before the unit's last S"
                    s_written[q] = n + 1
                elif op[0] == "PV":
                    _, q, n, half, un, acc, _ii = op
                    assert p_written[q][half] == n + 1, "P V read P before it was written"
                    p_read[q][half] = n + 1
                    if not acc:
                        assert o_read_done[q] >= un - 1, "O overwritten before its epilogue"
                        o_unit[q] = un
                else:
                    op[1].arrive()
            yield

    actors = [producer(), issuer(0), issuer(1), softmax(0), softmax(1)]
    alive = list(actors)
    pipe_actor = tensor_pipe()
    for _ in range(2_000_000):
        if not alive:
            return True
        a = rnd.choice(alive + [pipe_actor])
        try:
            next(a)
        except StopIteration:
            alive.remove(a)
    return False


@pytest.mark.parametrize("nslot", [3, 6])      # the bf16 ring and the E4M3 ring
def test_protocol_has_no_deadlock_no_parity_alias_and_no_hazard(nslot):
    cases = 0
    for (N, w, r) in [(1560, 3, 1), (1560, 3, 4), (1560, 4, 6), (130, 3, 1), (130, 4, 2),
                      (100, 2, 2), (1, 3, 2), (16, 2, 2), (200, 3, 2), (256, 2, 1)]:
        for T in (1, 2, 5, 21):
            rows = T * N
            walks = [unit_walk(l0, rows, N, w, r) for l0 in range(0, rows, 256)]
            for seed in range(6):
                rnd = random.Random(1000 * T + seed)
                n = rnd.randint(1, min(5, len(walks)))
                units = [walks[rnd.randrange(len(walks))] for _ in range(n)]
                assert simulate(units, seed, nslot), (N, w, r, T, seed)
                cases += 1
    assert cases == 240


def test_model_detects_a_planted_protocol_error():
    """The model is not vacuous: an issuer that issues the next S without waiting for its
    softmax to have read the previous one (the S-free wait removed) is caught. (Removing the
    wait for the previous unit's epilogue instead is not: the first P of a unit is written only
    after that epilogue, and its P V waits for it.)"""
    import inspect
    src = inspect.getsource(simulate)
    broken = src.replace("                        if ns > 0:\n"
                         "                            while not sfree[q].ready(ns - 1):\n"
                         "                                yield\n", "")
    assert broken != src
    ns = {}
    exec(compile("import random\n" + broken, "broken_model", "exec"), {**globals(), **ns}, ns)
    found = False
    walks = [unit_walk(l0, 3 * 200, 200, 2, 1) for l0 in range(0, 600, 256)]
    for seed in range(200):
        try:
            ns["simulate"]([walks[0], walks[1], walks[2], walks[0]], seed)
        except AssertionError as e:
            found = "S overwritten" in str(e) or "phase" in str(e)
            break
    assert found


def test_work_counter_shared_by_two_launches():
    """The persistent launches' work counter: CTAs take units by an atomic ticket until the
    tickets run past the units, then count themselves finished; the last of all CTAs (of the
    main launch and of the late CTAs queued behind another kernel, which may start at any
    time) puts both words back to zero. Every unit is processed exactly once, and the next
    launch on the counter finds it at zero."""
    rnd = random.Random(7)
    counter = [0, 0]
    for trial in range(300):
        nunits = rnd.randint(1, 60)
        grid = rnd.randint(1, 20)
        late = rnd.randint(0, 8)
        total = grid + late
        done = []

        def cta():
            while True:
                t = counter[0]
                counter[0] += 1                     # atomicAdd(&sched[0], 1)
                yield
                if t >= nunits:
                    break
                done.append(t)
                for _ in range(rnd.randint(0, 3)):
                    yield                           # the unit's work
            last = counter[1] == total - 1          # atomicAdd(&sched[1], 1) == total - 1
            counter[1] += 1
            if last:
                counter[0] = counter[1] = 0
            yield

        started = [cta() for _ in range(grid)]
        pending = [cta() for _ in range(late)]
        alive = list(started)
        while alive or pending:
            if pending and (not alive or rnd.random() < 0.1):
                alive.append(pending.pop())         # a late CTA starts
                continue
            a = rnd.choice(alive)
            try:
                next(a)
            except StopIteration:
                alive.remove(a)
        assert sorted(done) == list(range(nunits)), trial
        assert counter == [0, 0], trial
