"""Host models of the barrier protocols of the attention kernels and the fused prolog q kernel (no GPU).

The attention kernel (mla_prefill_sm100.cuh) streams key tiles through a ring of eight
16 KB chunks: key tile g, counted per CTA across its work units, occupies chunks
5g .. 5g + 4 (K_g in the first three, V_g in the last two; slot = chunk mod 8).  Four
barrier sets, indexed g mod 4, track the tiles:

  producer  K_g: waits v_empty(g - 2), arms k_full(g), issues the loads
            V_g: waits k_empty(g - 1), arms v_full(g), issues the loads
  MMA       per unit: wait k_full(first); S_0, S_1; release K(first)
            per key tile j: for t = 0, 1: wait P_t(j) (and v_full once), P V_t(j),
            release V when it is the last reader; wait k_full(j + 1) once, S_t(j + 1),
            release K(j + 1) when it is the last reader.  One thread issues every MMA;
            they complete in issue order, and a release (tcgen05.commit) completes once
            every MMA issued before it has.
  softmax   tile t: wait S_t(j) -> publish P_t(j)

This file re-states that protocol as Python coroutines and runs it under random
interleavings of the roles, the TMA completions and the in-order MMA completions, on
random unit sequences (including units where tile 1 has no rows or one key tile
fewer than tile 0).  It checks that nothing deadlocks, that no wait ever sees its
barrier more than one phase away from the intended one (mbarrier parity waits cannot
tell phases two apart), that no chunk is refilled while an MMA still reads it, and
that no MMA reads a chunk before its load has landed.  Planted protocol mistakes must
be caught, which shows the checks have teeth.  The model mirrors the kernel's logic
by hand: a change to the kernel's barrier protocol must be made here too.
"""
import random

import pytest

RING, TILE_SETS = 8, 4


class Barrier:
    """mbarrier with an arrival count; `done` counts completed phases."""

    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.done = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


class ProtocolError(AssertionError):
    pass


def ready(bar, phase):
    """A parity wait for completed phase `phase`; the barrier must be within one phase of it."""
    if bar.done not in (phase, phase + 1):
        raise ProtocolError("phase aliasing on %s: %d completed, waiting for %d" % (bar.name, bar.done, phase))
    return bar.done >= phase + 1


def simulate(units, seed, bug=None):
    """units: [(n0, n1)] key tiles of query tile 0 / 1 per unit (n_max = max(n0, n1) > 0)."""
    rnd = random.Random(seed)
    bars = {}
    for kind in ("k_full", "v_full", "k_empty", "v_empty"):
        for i in range(TILE_SETS):
            bars[kind, i] = Barrier("%s[%d]" % (kind, i))
    for t in range(2):
        bars["s_full", t] = Barrier("s_full[%d]" % t)
        bars["p_full", t] = Barrier("p_full[%d]" % t)
    slot_owner = {}   # ring slot -> (tile, "K" | "V") last loaded into it
    readers = {}      # (tile, kind) -> MMAs issued and not yet completed
    landed = set()
    tma = []          # loads in flight: (barrier, (tile, kind))
    mma_queue = []    # in issue order: ("mma", (tile, kind)) or ("commit", barrier)

    def b(kind, g):
        return bars[kind, g % TILE_SETS]

    def fill(g, kind, chunks):
        for c in chunks:
            slot = (5 * g + c) % RING
            prev = slot_owner.get(slot)
            if prev is not None and readers.get(prev, 0):
                raise ProtocolError("slot %d refilled with %s %d while an MMA reads %s" % (slot, kind, g, prev))
            slot_owner[slot] = (g, kind)

    def producer():
        g = 0
        for n0, n1 in units:
            for _ in range(max(n0, n1)):
                lag = 3 if bug == "k_waits_tile_g_minus_3" else 2
                if g >= lag:
                    while not ready(b("v_empty", g - lag), (g - lag) // TILE_SETS):
                        yield
                fill(g, "K", (0, 1, 2))
                tma.append((b("k_full", g), (g, "K")))
                if g >= 1 and bug != "no_v_slot_wait":
                    while not ready(b("k_empty", g - 1), (g - 1) // TILE_SETS):
                        yield
                fill(g, "V", (3, 4))
                tma.append((b("v_full", g), (g, "V")))
                g += 1
                yield

    def issue(operand):
        if operand not in landed:
            raise ProtocolError("MMA reads %s before it landed" % (operand,))
        readers[operand] = readers.get(operand, 0) + 1
        mma_queue.append(("mma", operand))

    def commit(bar):
        mma_queue.append(("commit", bar))

    def last_reader(t, j, n):
        if bug == "release_by_tile_0":
            return t == 0 or j >= n[1]
        return t == 1 or j >= n[1]

    def mma():
        tg, pf = 0, [0, 0]
        for n0, n1 in units:
            n = (n0, n1)
            while not ready(b("k_full", tg), tg // TILE_SETS):
                yield
            for t in range(2):
                if n[t] > 0:
                    issue((tg, "K"))
                    commit(bars["s_full", t])
            commit(b("k_empty", tg))
            for j in range(max(n)):
                g = tg + j
                v_ready = k_ready = False
                for t in range(2):
                    if j < n[t]:
                        while not ready(bars["p_full", t], pf[t]):
                            yield
                        pf[t] += 1
                        if not v_ready and bug != "no_v_full_wait":
                            while not ready(b("v_full", g), g // TILE_SETS):
                                yield
                            v_ready = True
                        issue((g, "V"))
                        if last_reader(t, j, n):
                            commit(b("v_empty", g))
                    if j + 1 < n[t]:
                        if not k_ready:
                            while not ready(b("k_full", g + 1), (g + 1) // TILE_SETS):
                                yield
                            k_ready = True
                        issue((g + 1, "K"))
                        commit(bars["s_full", t])
                        if last_reader(t, j + 1, n):
                            commit(b("k_empty", g + 1))
                    yield
            tg += max(n)

    def softmax(t):
        sf = 0
        for unit in units:
            for _ in range(unit[t]):
                while not ready(bars["s_full", t], sf):
                    yield
                sf += 1
                yield
                bars["p_full", t].arrive()

    roles = [producer(), mma(), softmax(0), softmax(1)]
    alive = [True] * len(roles)
    for _ in range(400000):
        if not (any(alive) or tma or mma_queue):
            return
        acts = [("role", i) for i, a in enumerate(alive) if a]
        if tma:
            acts.append(("tma", rnd.randrange(len(tma))))
        if mma_queue:
            acts.append(("mma", 0))
        act, arg = rnd.choice(acts)
        if act == "role":
            try:
                next(roles[arg])
            except StopIteration:
                alive[arg] = False
        elif act == "tma":
            bar, operand = tma.pop(arg)
            landed.add(operand)
            bar.arrive()
        else:
            op, x = mma_queue.pop(0)
            if op == "mma":
                readers[x] -= 1
            else:
                x.arrive()
    raise ProtocolError("deadlock")


def random_units(rng):
    units = []
    for _ in range(rng.randint(1, 7)):
        n1 = rng.randint(0, 8)
        n0 = rng.choice([n1, max(0, n1 - 1), 0, rng.randint(1, 6) if n1 == 0 else n1])
        if max(n0, n1):
            units.append((n0, n1))
    return units or [(1, 1)]


def test_protocol_holds_under_random_schedules():
    rng = random.Random(2024)
    for trial in range(400):
        simulate(random_units(rng), seed=trial)


@pytest.mark.parametrize("bug", ["no_v_slot_wait", "k_waits_tile_g_minus_3", "no_v_full_wait", "release_by_tile_0"])
def test_planted_protocol_mistakes_are_caught(bug):
    rng = random.Random(7)
    with pytest.raises(ProtocolError):
        for trial in range(400):
            simulate(random_units(rng), seed=trial, bug=bug)


# ---------------------------------------------------------------------------
# The CTA-pair kernel (mla_prefill_pair_sm100.cuh)
# ---------------------------------------------------------------------------
# Two CTAs (leader 0, follower 1) each stream their half of every 64-key tile through their own
# ring of six tile slots (K_g and V_g of key tile g in slot g mod 6, with a full and an empty
# barrier per slot for K and for V).  Each CTA also holds its 128 rows of Q for groups 0 and 1.
# Per group t, tensor memory holds O_t and two S buffers: S_t of the group's g-th tile (counted
# across units) goes to buffer g mod 2, and the softmax writes P_t(g) over the same buffer.
#
#   producer (each CTA)  per unit: Q_t for each group with key tiles: waits its own
#                        q_empty(t), arms its own q_full(t), loads; per key tile g:
#                        K_g waits its own k_empty(g - 6), V_g its own v_empty(g - 6)
#   relay (follower)     in the producer's order, waits for each of the follower's full
#                        barriers and arrives on the leader's matching one
#   helper t (leader)    for the group's g-th tile (unit step j): waits S_t(g) (issued after
#                        P V_t(g - 2), so the P-ready phase of tile g - 2 is complete and this
#                        arrival cannot fall into it; it also keeps the helper within one phase
#                        of the slots it checks next), then the leader's v_full(j) and, if the
#                        group has a tile j + 2, k_full(j + 2), then arrives on P_t[g mod 2]
#   MMA (leader)         per unit: waits q_full; S_t(0), S_t(1) (after k_full of tiles 0, 1);
#                        per step j and group t: waits P_t[g mod 2] (three arrivals: each CTA's
#                        softmax and the helper), issues P V_t(j), commits pv_done_t[g mod 2],
#                        then S_t(j + 2)
#                        into the buffer P_t(j) occupies (in-order completion: after P V_t(j)
#                        has read it) and commits s_full_t[buffer]; releases (q/k/v_empty)
#                        arrive in both CTAs.  The
#                        unit's first P V_t overwrites O_t with no O-free barrier: its P-ready
#                        phase needs every softmax warp of the group, and each has read its rows
#                        of O_t in the previous unit's epilogue before it starts the next unit
#   softmax (each CTA)   group t, tile g: waits its own s_full_t[g mod 2], reads S_t(g), writes
#                        P_t(g) over it; when its running max moved (modelled at random) waits
#                        pv_done_t[(g - 1) mod 2] and rescales O_t; arrives on the leader's
#                        P_t[g mod 2]; after the unit's last tile waits o_full_t and reads O_t.
#                        The S, P-ready and P V-done barriers come in pairs (tile parity): a
#                        barrier's next phase then needs this group's own next-but-one tile, so
#                        no role can fall two phases behind one it waits for, even where the
#                        softmax waits for P V-done only now and then
# Tensor-memory contents are tracked too: a write over data still to be read, or a read of the
# wrong tile's data, is a protocol error.
PAIR_SLOTS = 6


def simulate_pair(units, seed, bug=None):
    """units: [(n0, n1)] 64-key tiles of group 0 / 1 per 512-row unit (max > 0)."""
    rnd = random.Random(seed)
    bars = {}

    def mk(kind, cta, i, count=1):
        bars[kind, cta, i] = Barrier("%s[%d]@%d" % (kind, i, cta), count)

    for cta in range(2):
        full_count = 2 if cta == 0 else 1
        for i in range(PAIR_SLOTS):
            mk("k_full", cta, i, full_count)
            mk("v_full", cta, i, full_count)
            mk("k_empty", cta, i)
            mk("v_empty", cta, i)
        for t in range(2):
            mk("q_full", cta, t, full_count)
            mk("q_empty", cta, t)
            mk("o_full", cta, t)
            for buf in range(2):
                mk("s_full", cta, 2 * t + buf)
                mk("pv_done", cta, 2 * t + buf)
    for t in range(2):
        for buf in range(2):
            mk("p_full", 0, 2 * t + buf, 3)
    owner = {}     # (cta, ring slot part | ("Q", t)) -> operand last loaded there
    readers = {}   # operand -> MMAs issued and not yet completed
    landed = set()
    tma = []       # (cta, barrier, operand)
    mma_queue = []
    sbuf = {}      # (cta, t, buffer) -> ("S", g) | ("P", g) | ("X", g): written, P over it, P read
    otile = {}     # (cta, t) -> ("O", g) after P V(g), ("R", g) rescaled for g + 1, ("D",) drained

    def b(kind, cta, g):
        return bars[kind, cta, g % PAIR_SLOTS]

    def s_full(cta, t, g):
        if bug == "pair_one_s_full":
            return bars["s_full", cta, 2 * t]
        return bars["s_full", cta, 2 * t + g % 2]

    def p_full(t, g):
        if bug == "pair_one_p_full":
            return bars["p_full", 0, 2 * t]
        return bars["p_full", 0, 2 * t + g % 2]

    def pv_done(cta, t, g):
        return bars["pv_done", cta, 2 * t + g % 2]

    def phase(g):
        return g if bug == "pair_one_p_full" else g // 2

    def fill(cta, key, operand):
        prev = owner.get((cta, key))
        if prev is not None and readers.get(prev, 0):
            raise ProtocolError("%s refilled with %s while an MMA reads %s" % ((cta, key), operand, prev))
        owner[(cta, key)] = operand

    def producer(cta):
        g = 0
        ql = [0, 0]
        lag = 7 if bug == "pair_lag_7" else PAIR_SLOTS
        for n in units:
            for t in range(2):
                if n[t] == 0:
                    continue
                if ql[t] >= 1 and bug != "pair_no_q_empty_wait":
                    while not ready(bars["q_empty", cta, t], ql[t] - 1):
                        yield
                fill(cta, ("Q", t), (cta, "Q", t, ql[t]))
                tma.append((cta, bars["q_full", cta, t], (cta, "Q", t, ql[t])))
                ql[t] += 1
            for _ in range(max(n)):
                if g >= lag:
                    while not ready(b("k_empty", cta, g - lag), (g - lag) // PAIR_SLOTS):
                        yield
                fill(cta, ("K", g % PAIR_SLOTS), (cta, "K", g))
                tma.append((cta, b("k_full", cta, g), (cta, "K", g)))
                if g >= lag and bug != "pair_no_v_slot_wait":
                    while not ready(b("v_empty", cta, g - lag), (g - lag) // PAIR_SLOTS):
                        yield
                fill(cta, ("V", g % PAIR_SLOTS), (cta, "V", g))
                tma.append((cta, b("v_full", cta, g), (cta, "V", g)))
                g += 1
                yield

    def relay():
        g = 0
        qf = [0, 0]
        for n in units:
            for t in range(2):
                if n[t] == 0:
                    continue
                while not ready(bars["q_full", 1, t], qf[t]):
                    yield
                qf[t] += 1
                if bug != "pair_no_q_relay":
                    bars["q_full", 0, t].arrive()
            for _ in range(max(n)):
                for kind in ("k_full", "v_full"):
                    while not ready(b(kind, 1, g), g // PAIR_SLOTS):
                        yield
                    if not (bug == "pair_relay_skips_v" and kind == "v_full"):
                        b(kind, 0, g).arrive()
                g += 1
                yield

    def helper(t):
        tg, gt = 0, 0
        for n in units:
            for j in range(n[t]):
                kg = tg + j
                if bug != "pair_helper_runs_ahead":
                    while not ready(s_full(0, t, gt), gt // 2):
                        yield
                while not ready(b("v_full", 0, kg), kg // PAIR_SLOTS):
                    yield
                if j + 2 < n[t] and bug != "pair_helper_skips_k":
                    while not ready(b("k_full", 0, kg + 2), (kg + 2) // PAIR_SLOTS):
                        yield
                p_full(t, gt).arrive()
                gt += 1
                yield
            tg += max(n)

    def issue(effect, *operands):
        for op in operands:
            if op not in landed:
                raise ProtocolError("pair MMA reads %s before it landed" % (op,))
            readers[op] = readers.get(op, 0) + 1
        mma_queue.append(("mma", (effect, operands)))

    def commit_both(kind, idx):
        mma_queue.append(("commit", [bars[kind, 0, idx], bars[kind, 1, idx]]))

    def mma_effect(effect):
        kind, t, g, first = effect
        for cta in range(2):
            key = (cta, t, g % 2)
            if kind == "S":
                prev = sbuf.get(key)
                if prev is not None and prev != ("X", g - 2):
                    raise ProtocolError("S_%d(%d) overwrites %s in buffer %d" % (t, g, prev, g % 2))
                sbuf[key] = ("S", g)
            else:
                if sbuf.get(key) != ("P", g):
                    raise ProtocolError("P V_%d(%d) reads %s" % (t, g, sbuf.get(key)))
                sbuf[key] = ("X", g)
                o = otile.get((cta, t))
                want = [None, ("D",)] if first else [("O", g - 1), ("R", g - 1)]
                if o not in want:
                    raise ProtocolError("P V_%d(%d) on O_%d in state %s" % (t, g, t, o))
                otile[(cta, t)] = ("O", g)

    def mma():
        tg, qf, qn, gs = 0, [0, 0], [0, 0], [0, 0]
        ahead = 3 if bug == "pair_s_lookahead_3" else 2
        for n in units:
            for t in range(2):
                if n[t]:
                    while not ready(bars["q_full", 0, t], qf[t]):
                        yield
                    qf[t] += 1

            def issue_s(t, j):
                issue(("S", t, gs[t] + j, False), (0, "Q", t, qn[t]), (1, "Q", t, qn[t]), (0, "K", tg + j),
                      (1, "K", tg + j))
                mma_queue.append(("commit", [s_full(0, t, gs[t] + j), s_full(1, t, gs[t] + j)]))
                if j == n[t] - 1:
                    commit_both("q_empty", t)

            for j0 in range(min(ahead, max(n))):
                while not ready(b("k_full", 0, tg + j0), (tg + j0) // PAIR_SLOTS):
                    yield
                for t in range(2):
                    if j0 < n[t]:
                        issue_s(t, j0)
                commit_both("k_empty", (tg + j0) % PAIR_SLOTS)
            for j in range(max(n)):
                g = tg + j
                for t in range(2):
                    if j < n[t]:
                        while not ready(p_full(t, gs[t] + j), phase(gs[t] + j)):
                            yield
                        issue(("PV", t, gs[t] + j, j == 0), (0, "V", g), (1, "V", g))
                        mma_queue.append(("commit", [pv_done(0, t, gs[t] + j), pv_done(1, t, gs[t] + j)]))
                        if j == n[t] - 1:
                            commit_both("o_full", t)
                        if t == 1 or j >= n[1]:
                            commit_both("v_empty", g % PAIR_SLOTS)
                    if j + ahead < n[t]:
                        issue_s(t, j + ahead)
                        if t == 1 or j + ahead >= n[1]:
                            commit_both("k_empty", (g + ahead) % PAIR_SLOTS)
                    yield
            for t in range(2):
                if n[t]:
                    qn[t] += 1
                gs[t] += n[t]
            tg += max(n)

    def softmax(cta, t):
        gt, of = 0, 0
        for n in units:
            for j in range(n[t]):
                while not ready(s_full(cta, t, gt), gt // 2 if bug != "pair_one_s_full" else gt):
                    yield
                key = (cta, t, (gt + (bug == "pair_softmax_other_buffer")) % 2)
                if sbuf.get(key) != ("S", gt):
                    raise ProtocolError("softmax %d reads %s for S(%d)" % (t, sbuf.get(key), gt))
                yield
                sbuf[key] = ("P", gt)
                if j > 0 and rnd.random() < 0.3:  # the running max moved: rescale O_t
                    if bug != "pair_softmax_no_pv_wait":
                        while not ready(pv_done(cta, t, gt - 1), (gt - 1) // 2):
                            yield
                    o = otile.get((cta, t))
                    if o != ("O", gt - 1):
                        raise ProtocolError("rescale of O_%d(%d) sees %s" % (t, gt, o))
                    otile[(cta, t)] = ("R", gt - 1)
                p_full(t, gt).arrive()
                gt += 1
                yield
            if n[t]:
                while not ready(bars["o_full", cta, t], of):
                    yield
                of += 1
                if otile.get((cta, t)) != ("O", gt - 1):
                    raise ProtocolError("epilogue of O_%d sees %s" % (t, otile.get((cta, t))))
                otile[(cta, t)] = ("D",)

    roles = [producer(0), producer(1), relay(), helper(0), helper(1), mma()] + \
        [softmax(c, t) for c in range(2) for t in range(2)]
    alive = [True] * len(roles)
    for _ in range(800000):
        if not (any(alive) or tma or mma_queue):
            return
        acts = [("role", i) for i, a in enumerate(alive) if a]
        if tma:
            acts.append(("tma", rnd.randrange(len(tma))))
        if mma_queue:
            acts.append(("mma", 0))
        act, arg = rnd.choice(acts)
        if act == "role":
            try:
                next(roles[arg])
            except StopIteration:
                alive[arg] = False
        elif act == "tma":
            cta, bar, operand = tma.pop(arg)
            landed.add(operand)
            bar.arrive()
        else:
            op, x = mma_queue.pop(0)
            if op == "mma":
                effect, operands = x
                mma_effect(effect)
                for operand in operands:
                    readers[operand] -= 1
            else:
                for bar in x:
                    bar.arrive()
    raise ProtocolError("deadlock")


def test_pair_protocol_holds_under_random_schedules():
    rng = random.Random(4048)
    for trial in range(300):
        simulate_pair(random_units(rng), seed=trial)


@pytest.mark.parametrize("bug", ["pair_lag_7", "pair_no_v_slot_wait", "pair_no_q_empty_wait", "pair_no_q_relay",
                                 "pair_relay_skips_v", "pair_helper_skips_k", "pair_helper_runs_ahead",
                                 "pair_one_p_full",
                                 "pair_softmax_no_pv_wait", "pair_one_s_full", "pair_s_lookahead_3",
                                 "pair_softmax_other_buffer"])
def test_pair_planted_protocol_mistakes_are_caught(bug):
    rng = random.Random(11)
    with pytest.raises(ProtocolError):
        for trial in range(300):
            simulate_pair(random_units(rng), seed=trial, bug=bug)


# ---------------------------------------------------------------------------
# The fused MLA Prolog q kernel (prolog_q_sm100.cuh)
# ---------------------------------------------------------------------------
# Two CTAs (leader 0, follower 1).  Per tile (256 tokens x one head) the stages run N-chunk by
# N-chunk: chunk c takes k_stages stages of a ring of S slots; the accumulator's two channel halves
# (tensor memory) have their own barriers.
#
#   producer (each CTA)  stage i: waits its own empty(i - S), arms full(i), loads A and chunk c's B
#   relay (follower)     forwards each of the follower's full barriers to the leader's
#   MMA (leader)         before chunk c of a tile: waits half_free(h) of the previous tile for each
#                        half h the chunk writes (first time in the tile); per stage: waits full,
#                        MMAs, commits empty (both CTAs); after the chunk's last stage commits
#                        half_full(h) for the halves whose last chunk it is
#   epilogue half w      (the four warps summing half w's squares, modelled as one role per CTA):
#                        waits half_full(w), reads half w (pass 1), exchanges with the other half
#                        (xready), waits half_full(1 - w) (implied by the exchange, whose other side
#                        waited for it; the kernel waits too, for the tensor-memory ordering of its
#                        own reads), then per output block: reads its slice of
#                        the accumulator (first its share of half 0, then of half 1), releasing
#                        half_free(0) / (1) (leader, both CTAs' roles count) after its last read of
#                        the half; waits st_empty of the block's buffer, stages it, arrives st_full
#   store w (each CTA)   per block: waits st_full, issues the store (its read of the buffer happens
#                        later, at a random point); once every store but the newest has read its
#                        buffer, arrives the previous buffer's st_empty
# Tensor-memory halves and staging buffers are tracked: an MMA over a half the previous tile's
# epilogue still reads, a read of a half before its chunk completed, a staged buffer overwritten
# before its store read it, or a store of a buffer not yet staged are errors.


def simulate_prolog(n_tiles, chunks, halves_of_chunk, last_chunk_of_half, k_stages, blocks_per_half, seed,
                    slots=6, bug=None):
    rnd = random.Random(seed)
    bars = {}

    def mk(kind, cta, i, count=1):
        bars[kind, cta, i] = Barrier("%s[%d]@%d" % (kind, i, cta), count)

    for cta in range(2):
        for i in range(slots):
            mk("full", cta, i, 2 if cta == 0 else 1)
            mk("empty", cta, i)
        for h in range(2):
            mk("half_full", cta, h)
            mk("xready", cta, h, 2) if h == 0 else None
            for b in range(2):
                mk("st_full", cta, 2 * h + b)
                mk("st_empty", cta, 2 * h + b)
    for h in range(2):
        mk("half_free", 0, h, 4)  # both epilogue halves of both CTAs read part of every half
    owner, readers, landed, tma, mma_queue = {}, {}, set(), [], []
    acc = {}   # (cta, half) -> ("acc", tile, MMA stages done) | ("read", tile, readers left) | ("free", tile)
    buf = {}   # (cta, w, b) -> ("staged", block id) | ("free",)
    stage_order = [(t, c, ks) for t in range(n_tiles) for c in range(chunks) for ks in range(k_stages)]

    def producer(cta):
        for i, (t, c, ks) in enumerate(stage_order):
            lag = slots + 1 if bug == "prolog_lag" else slots
            if i >= slots:
                while not ready(bars["empty", cta, (i - lag) % slots if bug == "prolog_lag" else i % slots],
                                (i - slots) // slots):
                    yield
            prev = owner.get((cta, i % slots))
            if prev is not None and readers.get(prev, 0):
                raise ProtocolError("stage slot %d refilled while an MMA reads %s" % (i % slots, prev))
            owner[(cta, i % slots)] = (cta, i)
            tma.append((cta, bars["full", cta, i % slots], (cta, i)))
            yield

    def relay():
        for i in range(len(stage_order)):
            while not ready(bars["full", 1, i % slots], i // slots):
                yield
            bars["full", 0, i % slots].arrive()
            yield

    def mma():
        i = 0
        for t in range(n_tiles):
            waited = set()
            for c in range(chunks):
                for h in halves_of_chunk[c]:
                    if h not in waited and bug != "prolog_no_half_free_wait":
                        if t >= 1:
                            while not ready(bars["half_free", 0, h], t - 1):
                                yield
                        waited.add(h)
                for ks in range(k_stages):
                    while not ready(bars["full", 0, i % slots], i // slots):
                        yield
                    for op in ((0, i), (1, i)):
                        if op not in landed:
                            raise ProtocolError("MMA reads stage %s before it landed" % (op,))
                        readers[op] = readers.get(op, 0) + 1
                    mma_queue.append(("mma", (t, c, (0, i), (1, i))))
                    mma_queue.append(("commit", [bars["empty", 0, i % slots], bars["empty", 1, i % slots]]))
                    if ks == k_stages - 1:
                        for h in halves_of_chunk[c]:
                            if last_chunk_of_half[h] == c or (bug == "prolog_early_half_full" and h == 1):
                                mma_queue.append(("commit", [bars["half_full", 0, h], bars["half_full", 1, h]]))
                    i += 1
                    yield

    def mma_effect(t, c):
        for cta in range(2):
            for h in halves_of_chunk[c]:
                st = acc.get((cta, h))
                if st is not None and not (st[0] == "acc" and st[1] == t) and not (st[0] == "free" and st[1] == t - 1):
                    raise ProtocolError("chunk %d of tile %d writes half %d in state %s" % (c, t, h, st))
                done = st[2] + 1 if st is not None and st[0] == "acc" and st[1] == t else 1
                acc[(cta, h)] = ("acc", t, done)

    def epilogue(cta, w):
        kb = 0

        def check_read(t, part, what):
            st = acc.get((cta, part))
            need = k_stages * sum(1 for c in range(chunks) if part in halves_of_chunk[c])  # MMA stages
            if st is None or st[1] != t or st[0] not in ("acc", "read") or (st[0] == "acc" and st[2] != need):
                raise ProtocolError("%s of tile %d reads half %d in state %s" % (what, t, part, st))
            if st[0] == "acc":
                acc[(cta, part)] = ("read", t, 2)

        def release(t, part):
            st = acc[(cta, part)]
            left = st[2] - 1
            acc[(cta, part)] = ("read", t, left) if left else ("free", t)
            bars["half_free", 0, part].arrive()

        def stage():
            nonlocal kb
            b = kb & 1
            if kb >= 2 and bug != "prolog_no_st_empty_wait":
                while not ready(bars["st_empty", cta, 2 * w + b], (kb >> 1) - 1):
                    yield
            if buf.get((cta, w, b), ("free",))[0] == "staged":
                raise ProtocolError("staging buffer %s overwritten before its store read it" % ((cta, w, b),))
            buf[(cta, w, b)] = ("staged", kb)
            bars["st_full", cta, 2 * w + b].arrive()
            kb += 1
            yield

        for t in range(n_tiles):
            # half 0: this role's columns copied into registers, the half handed back at once
            while not ready(bars["half_full", cta, 0], t):
                yield
            if bug == "prolog_release_before_copy":
                release(t, 0)
                yield
                check_read(t, 0, "copy")
            else:
                check_read(t, 0, "copy")
                yield
                release(t, 0)
            yield
            # half 1: the squares of this role's columns
            if bug != "prolog_sum_before_full":
                while not ready(bars["half_full", cta, 1], t):
                    yield
            check_read(t, 1, "pass 1")
            yield
            bars["xready", cta, 0].arrive()
            while not ready(bars["xready", cta, 0], t):
                yield
            for _ in range(blocks_per_half):  # half 0 from registers
                yield from stage()
            # half 1, two blocks per load; the half goes back after the role's last load of it
            loads = (blocks_per_half + 1) // 2
            for i in range(loads):
                last = i == loads - 1
                if last and bug == "prolog_release_before_last_load":
                    release(t, 1)
                    yield
                check_read(t, 1, "pass 2")
                if last and bug != "prolog_release_before_last_load":
                    release(t, 1)
                for _ in range(min(2, blocks_per_half - 2 * i)):
                    yield from stage()
            yield

    store_reads = []  # TMA stores whose shared-memory read has not happened yet

    def store(cta, w):
        kb, inflight = 0, []
        for t in range(n_tiles):
            for _ in range(2 * blocks_per_half):
                b = kb & 1
                while not ready(bars["st_full", cta, 2 * w + b], kb >> 1):
                    yield
                if buf.get((cta, w, b)) != ("staged", kb):
                    raise ProtocolError("store of block %d sees buffer %s" % (kb, buf.get((cta, w, b))))
                ev = {"buf": (cta, w, b), "block": kb, "done": False}
                store_reads.append(ev)
                inflight.append(ev)
                if bug == "prolog_release_current":
                    buf[(cta, w, b)] = ("free",)
                    bars["st_empty", cta, 2 * w + b].arrive()
                else:
                    # wait_group.read 1: every store but the newest has read its buffer
                    while any(not e["done"] for e in inflight[:-1]):
                        yield
                    if len(inflight) > 1:
                        prev = inflight.pop(0)
                        buf[prev["buf"]] = ("free",)
                        bars["st_empty", cta, 2 * w + (prev["block"] & 1)].arrive()
                kb += 1
                yield

    roles = [producer(0), producer(1), relay(), mma()] + [epilogue(c, w) for c in range(2) for w in range(2)] + \
        [store(c, w) for c in range(2) for w in range(2)]
    alive = [True] * len(roles)
    for _ in range(400000):
        if not (any(alive) or tma or mma_queue or store_reads):
            return
        acts = [("role", i) for i, a in enumerate(alive) if a]
        if tma:
            acts.append(("tma", rnd.randrange(len(tma))))
        if mma_queue:
            acts.append(("mma", 0))
        if store_reads:
            acts.append(("read", rnd.randrange(len(store_reads))))
        act, arg = rnd.choice(acts)
        if act == "role":
            try:
                next(roles[arg])
            except StopIteration:
                alive[arg] = False
        elif act == "tma":
            cta, bar, operand = tma.pop(arg)
            landed.add(operand)
            bar.arrive()
        elif act == "read":
            ev = store_reads.pop(arg)
            if buf.get(ev["buf"]) != ("staged", ev["block"]):
                raise ProtocolError("store of block %d reads buffer %s" % (ev["block"], buf.get(ev["buf"])))
            ev["done"] = True
        else:
            op, x = mma_queue.pop(0)
            if op == "mma":
                t, c, o0, o1 = x
                mma_effect(t, c)
                readers[o0] -= 1
                readers[o1] -= 1
            else:
                for bar in x:
                    bar.arrive()
    raise ProtocolError("deadlock")


# (chunks, halves each chunk writes, last chunk of each half) for the head sizes the kernel takes
PROLOG_SHAPES = {
    512: (2, [[0], [1]], [0, 1]),          # nc = 256: chunk c is half c
    384: (3, [[0], [0, 1], [1]], [1, 2]),  # nc = 128: the middle chunk straddles the halves
    256: (1, [[0, 1]], [0, 0]),
    128: (1, [[0, 1]], [0, 0]),
}


@pytest.mark.parametrize("d", sorted(PROLOG_SHAPES))
def test_prolog_protocol_holds_under_random_schedules(d):
    chunks, hoc, loh = PROLOG_SHAPES[d]
    rng = random.Random(d)
    for trial in range(60):
        simulate_prolog(rng.randint(1, 4), chunks, hoc, loh, rng.randint(1, 4), d // 128, seed=trial)


@pytest.mark.parametrize("bug", ["prolog_lag", "prolog_no_half_free_wait", "prolog_early_half_full",
                                 "prolog_release_current", "prolog_no_st_empty_wait", "prolog_sum_before_full",
                                 "prolog_release_before_last_load", "prolog_release_before_copy"])
def test_prolog_planted_protocol_mistakes_are_caught(bug):
    rng = random.Random(3)
    with pytest.raises(ProtocolError):
        for trial in range(200):
            d = rng.choice(sorted(PROLOG_SHAPES))
            chunks, hoc, loh = PROLOG_SHAPES[d]
            simulate_prolog(rng.randint(2, 4), chunks, hoc, loh, rng.randint(1, 3), d // 128, seed=trial, bug=bug)
