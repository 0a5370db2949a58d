"""Randomised models of the mbarrier protocols of the two persistent attention
kernels (fa_fwd_persistent_kernel, fa_bwd_kernel), run on the CPU.

Each warp role of a kernel is a Python generator that performs the role's
waits, arrivals and issues in the kernel's order.  A scheduler picks one role,
the tensor pipe (which completes issued products and their commits in order)
or the TMA engine (which completes loads in order) at a time, with per-role
speeds drawn over three decades so that some roles lag far behind others.

An mbarrier wait with parity bit b passes when the barrier's completed-phase
count has the other parity; the model asserts that every wait passes exactly
when its intended phase is the most recently completed one.  A role more than
one phase behind would pass on a stale phase in hardware; the model reports it
as "run-ahead".  It also asserts that buffers (Q stages, K/V slots, unit-index
slots, TMEM accumulators) are refilled only after their last reader finished,
that no schedule deadlocks, and that every unit of work is done exactly once.

The models carry no attention arithmetic; a planted-mistake test for each
shows that a missing wait is caught.
"""

import random

import pytest


class _Bar:
    def __init__(self, count):
        self.count, self.arrived, self.phases = count, 0, 0

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count
        if self.arrived == self.count:
            self.arrived = 0
            self.phases += 1


def _waiter(bars):
    def wait(name, k):
        """Wait for the completion of phase k (0-based) of barrier ``name``."""
        b = bars[name]
        while True:
            if (b.phases & 1) != (k & 1):
                assert b.phases == k + 1, f"ambiguous pass {name}: wanted phase {k}, {b.phases} done"
                return
            if b.phases >= k + 2:
                raise AssertionError(f"run-ahead {name}: wanted phase {k}, {b.phases} done")
            yield
    return wait


def _run(gens, engines, rnd, max_steps=20_000_000):
    """Drive role generators and in-order engines ({key: (queue, complete_fn)})
    at random per-role speeds until all are finished."""
    alive = dict(gens)
    speed = {k: 10 ** rnd.uniform(-3, 0) for k in list(gens) + list(engines)}
    steps = 0
    while True:
        choices = list(alive) + [k for k, (q, _) in engines.items() if q]
        if not choices:
            return
        steps += 1
        assert steps < max_steps, "deadlock"
        ch = rnd.choices(choices, weights=[speed[c] for c in choices])[0]
        if ch in engines:
            q, complete = engines[ch]
            complete(q.pop(0))
        else:
            try:
                next(alive[ch])
            except StopIteration:
                del alive[ch]


# ---------------------------------------------------------------- backward
def simulate_bwd(unit_len, n_ctas, n_stage, lookahead, seed, mistake=None, halves=False, kt_tmem=False,
                 st_single=False, dk_ss=False):
    """fa_bwd_kernel: ``n_ctas`` persistent CTAs claim units (``unit_len[i]`` query
    steps each) from one counter.  Roles per CTA: the producer (lane 0 of warp
    0), the MMA warp, four compute warps and four drain warps.  ``lookahead`` is
    how many Sᵀ products run ahead (2 with several Q/dO stages, 1 with one).

    ``halves`` models the one-stage layout of d = 256, where a step's Q and dO
    tiles are loaded in two halves: half A (the head-dimension panels outside
    the CTA's own output columns, last read by dPᵀ) and half B (the CTA's own
    panels and the per-row statistics, last read by the dK product); half B's
    Q and dO complete on separate barriers.  Each step issues Sᵀ over half B,
    dPᵀ over half A and B, dV, then the next step's Sᵀ over half A, then dK and
    dQᵀ (a unit's first step issues its own Sᵀ over half A first).

    ``kt_tmem`` models Kᵀ in TMEM: at the start of each unit the four drain
    warps wait for the unit's K tile, write Kᵀ into TMEM and arrive on KTFULL,
    which the MMA warp waits for before the unit's first dQᵀ; the model checks
    that no dQᵀ reads a Kᵀ not yet fully written and that no Kᵀ is overwritten
    while a dQᵀ of the unit before may still read it.  ``st_single`` models one
    Sᵀ buffer (lookahead 1): each step's Sᵀ is issued right after the previous
    step's dV.  For both Sᵀ layouts the model checks that an Sᵀ product
    completes only after the compute warps handed over the Pᵀ it overwrites and
    the dV product that read it completed.  The compute warps overwrite the
    shared-memory dSᵀ tile of a step only after the previous step's readers of
    it completed: its dQᵀ product and, with ``dk_ss`` (dK reading dSᵀ from
    shared memory), its dK product."""
    rnd = random.Random(seed)
    counter = [0]
    done_units = []
    gens, engines = {}, {}
    # with halves, each unit owns one half of the output columns, chosen at random
    unit_dh = [rnd.randrange(2) for _ in unit_len]

    def make_cta(c):
        bars = {}
        for nm in ("KVFULL", "KVEMPTY", "DPFULL", "DQFULL", "ACC"):
            bars[nm] = _Bar(1)
        for nm in ("DSFULL", "DQEMPTY", "DKFREE", "DVFREE"):
            bars[nm] = _Bar(4)
        for i in range(n_stage):
            bars["QFULL", i] = _Bar(1)
            bars["QEMPTY", i] = _Bar(1)
        for nm in ("HAFULL", "HAEMPTY", "QBFULL", "DOBFULL", "HBEMPTY"):
            bars[nm] = _Bar(1)
        bars["KTFULL"] = _Bar(4)
        for i in range(2):
            bars["SFULL", i] = _Bar(1)
            bars["PFULL", i] = _Bar(4)
            bars["UNITFULL", i] = _Bar(1)
            bars["UNITEMPTY", i] = _Bar(9)
        wait = _waiter(bars)
        tc, tma = [], []            # in-order queues: tensor pipe, TMA
        completed = set()           # finished products
        loaded = set()              # finished loads
        slot = [None, None]         # unit-index ring
        slot_readers = [set(), set()]
        kv_readers, stage_readers, acc_writers = {}, {}, {}
        acc_read = {}               # (kind, uc) -> warps that read it out
        half_readers = {}           # (panel pair, g) -> products reading those panels of step g
        step_dh = {}                # g -> the output-column half of step g's unit
        stats_read = {}             # g -> compute warps done with step g's row statistics
        p_handed = {}               # g -> compute warps that handed over step g's Pᵀ
        dv_prod = {}                # g -> id of step g's dV product
        kt_writes = {}              # uc -> drain warps that wrote the unit's Kᵀ
        kt_readers = {}             # uc -> the unit's dQᵀ products
        ds_readers = {}             # g -> products reading step g's shared-memory dSᵀ tile
        prod_info = {}
        prod_id = [0]

        def issue(kind, uc, g):
            prod_id[0] += 1
            i = prod_id[0]
            tc.append(("mma", i))
            prod_info[i] = (kind, uc, g)
            if kind == "dV":
                dv_prod[g] = i
            if kind == "dQ" and kt_tmem:
                kt_readers.setdefault(uc, set()).add(i)
            if kind == "dQ" or (kind == "dK" and dk_ss):
                ds_readers.setdefault(g, set()).add(i)
            if kind in ("S", "dP", "dQ", "S_A", "S_B", "dP_A", "dP_B"):
                kv_readers.setdefault(uc, set()).add(i)
            if kind in ("S", "dP", "dV", "dK"):
                stage_readers.setdefault(g, set()).add(i)
            if kind in ("S_A", "dP_A"):
                half_readers.setdefault((1 - step_dh[g], g), set()).add(i)
            if kind in ("S_B", "dP_B") or (halves and kind in ("dV", "dK")):
                half_readers.setdefault((step_dh[g], g), set()).add(i)
            if kind in ("dV", "dK"):
                acc_writers.setdefault(uc, set()).add(i)
                if uc > 0:
                    assert acc_read.get((kind, uc - 1), 0) == 4, f"{kind} of unit {uc} overwrites unread TMEM"

        def commit(name):
            tc.append(("commit", name))

        def next_unit(uc, who):
            yield from wait(("UNITFULL", uc & 1), uc >> 1)
            entry = slot[uc & 1]
            assert entry is not None and entry[0] == uc, f"{who} read slot of unit {entry} for {uc}"
            assert who not in slot_readers[uc & 1]
            slot_readers[uc & 1].add(who)
            yield
            bars["UNITEMPTY", uc & 1].arrive()
            return entry[1]

        def producer():
            gs = uc = 0
            while True:
                idx = counter[0]
                counter[0] += 1
                yield
                if uc >= 2 and mistake != "no_unit_empty_wait":
                    yield from wait(("UNITEMPTY", uc & 1), (uc >> 1) - 1)
                    assert len(slot_readers[uc & 1]) == 9
                slot[uc & 1] = (uc, idx)
                slot_readers[uc & 1] = set()
                bars["UNITFULL", uc & 1].arrive()
                if idx >= len(unit_len):
                    return
                n = unit_len[idx]
                dh = unit_dh[idx]

                def load_halves(s):
                    # the unit's dh picks which panel pair is half A (1 - dh) and half B (dh)
                    g = gs + s
                    step_dh[g] = dh
                    if g >= 1:
                        yield from wait("HAEMPTY", g - 1)
                        if s == 0 and mistake != "no_unit_start_half_b_wait":
                            # the previous unit's half B may be this half A
                            yield from wait("HBEMPTY", g - 1)
                        assert half_readers.get((1 - dh, g - 1), set()) <= completed, \
                            f"panels {1 - dh} of step {g} reused"
                    tma.append(("HAFULL", ("QA", g)))
                    if g >= 1:
                        if mistake != "no_half_b_empty_wait":
                            yield from wait("HBEMPTY", g - 1)
                        assert half_readers.get((dh, g - 1), set()) <= completed, f"panels {dh} of step {g} reused"
                        assert stats_read.get(g - 1, 0) == 4, f"statistics of step {g} overwritten while read"
                    tma.append(("QBFULL", ("QB", g)))
                    tma.append(("DOBFULL", ("DOB", g)))

                def load_q(s):
                    if halves:
                        yield from load_halves(s)
                        return
                    g = gs + s
                    if g >= n_stage:
                        yield from wait(("QEMPTY", g % n_stage), g // n_stage - 1)
                        assert stage_readers.get(g - n_stage, set()) <= completed, f"stage of step {g} reused"
                    tma.append((("QFULL", g % n_stage), ("Q", g)))
                pre = min(1 if halves else n_stage, n)
                for s in range(pre):
                    yield from load_q(s)
                if uc > 0:
                    yield from wait("KVEMPTY", uc - 1)
                    assert kv_readers.get(uc - 1, set()) <= completed, "K/V reloaded while read"
                tma.append(("KVFULL", ("KV", uc)))
                for s in range(pre, n):
                    yield from load_q(s)
                gs += n
                uc += 1

        def mma():
            gs = uc = 0
            while True:
                idx = yield from next_unit(uc, "mma")
                if idx >= len(unit_len):
                    return
                n = unit_len[idx]
                yield from wait("KVFULL", uc)
                assert ("KV", uc) in loaded

                def wait_q(g):
                    yield from wait(("QFULL", g % n_stage), g // n_stage)
                    assert ("Q", g) in loaded
                if halves:
                    for s in range(n):
                        g = gs + s
                        if s == 0:
                            # later steps' Sᵀ over half A was issued during the previous step
                            yield from wait("HAFULL", g)
                            assert ("QA", g) in loaded
                            issue("S_A", uc, g)
                        yield from wait("QBFULL", g)
                        assert ("QB", g) in loaded
                        issue("S_B", uc, g)
                        commit(("SFULL", g & 1))
                        issue("dP_A", uc, g)
                        yield from wait("DOBFULL", g)
                        assert ("DOB", g) in loaded
                        issue("dP_B", uc, g)
                        commit("DPFULL")
                        commit("HAEMPTY")
                        yield from wait(("PFULL", g & 1), g >> 1)
                        if s == 0 and uc > 0 and mistake != "no_dvfree_wait":
                            yield from wait("DVFREE", uc - 1)
                        issue("dV", uc, g)
                        if s + 1 < n and mistake != "s_a_before_dv":
                            # the next step's Sᵀ over half A fills the wait for dSᵀ
                            yield from wait("HAFULL", g + 1)
                            assert ("QA", g + 1) in loaded
                            issue("S_A", uc, g + 1)
                        yield from wait("DSFULL", g)
                        if s == 0 and uc > 0:
                            yield from wait("DKFREE", uc - 1)
                        issue("dK", uc, g)
                        commit("HBEMPTY")
                        if g > 0:
                            yield from wait("DQEMPTY", g - 1)
                        issue("dQ", uc, g)
                        commit("DQFULL")
                    commit("ACC")
                    commit("KVEMPTY")
                    done_units.append(idx)
                    gs += n
                    uc += 1
                    continue
                for k in range(min(lookahead, n)):
                    yield from wait_q(gs + k)
                    issue("S", uc, gs + k)
                    commit(("SFULL", (gs + k) & 1))
                issue("dP", uc, gs)
                commit("DPFULL")
                for s in range(n):
                    g = gs + s
                    if st_single and mistake == "s_before_dv" and s + 1 < n:
                        yield from wait_q(g + 1)
                        issue("S", uc, g + 1)
                        commit(("SFULL", (g + 1) & 1))
                    yield from wait(("PFULL", g & 1), g >> 1)
                    if s == 0 and uc > 0 and mistake != "no_dvfree_wait":
                        yield from wait("DVFREE", uc - 1)
                    issue("dV", uc, g)
                    if st_single and mistake != "s_before_dv" and s + 1 < n:
                        # one Sᵀ buffer: the next step's Sᵀ right after dV
                        yield from wait_q(g + 1)
                        issue("S", uc, g + 1)
                        commit(("SFULL", (g + 1) & 1))
                    yield from wait("DSFULL", g)
                    if s == 0 and uc > 0:
                        yield from wait("DKFREE", uc - 1)
                    late_dk = mistake == "dk_after_next_dp"
                    if not late_dk:
                        issue("dK", uc, g)
                        commit(("QEMPTY", g % n_stage))
                    if g > 0:
                        yield from wait("DQEMPTY", g - 1)
                    if kt_tmem and s == 0 and mistake != "no_ktfull_wait":
                        yield from wait("KTFULL", uc)
                    issue("dQ", uc, g)
                    commit("DQFULL")
                    if s + 1 < n:
                        if lookahead == 1 and not st_single:
                            yield from wait_q(g + 1)
                        issue("dP", uc, g + 1)
                        commit("DPFULL")
                    if late_dk:
                        issue("dK", uc, g)
                        commit(("QEMPTY", g % n_stage))
                    if not st_single and s + lookahead < n:
                        g2 = g + lookahead
                        if lookahead > 1:
                            yield from wait_q(g2)
                        issue("S", uc, g2)
                        commit(("SFULL", g2 & 1))
                commit("ACC")
                commit("KVEMPTY")
                done_units.append(idx)
                gs += n
                uc += 1

        def epilogue_warp(w, kind, free_bar):
            # compute warps (kind "dK") or drain warps (kind "dV")
            gs = uc = 0
            while True:
                idx = yield from next_unit(uc, (kind, w))
                if idx >= len(unit_len):
                    return
                n = unit_len[idx]
                if kind == "dV" and kt_tmem:
                    if mistake != "kt_before_kvfull":
                        yield from wait("KVFULL", uc)
                    assert ("KV", uc) in loaded, f"Kᵀ of unit {uc} read from an unloaded K tile"
                    assert kt_readers.get(uc - 1, set()) <= completed, f"Kᵀ of unit {uc - 1} overwritten while read"
                    yield
                    kt_writes[uc] = kt_writes.get(uc, 0) + 1
                    bars["KTFULL"].arrive()
                for s in range(n):
                    g = gs + s
                    if kind == "dK":
                        if halves:
                            yield from wait("QBFULL", g)
                            assert ("QB", g) in loaded
                        else:
                            yield from wait(("QFULL", g % n_stage), g // n_stage)
                        yield from wait(("SFULL", g & 1), g >> 1)
                        yield
                        p_handed[g] = p_handed.get(g, 0) + 1
                        bars["PFULL", g & 1].arrive()
                        yield from wait("DPFULL", g)
                        if g > 0:
                            yield from wait("DQFULL", g - 1)
                            assert ds_readers.get(g - 1, set()) <= completed, f"dSᵀ tile of step {g - 1} overwritten while read"
                        yield
                        stats_read[g] = stats_read.get(g, 0) + 1
                        bars["DSFULL"].arrive()
                    else:
                        yield from wait("DQFULL", g)
                        yield
                        bars["DQEMPTY"].arrive()
                yield from wait("ACC", uc)
                assert acc_writers.get(uc, set()) <= completed
                yield
                acc_read[kind, uc] = acc_read.get((kind, uc), 0) + 1
                bars[free_bar].arrive()
                gs += n
                uc += 1

        nbuf = 1 if st_single else 2

        def tc_done(item):
            kind, x = item
            if kind == "commit":
                bars[x].arrive()
                return
            pk, puc, pg = prod_info[x]
            if pk == "S":
                # the Sᵀ buffer's previous content: Pᵀ of step pg - nbuf
                gp = pg - nbuf
                if gp in dv_prod or p_handed.get(gp, 0):
                    assert p_handed.get(gp, 0) == 4, f"Sᵀ of step {pg} overwrites Pᵀ of step {gp} being written"
                    assert dv_prod.get(gp) in completed, f"Sᵀ of step {pg} overwrites Pᵀ of step {gp} before dV read it"
            if pk == "dQ" and kt_tmem:
                assert kt_writes.get(puc, 0) == 4, f"dQᵀ of unit {puc} read a Kᵀ not fully written"
            completed.add(x)

        def tma_done(item):
            bar, what = item
            loaded.add(what)
            bars[bar].arrive()

        gens[c, "producer"] = producer()
        gens[c, "mma"] = mma()
        for w in range(4):
            gens[c, "compute", w] = epilogue_warp(w, "dK", "DKFREE")
            gens[c, "drain", w] = epilogue_warp(w, "dV", "DVFREE")
        engines[c, "tc"] = (tc, tc_done)
        engines[c, "tma"] = (tma, tma_done)

    for c in range(n_ctas):
        make_cta(c)
    _run(gens, engines, rnd)
    assert sorted(done_units) == list(range(len(unit_len))), "units lost or repeated"
    assert counter[0] == len(unit_len) + n_ctas


BWD_UNITS = ([1], [3, 1], [1, 1, 1, 1, 1], [5, 2, 8], [1, 7, 2, 1, 3], [2, 1, 3, 1, 1, 2, 5, 1])


@pytest.mark.parametrize("n_stage,lookahead", [(3, 2), (1, 1)])
@pytest.mark.parametrize("n_ctas", [1, 3])
def test_backward_protocol(n_stage, lookahead, n_ctas):
    for units in BWD_UNITS:
        for seed in range(4):
            simulate_bwd(units, n_ctas, n_stage, lookahead, seed)


@pytest.mark.parametrize("n_ctas", [1, 3])
def test_backward_protocol_half_stages(n_ctas):
    for units in BWD_UNITS:
        for seed in range(4):
            simulate_bwd(units, n_ctas, 1, 1, seed, halves=True)


@pytest.mark.parametrize("mistake", ["no_unit_empty_wait", "no_dvfree_wait"])
def test_backward_model_catches_a_missing_wait(mistake):
    caught = 0
    for seed in range(40):
        try:
            simulate_bwd([1, 1, 1, 1, 1, 1], 2, 3, 2, seed, mistake)
        except AssertionError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("n_stage,kt_tmem,st_single", [(4, True, False), (3, True, True), (3, False, True)])
@pytest.mark.parametrize("n_ctas", [1, 3])
def test_backward_protocol_kt_tmem_and_single_s_buffer(n_stage, kt_tmem, st_single, n_ctas):
    # d = 64: Kᵀ in TMEM, two Sᵀ buffers; d = 128: Kᵀ in TMEM, one Sᵀ buffer
    for units in BWD_UNITS:
        for seed in range(4):
            simulate_bwd(units, n_ctas, n_stage, 1 if st_single else 2, seed, kt_tmem=kt_tmem, st_single=st_single)


@pytest.mark.parametrize("n_ctas", [1, 3])
def test_backward_protocol_dk_from_shared_memory(n_ctas):
    # d = 64: dK reads dSᵀ from the shared-memory tile, Kᵀ in TMEM, two Sᵀ buffers
    for units in BWD_UNITS:
        for seed in range(4):
            simulate_bwd(units, n_ctas, 4, 2, seed, kt_tmem=True, dk_ss=True)


def test_backward_dk_from_shared_memory_model_catches_a_late_dk():
    caught = 0
    for seed in range(40):
        try:
            simulate_bwd([2, 1, 3, 1, 2, 1], 2, 4, 2, seed, "dk_after_next_dp", kt_tmem=True, dk_ss=True)
        except AssertionError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("mistake", ["no_ktfull_wait", "kt_before_kvfull", "s_before_dv"])
def test_backward_kt_tmem_model_catches_a_missing_wait(mistake):
    caught = 0
    for seed in range(40):
        try:
            simulate_bwd([2, 1, 3, 1, 2, 1], 2, 3, 1, seed, mistake, kt_tmem=True, st_single=True)
        except AssertionError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("mistake", ["no_half_b_empty_wait", "no_unit_start_half_b_wait"])
def test_backward_half_stage_model_catches_a_missing_wait(mistake):
    caught = 0
    for seed in range(40):
        try:
            simulate_bwd([2, 3, 1, 2, 1, 2], 2, 1, 1, seed, mistake, halves=True)
        except AssertionError:
            caught += 1
    assert caught > 0


# ----------------------------------------------------------------- forward
def simulate_fwd_single(n_qtiles, BH, causal, n_ctas, n_slot, seed, mistake=None):
    """fa_fwd_persistent_kernel at d = 128: items are pairs of 128-row query
    tiles of one (b, h), dealt to ``n_ctas`` CTAs in a fixed order.  Roles
    per CTA: the producer, one MMA warp for both tiles and the two softmax
    warpgroups (one per query tile).  K and V blocks are separate "units" streamed through ``n_slot``
    slots; with a causal mask the second tile's diagonal block comes first."""
    rnd = random.Random(seed)
    n_pairs = (n_qtiles + 1) // 2
    n_items = n_pairs * BH
    issued = {"S": [], "PV": []}

    def item(idx):
        if causal:
            pair, bh = n_pairs - 1 - idx // BH, idx % BH
        else:
            bh, pair = idx // n_pairs, idx % n_pairs
        qt0 = 2 * pair
        has1 = qt0 + 1 < n_qtiles
        n0 = qt0 + 1 if causal else n_qtiles
        n1 = (qt0 + 2 if causal else n_qtiles) if has1 else 0
        skew = 1 if (causal and has1) else 0
        return dict(qt0=qt0, n0=n0, n1=n1, skew=skew, nit=n0 + skew)

    def kv_block(w, jj):
        return w["qt0"] + 1 if (w["skew"] and jj == 0) else jj - w["skew"]

    def first(w, t):
        return w["skew"] if t == 0 else 0

    def has(w, t):
        return t == 0 or w["n1"] > 0

    def deal(k, c):
        return k * n_ctas + ((n_ctas - 1 - c) if (causal and (k & 1)) else c)

    n_rounds = (n_items + n_ctas - 1) // n_ctas
    gens, engines = {}, {}
    all_items = []

    def make_cta(c):
        items = [deal(k, c) for k in range(n_rounds) if deal(k, c) < n_items]
        all_items.extend(items)
        bars = {}
        for t in range(2):
            for nm in ("QFULL", "QEMPTY", "SFULL", "ODONE"):
                bars[nm, t] = _Bar(1)
            bars["PFULL", t] = _Bar(4)
            bars["PFULL2", t] = _Bar(4)
        for s in range(n_slot):
            bars["KVFULL", s] = _Bar(1)
            bars["KVEMPTY", s] = _Bar(1)
        wait = _waiter(bars)
        tc, tma = [], []
        slot_unit, released, loaded = {}, set(), set()
        q_tile = {0: None, 1: None}
        readers = {}
        unit_of = {}
        u_acc = 0
        for idx in items:
            for u in range(2 * item(idx)["nit"]):
                unit_of[u_acc + u] = (idx, u)
            u_acc += 2 * item(idx)["nit"]

        def producer():
            useq = 0
            q_loads = [0, 0]
            for idx in items:
                w = item(idx)
                for t in range(2):
                    if not has(w, t):
                        continue
                    if q_loads[t] > 0 and mistake != "no_qempty_wait":
                        yield from wait(("QEMPTY", t), q_loads[t] - 1)
                    q_tile[t] = (idx, t)
                    tma.append((("QFULL", t), None))
                    q_loads[t] += 1
                for u in range(2 * w["nit"]):
                    U = useq + u
                    s = U % n_slot
                    if U >= n_slot:
                        yield from wait(("KVEMPTY", s), U // n_slot - 1)
                    if s in slot_unit:
                        assert slot_unit[s] in released, f"slot {s} refilled while unit {slot_unit[s]} is read"
                    slot_unit[s] = U
                    tma.append((("KVFULL", s), U))
                useq += 2 * w["nit"]

        def mma():
            waited = [-1]
            q_seen = [0, 0]
            p_seen = [0, 0]

            def wait_upto(U):
                # K/V units are waited in load order, never skipping one
                while waited[0] < U:
                    waited[0] += 1
                    yield from wait(("KVFULL", waited[0] % n_slot), waited[0] // n_slot)
                    assert waited[0] in loaded

            def release(U, w, jj, t_read):
                readers.setdefault(U, set()).add(t_read)
                if t_read == 1 or w["n1"] == 0:
                    need = {t for t in range(2) if has(w, t) and jj >= first(w, t)}
                    assert readers[U] == need
                    released.add(U)
                    tc.append(("commit", ("KVEMPTY", U % n_slot)))

            def issue_s(t, w, idx, base, jj):
                if jj == first(w, t):
                    yield from wait(("QFULL", t), q_seen[t])
                    q_seen[t] += 1
                assert q_tile[t] == (idx, t), f"Q tile {t} overwritten: {q_tile[t]} for item {idx}"
                U = base + 2 * jj
                yield from wait_upto(U)
                assert unit_of[U] == (idx, 2 * jj) and U not in released
                issued["S"].append((idx, t, kv_block(w, jj)))
                tc.append(("commit", ("SFULL", t)))
                if jj == w["nit"] - 1:
                    tc.append(("commit", ("QEMPTY", t)))
                release(U, w, jj, t)

            if not items:
                return
            idx, w, base = items[0], item(items[0]), 0
            for t in range(2):
                if has(w, t):
                    yield from issue_s(t, w, idx, base, first(w, t))
            for pos in range(len(items)):
                nxt = items[pos + 1] if pos + 1 < len(items) else None
                w2 = item(nxt) if nxt is not None else None
                base2 = base + 2 * w["nit"]
                for jj in range(w["nit"]):
                    for t in range(2):
                        if not has(w, t) or jj < first(w, t):
                            continue
                        Uv = base + 2 * jj + 1
                        yield from wait(("PFULL", t), p_seen[t])
                        yield from wait_upto(Uv)
                        assert unit_of[Uv] == (idx, 2 * jj + 1) and Uv not in released
                        yield from wait(("PFULL2", t), p_seen[t])
                        issued["PV"].append((idx, t, kv_block(w, jj)))
                        tc.append(("commit", ("ODONE", t)))
                        p_seen[t] += 1
                        release(Uv, w, jj, t)
                        if jj + 1 < w["nit"]:
                            yield from issue_s(t, w, idx, base, jj + 1)
                        elif nxt is not None and has(w2, t):
                            # the next item's first QKᵀ right after this tile's last PV
                            yield from issue_s(t, w2, nxt, base2, first(w2, t))
                if nxt is None:
                    break
                if not has(w, 1) and has(w2, 1):
                    yield from issue_s(1, w2, nxt, base2, 0)
                idx, w, base = nxt, w2, base2

        def softmax(t):
            done = 0
            for idx in items:
                w = item(idx)
                if not has(w, t):
                    continue
                n = w["n0"] if t == 0 else w["n1"]
                for j in range(n):
                    yield from wait(("SFULL", t), done + j)
                    if j > 0 and rnd.random() < 0.3:   # conditional rescale of O
                        yield from wait(("ODONE", t), done + j - 1)
                    for _ in range(4):
                        bars["PFULL", t].arrive()
                    yield
                    for _ in range(4):
                        bars["PFULL2", t].arrive()
                yield from wait(("ODONE", t), done + n - 1)
                done += n

        def tc_done(entry):
            bars[entry[1]].arrive()

        def tma_done(entry):
            bar, unit = entry
            if unit is not None:
                loaded.add(unit)
            bars[bar].arrive()

        gens[c, "producer"] = producer()
        gens[c, "mma"] = mma()
        gens[c, "softmax", 0] = softmax(0)
        gens[c, "softmax", 1] = softmax(1)
        engines[c, "tc"] = (tc, tc_done)
        engines[c, "tma"] = (tma, tma_done)

    for c in range(n_ctas):
        make_cta(c)
    _run(gens, engines, rnd)
    assert sorted(all_items) == list(range(n_items))
    # every query tile met exactly the K/V blocks the mask leaves visible, once each
    for kind in ("S", "PV"):
        got = sorted(issued[kind])
        want = []
        for idx in range(n_items):
            w = item(idx)
            for t in range(2):
                if has(w, t):
                    qt = w["qt0"] + t
                    want += [(idx, t, j) for j in (range(qt + 1) if causal else range(n_qtiles))]
        assert got == sorted(want), kind


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_slot", [5, 8])
def test_forward_single_mma_warp_protocol(causal, n_slot):
    for n_qtiles in (1, 2, 3, 5, 8):
        for BH, n_ctas in ((1, 1), (3, 2), (5, 3)):
            simulate_fwd_single(n_qtiles, BH, causal, n_ctas, n_slot, seed=n_qtiles * 7 + BH)


def test_forward_single_mma_warp_model_catches_a_missing_wait():
    caught = 0
    for seed in range(20):
        try:
            simulate_fwd_single(4, 3, True, 1, 5, seed, mistake="no_qempty_wait")
        except AssertionError:
            caught += 1
    assert caught > 0


# ------------------------------------------------------------ forward, CTA pair
def simulate_fwd(n_qtiles, BH, causal, n_ctas, n_slot, seed, sep_p=False, mistake=None, max_steps=20_000_000):
    """fa_fwd_persistent_kernel: items are pairs of 128-row query tiles of one
    (b, h), dealt to ``n_ctas`` CTAs in a fixed order.  Roles per CTA: the
    producer, one MMA warp and one softmax warpgroup per query tile.  K and V
    blocks are separate "units" streamed through ``n_slot`` slots; with a
    causal mask the second tile's diagonal block comes first.

    At d = 64, MMA warp t issues tile t's QKᵀ and PV products only.  Both warps walk every K/V unit
    in load order and commit its release (the slot's empty barrier counts two
    arrivals), so the producer refills a slot only after both are done with
    it; a warp waits only for the units its tile reads.  ``sep_p`` (d = 64):
    P has its own TMEM columns, so a tile's next QKᵀ of the same item is
    issued as soon as the softmax has read S (SFREE), and the softmax waits
    for the previous PV before it writes P."""
    rnd = random.Random(seed)
    n_pairs = (n_qtiles + 1) // 2
    n_items = n_pairs * BH
    issued = {"S": [], "PV": []}

    def item(idx):
        if causal:
            pair, bh = n_pairs - 1 - idx // BH, idx % BH
        else:
            bh, pair = idx // n_pairs, idx % n_pairs
        qt0 = 2 * pair
        has1 = qt0 + 1 < n_qtiles
        n0 = qt0 + 1 if causal else n_qtiles
        n1 = (qt0 + 2 if causal else n_qtiles) if has1 else 0
        skew = 1 if (causal and has1) else 0
        return dict(qt0=qt0, n0=n0, n1=n1, skew=skew, nit=n0 + skew)

    def kv_block(w, jj):
        return w["qt0"] + 1 if (w["skew"] and jj == 0) else jj - w["skew"]

    def first(w, t):
        return w["skew"] if t == 0 else 0

    def has(w, t):
        return t == 0 or w["n1"] > 0

    def deal(k, c):
        return k * n_ctas + ((n_ctas - 1 - c) if (causal and (k & 1)) else c)

    n_rounds = (n_items + n_ctas - 1) // n_ctas
    gens, engines = {}, {}
    all_items = []

    def make_cta(c):
        items = [deal(k, c) for k in range(n_rounds) if deal(k, c) < n_items]
        all_items.extend(items)
        bars = {}
        for t in range(2):
            for nm in ("QFULL", "QEMPTY", "SFULL", "ODONE"):
                bars[nm, t] = _Bar(1)
            bars["PFULL", t] = _Bar(4)
            bars["PFULL2", t] = _Bar(4)
            bars["SFREE", t] = _Bar(4)
        for s in range(n_slot):
            bars["KVFULL", s] = _Bar(1)
            bars["KVEMPTY", s] = _Bar(2)
        wait = _waiter(bars)
        tc, tma = [], []
        slot_unit, loaded = {}, set()
        q_tile = {0: None, 1: None}
        unit_readers = {}           # unit -> ids of products that read it
        completed = set()
        commits = {}                # unit -> release commits that completed
        s_issued, s_read = [0, 0], [0, 0]
        p_written, pv_done = [0, 0], [0, 0]
        prod_id = [0]
        unit_of = {}
        u_acc = 0
        for idx in items:
            for u in range(2 * item(idx)["nit"]):
                unit_of[u_acc + u] = (idx, u)
            u_acc += 2 * item(idx)["nit"]

        def producer():
            useq = 0
            q_loads = [0, 0]
            for idx in items:
                w = item(idx)
                for t in range(2):
                    if not has(w, t):
                        continue
                    if q_loads[t] > 0 and mistake != "no_qempty_wait":
                        yield from wait(("QEMPTY", t), q_loads[t] - 1)
                    q_tile[t] = (idx, t)
                    tma.append((("QFULL", t), None))
                    q_loads[t] += 1
                for u in range(2 * w["nit"]):
                    U = useq + u
                    s = U % n_slot
                    if U >= n_slot:
                        yield from wait(("KVEMPTY", s), U // n_slot - 1)
                    if s in slot_unit:
                        old = slot_unit[s]
                        assert commits.get(old, 0) == 2, f"slot {s} refilled before both warps released unit {old}"
                        assert unit_readers.get(old, set()) <= completed, f"slot {s} refilled while unit {old} is read"
                    slot_unit[s] = U
                    tma.append((("KVFULL", s), U))
                useq += 2 * w["nit"]

        def mma(t):
            q_seen = [0]
            p_seen = [0]

            def wait_unit(U):
                yield from wait(("KVFULL", U % n_slot), U // n_slot)
                assert U in loaded and slot_unit[U % n_slot] == U

            def product(kind, U):
                prod_id[0] += 1
                unit_readers.setdefault(U, set()).add(prod_id[0])
                tc.append(("mma", prod_id[0]))

            def release(U):
                if mistake == "one_release_only" and t == 0:
                    return
                tc.append(("release", U))

            def issue_s(w, idx, base, jj):
                if sep_p and s_issued[t] > 0 and mistake != "no_sfree_wait":
                    yield from wait(("SFREE", t), s_issued[t] - 1)
                assert s_read[t] == s_issued[t], f"S buffer {t} overwritten before it was read"
                s_issued[t] += 1
                if jj == first(w, t):
                    yield from wait(("QFULL", t), q_seen[0])
                    q_seen[0] += 1
                assert q_tile[t] == (idx, t), f"Q tile {t} overwritten: {q_tile[t]} for item {idx}"
                U = base + 2 * jj
                yield from wait_unit(U)
                assert unit_of[U] == (idx, 2 * jj)
                product("S", U)
                issued["S"].append((idx, t, kv_block(w, jj)))
                tc.append(("commit", ("SFULL", t)))
                if jj == w["nit"] - 1:
                    tc.append(("commit", ("QEMPTY", t)))
                release(U)

            if not items:
                return
            idx, w, base = items[0], item(items[0]), 0
            if has(w, t):
                yield from issue_s(w, idx, base, first(w, t))
            for pos in range(len(items)):
                nxt = items[pos + 1] if pos + 1 < len(items) else None
                w2 = item(nxt) if nxt is not None else None
                base2 = base + 2 * w["nit"]
                for jj in range(w["nit"]):
                    if not has(w, t) or jj < first(w, t):
                        # units this tile does not read: release each once it
                        # holds this fill (a release ahead of the load would
                        # count towards the slot's previous fill)
                        for U in (base + 2 * jj, base + 2 * jj + 1):
                            if mistake != "release_before_load":
                                yield from wait_unit(U)
                            release(U)
                        continue
                    if sep_p and jj + 1 < w["nit"]:
                        yield from issue_s(w, idx, base, jj + 1)
                    Uv = base + 2 * jj + 1
                    yield from wait(("PFULL", t), p_seen[0])
                    yield from wait_unit(Uv)
                    yield from wait(("PFULL2", t), p_seen[0])
                    product("PV", Uv)
                    issued["PV"].append((idx, t, kv_block(w, jj)))
                    tc.append(("pv", t))
                    tc.append(("commit", ("ODONE", t)))
                    p_seen[0] += 1
                    release(Uv)
                    if jj + 1 < w["nit"]:
                        if not sep_p:
                            yield from issue_s(w, idx, base, jj + 1)
                    elif nxt is not None and has(w2, t):
                        yield from issue_s(w2, nxt, base2, first(w2, t))
                if nxt is None:
                    break
                if not has(w, t) and has(w2, t):
                    yield from issue_s(w2, nxt, base2, first(w2, t))
                idx, w, base = nxt, w2, base2

        def softmax(t):
            done = 0
            for idx in items:
                w = item(idx)
                if not has(w, t):
                    continue
                n = w["n0"] if t == 0 else w["n1"]
                for j in range(n):
                    yield from wait(("SFULL", t), done + j)
                    yield
                    s_read[t] += 1
                    if sep_p:
                        for _ in range(4):
                            bars["SFREE", t].arrive()
                        if j > 0:
                            yield from wait(("ODONE", t), done + j - 1)
                        assert pv_done[t] == p_written[t], f"P buffer {t} overwritten while a PV reads it"
                    elif j > 0 and rnd.random() < 0.3:
                        yield from wait(("ODONE", t), done + j - 1)
                    p_written[t] += 1
                    for _ in range(4):
                        bars["PFULL", t].arrive()
                    yield
                    for _ in range(4):
                        bars["PFULL2", t].arrive()
                yield from wait(("ODONE", t), done + n - 1)
                done += n

        def tc_done(entry):
            kind, x = entry
            if kind == "mma":
                completed.add(x)
            elif kind == "pv":
                pv_done[x] += 1
            elif kind == "release":
                commits[x] = commits.get(x, 0) + 1
                bars["KVEMPTY", x % n_slot].arrive()
            else:
                bars[x].arrive()

        def tma_done(entry):
            bar, unit = entry
            if unit is not None:
                loaded.add(unit)
            bars[bar].arrive()

        gens[c, "producer"] = producer()
        for t in range(2):
            gens[c, "mma", t] = mma(t)
            gens[c, "softmax", t] = softmax(t)
        engines[c, "tc"] = (tc, tc_done)
        engines[c, "tma"] = (tma, tma_done)

    for c in range(n_ctas):
        make_cta(c)
    _run(gens, engines, rnd, max_steps)
    assert sorted(all_items) == list(range(n_items))
    for kind in ("S", "PV"):
        got = sorted(issued[kind])
        want = []
        for idx in range(n_items):
            w = item(idx)
            for t in range(2):
                if has(w, t):
                    qt = w["qt0"] + t
                    want += [(idx, t, j) for j in (range(qt + 1) if causal else range(n_qtiles))]
        assert got == sorted(want), kind


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_slot", [8, 5])
def test_forward_per_tile_mma_warp_protocol(causal, n_slot):
    for n_qtiles in (1, 2, 3, 5, 8):
        for BH, n_ctas in ((1, 1), (3, 2), (5, 3)):
            simulate_fwd(n_qtiles, BH, causal, n_ctas, n_slot, seed=n_qtiles * 7 + BH, sep_p=True)


@pytest.mark.parametrize("mistake", ["no_qempty_wait", "no_sfree_wait", "one_release_only", "release_before_load"])
def test_forward_per_tile_model_catches_a_missing_wait(mistake):
    caught = 0
    for seed in range(30):
        try:
            simulate_fwd(3, 3, seed % 2 == 1, 1, 5, seed, True, mistake, max_steps=200_000)
        except AssertionError:
            caught += 1
    assert caught > 0


def simulate_fwd_pair(n0, n1, n_slot, seed, mistake=None, max_steps=20_000_000):
    """fa_fwd_pair_kernel: one cluster of two CTAs, each with two query tiles;
    tile pair t (one tile in each CTA) multiplies K/V blocks 0 .. n_t - 1,
    n0 <= n1.  Both CTAs' producers load their Q tiles and their halves of
    every K/V unit (K(0), V(0), K(1), V(1), ...), counted on the leader's
    barriers, which the leader's producer arms; the leader's MMA warp issues
    every product on one tensor pipe and commits to the barrier of the same
    name in both CTAs; the softmax warps of tile pair t in both CTAs (four per
    CTA, modelled as one role per CTA) arrive on the leader's P barriers of
    tile pair t."""
    assert 1 <= n0 <= n1
    rnd = random.Random(seed)
    n_of = (n0, n1)
    bars = {}
    for r in range(2):
        for s in range(n_slot):
            bars[r, "KVEMPTY", s] = _Bar(1)
        for t in range(2):
            bars[r, "SFULL", t] = _Bar(1)
            bars[r, "ODONE", t] = _Bar(1)
        bars[r, "DRAIN"] = _Bar(1)
    bars[0, "QFULL"] = _Bar(3)           # the leader's arming arrival + both CTAs' Q loads
    for s in range(n_slot):
        bars[0, "KVFULL", s] = _Bar(3)   # the leader's arming arrival + two halves
    for t in range(2):
        bars[0, "PFULL", t] = _Bar(8)
        bars[0, "PFULL2", t] = _Bar(8)
    wait = _waiter(bars)
    tc, tma = [], {0: [], 1: []}
    halves = {}                 # unit -> halves landed
    slot_unit = {}              # (cta, slot) -> unit
    read_done = set()           # units whose last reading product has completed
    p_phase_blocks = {}         # (name, t, phase) -> blocks of the arrivals
    p_count = {}
    issued = []

    def producer(r):
        if r == 0:
            bars[0, "QFULL"].arrive()
        tma[r].append(((0, "QFULL"), None))
        for u in range(2 * n1):
            s = u % n_slot
            if u >= n_slot and mistake != "no_kvempty_wait":
                yield from wait((r, "KVEMPTY", s), u // n_slot - 1)
            if (r, s) in slot_unit:
                assert slot_unit[r, s] in read_done, f"cta {r} slot {s} refilled while unit {slot_unit[r, s]} is read"
            slot_unit[r, s] = u
            if r == 0:
                bars[0, "KVFULL", s].arrive()
            tma[r].append(((0, "KVFULL", s), u))
            yield

    def mma():
        yield from wait((0, "QFULL"), 0)
        waited = [-1]

        def wait_upto(u):
            while waited[0] < u:
                waited[0] += 1
                yield from wait((0, "KVFULL", waited[0] % n_slot), waited[0] // n_slot)
                assert halves.get(waited[0]) == 2

        def issue_s(t, j):
            yield from wait_upto(2 * j)
            assert 2 * j not in read_done
            issued.append(("S", t, j))
            tc.append(("commit", "SFULL", t))
            if t == 1 and mistake != "release_k_early":
                tc.append(("release", 2 * j))
            if t == 0 and mistake == "release_k_early":
                tc.append(("release", 2 * j))

        yield from issue_s(0, 0)
        yield from issue_s(1, 0)
        for j in range(n1):
            for t in range(2):
                if j >= n_of[t]:
                    continue
                yield from wait((0, "PFULL", t), j)
                assert p_phase_blocks[("PFULL", t, j)] == {j}, "P barrier phase mixes blocks"
                yield from wait_upto(2 * j + 1)
                assert 2 * j + 1 not in read_done
                yield from wait((0, "PFULL2", t), j)
                assert p_phase_blocks[("PFULL2", t, j)] == {j}, "P barrier phase mixes blocks"
                issued.append(("PV", t, j))
                tc.append(("commit", "ODONE", t))
                if t == 1:
                    tc.append(("release", 2 * j + 1))
                if j + 1 < n_of[t]:
                    yield from issue_s(t, j + 1)
        tc.append(("commit", "DRAIN", None))
        yield from wait((0, "DRAIN"), 0)

    def softmax(r, t):
        n = n_of[t]
        for j in range(n):
            yield from wait((r, "SFULL", t), j)
            if j > 0 and rnd.random() < 0.3:      # conditional rescale of O_t
                yield from wait((r, "ODONE", t), j - 1)
            for name in ("PFULL", "PFULL2"):
                key = (name, t)
                ph = p_count.get(key, 0) // 8
                p_phase_blocks.setdefault((name, t, ph), set()).add(j)
                for _ in range(4):
                    p_count[key] = p_count.get(key, 0) + 1
                    bars[0, name, t].arrive()
                yield
        yield from wait((r, "ODONE", t), n - 1)

    def tc_done(entry):
        kind = entry[0]
        if kind == "commit":
            _, name, t = entry
            for r in range(2):                    # multicast to both CTAs
                bars[(r, name) if t is None else (r, name, t)].arrive()
        else:
            u = entry[1]
            read_done.add(u)
            for r in range(2):
                bars[r, "KVEMPTY", u % n_slot].arrive()

    def tma_done(entry):
        bar, unit = entry
        if unit is not None:
            halves[unit] = halves.get(unit, 0) + 1
        bars[bar].arrive()

    gens = {"producer0": producer(0), "producer1": producer(1), "mma": mma()}
    for r in range(2):
        for t in range(2):
            gens[f"softmax{r}{t}"] = softmax(r, t)
    engines = {"tc": (tc, tc_done), "tma0": (tma[0], tma_done), "tma1": (tma[1], tma_done)}
    _run(gens, engines, rnd, max_steps)
    for t in range(2):
        assert [x for x in issued if x[:2] == ("PV", t)] == [("PV", t, j) for j in range(n_of[t])]
        assert [x for x in issued if x[:2] == ("S", t)] == [("S", t, j) for j in range(n_of[t])]


@pytest.mark.parametrize("n_slot", [9, 3])
def test_forward_pair_protocol(n_slot):
    for n0, n1 in ((1, 1), (1, 3), (2, 4), (6, 6)):
        for seed in range(3):
            simulate_fwd_pair(n0, n1, n_slot, seed=seed * 31 + n1)


@pytest.mark.parametrize("mistake", ["no_kvempty_wait", "release_k_early"])
def test_forward_pair_model_catches_a_mistake(mistake):
    caught = 0
    for seed in range(12):
        try:
            simulate_fwd_pair(3, 5, 3, seed, mistake=mistake, max_steps=200_000)
        except AssertionError:
            caught += 1
            break
    assert caught > 0
