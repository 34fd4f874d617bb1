"""CPU test: the GEMM kernels' barrier protocols cannot deadlock, alias a phase or race on a
partial for the launch plans they use (every layer shape of the configurations, every ring
size the planner can pick, short and ragged stream-K ranges). The model lives in
schedule_model.py.

``simulate`` models the small-tile kernel as built (one A slot per residue) and the candidates
measured against it; ``simulate_large`` the large-tile kernel. ``simulate_ring`` (the
``test_ring_*`` tests) models a small-tile protocol that was built, run through every GPU
parity test and measured slower on B200: dequantised k-blocks in a ring of 4, 6 or 8 A slots
indexed by walk position, chunks fixed by walk position. Its tests keep the hazards that model
found before that kernel ran (a slot's consecutive uses by different issuers, a partial barrier
that the residue's next k-block completes first)."""
import pytest

from schedule_model import simulate

SHAPES = [(4096, 4096), (4096, 12288), (4096, 22016), (11008, 4096), (8192, 10240), (8192, 8192),
          (8192, 57344), (28672, 8192), (128, 128), (384, 1000), (1024, 136)]


def _plan(K, N):
    kbs = K // 128
    units = -(-N // 128) * kbs
    return units, min(148, units), kbs


@pytest.mark.parametrize("K,N", SHAPES)
@pytest.mark.parametrize("slots", [5, 9, 13, 16, 17, 18])
def test_no_deadlock(K, N, slots):
    units, grid, kbs = _plan(K, N)
    if K * N > 8192 * 10240 and slots not in (16, 17):
        pytest.skip("large shapes: the ring sizes the planner picks for them")
    stuck = simulate(units, grid, kbs, min(4, slots // 2), slots)
    assert not stuck, stuck[:5]


def test_model_catches_slot_indexed_barrier_hazard():
    # chunk barriers indexed by ring slot (instead of chunk number) let a barrier advance two
    # phases while a role still waits for the older one; the GPU showed it as expired waits on
    # the 8192 x 10240 layer with a 17-slot ring. Chunk-number indexing removes it.
    import schedule_model as sm
    orig = sm.chunks

    def slot_indexed(beg, end, kbs, chunk, slots):
        uses = [0] * slots
        for seg, pos, c, it0, ch in orig(beg, end, kbs, chunk, slots):
            if pos is None:
                yield seg, pos, c, it0, ch
                continue
            # barrier number = slot + 33 * (uses of that slot), so that mod 33 is the slot and
            # the phase parity is the slot's use count
            yield seg, pos, c, it0, pos + sm.NCB * uses[pos]
            uses[pos] += 1
    import random
    sm.chunks = slot_indexed
    try:
        units, grid, kbs = _plan(8192, 10240)
        assert simulate(units, grid, kbs, 4, 17, rng=random.Random(0))
    finally:
        sm.chunks = orig
    assert not simulate(units, grid, kbs, 4, 17, rng=random.Random(0))


class _Biased:
    """An interleaving that always moves the roles `first` picks before the others (random
    order within each group), each as far as it can: the extreme schedules that let one kind
    of warp run ahead of the rest."""

    def __init__(self, first, seed):
        import random
        self.r, self.first = random.Random(seed), first

    def shuffle(self, order):
        keyed = sorted((0 if self.first(x[1]) else 1, self.r.random(), k) for k, x in enumerate(order))
        order[:] = [order[k[2]] for k in keyed]

    def randint(self, a, b):
        return 1 << 30


_KINDS = ["dq", "iss", "prod", "acc"]
_BIASES = {f"{k}-first": (lambda k: lambda n: n.startswith(k))(k) for k in _KINDS}
_BIASES.update({f"{k}-last": (lambda k: lambda n: not n.startswith(k))(k) for k in _KINDS})
_BIASES["one-dq-warp-first"] = lambda n: n == "dq0"
_BIASES["one-dq-warp-last"] = lambda n: n != "dq1"


@pytest.mark.parametrize("K,N", [(8192, 57344), (4096, 22016), (8192, 10240), (1024, 136)])
@pytest.mark.parametrize("slots", [9, 16, 17])
def test_no_alias_or_deadlock_under_skewed_schedules(K, N, slots):
    import random
    units, grid, kbs = _plan(K, N)
    for cta in sorted({0, grid // 2, grid - 1}):
        for name, first in _BIASES.items():
            problems = simulate(units, grid, kbs, min(4, slots // 2), slots, rng=_Biased(first, cta), ctas_only=[cta])
            assert not problems, (name, cta, problems[:3])
        for seed in range(3):
            problems = simulate(units, grid, kbs, min(4, slots // 2), slots, rng=random.Random(seed), ctas_only=[cta])
            assert not problems, ("random", seed, cta, problems[:3])


def test_model_catches_period_mismatch():
    # every barrier needs fixed participants: A slots indexed with a period (6) other than
    # that of the dequant residues and issuers (4) let a role wait on a slot two phases early
    # and pass on the parity of an older phase. An earlier version of the kernel had such a
    # mismatch; the GPU showed it as expired waits on the 8192 x 57344 layer.
    import schedule_model as sm
    units, grid, kbs = _plan(8192, 57344)

    def aliases():
        found = []
        for name, first in _BIASES.items():
            for cta in (0, 1, 5):
                found += [p for p in simulate(units, grid, kbs, 4, 9, rng=_Biased(first, cta), ctas_only=[cta])
                          if p[0] == "alias"]
        return found
    saved = sm.NA
    sm.NA = 6
    try:
        old = aliases()
    finally:
        sm.NA = saved
    assert any(p[3].startswith(("afull", "aempty")) for p in old)
    assert not aliases()


def test_first_contributor_closed_form():
    # the owner finds the CTA holding its tile's first unit in closed form; it must be the CTA
    # whose range [unit_start(c), unit_start(c + 1)) contains that unit
    import random
    from schedule_model import first_contributor, unit_start
    r = random.Random(3)
    cases = [(units, grid) for units in (1, 7, 148, 149, 1024, 5504, 28672, 200000) for grid in (1, 3, 148)]
    cases += [(r.randint(1, 10 ** 6), r.randint(1, 148)) for _ in range(200)]
    for units, grid in cases:
        grid = min(grid, units)
        for t in {0, units - 1, units // 2, r.randrange(units)}:
            c = first_contributor(t, units, grid)
            assert 0 <= c < grid
            assert unit_start(c, units, grid) <= t < unit_start(c + 1, units, grid), (units, grid, t, c)


def _plan_large(K, N):
    kbs = K // 128
    units = -(-N // 128) * kbs
    return units, min(148, units), kbs


@pytest.mark.parametrize("K,N", [(4096, 22016), (8192, 8192), (1024, 1024), (4096, 2048)])
@pytest.mark.parametrize("slots,issuers", [(5, 2), (9, 4), (3, 1), (11, 4)])
def test_large_tiles_no_alias_deadlock_or_race(K, N, slots, issuers):
    import random
    from schedule_model import simulate_large
    units, grid, kbs = _plan_large(K, N)
    for cta in sorted({0, grid // 2, grid - 1}):
        for name, first in _BIASES.items():
            problems = simulate_large(units, grid, kbs, min(4, slots // 2), slots, issuers,
                                      rng=_Biased(first, cta), ctas_only=[cta])
            assert not problems, (name, cta, problems[:3])
        problems = simulate_large(units, grid, kbs, min(4, slots // 2), slots, issuers,
                                  rng=random.Random(cta), ctas_only=[cta])
        assert not problems, ("random", cta, problems[:3])


def test_large_model_catches_missing_epilogue_barrier():
    # the dequant warps of one residue may reach the next segment (and let the MMA start a
    # fresh accumulation) while the other residue still reads the accumulators, unless every
    # segment's epilogue ends with a barrier over all dequant warps. An earlier version had
    # no such barrier after a whole-tile owner epilogue; the GPU showed it as wrong results.
    from schedule_model import simulate_large
    units, grid, kbs = _plan_large(4096, 22016)  # 37 units per CTA: whole-tile owner segments
    races = []
    for cta in range(20):
        for name, first in _BIASES.items():
            races += [p for p in simulate_large(units, grid, kbs, 2, 5, 2, rng=_Biased(first, cta), ctas_only=[cta],
                                                owner_barrier=False) if p[0] == "race"]
    assert races


def test_model_catches_partial_read_too_late():
    # a residue's k-blocks alternate between two partial buffers, so a dequant warp must read a
    # partial before it hands the k-block two uses later to the MMA: with the read delayed by
    # one more k-block, the MMA may overwrite a partial that was never read
    import random
    import schedule_model as sm
    units, grid, kbs = _plan(4096, 22016)
    saved = sm.READ_DELAY
    sm.READ_DELAY = 2
    try:
        races = []
        for seed in range(4):
            races += [p for p in simulate(units, grid, kbs, 4, 16, rng=random.Random(seed), ctas_only=[3])
                      if p[0] == "race"]
    finally:
        sm.READ_DELAY = saved
    assert races
    for seed in range(4):
        assert not simulate(units, grid, kbs, 4, 16, rng=random.Random(seed), ctas_only=[3])


@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 22016), (8192, 57344), (1024, 136)])
def test_candidate_two_a_slots_per_residue(K, N):
    # the candidate next design: 3 residues, each alternating between two A slots and two
    # partial buffers (6 A slots, 3 issuers, chunks of at most 3 k-blocks): no alias, no stuck
    # role, no partial overwritten before it is read, under skewed and random interleavings
    import random
    import schedule_model as sm
    units, grid, kbs = _plan(K, N)
    saved = (sm.NA, sm.NQ, sm.DQ_PERIOD, sm.TWO_A_SLOTS)
    sm.NA, sm.NQ, sm.DQ_PERIOD, sm.TWO_A_SLOTS = 6, 3, 3, True
    try:
        for cta in sorted({0, grid // 2, grid - 1}):
            for name, first in _BIASES.items():
                problems = simulate(units, grid, kbs, 3, 17, rng=_Biased(first, cta), ctas_only=[cta])
                assert not problems, (name, cta, problems[:3])
            for seed in range(3):
                problems = simulate(units, grid, kbs, 3, 17, rng=random.Random(seed), ctas_only=[cta])
                assert not problems, ("random", seed, cta, problems[:3])
    finally:
        sm.NA, sm.NQ, sm.DQ_PERIOD, sm.TWO_A_SLOTS = saved


def test_candidate_two_a_slots_needs_the_partial_read_before_the_signal():
    # in the candidate design the partial of k-block u - 2 must be read before k-block u is
    # handed to the MMA; reading it one k-block later lets the MMA of u overwrite it
    import random
    import schedule_model as sm
    units, grid, kbs = _plan(4096, 22016)
    saved = (sm.NA, sm.NQ, sm.DQ_PERIOD, sm.TWO_A_SLOTS)
    sm.NA, sm.NQ, sm.DQ_PERIOD, sm.TWO_A_SLOTS = 6, 3, 3, True
    orig = sm._roles

    def late(*args, **kw):
        roles = orig(*args, **kw)
        for name, gen in list(roles.items()):
            if name.startswith("dq"):
                roles[name] = _delay_reads(gen)
        return roles
    sm._roles = late
    try:
        races = []
        for seed in range(4):
            races += [p for p in simulate(units, grid, kbs, 3, 17, rng=random.Random(seed), ctas_only=[3])
                      if p[0] == "race"]
    finally:
        sm._roles = orig
        sm.NA, sm.NQ, sm.DQ_PERIOD, sm.TWO_A_SLOTS = saved
    assert races


def _delay_reads(gen):
    """Moves every partial read after the dequant warp's next A-slot signal."""
    held = []
    for op in gen:
        if op[0] == "part_read":
            held.append(op)
            continue
        yield op
        if op[0] == "arrive" and op[1].name.startswith("afull") and held:
            yield from held
            held = []
    yield from held


@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 22016), (8192, 57344), (1024, 136)])
def test_candidate_two_issuers_per_residue(K, N):
    # another candidate: 4 residues, each k-block's 8 MMAs split between two issuers with
    # partials of their own; the A-slot and ring-slot barriers then count two commits
    import random
    import schedule_model as sm
    units, grid, kbs = _plan(K, N)
    saved = sm.ISSUERS_PER_RESIDUE
    sm.ISSUERS_PER_RESIDUE = 2
    try:
        for cta in sorted({0, grid // 2, grid - 1}):
            for name, first in _BIASES.items():
                problems = simulate(units, grid, kbs, 4, 17, rng=_Biased(first, cta), ctas_only=[cta])
                assert not problems, (name, cta, problems[:3])
            for seed in range(3):
                problems = simulate(units, grid, kbs, 4, 17, rng=random.Random(seed), ctas_only=[cta])
                assert not problems, ("random", seed, cta, problems[:3])
    finally:
        sm.ISSUERS_PER_RESIDUE = saved


def _plan_pairs(K, N):
    kbs = K // 128
    units = -(-N // 256) * kbs  # (256-column tile pair, k-block) units
    return units, min(74, units), kbs


@pytest.mark.parametrize("K,N", [(8192, 8192), (4096, 22016), (1024, 1024), (4096, 2048)])
@pytest.mark.parametrize("slots,issuers", [(3, 1), (5, 2), (9, 4)])
def test_planned_cta_pair_large_tiles(K, N, slots, issuers):
    # the planned 2-SM form of the large-tile kernel: the leader's barriers count both CTAs'
    # arrivals and its commits are multicast to both; no alias, stuck role or accumulator race
    import random
    from schedule_model import simulate_large_pair
    units, grid, kbs = _plan_pairs(K, N)
    for pair in sorted({0, grid // 2, grid - 1}):
        for name, first in _BIASES.items():
            problems = simulate_large_pair(units, grid, kbs, min(4, slots // 2), slots, issuers,
                                           rng=_Biased(first, pair), pairs_only=[pair])
            assert not problems, (name, pair, problems[:3])
        problems = simulate_large_pair(units, grid, kbs, min(4, slots // 2), slots, issuers,
                                       rng=random.Random(pair), pairs_only=[pair])
        assert not problems, ("random", pair, problems[:3])


def test_cta_pair_model_catches_a_commit_that_reaches_one_cta():
    # without the multicast, the follower's dequant warps never see their A slots freed
    import schedule_model as sm
    units, grid, kbs = _plan_pairs(4096, 22016)
    sm.PAIR_MULTICAST_COMMIT = False
    try:
        problems = sm.simulate_large_pair(units, grid, kbs, 2, 5, 2, pairs_only=[3])
    finally:
        sm.PAIR_MULTICAST_COMMIT = True
    assert any(isinstance(p[1], str) and p[1].startswith("dq1.") for p in problems)


# ------------------------------------------------------------------ the measured A-slot ring
from schedule_model import simulate_ring  # noqa: E402

RING_SHAPES = [(4096, 4096), (4096, 12288), (4096, 22016), (11008, 4096), (8192, 57344), (28672, 8192),
               (128, 128), (384, 1000), (1024, 136), (256, 8)]


def _ring_config(monkeypatch, na):
    import schedule_model as sm
    monkeypatch.setattr(sm, "RING_PARTIAL_WAIT", "slot" if na == 4 else "pfull")


@pytest.mark.parametrize("K,N", RING_SHAPES)
@pytest.mark.parametrize("slots,na", [(16, 4), (12, 4), (20, 4), (4, 4), (8, 6), (16, 6), (16, 8)])
def test_ring_no_deadlock_alias_or_race(K, N, slots, na, monkeypatch):
    # na = 4: one slot per residue (slots: multiples of 4, 16 at 16-row fp16 tiles, 12 at
    # 32-row, 20 for int8); 6 and 8 slots: the ring proper
    _ring_config(monkeypatch, na)
    units, grid, kbs = _plan(K, N)
    if K * N > 8192 * 10240 and (slots, na) not in ((16, 4), (12, 4)):
        pytest.skip("large shapes: the plans the planner picks for them")
    problems = simulate_ring(units, grid, kbs, slots, na)
    assert not problems, problems[:5]


_RING_BIASES = dict(_BIASES)
_RING_BIASES["one-issuer-first"] = lambda n: n == "iss3"
_RING_BIASES["one-issuer-last"] = lambda n: n != "iss0"


@pytest.mark.parametrize("K,N", [(8192, 57344), (4096, 22016), (4096, 4096), (1024, 136)])
@pytest.mark.parametrize("slots,na", [(16, 4), (12, 4), (8, 6), (16, 8)])
def test_ring_under_skewed_schedules(K, N, slots, na, monkeypatch):
    import random
    _ring_config(monkeypatch, na)
    units, grid, kbs = _plan(K, N)
    for cta in sorted({0, grid // 2, grid - 1}):
        for name, first in _RING_BIASES.items():
            problems = simulate_ring(units, grid, kbs, slots, na, rng=_Biased(first, cta), ctas_only=[cta])
            assert not problems, (name, cta, problems[:3])
        for seed in range(2):
            problems = simulate_ring(units, grid, kbs, slots, na, rng=random.Random(seed), ctas_only=[cta])
            assert not problems, ("random", seed, cta, problems[:3])


def _ring_problems_everywhere(slots=16, na=6):
    import random
    units, grid, kbs = _plan(8192, 57344)
    out = []
    for cta in (0, 1, grid // 2):
        for name, first in _RING_BIASES.items():
            out += simulate_ring(units, grid, kbs, slots, na, rng=_Biased(first, cta), ctas_only=[cta])
        out += simulate_ring(units, grid, kbs, slots, na, rng=random.Random(cta), ctas_only=[cta])
    return out


@pytest.mark.parametrize("na,flag,value", [
    (6, "RING_ONE_SLOT_BARRIER", True),       # one afull per A slot: an issuer passes on an older phase
    (6, "RING_ONE_PARTIAL_BARRIER", True),    # one pfull per residue: the next k-block completes it first
    (6, "RING_PARTIAL_WAIT", "slot"),         # 6 slots: the slot's barrier belongs to another residue's k-block
    (6, "RING_READ_DELAY", 2),                # a partial read after the next k-block was signalled
    (4, "RING_READ_DELAY", 2),
])
def test_ring_model_catches_planted_mistake(na, flag, value, monkeypatch):
    import schedule_model as sm
    _ring_config(monkeypatch, na)
    monkeypatch.setattr(sm, flag, value)
    assert _ring_problems_everywhere(na=na), f"{flag} = {value} went unnoticed at {na} slots"


# ---------------------------------------------------------------------------- register-operand tiles
_RF_BIASES = {
    "consumers-first": lambda n: n.startswith("cw"), "producers-first": lambda n: n.startswith("prod"),
    "non-epilogue-warps-first": lambda n: n.startswith("cw") and int(n[2:]) >= 4,  # run a segment ahead
    "one-residue-first": lambda n: n in ("cw12", "cw13", "cw14", "cw15"),
    "epilogue-warps-first": lambda n: n in ("cw0", "cw1", "cw2", "cw3"),
    "one-consumer-first": lambda n: n == "cw7", "one-consumer-last": lambda n: n != "cw0",
}


@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 264), (11008, 4096), (4096, 22016), (128, 8), (384, 1000)])
@pytest.mark.parametrize("slots", [2, 5, 13, 25])
def test_rf_no_alias_deadlock_or_race(K, N, slots):
    # a k-block is read by its residue's 4 warps; the residue sums share one buffer, and a second
    # barrier after the epilogue warps have read them keeps a warp that runs a segment ahead
    # from overwriting them
    import random
    from schedule_model import simulate_rf
    units, grid, kbs = _plan(K, N)
    chunk = max(1, min(4, slots // 2))
    assert not simulate_rf(units, grid, kbs, chunk, slots)
    for cta in sorted({0, 1, grid // 2, grid - 1}):
        for name, first in _RF_BIASES.items():
            problems = simulate_rf(units, grid, kbs, chunk, slots, rng=_Biased(first, cta), ctas_only=[cta])
            assert not problems, (name, cta, problems[:3])
        problems = simulate_rf(units, grid, kbs, chunk, slots, rng=random.Random(cta), ctas_only=[cta])
        assert not problems, ("random", cta, problems[:3])


def test_rf_model_catches_a_missing_second_barrier():
    # without the second barrier a consumer warp that has finished its next segment overwrites
    # the sums while the epilogue warps may still be reading them
    import schedule_model as sm
    units, grid, kbs = _plan(4096, 22016)  # several segments per CTA
    saved = sm.RED_SECOND_BARRIER
    sm.RED_SECOND_BARRIER = False
    try:
        races = []
        for cta in range(8):
            for name, first in _RF_BIASES.items():
                races += [p for p in sm.simulate_rf(units, grid, kbs, 4, 13, rng=_Biased(first, cta), ctas_only=[cta])
                          if p[0] == "race"]
    finally:
        sm.RED_SECOND_BARRIER = saved
    assert races

