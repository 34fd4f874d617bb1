"""A CPU model of the small-tile GEMM kernel's synchronisation protocol.

Every warp role of every CTA is a generator of barrier operations that follows the kernel's
walk over its (tile, k-block) units: segments last-first, k-blocks forward, chunks of up to
`chunk` k-blocks that never wrap the shared-memory ring, chunk barriers indexed by chunk
number modulo 33, ring slots. Walk index i belongs to residue i mod 4: a dequant warp per
lane quarter, tensor-memory A slot i mod 4 and MMA issuer i mod 4. The dequant warps also
add the MMA partials (the commit that frees an A slot also completes its partial), so at a
segment's end each waits for its last MMA; then the named barriers of the 4-way combine and of
the epilogue, and the stream-K publish flags.

A residue's k-blocks alternate between two partial buffers (its u-th k-block writes buffer
u % 2). A dequant warp reads the partial of its previous k-block after it has handed the next
one to the MMA (afull); the model records each read and reports a "race" when an MMA starts
writing a buffer whose previous partial (two k-blocks of the residue back) has not been read
by all four lane quarters.

With TWO_A_SLOTS (and NA = 2 * DQ_PERIOD = 2 * NQ) the model describes a candidate design in
which every residue alternates between two A slots as well: the dequant warps of k-block u
wait only for the MMAs of k-block u - 2 (which frees the slot and completes the partial
buffer that k-block u will write), read that partial, dequantise into the slot and signal it,
so that they work on k-block u while the MMAs of k-block u - 1 run. At a segment's end they
wait for, and read, the partials of the last two k-blocks.

With ISSUERS_PER_RESIDUE = 2 (another candidate) two issuers serve each residue, each issuing
half of every k-block's MMAs into a partial of its own; both wait for the same A-slot signal
and both commit to the slot's barrier and to the ring slot (counts 2).
mbarriers follow the PTX phase/parity rules: a wait on parity p passes once the phase with
that parity has completed, i.e. while the current phase's parity differs from p.

Every wait also carries the number of completed phases its role means to wait for. A parity
wait cannot tell phase n from phase n - 2 (or n + 2), so a wait that passes while the barrier
has completed any other number of phases is a protocol error (an "alias") even when nothing
deadlocks: the role would read a slot before it was written, or after it was overwritten.

`simulate` runs all roles of all CTAs until nothing can move and returns the aliased waits and
the roles still blocked: an empty list means the protocol is sound for that launch plan and
that interleaving. The module constants NA (A slots), DQ_PERIOD (dequant residues) and NQ
(issuers) are all 4 in the kernel; tests change them to check that the model catches a
mismatch.
"""
from collections import defaultdict

NCB = 33          # chunk barriers
NA = 4            # tensor-memory A slots: k-block i uses slot i % NA
NQ = 4            # MMA issuers: issuer i % NQ
DQ_PERIOD = 4     # dequant warps per lane quarter: warp (quarter, i % DQ_PERIOD)
READ_DELAY = 1    # a dequant warp reads a partial after handing this many later k-blocks to the MMA
TWO_A_SLOTS = False  # a design with two A slots per residue (NA = 2 * DQ_PERIOD); see below
ISSUERS_PER_RESIDUE = 1  # 2: a design in which two issuers split each k-block's MMAs (K halves)
PAIR_MULTICAST_COMMIT = True  # CTA-pair model: the leader's commits reach both CTAs' barriers


class Bar:
    def __init__(self, count, name):
        self.count, self.pending, self.phase, self.name = count, count, 0, name

    def arrive(self):
        self.pending -= 1
        if self.pending < 0:
            raise AssertionError(f"over-arrival on {self.name} phase {self.phase}")
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def ready(self, need):
        # the role waits on parity (need - 1) & 1, the parity of the phase whose completion it wants
        return ((need - 1) & 1) != (self.phase & 1)


def unit_start(c, units, grid):
    return c * units // grid


def first_contributor(tbase, units, grid):
    """The CTA holding unit `tbase` (a tile's first unit): the smallest c with
    unit_start(c + 1) > tbase, in closed form."""
    return ((tbase + 1) * grid + units - 1) // units - 1


def segments(beg, end, kbs):
    it = end - 1
    while it >= beg:
        tile = it // kbs
        tbase = tile * kbs
        lo = max(beg, tbase)
        yield tile, lo - tbase, it - tbase, (it - tbase) == kbs - 1, (it - tbase) == kbs - 1 and lo == tbase
        it = lo - 1


FIRST_CHUNK = 1  # the CTA's first chunk is one k-block (the kernels' chunk_len)


def chunks(beg, end, kbs, chunk, slots):
    pos = it = ch = 0
    for seg in segments(beg, end, kbs):
        _, kb_lo, kb_hi, _, _ = seg
        kb = kb_lo
        while kb <= kb_hi:
            c = min(chunk, kb_hi - kb + 1, slots - pos)
            if ch == 0:
                c = min(c, FIRST_CHUNK)
            yield seg, pos, c, it, ch
            ch += 1
            it += c
            kb += c
            pos = (pos + c) % slots
        yield seg, None, None, it, ch


def _roles(cta, units, grid, kbs, chunk, slots, B):
    """Operations: ("wait", bar, need, walk index), ("arrive", bar), ("nbar", name, count),
    ("flag_set", cta), ("flag_wait", cta)."""
    beg, end = unit_start(cta, units, grid), unit_start(cta + 1, units, grid)

    def has(it0, c, period, residue):
        return ((residue + period - it0 % period) % period) < c

    def dq(quarter, residue):
        last = None  # walk index of this residue's last k-block in the current segment
        unread = []  # this segment's k-blocks of the residue whose partial is not read yet
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                if TWO_A_SLOTS:  # the MMAs of the residue's last two k-blocks, then their partials
                    for j in unread:
                        yield ("wait", B["aempty"][j % NA], j // NA + 1, j)
                        yield ("part_read", j)
                else:
                    if last is not None:  # the segment's last k-block of this residue: its MMAs
                        yield ("wait", B["aempty"][last % NA], last // NA + 1, last)
                    for j in unread:
                        yield ("part_read", j)
                unread = []
                yield ("nbar", f"comb{quarter}", DQ_PERIOD)
                yield ("nbar", f"comb{quarter}", DQ_PERIOD)
                tile, kb_lo, kb_hi, owner, whole = seg
                if not owner:
                    yield ("nbar", "epi", 4 * DQ_PERIOD)
                    if quarter == 0 and residue == 0:
                        yield ("flag_set", cta)
                elif not whole:
                    for cc in range(cta - 1, first_contributor(tile * kbs, units, grid) - 1, -1):
                        yield ("flag_wait", cc)
                    yield ("nbar", "epi", 4 * DQ_PERIOD)
                last = None
                continue
            if not has(it0, c, DQ_PERIOD, residue):
                continue
            yield ("wait", B["full"][ch % NCB], ch // NCB + 1, it0)
            for t in range(c):
                i = it0 + t
                if i % DQ_PERIOD == residue:
                    yield ("arrive", B["empty_w"][pos + t])
                    yield ("wait", B["aempty"][i % NA], i // NA, i)
                    if TWO_A_SLOTS and unread and unread[0] == i - NA:
                        yield ("part_read", unread.pop(0))  # completed by the MMAs just waited for
                    yield ("arrive", B["afull"][i % NA])
                    unread.append(i)
                    while not TWO_A_SLOTS and len(unread) > READ_DELAY:
                        yield ("part_read", unread.pop(0))
                    last = i

    def issuer(q):
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None or not has(it0, c, NQ, q):
                continue
            yield ("wait", B["full"][ch % NCB], ch // NCB + 1, it0)
            for t in range(c):
                i = it0 + t
                if i % NQ == q:
                    yield ("wait", B["afull"][i % NA], i // NA + 1, i)
                    yield ("part_write", i)
                    yield ("arrive", B["aempty"][i % NA])
                    yield ("arrive", B["empty_a"][pos + t])

    def producer(which):
        uses = [0] * slots
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                continue
            for t in range(c):
                yield ("wait", B[which][pos + t], uses[pos + t], it0 + t)
                uses[pos + t] += 1
            yield ("arrive", B["full"][ch % NCB])

    roles = {}
    for w in range(4 * DQ_PERIOD):
        roles[f"dq{w}"] = dq(w & 3, w >> 2)
    for q in range(NQ):
        for h in range(ISSUERS_PER_RESIDUE):
            roles[f"iss{q}" + (f".{h}" if ISSUERS_PER_RESIDUE > 1 else "")] = issuer(q)
    roles["prod_w"] = producer("empty_w")
    roles["prod_a"] = producer("empty_a")
    return roles


def simulate(units, grid, kbs, chunk, slots, rng=None, ctas_only=None):
    """Runs the roles of the CTAs (all, or `ctas_only`) to a standstill. With `rng` the roles
    move in a random order and a random number of operations at a time (any object with
    `shuffle(list)` and `randint(a, b)` can bias the interleaving). Returns a list of problems:
    ("alias", cta, role, barrier, phases needed, phases completed) for each wait that passed on
    the wrong phase, ("race", cta, walk index) for each partial overwritten before all four
    lane quarters read it, and (cta, role, pending operation) for each role left blocked."""
    flags = {}
    if ctas_only is not None:  # CTAs outside the subset count as having published
        flags = {c: 1 for c in range(grid) if c not in ctas_only}
    ctas = []
    for cta in (range(grid) if ctas_only is None else ctas_only):
        B = {"full": [Bar(2, f"full{k}") for k in range(NCB)],
             "empty_w": [Bar(4, f"empty_w{s}") for s in range(slots)],
             "empty_a": [Bar(ISSUERS_PER_RESIDUE, f"empty_a{s}") for s in range(slots)],
             "afull": [Bar(4, f"afull{a}") for a in range(NA)],
             "aempty": [Bar(ISSUERS_PER_RESIDUE, f"aempty{a}") for a in range(NA)]}
        roles = _roles(cta, units, grid, kbs, chunk, slots, B)
        ctas.append({"cta": cta, "roles": roles, "cur": dict.fromkeys(roles), "done": set(),
                     "nbar": defaultdict(list), "reads": defaultdict(int)})
    problems = []
    moved = True
    while moved:
        moved = False
        order = [(st, name) for st in ctas for name in st["roles"]]
        if rng is not None:
            rng.shuffle(order)
        for st, name in order:
            gen = st["roles"][name]
            steps = 0
            while name not in st["done"]:
                if rng is not None and steps >= rng.randint(1, 4):
                    moved = True
                    break
                steps += 1
                op = st["cur"][name]
                if op is None:
                    try:
                        op = st["cur"][name] = next(gen)
                    except StopIteration:
                        st["done"].add(name)
                        break
                kind = op[0]
                if kind == "wait":
                    if not op[1].ready(op[2]):
                        break
                    if op[1].phase != op[2]:
                        problems.append(("alias", st["cta"], name, op[1].name, op[2], op[1].phase))
                elif kind == "flag_wait":
                    if not flags.get(op[1]):
                        break
                elif kind == "arrive":
                    op[1].arrive()
                elif kind == "flag_set":
                    flags[op[1]] = 1
                elif kind == "part_read":
                    st["reads"][op[1]] += 1
                elif kind == "part_write":
                    # the buffer's previous partial: two k-blocks of the residue back
                    if op[1] >= 2 * NQ and st["reads"][op[1] - 2 * NQ] < 4:
                        problems.append(("race", st["cta"], op[1] - 2 * NQ))
                elif kind == "nbar":
                    waiting = st["nbar"][op[1]]
                    if name not in waiting:
                        waiting.append(name)
                    if len(waiting) < op[2]:
                        break
                    for other in waiting:
                        st["cur"][other] = None
                    st["nbar"][op[1]] = []
                st["cur"][name] = None
                moved = True
    stuck = [(st["cta"], name, st["cur"][name]) for st in ctas for name in st["roles"] if name not in st["done"]]
    return problems + stuck


# ---------------------------------------------------------------------------- large tiles
def _roles_large(cta, units, grid, kbs, chunk, slots, issuers, B, state, owner_barrier=True):
    """The large-tile kernel: 16 dequant warps in 2 residues (walk index mod 2) x 2 halves of
    a k-block x 4 lane quarters; A slot i mod 4; `issuers` MMA issuers splitting every
    k-block's K range, each accumulating the whole segment into its own accumulator; the
    segment-done barrier; the epilogue in the dequant warps. Besides barrier operations the
    roles report ("acc_read_done", segment) once a dequant warp has read the segment's
    accumulators and ("acc_overwrite", segment) when an issuer starts a segment's fresh
    accumulation: an overwrite before all 16 reads of the previous segment is a race."""
    beg, end = unit_start(cta, units, grid), unit_start(cta + 1, units, grid)

    def has(it0, c, residue):
        return ((residue + 2 - it0 % 2) % 2) < c

    def dq(quarter, half, residue):
        seg_index = 0
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                yield ("wait", B["dfull"], seg_index + 1, seg_index)
                tile, kb_lo, kb_hi, owner, whole = seg
                if not owner:
                    yield ("acc_read_done", seg_index)
                    yield ("nbar", "epi", 16)
                    if quarter == 0 and half == 0 and residue == 0:
                        yield ("flag_set", cta)
                else:
                    if not whole:
                        for cc in range(cta - 1, first_contributor(tile * kbs, units, grid) - 1, -1):
                            yield ("flag_wait", cc)
                    yield ("acc_read_done", seg_index)
                    if owner_barrier or not whole:
                        yield ("nbar", "epi", 16)
                seg_index += 1
                continue
            if not has(it0, c, residue):
                continue
            yield ("wait", B["full"][ch % NCB], ch // NCB + 1, it0)
            for t in range(c):
                i = it0 + t
                if i % 2 == residue:
                    yield ("arrive", B["empty_w"][pos + t])
                    yield ("wait", B["aempty"][i % 4], i // 4, i)
                    yield ("arrive", B["afull"][i % 4][half])

    def issuer(q):
        halves = [0, 1] if issuers == 1 else [(q * (8 // issuers) * 16) // 64]
        seg_index = 0
        first = True
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                yield ("arrive", B["dfull"])
                seg_index += 1
                first = True
                continue
            yield ("wait", B["full"][ch % NCB], ch // NCB + 1, it0)
            for t in range(c):
                i = it0 + t
                for h in halves:
                    yield ("wait", B["afull"][i % 4][h], i // 4 + 1, i)
                if first:
                    yield ("acc_overwrite", seg_index)
                    first = False
                yield ("arrive", B["aempty"][i % 4])
                yield ("arrive", B["empty_a"][pos + t])

    def producer(which):
        uses = [0] * slots
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                continue
            for t in range(c):
                yield ("wait", B[which][pos + t], uses[pos + t], it0 + t)
                uses[pos + t] += 1
            yield ("arrive", B["full"][ch % NCB])

    roles = {}
    for w in range(16):
        roles[f"dq{w}"] = dq(w & 3, (w >> 2) & 1, w >> 3)
    for q in range(issuers):
        roles[f"iss{q}"] = issuer(q)
    roles["prod_w"] = producer("empty_w")
    roles["prod_a"] = producer("empty_a")
    return roles


def simulate_large(units, grid, kbs, chunk, slots, issuers, rng=None, ctas_only=None, owner_barrier=True):
    """Like simulate, for the large-tile kernel; problems also include ("race", cta, segment)
    for an accumulator overwrite before the previous segment's reads were done."""
    flags = {}
    if ctas_only is not None:
        flags = {c: 1 for c in range(grid) if c not in ctas_only}
    ctas = []
    for cta in (range(grid) if ctas_only is None else ctas_only):
        B = {"full": [Bar(2, f"full{k}") for k in range(NCB)],
             "empty_w": [Bar(8, f"empty_w{s}") for s in range(slots)],
             "empty_a": [Bar(issuers, f"empty_a{s}") for s in range(slots)],
             "afull": [[Bar(4, f"afull{a}.{h}") for h in range(2)] for a in range(4)],
             "aempty": [Bar(issuers, f"aempty{a}") for a in range(4)],
             "dfull": Bar(issuers, "dfull")}
        state = {"reads": defaultdict(int)}
        roles = _roles_large(cta, units, grid, kbs, chunk, slots, issuers, B, state, owner_barrier)
        ctas.append({"cta": cta, "roles": roles, "cur": dict.fromkeys(roles), "done": set(),
                     "nbar": defaultdict(list), "state": state})
    problems = []
    moved = True
    while moved:
        moved = False
        order = [(st, name) for st in ctas for name in st["roles"]]
        if rng is not None:
            rng.shuffle(order)
        for st, name in order:
            gen = st["roles"][name]
            steps = 0
            while name not in st["done"]:
                if rng is not None and steps >= rng.randint(1, 4):
                    moved = True
                    break
                steps += 1
                op = st["cur"][name]
                if op is None:
                    try:
                        op = st["cur"][name] = next(gen)
                    except StopIteration:
                        st["done"].add(name)
                        break
                kind = op[0]
                if kind == "wait":
                    if not op[1].ready(op[2]):
                        break
                    if op[1].phase != op[2]:
                        problems.append(("alias", st["cta"], name, op[1].name, op[2], op[1].phase))
                elif kind == "flag_wait":
                    if not flags.get(op[1]):
                        break
                elif kind == "arrive":
                    op[1].arrive()
                elif kind == "flag_set":
                    flags[op[1]] = 1
                elif kind == "acc_read_done":
                    st["state"]["reads"][op[1]] += 1
                elif kind == "acc_overwrite":
                    if op[1] > 0 and st["state"]["reads"][op[1] - 1] < 16:
                        problems.append(("race", st["cta"], op[1]))
                elif kind == "nbar":
                    waiting = st["nbar"][op[1]]
                    if name not in waiting:
                        waiting.append(name)
                    if len(waiting) < op[2]:
                        break
                    for other in waiting:
                        st["cur"][other] = None
                    st["nbar"][op[1]] = []
                st["cur"][name] = None
                moved = True
    stuck = [(st["cta"], name, st["cur"][name]) for st in ctas for name in st["roles"] if name not in st["done"]]
    return problems + stuck


# ---------------------------------------------------------------------------- large tiles, CTA pairs
def _roles_large_pair(pair, units, grid, kbs, chunk, slots, issuers, B, state):
    """The planned 2-SM form of the large-tile kernel: a pair of CTAs (k = 0 leader, 1 follower)
    walks the same (tile pair, k-block) units. Each CTA dequantises its own 128 weight columns
    into its own A slots and loads half of the activation rows. The leader's issuers issue the
    paired MMAs: they wait on the leader's barriers, which count arrivals from both CTAs (the
    follower's dequant warps arrive remotely, its activation copy signals the leader's barrier),
    and their commits are multicast to the same barrier in both CTAs. Both CTAs' accumulators are
    written by every MMA, so a segment's fresh accumulation must wait for all 32 dequant warps
    of the pair to have read the previous segment's accumulators."""
    beg, end = unit_start(pair, units, grid), unit_start(pair + 1, units, grid)
    L = B[0]  # the leader's barriers

    def has(it0, c, residue):
        return ((residue + 2 - it0 % 2) % 2) < c

    def dq(k, quarter, half, residue):
        seg_index = 0
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                yield ("wait", B[k]["dfull"], seg_index + 1, seg_index)
                tile, kb_lo, kb_hi, owner, whole = seg
                if not owner:
                    yield ("acc_read_done", seg_index)
                    yield ("nbar", f"epi{k}", 16)
                    if quarter == 0 and half == 0 and residue == 0:
                        yield ("flag_set", (pair, k))
                else:
                    if not whole:
                        for cc in range(pair - 1, first_contributor(tile * kbs, units, grid) - 1, -1):
                            yield ("flag_wait", (cc, k))
                    yield ("acc_read_done", seg_index)
                    yield ("nbar", f"epi{k}", 16)
                seg_index += 1
                continue
            if not has(it0, c, residue):
                continue
            yield ("wait", B[k]["full_w"][ch % NCB], ch // NCB + 1, it0)
            for t in range(c):
                i = it0 + t
                if i % 2 == residue:
                    yield ("arrive", B[k]["empty_w"][pos + t])
                    yield ("wait", B[k]["aempty"][i % 4], i // 4, i)
                    yield ("arrive", L["afull"][i % 4][half])  # remote for the follower

    def issuer(q):
        halves = [0, 1] if issuers == 1 else [(q * (8 // issuers) * 16) // 64]
        seg_index = 0
        first = True
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                for kk in ((0, 1) if PAIR_MULTICAST_COMMIT else (0,)):  # multicast commit
                    yield ("arrive", B[kk]["dfull"])
                seg_index += 1
                first = True
                continue
            yield ("wait", L["full_a"][ch % NCB], ch // NCB + 1, it0)
            for t in range(c):
                i = it0 + t
                for h in halves:
                    yield ("wait", L["afull"][i % 4][h], i // 4 + 1, i)
                if first:
                    yield ("acc_overwrite", seg_index)
                    first = False
                for kk in ((0, 1) if PAIR_MULTICAST_COMMIT else (0,)):
                    yield ("arrive", B[kk]["aempty"][i % 4])
                    yield ("arrive", B[kk]["empty_a"][pos + t])

    def producer(k, which):
        uses = [0] * slots
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                continue
            empty = "empty_w" if which == "w" else "empty_a"
            for t in range(c):
                yield ("wait", B[k][empty][pos + t], uses[pos + t], it0 + t)
                uses[pos + t] += 1
            yield ("arrive", B[k]["full_w"][ch % NCB] if which == "w" else L["full_a"][ch % NCB])

    roles = {}
    for k in (0, 1):
        for w in range(16):
            roles[f"dq{k}.{w}"] = dq(k, w & 3, (w >> 2) & 1, w >> 3)
        roles[f"prod_w{k}"] = producer(k, "w")
        roles[f"prod_a{k}"] = producer(k, "a")
    for q in range(issuers):
        roles[f"iss{q}"] = issuer(q)
    return roles


def simulate_large_pair(units, grid, kbs, chunk, slots, issuers, rng=None, pairs_only=None):
    """Like simulate_large, for CTA pairs (`grid` pairs over `units` (tile pair, k-block) units)."""
    flags = {}
    if pairs_only is not None:
        flags = {(c, k): 1 for c in range(grid) if c not in pairs_only for k in (0, 1)}
    pairs = []
    for pair in (range(grid) if pairs_only is None else pairs_only):
        B = []
        for k in (0, 1):
            b = {"full_w": [Bar(1, f"full_w{k}.{x}") for x in range(NCB)],
                 "empty_w": [Bar(8, f"empty_w{k}.{s}") for s in range(slots)],
                 "empty_a": [Bar(issuers, f"empty_a{k}.{s}") for s in range(slots)],
                 "aempty": [Bar(issuers, f"aempty{k}.{a}") for a in range(4)],
                 "dfull": Bar(issuers, f"dfull{k}")}
            if k == 0:
                b["full_a"] = [Bar(2, f"full_a.{x}") for x in range(NCB)]
                b["afull"] = [[Bar(8, f"afull{a}.{h}") for h in range(2)] for a in range(4)]
            B.append(b)
        state = {"reads": defaultdict(int)}
        roles = _roles_large_pair(pair, units, grid, kbs, chunk, slots, issuers, B, state)
        pairs.append({"cta": pair, "roles": roles, "cur": dict.fromkeys(roles), "done": set(),
                      "nbar": defaultdict(list), "state": state})
    problems = []
    moved = True
    while moved:
        moved = False
        order = [(st, name) for st in pairs for name in st["roles"]]
        if rng is not None:
            rng.shuffle(order)
        for st, name in order:
            gen = st["roles"][name]
            steps = 0
            while name not in st["done"]:
                if rng is not None and steps >= rng.randint(1, 4):
                    moved = True
                    break
                steps += 1
                op = st["cur"][name]
                if op is None:
                    try:
                        op = st["cur"][name] = next(gen)
                    except StopIteration:
                        st["done"].add(name)
                        break
                kind = op[0]
                if kind == "wait":
                    if not op[1].ready(op[2]):
                        break
                    if op[1].phase != op[2]:
                        problems.append(("alias", st["cta"], name, op[1].name, op[2], op[1].phase))
                elif kind == "flag_wait":
                    if not flags.get(op[1]):
                        break
                elif kind == "arrive":
                    op[1].arrive()
                elif kind == "flag_set":
                    flags[op[1]] = 1
                elif kind == "acc_read_done":
                    st["state"]["reads"][op[1]] += 1
                elif kind == "acc_overwrite":
                    if op[1] > 0 and st["state"]["reads"][op[1] - 1] < 32:
                        problems.append(("race", st["cta"], op[1]))
                elif kind == "nbar":
                    waiting = st["nbar"][op[1]]
                    if name not in waiting:
                        waiting.append(name)
                    if len(waiting) < op[2]:
                        break
                    for other in waiting:
                        st["cur"][other] = None
                    st["nbar"][op[1]] = []
                st["cur"][name] = None
                moved = True
    stuck = [(st["cta"], name, st["cur"][name]) for st in pairs for name in st["roles"] if name not in st["done"]]
    return problems + stuck


# ---------------------------------------------------------------------------- small tiles, A-slot ring
# A small-tile protocol that was built, passed every GPU parity test and was measured slower
# than the kernel as built (kept here with its tests as the record of the hazards it needed
# to avoid): walk index j belongs to residue j % 4 (dequant warp
# per lane quarter, issuer j % 4, partial buffers 2r, 2r + 1 by the residue's use count); the
# dequantised k-block goes to A slot j % na. Chunks are fixed by walk position: {0}, {1},
# {2, 3}, then runs of four; ring slot j % slots with slots a multiple of 4; chunk barrier
# chunk % NCB. A split tile is finished by the CTA holding its last k-block, which waits for
# the publish flags of the CTAs holding its other k-blocks (stream-K).
#
# na = 4: a slot's previous user is the residue's own previous k-block,
# so the wait that frees the slot also completes that k-block's partial (RING_PARTIAL_WAIT =
# "slot"). na = 6 or 8: the partial is
# signalled on the barrier of its partial buffer, pfull[r][u % 2] ("pfull"); with a single
# barrier per residue the issuer could complete the residue's next k-block (which the dequant
# warps signal before reading the previous partial) before the warps wait: two phases ahead.
# With na not a multiple of 4 a slot's consecutive uses belong to different issuers, so an
# issuer can reach a slot's use u + 1 before use u was signalled; the slot's full barrier is
# therefore a pair, afull[a][use % 2], so that a waiter is never two phases behind either.
RING_READ_DELAY = 1  # the kernel reads a residue's partial after signalling 1 later k-block; 2 is a planted mistake
RING_PARTIAL_WAIT = "slot"  # "slot" (na = 4) or "pfull" (na = 6, 8); "slot" with na = 6 is a planted mistake
RING_ONE_PARTIAL_BARRIER = False  # planted mistake: one partial barrier per residue, not one per buffer
RING_ONE_SLOT_BARRIER = False  # planted mistake: one afull barrier per A slot, not one per use parity


def ring_chunk(j):
    return j if j < 2 else (2 if j < 4 else j // 4 + 2)


def ring_chunk_len(c):
    return 1 if c < 2 else (2 if c == 2 else 4)


def _segment_bounds(beg, end, kbs):
    """(segment, walk index where it ends) for the CTA's walk, last segment first."""
    out, se = [], 0
    for seg in segments(beg, end, kbs):
        se += seg[2] - seg[1] + 1
        out.append((seg, se))
    return out


def _roles_ring(cta, units, grid, kbs, slots, na, B):
    beg, end = unit_start(cta, units, grid), unit_start(cta + 1, units, grid)
    L = end - beg
    segs = _segment_bounds(beg, end, kbs)

    def _afull(j):
        return B["afull"][j % na][0 if RING_ONE_SLOT_BARRIER else (j // na) % 2]

    def dq(quarter, r):
        j, u = r, 0
        for seg, se in segs:
            unread = []  # (walk index, use count) of this segment's k-blocks whose partial is unread

            def read(pj, pu, covered):
                # covered: with 4 slots the wait that freed this k-block's slot for the residue's next
                # k-block already saw these MMAs complete; the kernel reads without waiting again,
                # and the model only checks that the phase is indeed complete
                if RING_PARTIAL_WAIT == "slot" and covered:
                    yield ("check", B["aempty"][pj % na], pj // na + 1, pj)
                elif RING_PARTIAL_WAIT == "slot":
                    yield ("wait", B["aempty"][pj % na], pj // na + 1, pj)
                elif RING_ONE_PARTIAL_BARRIER:
                    yield ("wait", B["pfull"][r][0], pu + 1, pj)
                else:
                    yield ("wait", B["pfull"][r][pu % 2], pu // 2 + 1, pj)
                yield ("part_read", pj)

            while j < se and j < L:
                c = ring_chunk(j)
                yield ("wait", B["full"][c % NCB], c // NCB + 1, j)
                yield ("arrive", B["empty_w"][j % slots])
                yield ("wait", B["aempty"][j % na], j // na, j)
                yield ("arrive", _afull(j))
                unread.append((j, u))
                while len(unread) > RING_READ_DELAY:
                    yield from read(*unread.pop(0), covered=True)
                u += 1
                j += 4
            for pj, pu in unread:
                yield from read(pj, pu, covered=False)
            yield ("nbar", f"comb{quarter}", 4)
            yield ("nbar", f"comb{quarter}", 4)
            tile, kb_lo, kb_hi, owner, whole = seg
            if not owner:
                yield ("nbar", "epi", 16)
                if quarter == 0 and r == 0:
                    yield ("flag_set", cta)
            elif not whole:
                for cc in range(cta - 1, first_contributor(tile * kbs, units, grid) - 1, -1):
                    yield ("flag_wait", cc)
                yield ("nbar", "epi", 16)

    def issuer(q):
        for u, j in enumerate(range(q, L, 4)):
            c = ring_chunk(j)
            yield ("wait", B["full"][c % NCB], c // NCB + 1, j)
            if RING_ONE_SLOT_BARRIER:
                yield ("wait", _afull(j), j // na + 1, j)
            else:
                yield ("wait", _afull(j), (j // na) // 2 + 1, j)
            yield ("part_write", j)
            yield ("arrive", B["aempty"][j % na])
            yield ("arrive", B["empty_a"][j % slots])
            if RING_PARTIAL_WAIT == "pfull":
                yield ("arrive", B["pfull"][q][0 if RING_ONE_PARTIAL_BARRIER else u % 2])

    def producer(which):
        uses = [0] * slots
        j, c = 0, 0
        while j < L:
            n = min(ring_chunk_len(c), L - j)
            for t in range(n):
                s = (j + t) % slots
                yield ("wait", B[which][s], uses[s], j + t)
                uses[s] += 1
            yield ("arrive", B["full"][c % NCB])
            j += n
            c += 1

    roles = {}
    for w in range(16):
        roles[f"dq{w}"] = dq(w & 3, w >> 2)
    for q in range(4):
        roles[f"iss{q}"] = issuer(q)
    roles["prod_w"] = producer("empty_w")
    roles["prod_a"] = producer("empty_a")
    return roles


def simulate_ring(units, grid, kbs, slots, na, rng=None, ctas_only=None):
    """Like simulate, for the small-tile kernel with the A-slot ring: ("alias", ...) for a wait
    that passed on the wrong phase, ("race", cta, walk index) for a partial overwritten before
    all four lane quarters read it, ("unsynchronised", ...) for a partial read whose MMAs were
    not known to be complete, and the roles left blocked."""
    assert slots % 4 == 0 and slots >= 4
    flags = {}
    if ctas_only is not None:  # CTAs outside the subset count as having published
        flags = {c: 1 for c in range(grid) if c not in ctas_only}
    ctas = []
    for cta in (range(grid) if ctas_only is None else ctas_only):
        B = {"full": [Bar(2, f"full{k}") for k in range(NCB)],
             "empty_w": [Bar(4, f"empty_w{s}") for s in range(slots)],
             "empty_a": [Bar(1, f"empty_a{s}") for s in range(slots)],
             "afull": [[Bar(4, f"afull{a}.{b}") for b in range(2)] for a in range(na)],
             "aempty": [Bar(1, f"aempty{a}") for a in range(na)],
             "pfull": [[Bar(1, f"pfull{r}.{b}") for b in range(2)] for r in range(4)]}
        roles = _roles_ring(cta, units, grid, kbs, slots, na, B)
        ctas.append({"cta": cta, "roles": roles, "cur": dict.fromkeys(roles), "done": set(),
                     "nbar": defaultdict(list), "reads": defaultdict(int)})
    problems = []
    moved = True
    while moved:
        moved = False
        order = [(st, name) for st in ctas for name in st["roles"]]
        if rng is not None:
            rng.shuffle(order)
        for st, name in order:
            gen = st["roles"][name]
            steps = 0
            while name not in st["done"]:
                if rng is not None and steps >= rng.randint(1, 4):
                    moved = True
                    break
                steps += 1
                op = st["cur"][name]
                if op is None:
                    try:
                        op = st["cur"][name] = next(gen)
                    except StopIteration:
                        st["done"].add(name)
                        break
                kind = op[0]
                if kind == "wait":
                    if not op[1].ready(op[2]):
                        break
                    if op[1].phase != op[2]:
                        problems.append(("alias", st["cta"], name, op[1].name, op[2], op[1].phase))
                elif kind == "flag_wait":
                    if not flags.get(op[1]):
                        break
                elif kind == "arrive":
                    op[1].arrive()
                elif kind == "flag_set":
                    flags[op[1]] = 1
                elif kind == "check":
                    if op[1].phase < op[2]:
                        problems.append(("unsynchronised", st["cta"], name, op[1].name, op[2], op[1].phase))
                elif kind == "part_read":
                    st["reads"][op[1]] += 1
                elif kind == "part_write":
                    if op[1] >= 8 and st["reads"][op[1] - 8] < 4:
                        problems.append(("race", st["cta"], op[1] - 8))
                elif kind == "nbar":
                    waiting = st["nbar"][op[1]]
                    if name not in waiting:
                        waiting.append(name)
                    if len(waiting) < op[2]:
                        break
                    for other in waiting:
                        st["cur"][other] = None
                    st["nbar"][op[1]] = []
                st["cur"][name] = None
                moved = True
    stuck = [(st["cta"], name, st["cur"][name]) for st in ctas for name in st["roles"] if name not in st["done"]]
    return problems + stuck


# ---------------------------------------------------------------------------- register-operand tiles
RED_SECOND_BARRIER = True  # the residue sums: one buffer, a second barrier once they are read


def _roles_rf(cta, units, grid, kbs, chunk, slots, B):
    """The register-operand kernel: 16 consumer warps in 4 residues (walk index mod 4) x 4 column
    groups; the 4 warps of a k-block's residue read it (empty_w and empty_a count 4 arrivals).
    At a segment's end every warp writes its sums into the one buffer, all meet at a 16-warp
    barrier, warps 0..3 read the four residues' sums, all meet again (RED_SECOND_BARRIER) and
    warps 0..3 run the stream-K epilogue (a 4-warp barrier). Besides barrier operations the
    roles report ("red_write", segment) and ("red_read", segment): a write while the previous
    segment's sums have not been read by all four epilogue warps is a race."""
    beg, end = unit_start(cta, units, grid), unit_start(cta + 1, units, grid)

    def has(it0, c, residue):
        return ((residue + 4 - it0 % 4) % 4) < c

    def consumer(w):
        residue = w >> 2
        seg_no = 0
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                yield ("red_write", seg_no)
                yield ("nbar", "red", 16)
                if w < 4:
                    yield ("red_read", seg_no)
                if RED_SECOND_BARRIER:
                    yield ("nbar", "red", 16)
                if w < 4:
                    tile, kb_lo, kb_hi, owner, whole = seg
                    if not owner:
                        yield ("nbar", "epi", 4)
                        if w == 0:
                            yield ("flag_set", cta)
                    elif not whole:
                        for cc in range(cta - 1, first_contributor(tile * kbs, units, grid) - 1, -1):
                            yield ("flag_wait", cc)
                        yield ("nbar", "epi", 4)
                seg_no += 1
                continue
            if not has(it0, c, residue):
                continue
            yield ("wait", B["full"][ch % NCB], ch // NCB + 1, it0)
            for t in range(c):
                if (it0 + t) % 4 == residue:
                    yield ("arrive", B["empty_w"][pos + t])
                    yield ("arrive", B["empty_a"][pos + t])

    def producer(which):
        uses = [0] * slots
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                continue
            for t in range(c):
                yield ("wait", B[which][pos + t], uses[pos + t], it0 + t)
                uses[pos + t] += 1
            yield ("arrive", B["full"][ch % NCB])

    roles = {f"cw{w}": consumer(w) for w in range(16)}
    roles["prod_w"] = producer("empty_w")
    roles["prod_a"] = producer("empty_a")
    return roles


def simulate_rf(units, grid, kbs, chunk, slots, rng=None, ctas_only=None):
    """Like simulate, for the register-operand kernel; problems also include ("race", cta,
    segment) for a residue sum overwritten before the epilogue warps read it."""
    flags = {}
    if ctas_only is not None:
        flags = {c: 1 for c in range(grid) if c not in ctas_only}
    ctas = []
    for cta in (range(grid) if ctas_only is None else ctas_only):
        B = {"full": [Bar(2, f"full{k}") for k in range(NCB)],
             "empty_w": [Bar(4, f"empty_w{s}") for s in range(slots)],
             "empty_a": [Bar(4, f"empty_a{s}") for s in range(slots)]}
        roles = _roles_rf(cta, units, grid, kbs, chunk, slots, B)
        ctas.append({"cta": cta, "roles": roles, "cur": dict.fromkeys(roles), "done": set(),
                     "nbar": defaultdict(list), "reads": defaultdict(int)})
    problems = []
    moved = True
    while moved:
        moved = False
        order = [(st, name) for st in ctas for name in st["roles"]]
        if rng is not None:
            rng.shuffle(order)
        for st, name in order:
            gen = st["roles"][name]
            steps = 0
            while name not in st["done"]:
                if rng is not None and steps >= rng.randint(1, 4):
                    moved = True
                    break
                steps += 1
                op = st["cur"][name]
                if op is None:
                    try:
                        op = st["cur"][name] = next(gen)
                    except StopIteration:
                        st["done"].add(name)
                        break
                kind = op[0]
                if kind == "wait":
                    if not op[1].ready(op[2]):
                        break
                    if op[1].phase != op[2]:
                        problems.append(("alias", st["cta"], name, op[1].name, op[2], op[1].phase))
                elif kind == "flag_wait":
                    if not flags.get(op[1]):
                        break
                elif kind == "arrive":
                    op[1].arrive()
                elif kind == "flag_set":
                    flags[op[1]] = 1
                elif kind == "red_read":
                    st["reads"][op[1]] += 1
                elif kind == "red_write":
                    prev = op[1] - 1  # the segment that last used the buffer
                    if prev >= 0 and st["reads"][prev] < 4:
                        problems.append(("race", st["cta"], prev))
                elif kind == "nbar":
                    waiting = st["nbar"][op[1]]
                    if name not in waiting:
                        waiting.append(name)
                    if len(waiting) < op[2]:
                        break
                    for other in waiting:
                        st["cur"][other] = None
                    st["nbar"][op[1]] = []
                st["cur"][name] = None
                moved = True
    stuck = [(st["cta"], name, st["cur"][name]) for st in ctas for name in st["roles"] if name not in st["done"]]
    return problems + stuck

