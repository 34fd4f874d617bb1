"""A CPU model of the small-tile GEMM kernel's synchronisation protocol.

Every warp role of every CTA is a generator of barrier operations that follows the kernel's
walk over its (tile, k-block) units: segments last-first, k-blocks forward, chunks of up to
`chunk` k-blocks that never wrap the shared-memory ring, chunk barriers indexed by chunk
number modulo 33, ring slots, tensor-memory A slots (6), partial buffers (4 issuers), the
two accumulate parities, the named barriers of the epilogue and the stream-K publish flags.
mbarriers follow the PTX phase/parity rules: a wait on parity p passes once the phase with
that parity has completed, i.e. while the current phase's parity differs from p.

`simulate` runs all roles of all CTAs until nothing can move and returns the roles still
blocked: an empty list means the protocol cannot deadlock for that launch plan.
"""
from collections import defaultdict

NCB = 33          # chunk barriers
NA = 6            # tensor-memory A slots
NQ = 4            # MMA issuers


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

    def ready(self, parity):
        return parity != (self.phase & 1)


def unit_start(c, units, grid):
    return c * units // grid


def segments(beg, end, kbs):
    it = end - 1
    while it >= beg:
        tile = it // kbs
        tbase = tile * kbs
        lo = max(beg, tbase)
        yield tile, lo - tbase, it - tbase, (it - tbase) == kbs - 1, (it - tbase) == kbs - 1 and lo == tbase
        it = lo - 1


def chunks(beg, end, kbs, chunk, slots):
    pos = it = ch = 0
    for seg in segments(beg, end, kbs):
        _, kb_lo, kb_hi, _, _ = seg
        kb = kb_lo
        while kb <= kb_hi:
            c = min(chunk, kb_hi - kb + 1, slots - pos)
            yield seg, pos, c, it, ch
            ch += 1
            it += c
            kb += c
            pos = (pos + c) % slots
        yield seg, None, None, it, ch


def _roles(cta, units, grid, kbs, chunk, slots, B):
    beg, end = unit_start(cta, units, grid), unit_start(cta + 1, units, grid)

    def has(it0, c, period, residue):
        return ((residue + period - it0 % period) % period) < c

    def dq(residue):
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None or not has(it0, c, 3, residue):
                continue
            yield ("wait", B["full"][ch % NCB], (ch // NCB) & 1)
            for t in range(c):
                i = it0 + t
                if i % 3 == residue:
                    yield ("arrive", B["empty_w"][pos + t])
                    yield ("wait", B["aempty"][i % NA], ((i // NA) & 1) ^ 1)
                    yield ("arrive", B["afull"][i % NA])

    def issuer(q):
        j = 0
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None or not has(it0, c, NQ, q):
                continue
            yield ("wait", B["full"][ch % NCB], (ch // NCB) & 1)
            for t in range(c):
                i = it0 + t
                if i % NQ == q:
                    yield ("wait", B["afull"][i % NA], (i // NA) & 1)
                    yield ("wait", B["pempty"][q], (j & 1) ^ 1)
                    j += 1
                    yield ("arrive", B["aempty"][i % NA])
                    yield ("arrive", B["empty_a"][pos + t])
                    yield ("arrive", B["pfull"][q])

    def producer(which):
        ebits = [0] * slots
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                continue
            for t in range(c):
                yield ("wait", B[which][pos + t], ebits[pos + t] ^ 1)
                ebits[pos + t] ^= 1
            yield ("arrive", B["full"][ch % NCB])

    def acc(quarter, parity):
        for seg, pos, c, it0, ch in chunks(beg, end, kbs, chunk, slots):
            if pos is None:
                yield ("nbar", f"comb{quarter}", 2)
                if parity == 0:
                    tile, kb_lo, kb_hi, owner, whole = seg
                    if not owner:
                        yield ("nbar", "epi", 4)
                        if quarter == 0:
                            yield ("flag_set", cta)
                    elif not whole:
                        cc = cta - 1
                        while cc >= 0:
                            yield ("flag_wait", cc)
                            if unit_start(cc, units, grid) <= tile * kbs:
                                break
                            cc -= 1
                        yield ("nbar", "epi", 4)
                continue
            if not has(it0, c, 2, parity):
                continue
            yield ("wait", B["full"][ch % NCB], (ch // NCB) & 1)
            for t in range(c):
                i = it0 + t
                if i % 2 == parity:
                    yield ("wait", B["pfull"][i % NQ], (i // NQ) & 1)
                    yield ("arrive", B["pempty"][i % NQ])
                    yield ("arrive", B["empty_w"][pos + t])

    roles = {}
    for w in range(12):          # 3 dequant warps per lane quarter; the quarters move together
        roles[f"dq{w}"] = dq(w >> 2)
    for q in range(NQ):
        roles[f"iss{q}"] = issuer(q)
    roles["prod_w"] = producer("empty_w")
    roles["prod_a"] = producer("empty_a")
    for w in range(8):
        roles[f"acc{w}"] = acc(w & 3, w >> 2)
    return roles


def simulate(units, grid, kbs, chunk, slots):
    flags = {}
    ctas = []
    for cta in range(grid):
        B = {"full": [Bar(2, f"full{k}") for k in range(NCB)],
             "empty_w": [Bar(8, f"empty_w{s}") for s in range(slots)],
             "empty_a": [Bar(1, f"empty_a{s}") for s in range(slots)],
             "afull": [Bar(4, f"afull{a}") for a in range(NA)],
             "aempty": [Bar(1, f"aempty{a}") for a in range(NA)],
             "pfull": [Bar(1, f"pfull{q}") for q in range(NQ)],
             "pempty": [Bar(4, f"pempty{q}") for q in range(NQ)]}
        roles = _roles(cta, units, grid, kbs, chunk, slots, B)
        ctas.append({"cta": cta, "roles": roles, "cur": dict.fromkeys(roles), "done": set(),
                     "nbar": defaultdict(list)})
    moved = True
    while moved:
        moved = False
        for st in ctas:
            for name, gen in st["roles"].items():
                while name not in st["done"]:
                    op = st["cur"][name]
                    if op is None:
                        try:
                            op = st["cur"][name] = next(gen)
                        except StopIteration:
                            st["done"].add(name)
                            break
                    kind = op[0]
                    if kind == "wait" and not op[1].ready(op[2]):
                        break
                    if kind == "flag_wait" and not flags.get(op[1]):
                        break
                    if kind == "arrive":
                        op[1].arrive()
                    elif kind == "flag_set":
                        flags[op[1]] = 1
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
    return [(st["cta"], name, st["cur"][name]) for st in ctas for name in st["roles"] if name not in st["done"]]
