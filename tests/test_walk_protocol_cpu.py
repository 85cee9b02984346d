"""The synchronisation of the backward's dk/dv walk (bwd_walk_kernel in
linear_attention_11_b200/csrc/la_backward_walk.cu), modelled on the CPU.

Every role of one CTA (key-block copies, K/V copies, MMA issue, the two math
warpgroups) is written out as the sequence of waits, arrivals, copies and
MMAs it performs in the kernel, over the same cursor of (item, chunk, key
block).  MMAs and commits execute in issue order in a tensor-pipe queue at
random times; bulk copies land at random times in any order; a randomised
scheduler interleaves the roles.  Checked for many shapes and interleavings:

  - progress: some role can always move until every role has finished (a
    deadlock here would be a kernel timeout on the GPU);
  - parity: a wait for phase k of a barrier only starts, or stays blocked,
    while at most k + 1 phases have completed (a parity wait cannot tell
    phase k from phase k + 2);
  - data: every operand an MMA reads (ring slot, K/V slot, P over its scores
    in tensor memory, bf16 state copy) holds the version it was issued for
    when the MMA executes, and no copy, P store or state conversion
    overwrites a version a queued MMA still needs; each score buffer's P is
    multiplied before the next scores of its stream land; the state D is
    reloaded or converted before the next chunk's updates; dk, dv are read
    out before the next chunk starts them;
  - coverage: every (group, chunk, key block) is multiplied exactly once and
    every chunk's dk, dv are written exactly once.

The model mirrors the kernel as written; a change to the kernel's
synchronisation must be made here too.
"""
import random

import pytest

RING = 4
CHUNK, KEYBLK = 128, 64


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.done = 0      # completed phases
        self.pending = 0   # arrivals in the current phase

    def arrive(self):
        self.pending += 1
        assert self.pending <= self.count, f"{self.name}: too many arrivals"
        if self.pending == self.count:
            self.pending = 0
            self.done += 1


class Model:
    def __init__(self, B, Hq, Hkv, N, nspan, grid, cta, seed):
        self.G, self.Hkv, self.N, self.nspan = Hq // Hkv, Hkv, N, nspan
        self.tiles = (N + CHUNK - 1) // CHUNK
        self.items = B * Hkv * nspan
        self.grid, self.cta = grid, cta
        self.rng = random.Random(seed)
        mk = Barrier
        self.ring_full = [mk(f"ring_full{s}", 1) for s in range(RING)]
        self.ring_empty = [mk(f"ring_empty{s}", 1) for s in range(RING)]
        # K_n and the bf16 copy of D take turns in two regions (K_n in region
        # n % 2, D's copy for chunk n in region (n + 1) % 2); V has its own
        self.k_full, self.v_full = mk("k_full", 1), mk("v_full", 1)
        self.d_free, self.v_free = mk("d_free", 1), mk("v_free", 1)
        # two score streams, each in its own tensor-memory buffer: S1 = K_c Q^T
        # (masked by warpgroup 1 into P1, for dv) and S2 = V_c dO^T (warpgroup
        # 2, P2, for dk); each P is written over its own scores
        self.a_full = [mk("a_full1", 1), mk("a_full2", 1)]
        self.p_full = [mk("p_full1", 1), mk("p_full2", 1)]
        self.o_full = mk("o_full", 1)
        self.o_empty = [mk("o_empty0", 1), mk("o_empty1", 1)]
        self.s_full, self.sb_full = mk("s_full", 1), mk("sb_full", 1)
        self.waiting = {}      # role -> (barrier, phase)
        self.tensor = []       # queued MMAs and commits, executed in order
        self.copies = []       # (barrier, resource, version), landing in any order
        # resource versions
        self.ver = {("ring", s): None for s in range(RING)}
        self.ver.update({("R", 0): None, ("R", 1): None, "V": None, ("S", 0): None,
                         ("S", 1): None})
        self.sc_need = {0: None, 1: None}  # scores or P a buffer still owes its reader
        self.d_ready = 0              # D holds what chunk d_ready's updates need
        self.d_done = -1              # last chunk whose every update of D has executed
        self.acc = {1: None, 2: None}      # chunk of the last product into dv (1), dk (2)
        self.acc_read = {1: -1, 2: -1}     # last chunk each warpgroup wrote out
        self.multiplied, self.written = [], []

    # ----------------------------------------------------------- cursor
    def span_of(self, it):
        j = it % self.nspan
        return it // self.nspan, j * self.tiles // self.nspan, (j + 1) * self.tiles // self.nspan

    def halves(self, cs):
        return 2 if self.N - cs * CHUNK > KEYBLK else 1

    def blocks(self):
        """Blocks in the order every role walks them."""
        i = gc = 0
        for it in range(self.cta, self.items, self.grid):
            bg, tb, te = self.span_of(it)
            for n in range(te - tb):
                cs = te - 1 - n
                nb = self.G * self.halves(cs)
                for blk in range(nb):
                    yield dict(it=it, bg=bg, n=n, cs=cs, blk=blk, nb=nb, gc=gc, i=i)
                    i += 1
                gc += 1

    # ----------------------------------------------------------- primitives
    def wait(self, role, bar, phase):
        assert bar.done <= phase + 1, (
            f"{role}: waits for phase {phase} of {bar.name} after {bar.done} completed")
        self.waiting[role] = (bar, phase)
        while bar.done <= phase:
            yield
        del self.waiting[role]

    def mma(self, name, reads=(), run=None):
        self.tensor.append(("mma", name, tuple(reads), run))

    def commit(self, bar):
        self.tensor.append(("commit", bar))

    def queued_reads(self, res):
        return [v for e in self.tensor if e[0] == "mma" for r, v in e[2] if r == res]

    def overwrite(self, res, version, who):
        stale = [v for v in self.queued_reads(res) if v != version]
        assert not stale, f"{who}: overwrites {res} while queued MMAs still need {stale}"
        self.ver[res] = version

    def expect(self, res, v, who):
        assert self.ver[res] == v, f"{who}: {res} holds {self.ver[res]}, wants {v}"

    def land(self, res, v):
        self.overwrite(res, v, f"copy into {res}")

    def execute(self):
        e = self.tensor.pop(0)
        if e[0] == "commit":
            e[1].arrive()
            return
        _, name, reads, run = e
        for res, v in reads:
            assert self.ver[res] == v, f"{name}: reads {res} = {self.ver[res]}, issued for {v}"
        if run:
            run()

    # ----------------------------------------------------------- roles
    def producer_ring(self):
        for x in self.blocks():
            s = x["i"] % RING
            if x["i"] >= RING:
                yield from self.wait("ring", self.ring_empty[s], x["i"] // RING - 1)
            self.copies.append((self.ring_full[s], ("ring", s), x["i"]))
            yield

    def producer_kv(self):
        gc = 0
        for it in range(self.cta, self.items, self.grid):
            _, tb, te = self.span_of(it)
            for _n in range(te - tb):
                # K into the region the previous chunk's D copy held, then V
                if gc >= 1:
                    yield from self.wait("kv", self.d_free, gc - 1)
                self.copies.append((self.k_full, ("R", gc % 2), ("K", gc)))
                yield
                if gc >= 1:
                    yield from self.wait("kv", self.v_free, gc - 1)
                self.copies.append((self.v_full, "V", gc))
                gc += 1
                yield

    def mma_role(self):
        # Per block k: dv += P1(k) dO(k), the next block's S1, dk += P2(k) Q(k),
        # the next block's S2, at a chunk's first block K_c D and V_c D^T, then
        # D += Q(k)^T dO(k).  A stream's next scores follow its product, so the
        # tensor pipe's order keeps them off P until P has been used, and each
        # mask has the other stream's product and scores and D's update to run
        # under it.
        seq = list(self.blocks())
        st = {"inter_gc": -1, "kv_pending": -1}

        def scores(t, i):
            def run():
                assert self.sc_need[t] is None, (
                    f"S{t + 1}({i}) lands on {self.sc_need[t]} before it was used")
                self.ver[("S", t)] = ("A", i)
                self.sc_need[t] = ("A", i)
            return run

        def product(wg, gc, first, t=None):
            def run():
                if first:
                    assert self.acc_read[wg] >= gc - 1, (
                        f"chunk {gc} starts accumulator {wg} before chunk {gc - 1} was read out")
                self.acc[wg] = gc
                if t is not None:
                    self.sc_need[t] = None
            return run

        def update(gc, last):
            def run():
                assert self.d_ready >= gc, f"update of chunk {gc} before D was ready for it"
                if last:
                    self.d_done = gc
            return run

        def issue_s(t, x):
            gc = x["gc"]
            if x["blk"] == 0:
                yield from self.wait("mma", self.k_full if t == 0 else self.v_full, gc)
            s = x["i"] % RING
            yield from self.wait("mma", self.ring_full[s], x["i"] // RING)
            src = (("R", gc % 2), ("K", gc)) if t == 0 else ("V", gc)
            self.mma(f"S{t + 1}({x['i']})", [(("ring", s), x["i"]), src], scores(t, x["i"]))
            self.commit(self.a_full[t])
            # S2 of a chunk's last block is V's last score reader
            if t == 1 and x["blk"] == x["nb"] - 1:
                if st["inter_gc"] >= x["gc"]:
                    self.commit(self.v_free)
                else:
                    st["kv_pending"] = x["gc"]

        if seq:
            yield from issue_s(0, seq[0])
            yield from issue_s(1, seq[0])
        for idx, c in enumerate(seq):
            k, gc, s = c["i"], c["gc"], c["i"] % RING
            nxt = seq[idx + 1] if idx + 1 < len(seq) else None
            first, last = c["blk"] == 0, c["blk"] == c["nb"] - 1
            yield from self.wait("mma", self.p_full[0], k)
            # (implied by P1 since warpgroup 1 reads dv out before this mask;
            # the kernel keeps the direct wait as well)
            if first and gc >= 1:
                yield from self.wait("mma", self.o_empty[0], gc - 1)
            self.mma(f"dv+=P1dO({k})", [(("ring", s), k), (("S", 0), ("P", k))],
                     product(1, gc, first, 0))
            # a next chunk's scores wait for its K and V, whose regions free up
            # with this chunk's K_c D, V_c D^T and last S2: at a chunk
            # boundary they go last
            if nxt and nxt["blk"] != 0:
                yield from issue_s(0, nxt)
            yield from self.wait("mma", self.p_full[1], k)
            if first and gc >= 1:
                yield from self.wait("mma", self.o_empty[1], gc - 1)
            self.mma(f"dk+=P2Q({k})", [(("ring", s), k), (("S", 1), ("P", k))],
                     product(2, gc, first, 1))
            if nxt and nxt["blk"] != 0:
                yield from issue_s(1, nxt)
            if first:
                # the bf16 copy of D for this chunk; D's first update of the
                # chunk waits for it too (the conversion reads D)
                yield from self.wait("mma", self.sb_full, gc)
                kreg, dreg = (("R", gc % 2), ("K", gc)), (("R", (gc + 1) % 2), ("D", gc))
                self.mma(f"dv+=KD({gc})", [kreg, dreg], product(1, gc, False))
                self.mma(f"dk+=VD^T({gc})", [("V", gc), dreg], product(2, gc, False))
                self.commit(self.d_free)
                st["inter_gc"] = gc
                if st["kv_pending"] == gc:
                    self.commit(self.v_free)
                    st["kv_pending"] = -1
            self.mma(f"D+=QdO({k})", [(("ring", s), k)], update(gc, last))
            self.commit(self.ring_empty[s])
            if last:
                self.commit(self.o_full)
                self.commit(self.s_full)
            self.multiplied.append((c["bg"], c["cs"], c["blk"]))
            if nxt and nxt["blk"] == 0:
                yield from issue_s(0, nxt)
                yield from issue_s(1, nxt)
            yield

    def warpgroup(self, wg):
        role = f"wg{wg}"
        prev = None

        def write_out(p):
            # the accumulator is read into registers and released; the rows
            # go to global memory later (a quarter after each of the next four
            # masks), outside the protocol
            yield from self.wait(role, self.o_full, p["gc"])
            assert self.acc[wg] == p["gc"], f"{role}: reads chunk {p['gc']}, holds {self.acc[wg]}"
            self.acc_read[wg] = p["gc"]
            self.o_empty[wg - 1].arrive()
            self.written.append((role, p["bg"], p["cs"]))

        def state_ready(gc):
            # D after chunk gc - 1 is read (converted, or the final state at
            # an item's end); the bf16 copy (and at an item start D itself)
            # now serve chunk gc
            if gc > 0:
                assert self.d_done == gc - 1, f"{role}: reads D for chunk {gc} after chunk {self.d_done}"
            d_region = ("R", (gc + 1) % 2)
            self.overwrite(d_region, ("D", gc), role)
            self.d_ready = gc
            self.sb_full.arrive()

        if wg == 1:
            state_ready(0)
        t = wg - 1
        for c in self.blocks():
            k = c["i"]
            # at a chunk boundary the previous chunk's accumulator is read out
            # first (the chunk's first product waits for it), the state
            # converted after the mask (its first use comes later)
            boundary = c["blk"] == 0 and prev is not None
            if boundary:
                yield from write_out(prev)
            yield from self.wait(role, self.a_full[t], k)
            self.expect(("S", t), ("A", k), f"{role}: mask({k})")
            self.overwrite(("S", t), ("P", k), role)  # P over its scores
            self.sc_need[t] = ("P", k)
            self.p_full[t].arrive()
            yield
            if boundary and wg == 1:
                yield from self.wait(role, self.s_full, prev["gc"])
                state_ready(c["gc"])
            prev = c
        if prev is not None:
            if wg == 1:
                yield from self.wait(role, self.s_full, prev["gc"])
                assert self.d_done == prev["gc"], f"{role}: final state read early"
            yield from write_out(prev)

    # ----------------------------------------------------------- scheduler
    def run(self):
        live = {"ring": self.producer_ring(), "kv": self.producer_kv(), "mma": self.mma_role(),
                "wg1": self.warpgroup(1), "wg2": self.warpgroup(2)}
        idle = 0
        # random speeds per run, so that some runs leave a role or a queue
        # nearly frozen while the others race ahead
        speed = {name: self.rng.choice((0.02, 0.3, 1.0, 1.0, 4.0)) for name in live}
        p_tensor = self.rng.choice((0.05, 0.3, 0.6))
        p_copy = self.rng.choice((0.05, 0.3, 0.6))
        while live or self.tensor or self.copies:
            moved = False
            choice = self.rng.random()
            if self.tensor and choice < p_tensor:
                self.execute()
                moved = True
            elif self.copies and choice < p_tensor + p_copy * (1 - p_tensor):
                bar, res, v = self.copies.pop(self.rng.randrange(len(self.copies)))
                self.land(res, v)
                bar.arrive()
                moved = True
            elif live:
                names = list(live)
                name = self.rng.choices(names, weights=[speed[n] for n in names])[0]
                before = self.waiting.get(name)
                try:
                    next(live[name])
                except StopIteration:
                    del live[name]
                    moved = True
                else:
                    moved = before is None or self.waiting.get(name) != before
            for role, (bar, phase) in self.waiting.items():
                assert bar.done <= phase + 1, (
                    f"{role}: blocked on phase {phase} of {bar.name}, {bar.done} completed")
            idle = 0 if moved else idle + 1
            if idle > 20000:
                blocked = {r: (b.name, p, b.done) for r, (b, p) in self.waiting.items()}
                raise AssertionError(f"no progress: {blocked}, live {sorted(live)}")
        return self


def _walk_spans(units, tiles, sms, G):
    """The host planner's span choice (walk_spans in la_backward_walk.cu)."""
    r_span = (2.0 * G) / (2.0 * G + 4.0)
    best, best_cost = 1, float("inf")
    for ns in range(1, min(tiles, 256) + 1):
        rounds = -(-units * ns // sms)
        cost = rounds * -(-tiles // ns)
        if ns > 1:
            cost += (ns - 1) / ns * units * tiles * r_span / sms + 1.0
        if cost < best_cost - 1e-9:
            best, best_cost = ns, cost
    return best


SHAPES = [
    # B, Hq, Hkv, N, nspan, grid
    (1, 1, 1, 1, 1, 1),         # one token: one chunk with one key block
    (1, 1, 1, 129, 2, 2),       # G = 1, a one-block chunk at an item start
    (1, 1, 1, 300, 1, 1),       # G = 1, one-block chunk after two full ones
    (1, 1, 1, 64, 1, 1),        # exactly one half chunk
    (1, 3, 1, 385, 2, 1),       # both spans on one CTA, ragged last chunk
    (2, 4, 2, 777, 3, 5),       # several items per CTA, G = 4
    (1, 16, 1, 500, 2, 1),      # G = 16
    (4, 8, 8, 200, 1, 3),       # many groups, one span each
    (1, 8, 1, 2000, 4, 3),      # many spans of a long sequence
    (3, 2, 1, 129, 2, 4),       # G = 2 with one-block chunks, items over CTAs
]


@pytest.mark.parametrize("B,Hq,Hkv,N,nspan,grid", SHAPES)
def test_walk_protocol(B, Hq, Hkv, N, nspan, grid):
    items = B * Hkv * nspan
    grid = min(grid, items)
    tiles = (N + CHUNK - 1) // CHUNK
    assert 1 <= nspan <= tiles
    multiplied, written = [], []
    for cta in range(grid):
        for seed in range(10):
            m = Model(B, Hq, Hkv, N, nspan, grid, cta, seed=1000 * cta + seed).run()
            if seed == 0:
                multiplied += m.multiplied
                written += m.written
    G = Hq // Hkv
    want = [(bg, cs, blk) for bg in range(B * Hkv) for cs in range(tiles)
            for blk in range(G * (2 if N - cs * CHUNK > KEYBLK else 1))]
    assert sorted(multiplied) == sorted(want)
    chunks = sorted((bg, cs) for bg in range(B * Hkv) for cs in range(tiles))
    for role in ("wg1", "wg2"):
        assert sorted((bg, cs) for r, bg, cs in written if r == role) == chunks


def test_planner_spans_fit_the_chunks():
    """The span counts the host planner can pick leave every span a chunk."""
    for units in (1, 3, 32, 200):
        for tiles in (1, 2, 9, 256, 8192):
            for G in (1, 4, 16):
                ns = _walk_spans(units, tiles, 148, G)
                assert 1 <= ns <= tiles


# Planted mistakes: each removes or weakens one wait, moves one issue, or
# merges two barriers, as a plausible slip would, and must fail the model.
MUTANTS = {
    "dv without its P1": (
        "            yield from self.wait(\"mma\", self.p_full[0], k)\n", ""),
    "dk without its P2": (
        "            yield from self.wait(\"mma\", self.p_full[1], k)\n", ""),
    "mask without its scores": (
        "            yield from self.wait(role, self.a_full[t], k)\n", ""),
    "state terms before the bf16 copy of D": (
        "                yield from self.wait(\"mma\", self.sb_full, gc)\n", ""),
    "key block copied into a busy stage": (
        "                yield from self.wait(\"ring\", self.ring_empty[s], x[\"i\"] // RING - 1)\n",
        "                pass\n"),
    "K copied over D's copy before its readers ran": (
        "                    yield from self.wait(\"kv\", self.d_free, gc - 1)\n",
        "                    pass\n"),
    "V copied into the busy region": (
        "                    yield from self.wait(\"kv\", self.v_free, gc - 1)\n",
        "                    pass\n"),
    "D's copy written over the chunk's own K": (
        "            d_region = (\"R\", (gc + 1) % 2)\n",
        "            d_region = (\"R\", gc % 2)\n"),
    "next S1 ahead of the dv that reads P1": (
        "            self.mma(f\"dv+=P1dO({k})\", [((\"ring\", s), k), ((\"S\", 0), (\"P\", k))],\n"
        "                     product(1, gc, first, 0))\n"
        "            # a next chunk's scores wait for its K and V, whose regions free up\n"
        "            # with this chunk's K_c D, V_c D^T and last S2: at a chunk\n"
        "            # boundary they go last\n"
        "            if nxt and nxt[\"blk\"] != 0:\n"
        "                yield from issue_s(0, nxt)\n",
        "            if nxt and nxt[\"blk\"] != 0:\n"
        "                yield from issue_s(0, nxt)\n"
        "            self.mma(f\"dv+=P1dO({k})\", [((\"ring\", s), k), ((\"S\", 0), (\"P\", k))],\n"
        "                     product(1, gc, first, 0))\n"),
    "V released at the last S1 instead of the last S2": (
        "            if t == 1 and x[\"blk\"] == x[\"nb\"] - 1:\n",
        "            if t == 0 and x[\"blk\"] == x[\"nb\"] - 1:\n"),
    "one p_full barrier for both streams": (
        "        self.p_full = [mk(\"p_full1\", 1), mk(\"p_full2\", 1)]",
        "        self.p_full = [mk(\"p_full\", 1)] * 2"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_walk_mistakes(name):
    import inspect
    import sys
    old, new = MUTANTS[name]
    src = inspect.getsource(sys.modules[__name__])
    src = src[:src.index("\n# Planted mistakes")]
    assert src.count(old) == 1, name
    ns = {"__name__": f"walk_mutant_{abs(hash(name))}"}
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    caught = False
    for shape in ns["SHAPES"]:
        try:
            ns["test_walk_protocol"](*shape)
        except AssertionError:
            caught = True
            break
    assert caught, f"planted mistake '{name}' passed the model"
