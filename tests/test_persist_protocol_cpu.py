"""The synchronisation of the prefill's persistent chunk-loop kernel
(prefill_persist_kernel in linear_attention_11_b200/csrc/la_prefill_persist.cu),
modelled on the CPU, for the four forward configurations the launcher
instantiates: 64-token tiles with a dedicated output tile, 64-token tiles with
staged states (output through the Q slot), 128-token tiles with one tile per
chunk step (K and V tiles together in two slots), and 128-token tiles with
several (K and V tiles apart in a three-slot ring, three Q slots, the state
update ahead of the step's last P V).

Each role of one CTA (Q copies, K/V copies, staged-state copies, MMA issue,
the mask warpgroup, the output warpgroup; both warpgroups convert the state)
is written out as its sequence of barrier waits, arrivals, copies and MMAs
over the same items, chunk steps and head subsets as the kernel.  MMAs and
commits execute in issue order at random times, copies land at random times,
and a randomised scheduler interleaves the roles.  The bulk store of a
staged final state reads the staging tile at a random later time, and the
tile is released only then: the other warps do not wait for that store, so
they may reach the next hand-over first.  Checked: progress; that
no parity wait can see its barrier two phases ahead; that every operand an
MMA reads (Q slot, K/V slot, bf16 state copy, score/output buffer, P buffer)
holds the version it was issued for when it executes and that nothing
overwrites a version a queued MMA or a pending store still needs; that the
state is read after its update and reloaded before the next one; and that
every tile is written out once.  A change to the kernel's synchronisation
must be made here too.
"""
import random

import pytest

from test_walk_protocol_cpu import Barrier


class Model:
    def __init__(self, T, QST, KVST, out, staged, G, units, nspan, tiles, grid, cta, s_out,
                 seed, halfkv=False):
        # out: "dedicated" (output tile of its own), "qslot" (output staged in
        # the tile's Q slot), "direct" (registers to global memory, no staging)
        self.T, self.QST, self.KVST, self.out, self.staged = T, QST, KVST, out, staged
        # halfkv: K of chunk step c is copy 2c of the K/V ring, V copy 2c + 1
        # (else one copy c holds both)
        self.halfkv = halfkv
        self.dedo = out == "dedicated"
        self.nsub = G // (128 // T)
        self.nspan, self.tiles, self.items = nspan, tiles, units * nspan
        self.grid, self.cta, self.s_out = grid, cta, s_out
        # score buffers in tensor memory (P is written over its scores): two
        # of 64 columns at T = 64, which lets QK of the next tile go ahead of
        # PV; one of 128 at T = 128
        self.nsc = 2 if T == 64 else 1
        # at T = 128 the mask hands P over in two halves of 64 keys, each
        # multiplied by V (P V in two halves) as soon as it is written
        self.halves = 2 if T == 128 else 1
        self.rng = random.Random(seed)
        mk = Barrier
        self.q_full = [mk(f"q_full{s}", 1) for s in range(QST)]
        self.q_empty = [mk(f"q_empty{s}", 2 if out == "qslot" else 1) for s in range(QST)]
        self.kv_full = [mk(f"kv_full{s}", 1) for s in range(KVST)]
        self.kv_empty = [mk(f"kv_empty{s}", 1) for s in range(KVST)]
        self.a_full = [mk(f"a_full{b}", 1) for b in range(self.nsc)]
        # per score buffer at T = 64; per half of the one buffer at T = 128
        self.p_full = [mk(f"p_full{b}", 1) for b in range(max(self.nsc, self.halves))]
        self.o_full = [mk("o_full0", 1), mk("o_full1", 1)]
        self.o_empty = [mk("o_empty0", 1), mk("o_empty1", 1)]
        self.s_full, self.sb_full = mk("s_full", 1), mk("sb_full", 2)
        self.store_ready, self.ostage_free = mk("store_ready", 1), mk("ostage_free", 1)
        self.st_full, self.st_empty, self.stage_done = (mk("st_full", 1), mk("st_empty", 1),
                                                       mk("stage_done", 2))
        self.waiting, self.tensor, self.copies = {}, [], []
        # final-state stores in flight: a bulk store reads the staging tile at
        # some later time, then warp 6 releases the tile (st_empty); the other
        # warps of both warpgroups do not wait for it
        self.state_stores = []
        self.ver = {("q", s): None for s in range(QST)}
        self.ver.update({("kv", s): None for s in range(KVST)})
        self.ver.update({("obuf", 0): None, ("obuf", 1): None, ("sc", 0): None, ("sc", 1): None,
                         "sS": 0, "ostage": None, ("staging", 0): None, ("staging", 1): None})
        self.ver.update({("ph", b, h): None for b in range(2) for h in range(2)})
        self.stage_need = {0: None, 1: None}  # what each half of the staging tile still owes
        self.obuf_need = {0: None, 1: None}   # output a buffer still owes the epilogue
        self.sc_need = {0: None, 1: None}     # scores the mask, or P the PV, has yet to read
        self.state_chunk = None   # the chunk step after which the state in TMEM is final
        self.state_ready = 0      # the chunk step whose update may run next
        self.stored = []

    # ----------------------------------------------------------- schedule
    def next_item(self, it):
        return it + self.grid if it + self.grid < self.items else -1

    def steps(self):
        """(k, it, n, hs, i, gc, last_hs, item_end, has_next) as every role walks them."""
        i = gc = 0
        for k, it in enumerate(range(self.cta, self.items, self.grid)):
            j = it % self.nspan
            tb, te = j * self.tiles // self.nspan, (j + 1) * self.tiles // self.nspan
            last_item = self.next_item(it) < 0
            for n in range(te - tb):
                for hs in range(self.nsub):
                    last_hs = hs == self.nsub - 1
                    item_end = last_hs and n == te - tb - 1
                    yield dict(k=k, it=it, n=n, hs=hs, i=i, gc=gc, last_hs=last_hs,
                               item_end=item_end, has_next=not (last_item and item_end))
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

    def mma(self, name, reads, run=None):
        self.tensor.append(("mma", name, tuple(reads), run))

    def commit(self, bar):
        self.tensor.append(("commit", bar))

    def overwrite(self, res, version, who):
        stale = [v for e in self.tensor if e[0] == "mma" for r, v in e[2]
                 if r == res and v != version]
        assert not stale, f"{who}: overwrites {res} while queued MMAs still need {stale}"
        self.ver[res] = version

    def expect(self, res, version, who):
        assert self.ver[res] == version, f"{who}: {res} holds {self.ver[res]}, wants {version}"

    def land(self, res, v):
        if res != "staging":
            self.overwrite(res, v, f"copy into {res}")
            return
        for h in (0, 1):
            assert self.stage_need[h] is None, (
                f"state copy {v[1]} overwrites {self.stage_need[h]} of half {h}")
            self.ver[("staging", h)] = v
            self.stage_need[h] = v

    def store_state(self):
        k = self.state_stores.pop(0)
        for h in (0, 1):
            self.expect(("staging", h), ("out", k), "final-state store")
            self.stage_need[h] = None
        self.st_empty.arrive()

    def execute(self):
        e = self.tensor.pop(0)
        if e[0] == "commit":
            e[1].arrive()
            return
        _, name, reads, run = e
        for res, v in reads:
            self.expect(res, v, name)
        if run:
            run()

    # ----------------------------------------------------------- copy lanes
    def q_lane(self):
        for x in self.steps():
            i, s = x["i"], x["i"] % self.QST
            if i >= self.QST:
                yield from self.wait("q", self.q_empty[s], i // self.QST - 1)
            self.copies.append((self.q_full[s], ("q", s), ("Q", i)))
            yield

    def kcopy(self, gc):
        return 2 * gc if self.halfkv else gc

    def vcopy(self, gc):
        return 2 * gc + 1 if self.halfkv else gc

    def kver(self, gc):
        return ("K", gc) if self.halfkv else gc

    def vver(self, gc):
        return ("V", gc) if self.halfkv else gc

    def kv_lane(self):
        u = 0
        for x in self.steps():
            if not x["last_hs"]:
                continue
            gc = x["gc"]
            for ver in ((self.kver(gc), self.vver(gc)) if self.halfkv else (gc,)):
                s = u % self.KVST
                if u >= self.KVST:
                    yield from self.wait("kv", self.kv_empty[s], u // self.KVST - 1)
                self.copies.append((self.kv_full[s], ("kv", s), ver))
                u += 1
                yield

    def stage_lane(self):
        for k, _it in enumerate(range(self.cta, self.items, self.grid)):
            if k >= 1:
                yield from self.wait("st", self.st_empty, k - 1)
            self.copies.append((self.st_full, "staging", ("in", k)))  # both halves
            yield

    # ----------------------------------------------------------- MMA
    def mma_role(self):
        seq = list(self.steps())

        def qk(i, gci):
            sc = i % self.nsc
            ku = self.kcopy(gci)
            yield from self.wait("mma", self.q_full[i % self.QST], i // self.QST)
            yield from self.wait("mma", self.kv_full[ku % self.KVST], ku // self.KVST)

            def run():
                assert self.sc_need[sc] is None, (
                    f"QK({i}) overwrites {self.sc_need[sc]} before it was read")
                self.ver[("sc", sc)] = ("A", i)
                self.sc_need[sc] = ("A", i)
            self.mma(f"QK({i})", [(("q", i % self.QST), ("Q", i)),
                                  (("kv", ku % self.KVST), self.kver(gci))], run)
            self.commit(self.a_full[sc])

        def wait_v(gci):
            vu = self.vcopy(gci)
            yield from self.wait("mma", self.kv_full[vu % self.KVST], vu // self.KVST)

        def kv(gci):
            if self.halfkv:
                yield from wait_v(gci)

            def run():
                assert self.state_ready >= gci, f"KV({gci}) before the state was ready"
                self.state_chunk = gci
            ku, vu = self.kcopy(gci), self.vcopy(gci)
            self.mma(f"KV({gci})", [(("kv", ku % self.KVST), self.kver(gci)),
                                    (("kv", vu % self.KVST), self.vver(gci))], run)
            self.commit(self.s_full)
            self.commit(self.kv_empty[ku % self.KVST])  # K's last reader

        yield from qk(0, 0)
        for x in seq:
            i, gc, ob, sc = x["i"], x["gc"], x["i"] & 1, x["i"] % self.nsc
            if x["hs"] == 0:
                yield from self.wait("mma", self.sb_full, gc)
            if i >= 2:
                yield from self.wait("mma", self.o_empty[ob], (i >> 1) - 1)

            def qs_run(ob=ob, i=i):
                assert self.obuf_need[ob] is None, f"QS({i}) overwrites unread output"
                self.ver[("obuf", ob)] = ("O", i)

            def pv_run(ob=ob, i=i, sc=sc):
                self.sc_need[sc] = None
                self.obuf_need[ob] = ("O", i)

            def pv_half_run():
                pass
            self.mma(f"QS({i})", [(("q", i % self.QST), ("Q", i)), ("sS", gc)], qs_run)
            self.commit(self.q_empty[i % self.QST])
            nxt = gc + 1 if x["last_hs"] else gc
            # with two score buffers the next tile's scores go ahead of PV
            # (inside an item; at its end the state update goes first)
            early = self.nsc == 2 and not self.staged and not x["item_end"]
            if early:
                yield from qk(i + 1, nxt)
            vu = self.vcopy(gc)
            # with K and V apart the update goes before the step's last P V
            if self.halfkv and x["last_hs"]:
                yield from kv(gc)
            if self.halfkv:
                yield from wait_v(gc)
            release_v_early = False
            if release_v_early and self.halfkv and x["last_hs"]:
                self.commit(self.kv_empty[vu % self.KVST])
            for h in range(self.halves):
                pf = self.p_full[h] if self.halves == 2 else self.p_full[sc]
                yield from self.wait("mma", pf, i // self.nsc)
                last_half = h == self.halves - 1
                self.mma(f"PV{h}({i})", [(("ph", sc, h), ("P", i)),
                                         (("kv", vu % self.KVST), self.vver(gc)),
                                         (("obuf", ob), ("O", i))],
                         pv_run if last_half else pv_half_run)
            self.commit(self.o_full[ob])
            if self.halfkv and x["last_hs"] and not release_v_early:
                self.commit(self.kv_empty[vu % self.KVST])  # V's last reader
            if not self.halfkv and x["last_hs"]:
                yield from kv(gc)
            if not early and x["has_next"]:
                yield from qk(i + 1, nxt)
            yield

    # ----------------------------------------------------------- warpgroups
    def state_in(self, role, gc):
        """A new state version (the next chunk's bf16 copy, or an item's
        entering state) for chunk step gc."""
        self.overwrite("sS", gc, role)
        self.state_ready = gc
        self.sb_full.arrive()

    def stage_swap(self, role, have_in, have_out, k, gc):
        h = 0 if role == "mask" else 1  # each warpgroup swaps its own columns
        if have_in:
            self.expect(("staging", h), ("in", k), role)
            self.stage_need[h] = None
        if have_out:
            assert self.state_chunk == gc - 1, f"{role}: final state of {gc - 1} read early"
            assert self.stage_need[h] is None, (
                f"{role}: final state {k - 1} overwrites {self.stage_need[h]} of half {h}")
            self.ver[("staging", h)] = ("out", k - 1)
            self.stage_need[h] = ("out", k - 1)
        if have_in:
            self.state_in(role, gc)
        self.stage_done.arrive()

    def state_step(self, role, x, nx):
        gc, k = x["gc"], x["k"]
        yield from self.wait(role, self.s_full, gc)
        assert self.state_chunk == gc, f"{role}: state of chunk step {gc} read early"
        if x["item_end"] and self.staged:
            if nx >= 0:
                yield from self.wait(role, self.st_full, k + 1)
            elif self.s_out:
                # no state comes in to order the reuse: wait until the
                # previous final state's store has read the tile
                yield from self.wait(role, self.st_empty, k)
            self.stage_swap(role, nx >= 0, self.s_out, k + 1, gc + 1)
        elif not x["item_end"]:
            self.state_in(role, gc + 1)
        elif nx >= 0:
            self.state_in(role, gc + 1)

    def first_state(self, role):
        # both warpgroups bring in half of the CTA's first entering state
        if self.staged:
            yield from self.wait(role, self.st_full, 0)
            self.stage_swap(role, True, False, 0, 0)
        else:
            self.state_in(role, 0)

    def mask_role(self):
        role = "mask"
        yield from self.first_state(role)

        def mask_tile(i):
            sc = i % self.nsc
            yield from self.wait(role, self.a_full[sc], i // self.nsc)
            self.expect(("sc", sc), ("A", i), f"mask({i})")
            self.sc_need[sc] = ("P", i)
            for h in range(self.halves):  # P over its scores, half by half
                self.overwrite(("ph", sc, h), ("P", i), f"mask({i})")
                (self.p_full[h] if self.halves == 2 else self.p_full[sc]).arrive()
                if h + 1 < self.halves:
                    yield

        yield from mask_tile(0)
        for x in self.steps():
            nx = self.next_item(x["it"])
            # the MMA order decides which is ready first: with the next tile's
            # scores ahead of PV (two score buffers, inside an item) the mask
            # comes before the state step
            mask_first = self.nsc == 2 and not self.staged and not x["item_end"]
            for ph in (0, 1):
                do_step = x["last_hs"] and ph == (1 if mask_first else 0)
                do_mask = x["has_next"] and ph == (0 if mask_first else 1)
                if do_mask:
                    yield from mask_tile(x["i"] + 1)
                if do_step:
                    yield from self.state_step(role, x, nx)
            yield

    def out_role(self):
        role = "out"
        yield from self.first_state(role)
        if self.staged:
            yield from self.wait(role, self.stage_done, 0)
            self.st_empty.arrive()
        for x in self.steps():
            i, ob, k = x["i"], x["i"] & 1, x["k"]
            nx = self.next_item(x["it"])
            if x["last_hs"]:
                yield from self.state_step(role, x, nx)
            if self.staged and x["item_end"]:
                yield from self.wait(role, self.stage_done, k + 1)
                if self.s_out:
                    self.state_stores.append(k)
                else:
                    self.st_empty.arrive()
            yield from self.wait(role, self.o_full[ob], i >> 1)
            if self.out == "direct":  # registers to global memory, no tile to stage in
                self.expect(("obuf", ob), ("O", i), f"epilogue({i})")
                self.obuf_need[ob] = None
                self.o_empty[ob].arrive()
                self.stored.append((x["it"], x["n"], x["hs"]))
                yield
                continue
            if self.dedo and i > 0:
                yield from self.wait(role, self.ostage_free, i - 1)
            self.expect(("obuf", ob), ("O", i), f"epilogue({i})")
            self.obuf_need[ob] = None
            stage = "ostage" if self.dedo else ("q", i % self.QST)
            self.overwrite(stage, ("out", i), f"epilogue({i})")
            self.o_empty[ob].arrive()
            self.store_ready.arrive()
            yield from self.wait(role, self.store_ready, i)
            self.expect(stage, ("out", i), f"store({i})")   # the store reads the tile
            self.stored.append((x["it"], x["n"], x["hs"]))
            (self.ostage_free if self.dedo else self.q_empty[i % self.QST]).arrive()
            yield

    # ----------------------------------------------------------- scheduler
    def run(self):
        live = {"q": self.q_lane(), "kv": self.kv_lane(), "mma": self.mma_role(),
                "mask": self.mask_role(), "out": self.out_role()}
        if self.staged:
            live["st"] = self.stage_lane()
        idle = 0
        # random speeds per run, so that some runs leave a role or a queue
        # nearly frozen while the others race ahead
        speed = {name: self.rng.choice((0.02, 0.3, 1.0, 1.0, 4.0)) for name in live}
        p_tensor = self.rng.choice((0.05, 0.3, 0.6))
        p_copy = self.rng.choice((0.05, 0.3, 0.6))
        while live or self.tensor or self.copies or self.state_stores:
            moved = False
            choice = self.rng.random()
            if self.state_stores and self.rng.random() < p_copy:
                self.store_state()
                moved = True
            elif self.tensor and choice < p_tensor:
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


CONFIGS = {
    "t64_dedicated_out": dict(T=64, QST=3, KVST=2, out="dedicated", staged=False),
    "t64_staged": dict(T=64, QST=2, KVST=2, out="qslot", staged=True),
    "t128": dict(T=128, QST=2, KVST=2, out="qslot", staged=False),
    "t128_half_kv": dict(T=128, QST=3, KVST=3, out="qslot", staged=False, halfkv=True),
}

SHAPES = [
    # G, units, nspan, tiles, grid, s_out
    (2, 1, 1, 1, 1, True),
    (2, 3, 1, 1, 2, True),      # one-tile items, several per CTA (the staged case)
    (2, 9, 1, 1, 2, True),      # the same with more items per CTA
    (4, 2, 1, 4, 1, False),
    (4, 1, 3, 7, 2, False),     # spans of unequal length
    (8, 5, 1, 2, 3, True),
    (2, 2, 4, 9, 3, False),
]


@pytest.mark.parametrize("config", sorted(CONFIGS))
@pytest.mark.parametrize("G,units,nspan,tiles,grid,s_out", SHAPES)
def test_persist_protocol(config, G, units, nspan, tiles, grid, s_out):
    cfg = CONFIGS[config]
    if cfg["staged"] and nspan != 1:
        pytest.skip("states are staged with one span per sequence only")
    items = units * nspan
    grid = min(grid, items)
    stored = []
    # short one-span items (the staged case) get more interleavings
    seeds = 48 if nspan == 1 and tiles <= 2 else 8
    for cta in range(grid):
        for seed in range(seeds):
            m = Model(G=G, units=units, nspan=nspan, tiles=tiles, grid=grid, cta=cta,
                      s_out=s_out, seed=100 * cta + seed, **cfg).run()
            if seed == 0:
                stored += [(it, n, hs) for it, n, hs in m.stored]
    nsub = G // (128 // cfg["T"])
    want = []
    for it in range(items):
        j = it % nspan
        steps = (j + 1) * tiles // nspan - j * tiles // nspan
        want += [(it, n, hs) for n in range(steps) for hs in range(nsub)]
    assert sorted(stored) == sorted(want)


# Planted mistakes: each removes or weakens one wait or barrier count of the
# kernel's protocol, as a plausible slip would, and must fail the model.
MUTANTS = {
    "epilogue without o_full": (
        "            yield from self.wait(role, self.o_full[ob], i >> 1)\n", ""),
    "QS without o_empty": (
        "            if i >= 2:\n"
        "                yield from self.wait(\"mma\", self.o_empty[ob], (i >> 1) - 1)\n", ""),
    "mask without a_full": (
        "            yield from self.wait(role, self.a_full[sc], i // self.nsc)\n", ""),
    "PV without p_full": (
        "                yield from self.wait(\"mma\", pf, i // self.nsc)\n", ""),
    "next scores ahead of PV with one score buffer": (
        "            early = self.nsc == 2 and not self.staged and not x[\"item_end\"]\n",
        "            early = not x[\"item_end\"]\n"),
    "one a_full barrier for two score buffers": (
        "        self.a_full = [mk(f\"a_full{b}\", 1) for b in range(self.nsc)]",
        "        self.a_full = [mk(\"a_full\", 1)] * self.nsc"),
    "K/V copy without kv_empty": (
        "                if u >= self.KVST:\n"
        "                    yield from self.wait(\"kv\", self.kv_empty[s], u // self.KVST - 1)\n",
        ""),
    "P V without its V tile": (
        "            if self.halfkv:\n"
        "                yield from wait_v(gc)\n", ""),
    "V tile released before its last P V": (
        "            release_v_early = False\n", "            release_v_early = True\n"),
    "Q copy without q_empty": (
        "            if i >= self.QST:\n"
        "                yield from self.wait(\"q\", self.q_empty[s], i // self.QST - 1)\n", ""),
    "state copy without st_empty": (
        "            if k >= 1:\n"
        "                yield from self.wait(\"st\", self.st_empty, k - 1)\n", ""),
    "last final state without st_empty": (
        "                yield from self.wait(role, self.st_empty, k)\n", "                pass\n"),
    "state step without s_full": (
        "        yield from self.wait(role, self.s_full, gc)\n        assert self.state_chunk == gc",
        "        assert self.state_chunk == gc"),
    "QS without sb_full": (
        "            if x[\"hs\"] == 0:\n"
        "                yield from self.wait(\"mma\", self.sb_full, gc)\n", ""),
    "q_empty released by the MMA alone": (
        "self.q_empty = [mk(f\"q_empty{s}\", 2 if out == \"qslot\" else 1) for s in range(QST)]",
        "self.q_empty = [mk(f\"q_empty{s}\", 1) for s in range(QST)]"),
    "second half of P V before its half of P": (
        "                pf = self.p_full[h] if self.halves == 2 else self.p_full[sc]\n",
        "                pf = self.p_full[0] if self.halves == 2 else self.p_full[sc]\n"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_protocol_mistakes(name):
    import inspect
    import sys
    old, new = MUTANTS[name]
    src = inspect.getsource(sys.modules[__name__])
    src = src[:src.index("\n# Planted mistakes")]
    assert src.count(old) == 1, name
    ns = {"__name__": f"mutant_{abs(hash(name))}"}
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    caught = False
    for config in sorted(ns["CONFIGS"]):
        for shape in ns["SHAPES"]:
            try:
                ns["test_persist_protocol"](config, *shape)
            except AssertionError:
                caught = True
                break
            except pytest.skip.Exception:
                continue
        if caught:
            break
    assert caught, f"planted mistake '{name}' passed the model"
