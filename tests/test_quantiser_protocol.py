"""Randomised model of the FP8 quantiser's staging protocol (no GPU).

The quantiser (`quantize_qkv` in csrc/fp8_prologue.cu) is one persistent CTA
per SM: a producer warp and 16 converting warps.  Work item n (one 128-token
block of one (b,h)) is three tiles, Q, V and K, each staged by a bulk copy into
a slot of its own (three tile slots), and the item's rotary rows, staged into
table slot n % 2.  The converting warps read a tile after its copy has landed
(a full mbarrier: the producer's arrive.expect_tx, completed by the copy's
bytes), release it with one arrival per warp on the slot's empty mbarrier (K,
the last reader of an item's rows, also releases the table slot), and meet
once per tile on a named barrier that ORs their failure flags.  The producer
stages item n's table once item n - 2 has released it and each tile of item n
once item n - 1 has released that slot.

Semantics modelled: an mbarrier phase completes after `count` arrivals (for a
full barrier: the producer's arrival and its copy's landing); a parity wait
succeeds while the completed-phase count has the other parity; copies land in
any order; the named barrier completes when all 16 warps have arrived.

Failure path (as in the kernel): every mbarrier wait is bounded; a wait that
times out raises the CTA's abort flag, and the waits that watch the flag give
up once it is raised.  A converting warp whose wait failed still releases its
slots and meets the others at the tile's named barrier, where all 16 learn of
the failure and stop; warp 0 raises the abort flag.  The producer, once a wait
leaves, waits (bounded, not watching the flag) for every copy it staged
before the CTA's shared memory is released; on every exit, since the
converting warps' releases on their failure path can let its last stagings
through after they have stopped.  A fault is a copy that
never lands or a release that never comes: each one must end every role, and
every copy still in flight at the end must be the lost one.

Checks: no deadlock; every role finishes; a warp reads a slot only after the
copy of the tile it expects has landed there; no copy is staged into a slot a
warp is still reading; nothing is in flight at the end of a fault-free run.
Planted mistakes (negative controls) must each be caught.
"""
import random

import pytest

WARPS = 16
KINDS = ("Q", "V", "K")


class MBar:
    def __init__(self, count):
        self.count, self.pending, self.completed = count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count

    def done(self, parity):
        return (self.completed & 1) != parity


class Hazard(Exception):
    pass


class Deadlock(Exception):
    pass


class Sim:
    """One CTA.  `fault`: ("copy", k) loses the k-th staged copy; ("late", k)
    delays it past a wait's time limit (it lands only once the abort flag is up,
    so warps waiting for it may decide differently); ("release", k) loses the
    k-th empty arrival.  `mistake`: a planted protocol error."""

    def __init__(self, items, rope, seed, fault=None, mistake=None):
        self.items, self.rope, self.rng = items, rope, random.Random(seed)
        self.fault, self.mistake = fault, mistake
        self.full = {("tile", k): MBar(1) for k in KINDS}
        self.full.update({("tab", s): MBar(1) for s in (0, 1)})
        self.empty = {("tile", k): MBar(WARPS) for k in KINDS}
        self.empty.update({("tab", s): MBar(WARPS) for s in (0, 1)})
        self.content = {}        # slot -> (what, landed)
        self.readers = {slot: set() for slot in self.full}
        self.inflight = []       # [slot, what, lost]
        self.copies = 0
        self.releases = 0
        self.abort = False
        self.named = {"gen": 0, "arrived": 0, "any": False, "result": {}}
        self.finished = set()
        self.read_log = []

    # ---- actions -------------------------------------------------------------
    def stage(self, slot, what):
        if self.readers[slot]:
            raise Hazard(f"copy of {what} staged into {slot} while warps {sorted(self.readers[slot])} read it")
        lost = self.fault == ("copy", self.copies)
        late = self.fault == ("late", self.copies)
        self.copies += 1
        self.content[slot] = (what, False)
        self.inflight.append([slot, what, lost, late])
        # arrive.expect_tx: the phase completes when the bytes land

    def land(self, i):
        slot, what, lost, late = self.inflight.pop(i)
        self.content[slot] = (what, True)
        self.full[slot].arrive()

    def release(self, slot):
        lost = self.fault == ("release", self.releases)
        self.releases += 1
        if not lost:
            self.empty[slot].arrive()

    # ---- roles (generators yielding waits) -----------------------------------
    def producer(self):
        staged = {}  # full barrier -> parity of the last staged phase
        ok = True
        # The kernel stages item n's rows just after item n - 1's K tile, whose wait
        # already implies that item n - 2 released the table slot.  The variant
        # "table_ahead" stages them one item earlier (before item n - 1's tiles),
        # where only the table slot's own release protects them.
        ahead = self.mistake in ("table_ahead", "table_ahead_no_wait", "table_ahead_q")
        for n in range(self.items):
            for m in ((n,) if not ahead else ((0, 1) if n == 0 else (n + 1,))):
                if not self.rope or m >= self.items:
                    continue
                ts = m & 1
                if m >= 2 and self.mistake != "table_ahead_no_wait":
                    ok = yield ("bwait", lambda ts=ts, m=m: self.empty[("tab", ts)].done(((m - 2) >> 1) & 1), True)
                    if not ok:
                        break
                self.stage(("tab", ts), (m, "tab"))
                staged[("tab", ts)] = (m >> 1) & 1
            if not ok:
                break
            for kind in KINDS:
                if n >= 1 and self.mistake != "tile_no_wait":
                    ok = yield ("bwait", lambda kind=kind, n=n: self.empty[("tile", kind)].done((n - 1) & 1), True)
                    if not ok:
                        break
                self.stage(("tile", kind), (n, kind))
                staged[("tile", kind)] = n & 1
            if not ok:
                break
        # the drain, on every exit (the planted mistake: only after a failed wait of its own)
        if not (self.mistake == "drain_on_own_failure_only" and ok):
            for slot, par in staged.items():
                yield ("bwait", lambda slot=slot, par=par: self.full[slot].done(par), False)
        self.finished.add("producer")

    def warp(self, w):
        for n in range(self.items):
            for kind in KINDS:
                tile = ("tile", kind)
                tab = ("tab", n & 1)
                rot = self.rope and kind != "V"
                ok = yield ("bwait", lambda tile=tile, n=n: self.full[tile].done(n & 1), True)
                if rot and ok:
                    ok = yield ("bwait", lambda tab=tab, n=n: self.full[tab].done((n >> 1) & 1), True)
                if ok:
                    for slot, want in ((tile, (n, kind)),) + (((tab, (n, "tab")),) if rot else ()):
                        got = self.content.get(slot)
                        if got != (want, True):
                            raise Hazard(f"warp {w} read {slot} for {want}, found {got}")
                        self.readers[slot].add(w)
                    yield ("step",)  # the reads take time
                    for slot in (tile,) + ((tab,) if rot else ()):
                        self.readers[slot].discard(w)
                    self.read_log.append((w, n, kind))
                elif self.mistake == "early_exit":  # leaves without its releases and the named barrier
                    self.finished.add(f"warp{w}")
                    return
                self.release(tile)
                releases_tab = (kind == "K") if self.mistake != "table_ahead_q" else (kind == "Q")
                if rot and releases_tab:
                    self.release(tab)
                failed = yield ("named", not ok)
                if failed:
                    if w == 0:
                        self.abort = True
                    self.finished.add(f"warp{w}")
                    return
        self.finished.add(f"warp{w}")

    # ---- scheduler -----------------------------------------------------------
    def run(self, max_steps=200000):
        roles = {"producer": self.producer()}
        roles.update({f"warp{w}": self.warp(w) for w in range(WARPS)})
        state = {}  # role -> current request
        for name, g in list(roles.items()):
            try:
                state[name] = next(g)
            except StopIteration:  # nothing to wait for (the producer of a single item)
                del roles[name]
        for _ in range(max_steps):
            if not roles:
                break
            runnable = []
            for name, req in state.items():
                if req[0] == "step":
                    runnable.append(name)
                elif req[0] == "bwait":
                    if req[1]() or (req[2] and self.abort):
                        runnable.append(name)
                elif req[0] == "named":
                    gen = req[2] if len(req) > 2 else None
                    if gen is not None and gen in self.named["result"]:
                        runnable.append(name)
            # named-barrier arrivals are actions too
            arrivals = [n for n, r in state.items() if r[0] == "named" and len(r) == 2]
            landings = [i for i, c in enumerate(self.inflight) if not c[2] and not (c[3] and not self.abort)]
            choices = [("role", n) for n in runnable] + [("arrive", n) for n in arrivals] + \
                      [("land", i) for i in landings]
            if not choices:
                # every role is blocked: a bounded wait times out (raising the abort flag)
                bounded = [n for n, r in state.items() if r[0] == "bwait"]
                if not bounded:
                    raise Deadlock(f"blocked on named barriers only: {sorted(state)}")
                name = self.rng.choice(bounded)
                if state[name][2]:
                    self.abort = True
                self._resume(roles, state, name, False)
                continue
            kind, x = self.rng.choice(choices)
            if kind == "land":
                self.land(x)
            elif kind == "arrive":
                req = state[x]
                nb = self.named
                nb["arrived"] += 1
                nb["any"] = nb["any"] or req[1]
                gen = nb["gen"]
                state[x] = ("named", req[1], gen)
                if nb["arrived"] == WARPS:
                    nb["result"][gen] = nb["any"]
                    nb["gen"] += 1
                    nb["arrived"], nb["any"] = 0, False
            else:
                req = state[x]
                if req[0] == "step":
                    val = None
                elif req[0] == "bwait":
                    val = bool(req[1]())
                else:
                    val = self.named["result"][req[2]]
                self._resume(roles, state, x, val)
        else:
            raise Deadlock("step limit")
        return self

    def _resume(self, roles, state, name, val):
        try:
            state[name] = roles[name].send(val)
        except StopIteration:
            del roles[name]
            del state[name]


def run(items, rope, seed, **kw):
    return Sim(items, rope, seed, **kw).run()


@pytest.mark.parametrize("rope", [True, False])
@pytest.mark.parametrize("items", [1, 2, 3, 5])
def test_fault_free_interleavings(items, rope):
    for seed in range(60):
        s = run(items, rope, seed)
        assert s.finished == {"producer"} | {f"warp{w}" for w in range(WARPS)}
        assert not s.inflight
        assert not s.abort
        assert len(s.read_log) == WARPS * 3 * items


@pytest.mark.parametrize("rope", [True, False])
def test_every_lost_copy_or_release_ends_every_role(rope):
    items = 3
    n_copies = items * (3 + (1 if rope else 0))
    n_releases = items * 3 * WARPS + (items * WARPS if rope else 0)
    faults = [("copy", k) for k in range(n_copies)] + [("late", k) for k in range(n_copies)] + \
             [("release", k) for k in range(0, n_releases, 7)]
    for fault in faults:
        for seed in range(6):
            s = run(items, rope, seed, fault=fault)
            assert s.finished == {"producer"} | {f"warp{w}" for w in range(WARPS)}, (fault, seed)
            # whatever is still in flight is the copy that was lost
            assert all(c[2] for c in s.inflight), (fault, seed, s.inflight)


def _caught(mistake, fault=None, items=3, rope=True, seeds=60):
    """A hazard, a deadlock, or (with no fault injected) a wait that had to time out."""
    for seed in range(seeds):
        try:
            s = Sim(items, rope, seed, mistake=mistake, fault=fault).run()
        except (Hazard, Deadlock):
            return True
        if fault is None and s.abort:
            return True
    return False


def test_tables_staged_an_item_earlier_are_safe_with_their_own_release():
    for seed in range(60):
        s = Sim(4, True, seed, mistake="table_ahead").run()
        assert not s.inflight and not s.abort and len(s.read_log) == WARPS * 3 * 4


@pytest.mark.parametrize("mistake", ["tile_no_wait", "table_ahead_no_wait", "table_released_by_q"])
def test_planted_protocol_mistakes_are_caught(mistake):
    # the table mistakes matter once the rows are staged an item earlier
    assert _caught(mistake, items=4) if mistake == "tile_no_wait" else _caught_ahead(mistake)


def _caught_ahead(mistake):
    return _caught(mistake if mistake != "table_released_by_q" else "table_ahead_q", items=4)


def test_planted_early_exit_is_caught():
    # a warp that leaves on a failed wait strands the others on the named barrier
    # (a late copy: some warps give up on it, others see it land)
    assert any(_caught("early_exit", fault=("late", k)) for k in range(4))


def test_planted_drain_only_after_own_failure_is_caught():
    # the converting warps stop on a lost release; their releases on the failure path
    # complete the phase the producer waits for, it stages the last item and leaves
    # normally: without a drain on that exit its copies are still in flight
    caught = False
    for fault in [("release", k) for k in range(40, 60)]:
        for seed in range(10):
            s = Sim(3, False, seed, mistake="drain_on_own_failure_only", fault=fault).run()
            if any(not c[2] for c in s.inflight):
                caught = True
    assert caught


def test_model_matches_the_kernel_source():
    """The model's shape is the kernel's: 16 converting warps (512 threads), three
    tile slots and two table slots, full barriers with one arrival and empty
    barriers with one arrival per converting warp, tiles in the order Q, V, K."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "diffusion_transformer_denoising_dit_b200", "csrc", "fp8_prologue.cu")).read()
    assert int(re.search(r"constexpr int kQzThreads = (\d+);", src).group(1)) == 32 * WARPS
    assert "constexpr int kQzBarOff = 3 * kTileBytes + 2 * kTabBytes;" in src
    kern = src[src.index("quantize_qkv(Fp8Prep p)"):]
    assert "for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);" in kern            # tile_full[3], tab_full[2]
    assert "for (int i = 5; i < 10; ++i) mbar_init(&bars[i], kQzThreads / 32);" in kern  # the empties
    order = [kern.index(f"qz_tile<kQz{k}, INT8>") for k in KINDS]
    assert order == sorted(order)
    # the producer stages the table of item n after item n - 2 released it, and
    # each tile of item n after item n - 1 released that slot; it drains on every exit
    assert "static_cast<uint32_t>((n - 2) >> 1) & 1u" in kern
    assert "static_cast<uint32_t>(n - 1) & 1u" in kern
    producer = kern[kern.index("if (threadIdx.x >= kQzThreads) {"):kern.index("    return;\n  }")]
    guard = producer[:producer.index("mbar_wait_until")].rsplit("\n    if (", 1)[1].split("\n", 1)[0]
    assert guard == "(threadIdx.x & 31) == 0) {", guard  # no "!ok": the drain runs whichever way the loop ended
