"""Randomised model of the attention kernel's synchronisation protocol (no GPU).

The attention kernel (csrc/attn_kernel.cuh) is four cooperating roles per CTA:
a TMA producer, an MMA issuer and two softmax warpgroups, linked by mbarriers
(signalled by the TMA unit and by tcgen05.commit) and by named barriers
(thread-to-thread hand-offs).  A wait that never completes is a GPU hang and a
buffer overwritten too early is a silent wrong answer, so the protocol is
modelled here step by step as the kernel performs it and run under many random
interleavings, with the kernel's three configurations (BF16 d=128: K ring 3, V
ring 2, P handed over in two halves in TMEM, ping-pong turns; BF16 d=64: rings
4/4; FP8: rings 4/4, no turns and no named barriers: P in a shared-memory tile
of its own, handed over through a p_ready mbarrier; the MMA thread polls four
event streams and issues S_i(j) once softmax i has read S_i(j-1) and PV_i(j)
once P_i(j) is stored, whichever is ready first; every PV is committed to
pv_done, which softmax i waits for before it overwrites P_i or rescales O_i).

Semantics modelled:
* mbarrier: a phase completes after `count` arrivals; a parity wait succeeds
  while the barrier's completed-phase count has the other parity (PTX
  try_wait.parity), so a barrier that runs two phases ahead of its waiter
  blocks it, as on the hardware.
* tcgen05 MMAs from the issuing thread execute in issue order; a commit
  arrives on its mbarrier once every MMA issued before it has completed; an
  issued MMA may read or write its operands at any moment until it completes.
* TMA loads land in any order; each arrives on its stage's mbarrier.
* A named barrier counts arrivals warp by warp (32 threads each); a generation
  completes the moment its count is reached and the count starts again from
  zero, so arrivals made ahead of a syncing partner are carried into the next
  generation as on the hardware.  A second arrival by the same role within one
  generation is an error on the fault-free path.

Checks: no deadlock; every role finishes; an MMA reads the K/V tile, the Q tile
(rotated, for BF16) and the half of P it was issued for; no TMA load lands in a
stage an issued MMA still reads; the softmax reads S and writes P only while no
issued MMA touches that half of the buffer (FP8: reads S while no S MMA of its
tile is outstanding, writes its P tile while no PV reads it); O is rescaled and
read only while no PV into it is outstanding; nothing is in flight when the
CTA ends.  Planted
protocol mistakes (negative controls) must each be caught.

Failure path (as in the kernel): every mbarrier wait is bounded; the first one
that gives up raises the CTA's abort flag, after which every other bounded wait
gives up as well.  A role that gives up performs the rest of its named-barrier
schedule without the work between (the MMA warp its syncs, a softmax
warpgroup its arrivals and ping-pong turns), so no partner is left on a named
barrier, which cannot time out.  The BF16 softmax hands its Q tile on only when
the tile came; the producer waits, bounded, for the last load it issued into
every stage before it leaves; after a failure the MMA thread waits, bounded,
for its own MMAs before TMEM is released.  A fault is a load or an arrival that
never comes: each one, in every configuration, must end every role.  A softmax
warpgroup is modelled as one role: its four warps each take the same decision
at every bounded wait or, where they differ, each completes the same schedule
of named-barrier operations, which is what the dry schedule guarantees.
"""
import random

import pytest


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


class Named:
    """A named barrier of `count` threads: arrivals are counted warp by warp and a
    generation completes the moment the count is reached."""

    def __init__(self, name, count, errors):
        self.name, self.count, self.errors = name, count, errors
        self.arrived, self.gen, self.who = 0, 0, set()
        self.strict = True  # fault-free runs: no role arrives twice in one generation

    def arrive(self, who, n):
        """Arrive with n threads (n/32 warps); returns the generation of the last warp."""
        if who in self.who and self.strict:
            self.errors.append(f"{who} arrives twice at {self.name} in generation {self.gen}")
        self.who.add(who)
        g = self.gen
        for _ in range(n // 32):
            g = self.gen
            self.arrived += 32
            if self.arrived == self.count:
                self.arrived, self.gen, self.who = 0, self.gen + 1, set()
        return g


CONFIGS = {
    "bf16_d128": dict(fp8=False, NK=3, NV=2),
    "bf16_d64": dict(fp8=False, NK=4, NV=4),
    "fp8_d128": dict(fp8=True, NK=4, NV=4),
}


def simulate(fp8, NK, NV, nkv, seed, mistake=None, lost=None, report=None):
    """Run one random interleaving; returns (errors, finished, timeouts).  With a
    fault injected the result is already invalid once a wait has given up, so
    data hazards no longer stop the run and `errors` holds only a hang.

    lost: a fault to inject -- ("load", kind, tile) for a TMA load that never
    lands (issued and in flight), or ("commit", barrier name, index, nth) for a
    commit arrival that never comes.  Without a fault no wait may give up.
    report: a dict that receives the loads still in flight when every role has
    ended, the stages whose drain wait gave up, and whether the abort flag rose.
    """
    rng = random.Random(seed)
    split = pingpong = not fp8
    psmem = fp8  # P in shared memory, S freed once read
    errors = []
    q_full = [MBar(1), MBar(1)]
    q_ready = [MBar(1), MBar(1)]  # 128 arrivals in the kernel: one per softmax thread, modelled as one
    k_full = [MBar(1) for _ in range(NK)]
    k_empty = [MBar(1 if mistake == "k_empty_single_release" else 2) for _ in range(NK)]
    v_full = [MBar(1) for _ in range(NV)]
    v_empty = [MBar(2) for _ in range(NV)]
    s_full = [MBar(1), MBar(1)]
    pv_done = [MBar(1), MBar(1)]
    s_free = [MBar(1), MBar(1)]  # FP8: one arrival per softmax warp in the kernel, modelled as one
    p_ready_m = [MBar(1), MBar(1)]  # FP8: likewise
    bars = {"s_full": s_full, "pv_done": pv_done, "k_empty": k_empty, "v_empty": v_empty}
    p_ready = [Named(f"PReady{i}", 160, errors) for i in range(2)]
    p_half = [Named(f"PHalf{i}", 160, errors) for i in range(2)]
    turn = [Named(f"Turn{i}", 256, errors) for i in range(2)]
    if lost is not None:
        for b in p_ready + p_half + turn:
            b.strict = False
    abort = [False]
    mma_done = [0, 0]     # PReady_i generations the MMA warp has passed (published after each)

    qstate = ["none", "none"]
    kstage, vstage = {}, {}
    buf = [[None, None], [None, None]]  # S_i buffer halves: ("S", j) or ("P", j)
    psm = [None, None]                  # FP8: P_i shared-memory tile, ("P", j)
    tma = []                            # loads in flight: (kind, slot, tile)
    queue, issued, completed = [], [0], [0]
    commits = []                        # (MMAs that must have completed, barrier)
    commit_count = {}

    def fire_commits():
        while commits and commits[0][0] <= completed[0]:
            commits.pop(0)[1].arrive()

    def commit(name, idx):
        n = commit_count.get((name, idx), 0)
        commit_count[(name, idx)] = n + 1
        if lost == ("commit", name, idx, n):
            return  # this arrival never comes
        commits.append((issued[0], bars[name][idx]))
        fire_commits()

    stalled = set()
    drain_gave_up = set()

    def load(kind, slot, tile):
        tma.append((kind, slot, tile))
        if lost == ("load", kind, tile):
            stalled.add((kind, slot, tile))  # issued, never lands

    def issue(kind, i, tile, stage, halves):
        queue.append(dict(kind=kind, i=i, tile=tile, stage=stage, halves=halves))
        issued[0] += 1

    def touching(i, half):
        return [m for m in queue if m["i"] == i and (m["kind"] == "S" or half in m["halves"])]

    def s_pending(i):
        return any(m["kind"] == "S" and m["i"] == i for m in queue)

    def pv_pending(i):
        return any(m["kind"] == "PV" and m["i"] == i for m in queue)

    def complete_mma():
        m = queue.pop(0)
        i, j = m["i"], m["tile"]
        if m["kind"] == "S":
            if kstage.get(m["stage"]) != j:
                errors.append(f"S{i}({j}) read K stage {m['stage']} holding {kstage.get(m['stage'])}")
            want = "loaded" if fp8 else "rotated"
            if qstate[i] != want:
                errors.append(f"S{i}({j}) read Q{i} {qstate[i]}")
            buf[i] = [("S", j), ("S", j)]
        else:
            if vstage.get(m["stage"]) != j:
                errors.append(f"PV{i}({j}) read V stage {m['stage']} holding {vstage.get(m['stage'])}")
            if psmem:
                if psm[i] != ("P", j):
                    errors.append(f"PV{i}({j}) read the P tile holding {psm[i]}")
            else:
                for h in m["halves"]:
                    if buf[i][h] != ("P", j):
                        errors.append(f"PV{i}({j}) read half {h} holding {buf[i][h]}")
        completed[0] += 1
        fire_commits()

    def land(ld):
        tma.remove(ld)
        kind, slot, tile = ld
        if kind == "Q":
            qstate[slot] = "loaded"
            q_full[slot].arrive()
            return
        stages, full = (kstage, k_full) if kind == "K" else (vstage, v_full)
        mk = "S" if kind == "K" else "PV"
        if any(m["kind"] == mk and m["stage"] == slot for m in queue):
            errors.append(f"{kind} tile {tile} lands in stage {slot} while an issued MMA reads it")
        stages[slot] = tile
        full[slot].arrive()

    # ------------------------------------------------------------------ roles
    # A role yields ("mbar", pred) for a bounded, abort-aware mbarrier wait (sent
    # back True when it completes, False when it gives up: on its own limit, which
    # raises the abort flag, or once the flag is up), ("deadline", pred) for a
    # bounded wait that ignores the flag (the drains), or a bare predicate for a
    # wait that cannot time out (named barriers) or a plain scheduling point.
    def named_sync(bar, who, n):
        g = bar.arrive(who, n)
        return lambda: bar.gen > g

    def producer():
        for i in range(2):
            load("Q", i, i)  # Q tile i (the tile index names which Q load a fault drops)
        nk_issued = nv_issued = 0
        for j in range(nkv):
            sk, sv = j % NK, j % NV
            if j >= NK:
                par = ((j // NK) & 1) if mistake == "producer_parity_without_xor" else ((j // NK) & 1) ^ 1
                if not (yield ("mbar", lambda sk=sk, par=par: k_empty[sk].done(par))):
                    break
            load("K", sk, j)
            nk_issued += 1
            if j >= NV:
                if not (yield ("mbar", lambda sv=sv, j=j: v_empty[sv].done(((j // NV) & 1) ^ 1))):
                    break
            load("V", sv, j)
            nv_issued += 1
        if mistake == "no_drain":
            return
        # drain: the last load issued into each stage has landed (phase index = tile // ring)
        for i in range(2):
            if not (yield ("deadline", lambda i=i: q_full[i].done(0))):
                drain_gave_up.add(("Q", i))
        for kind, ring, issued_n, full in (("K", NK, nk_issued, k_full), ("V", NV, nv_issued, v_full)):
            for st in range(min(ring, issued_n)):
                last = st + ((issued_n - 1 - st) // ring) * ring
                if not (yield ("deadline", lambda full=full, st=st, last=last, ring=ring:
                               full[st].done((last // ring) & 1))):
                    drain_gave_up.add((kind, st))

    def mma():
        q_in = q_full if (fp8 or mistake == "mma_waits_unrotated_q") else q_ready
        halves_all = (0, 1)
        ok = (yield ("mbar", lambda: q_in[0].done(0))) and (yield ("mbar", lambda: k_full[0].done(0)))
        if ok:
            issue("S", 0, 0, 0, halves_all)
            commit("s_full", 0)
            commit("k_empty", 0)
            ok = yield ("mbar", lambda: q_in[1].done(0))
        if ok:
            issue("S", 1, 0, 0, halves_all)
            commit("s_full", 1)
            commit("k_empty", 0)
        if psmem:
            # event-driven: each pass issues every S and PV whose inputs are ready
            ns, npv = [1, 1], [0, 0]

            def s_ready(i):
                t = ns[i]
                return (t < nkv and (mistake == "s_before_read" or s_free[i].done((t - 1) & 1))
                        and k_full[t % NK].done((t // NK) & 1))

            def pv_ready(i):
                t = npv[i]
                return t < nkv and p_ready_m[i].done(t & 1) and v_full[t % NV].done((t // NV) & 1)

            while ok and (npv[0] < nkv or npv[1] < nkv):
                cond = lambda: any(s_ready(i) or pv_ready(i) for i in range(2))
                if mistake == "mma_poll_unbounded":
                    yield cond
                else:
                    ok = yield ("mbar", cond)
                if not ok:
                    break
                for i in range(2):
                    if s_ready(i):
                        t = ns[i]
                        issue("S", i, t, t % NK, halves_all)
                        commit("s_full", i)
                        commit("k_empty", t % NK)
                        ns[i] += 1
                    if pv_ready(i):
                        t = npv[i]
                        issue("PV", i, t, t % NV, halves_all)
                        commit("pv_done", i)
                        commit("v_empty", t % NV)
                        npv[i] += 1
                    yield lambda: True  # other roles run between the checks
            return
        j = 1
        while ok and j <= nkv:
            jj, sv, sk = j - 1, (j - 1) % NV, j % NK
            ok = not abort[0]
            if ok:
                ok = yield ("mbar", lambda sv=sv, jj=jj: v_full[sv].done((jj // NV) & 1))
            if ok and j < nkv:
                ok = yield ("mbar", lambda sk=sk, j=j: k_full[sk].done((j // NK) & 1))
            if not ok:
                break
            for i in range(2):
                early_s = mistake == "s_before_pv" and j < nkv
                if early_s:
                    issue("S", i, j, sk, halves_all)
                if split:
                    yield named_sync(p_half[i], "mma", 32)
                    issue("PV", i, jj, sv, (0,))
                yield named_sync(p_ready[i], "mma", 32)
                issue("PV", i, jj, sv, (1,) if split else halves_all)
                if j == nkv:  # the epilogue waits for the last PV only
                    commit("pv_done", i)
                commit("v_empty", sv)
                if j < nkv and not early_s:
                    issue("S", i, j, sk, halves_all)
                if j < nkv:
                    commit("s_full", i)
                    commit("k_empty", sk)
                mma_done[i] = j
            j += 1
        if not ok and mistake != "mma_leaves_without_schedule":
            # the rest of the named-barrier schedule, no MMAs, from the iteration after
            # the last one whose progress was published for warpgroup 1
            assert mma_done[1] + 1 == j
            for jd in range(mma_done[1] + 1, nkv + 1):
                for i in range(2):
                    if split:
                        yield named_sync(p_half[i], "mma", 32)
                    yield named_sync(p_ready[i], "mma", 32)
                    mma_done[i] = jd

    def softmax(i):
        who = f"softmax{i}"
        ok = True
        if not fp8:
            ok = yield ("mbar", lambda: q_full[i].done(0))
            if ok:
                if touching(i, 0):
                    errors.append(f"Q{i} rotated while an MMA reads it")
                qstate[i] = "rotated"
                q_ready[i].arrive()  # only a tile that came is handed on
        j = 0
        while ok and j < nkv:
            ok = yield ("mbar", lambda j=j: s_full[i].done(j & 1))
            if not ok:
                break
            if s_pending(i) or buf[i] != [("S", j), ("S", j)]:
                errors.append(f"softmax{i}({j}) reads S holding {buf[i]} with MMAs {len(queue)} in flight")
            grow = j > 0 and rng.random() < 0.5
            if psmem:
                s_free[i].arrive()  # S_i is in registers
                yield lambda: True  # the exponentials: anything may run meanwhile
                if j > 0 and mistake != "p_store_without_pv_wait":
                    ok = yield ("mbar", lambda j=j: pv_done[i].done((j - 1) & 1))
                    if not ok:
                        break
                if pv_pending(i):
                    errors.append(f"softmax{i}({j}) writes its P tile while a PV reads it")
                psm[i] = ("P", j)
                if grow and mistake != "rescale_after_release" and pv_pending(i):
                    errors.append(f"softmax{i}({j}) rescales O while a PV writes it")
                p_ready_m[i].arrive()
                if grow and mistake == "rescale_after_release":
                    yield lambda: True
                    if pv_pending(i):
                        errors.append(f"softmax{i}({j}) rescales O while a PV writes it")
                j += 1
                continue
            if pingpong:
                if i == 1:
                    yield named_sync(turn[1], who, 128)
                elif j > 0 and mistake != "softmax0_skips_turn":
                    yield named_sync(turn[0], who, 128)
            for h in (0, 1):
                if touching(i, h):
                    errors.append(f"softmax{i}({j}) writes P half {h} while an MMA touches it")
                buf[i][h] = ("P", j)
                if split and h == 0:
                    if grow and mistake != "rescale_after_release" and pv_pending(i):
                        errors.append(f"softmax{i}({j}) rescales O while a PV writes it")
                    p_half[i].arrive(who, 128)
                    yield lambda: True  # the MMA warp may run between the halves
            if pingpong:
                if i == 0:
                    turn[1].arrive(who, 128)
                elif j + 1 < nkv and mistake != "softmax0_skips_turn":
                    turn[0].arrive(who, 128)
            if not split and grow and mistake != "rescale_after_release" and pv_pending(i):
                errors.append(f"softmax{i}({j}) rescales O while a PV writes it")
            p_ready[i].arrive(who, 128)
            if grow and mistake == "rescale_after_release":
                yield lambda: True
                if pv_pending(i):
                    errors.append(f"softmax{i}({j}) rescales O while a PV writes it")
            j += 1
        if not ok and not psmem and mistake != "softmax_leaves_without_schedule":
            # the rest of the named-barrier schedule, no work; each arrival waits until its
            # partner has passed the previous generation (the pacing the data
            # dependencies give on the normal path), so arrivals never run a generation
            # ahead.  Only the MMA warp's progress is published: it passing PReady_1(t-1)
            # means warpgroup 1 passed Turn_1(t-1) before arriving there, and it passing
            # PReady_0(t) means warpgroup 0 passed Turn_0(t-1).
            paced = mistake != "dry_without_pacing"
            for t in range(j, nkv):
                turns = pingpong and mistake != "dry_schedule_without_turns"
                if turns:
                    if i == 1:
                        yield named_sync(turn[1], who, 128)
                    elif t > 0:
                        yield named_sync(turn[0], who, 128)
                if paced:
                    yield lambda t=t: mma_done[i] >= t
                if split:
                    p_half[i].arrive(who, 128)
                if turns:
                    if i == 0:
                        if paced:
                            yield lambda t=t: mma_done[1] >= t
                        turn[1].arrive(who, 128)
                    elif t + 1 < nkv:
                        if paced:
                            yield lambda t=t: mma_done[0] >= t + 1
                        turn[0].arrive(who, 128)
                p_ready[i].arrive(who, 128)
                yield lambda: True
        if ok:  # BF16 commits pv_done after the last PV only, FP8 after every PV
            last = (nkv - 1) & 1 if psmem else 0
            ok = yield ("mbar", lambda: pv_done[i].done(last))
        if ok and pv_pending(i):
            errors.append(f"softmax{i} reads O while a PV writes it")

    roles = {"producer": producer(), "mma": mma(), "softmax0": softmax(0), "softmax1": softmax(1)}
    waiting = {name: None for name in roles}   # None: about to start
    finished = set()
    timeouts = []

    def ready(name):
        w = waiting[name]
        if w is None:
            return True
        return (w[1] if isinstance(w, tuple) else w)()

    def step(name, value):
        try:
            waiting[name] = roles[name].send(value)
        except StopIteration:
            finished.add(name)

    hang = []
    for _ in range(200000):
        if errors and lost is None:
            break
        if len(finished) == len(roles):
            break  # every role has ended: the CTA reaches its last barrier
        options = [("role", n) for n in roles if n not in finished and ready(n)]
        options += [("tma", ld) for ld in tma if ld not in stalled]
        if queue:
            options.append(("mma", None))
        if abort[0]:  # a waiting role sees the flag and gives up
            options += [("abort", n) for n in roles if n not in finished and not ready(n)
                        and isinstance(waiting[n], tuple) and waiting[n][0] == "mbar"]
        if not options:
            blocked = sorted(set(roles) - finished)
            bounded = [n for n in blocked if isinstance(waiting[n], tuple)]
            if lost is None or not bounded:
                hang.append(", ".join(blocked) + " blocked" + ("" if bounded else " on named barriers"))
                errors.append(("deadlock: " if lost is None else "hang: ") + hang[-1])
                break
            name = rng.choice(bounded)
            timeouts.append(name)
            if waiting[name][0] == "mbar":
                abort[0] = True
            step(name, False)
            continue
        kind, what = rng.choice(options)
        if kind == "tma":
            land(what)
        elif kind == "mma":
            complete_mma()
        elif kind == "abort":
            step(what, False)
        else:
            step(what, None if waiting[what] is None else True)
    else:
        errors.append("no progress bound reached")
    # CTA exit: after a failure the MMA thread waits for its own MMAs (they always
    # complete); on the fault-free path nothing may still be running
    if abort[0]:
        while queue:
            complete_mma()
    elif lost is None and len(finished) == len(roles) and queue:
        errors.append(f"{len(queue)} MMAs still running when TMEM is released")
    if report is not None:
        report["in_flight_at_exit"] = list(tma)
        report["drain_gave_up"] = set(drain_gave_up)
        report["abort"] = abort[0]
    if lost is not None:
        return hang, len(finished) == len(roles), timeouts
    return errors, len(finished) == len(roles), timeouts


@pytest.mark.parametrize("name", sorted(CONFIGS))
@pytest.mark.parametrize("nkv", [1, 2, 3, 4, 5, 9])
def test_protocol_completes_without_hazards(name, nkv):
    cfg = CONFIGS[name]
    for seed in range(400):
        errors, finished, timeouts = simulate(nkv=nkv, seed=seed, **cfg)
        assert not errors and finished and not timeouts, (name, nkv, seed, errors[:3])


PLANTED = [
    ("k_empty_single_release", "bf16_d128"),      # K stage freed after S0 alone
    ("producer_parity_without_xor", "fp8_d128"),  # waits for the wrong phase: hangs
    ("s_before_pv", "bf16_d128"),                 # next S overwrites P before PV read it
    ("s_before_read", "fp8_d128"),                # next S issued before the softmax read S
    ("p_store_without_pv_wait", "fp8_d128"),      # P tile overwritten while the last PV reads it
    ("mma_waits_unrotated_q", "bf16_d128"),       # S reads Q before its rotation
    ("rescale_after_release", "fp8_d128"),        # O rescaled after P was handed over
    ("rescale_after_release", "bf16_d64"),
    ("softmax0_skips_turn", "bf16_d128"),         # a second arrival at Turn1 within one generation
]


@pytest.mark.parametrize("mistake,name", PLANTED)
def test_planted_protocol_mistakes_are_caught(mistake, name):
    cfg = CONFIGS[name]
    for seed in range(400):
        errors, finished, _ = simulate(nkv=7, seed=seed, mistake=mistake, **cfg)
        if errors or not finished:
            return
    pytest.fail(f"{mistake} not caught in 400 interleavings")


def _faults(cfg):
    """Every single loss the model can inject for a 7-tile run: each TMA load (Q, K,
    V), each stage release and each S / PV completion signal."""
    out = [("load", "Q", 0), ("load", "Q", 1)]
    out += [("load", kind, t) for kind in ("K", "V") for t in range(7)]
    if cfg["fp8"]:  # one pv_done commit per tile
        out += [("commit", "pv_done", i, n) for i in range(2) for n in (0, 3, 6)]
    else:
        out += [("commit", "pv_done", 0, 0), ("commit", "pv_done", 1, 0)]
    for name, n, per in (("k_empty", cfg["NK"], 2), ("v_empty", cfg["NV"], 2), ("s_full", 2, 1)):
        for idx in range(n):
            uses = 7 if name == "s_full" else -(-7 // n) * per
            out += [("commit", name, idx, k) for k in sorted({0, uses // 2, uses - 2, uses - 1})]
    return out


def _waited_on(fault, cfg, nkv):
    """Whether some wait depends on the lost arrival: every load, S completion and
    the (single) completion of the last PV; the stage release of tile t only if
    tile t + ring is loaded into that stage."""
    if fault[0] == "load" or fault[1] in ("s_full", "pv_done"):
        return True
    _, name, idx, n = fault
    ring = cfg["NK"] if name == "k_empty" else cfg["NV"]
    return idx + (n // 2) * ring + ring < nkv


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_every_single_loss_ends_every_role(name):
    """Whatever arrival is lost, every role ends (the loss is reported through a
    bounded wait that gives up, never absorbed silently into a hang), and a load
    still in flight when the CTA ends is one the producer's drain waited for."""
    cfg = CONFIGS[name]
    faults = _faults(cfg)
    assert len(faults) > 30
    for fault in faults:
        for seed in range(40):
            rep = {}
            hang, finished, timeouts = simulate(nkv=7, seed=seed, lost=fault, report=rep, **cfg)
            assert finished and not hang, (name, fault, seed, hang)
            for kind, slot, _ in rep["in_flight_at_exit"]:
                assert (kind, slot) in rep["drain_gave_up"], (fault, seed, rep)
            if _waited_on(fault, cfg, 7):
                assert timeouts and rep["abort"], (name, fault, seed)
            else:  # nothing waits for it: the loss changes nothing
                assert not timeouts and not rep["abort"], (name, fault, seed)


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_fault_free_runs_raise_no_abort_and_leave_nothing_in_flight(name):
    cfg = CONFIGS[name]
    for nkv in (1, 2, 3, 5, 9):
        for seed in range(150):
            rep = {}
            errors, finished, timeouts = simulate(nkv=nkv, seed=seed, report=rep, **cfg)
            assert not errors and finished and not timeouts, (nkv, seed, errors)
            assert not rep["in_flight_at_exit"] and not rep["abort"], (nkv, seed, rep)


# Planted mistakes in the failure path: each leaves some role on a named barrier
# (or exits with a load in flight) under some single loss.
FAILURE_PATH_MISTAKES = [
    ("dry_without_pacing", "bf16_d128", ("load", "Q", 0)),
    ("dry_without_pacing", "bf16_d64", ("load", "V", 2)),
    ("softmax_leaves_on_timeout", "bf16_d64", ("commit", "s_full", 0, 2)),
    ("mma_poll_unbounded", "fp8_d128", ("load", "K", 3)),      # FP8's issuer without its time limit
    ("softmax_leaves_on_timeout", "bf16_d128", ("commit", "s_full", 1, 2)),
    ("dry_schedule_without_turns", "bf16_d128", ("commit", "s_full", 0, 2)),
    ("mma_leaves_without_schedule", "bf16_d64", ("load", "V", 3)),
]


@pytest.mark.parametrize("mistake,name,fault", FAILURE_PATH_MISTAKES)
def test_planted_failure_path_mistakes_hang(mistake, name, fault):
    m = {"softmax_leaves_on_timeout": "softmax_leaves_without_schedule"}.get(mistake, mistake)
    for seed in range(200):
        hang, finished, _ = simulate(nkv=7, seed=seed, lost=fault, mistake=m, **CONFIGS[name])
        if hang or not finished:
            return
    pytest.fail(f"{mistake} under {fault} never hung in 200 interleavings")


def test_without_the_drain_a_stalled_load_is_left_behind():
    rep = {}
    for seed in range(50):
        hang, finished, _ = simulate(nkv=7, seed=seed, lost=("load", "K", 2), mistake="no_drain", report=rep,
                                     **CONFIGS["bf16_d128"])
        assert finished and not hang
        if ("K", 2 % 3, 2) in rep["in_flight_at_exit"] and not rep["drain_gave_up"]:
            return
    pytest.fail("a stalled load was never left in flight without the drain")
