"""Randomised model of the attention kernel's synchronisation protocol (no GPU).

The attention kernel (csrc/attn_kernel.cuh) is four cooperating roles per CTA:
a TMA producer, an MMA issuer and two softmax warpgroups, linked by mbarriers
(signalled by the TMA unit and by tcgen05.commit) and by named barriers
(thread-to-thread hand-offs).  A wait that never completes is a GPU hang and a
buffer overwritten too early is a silent wrong answer, so the protocol is
modelled here step by step as the kernel performs it and run under many random
interleavings, with the kernel's three configurations (BF16 d=128: K ring 3, V
ring 2, P handed over in two halves, ping-pong turns; BF16 d=64: rings 4/4;
FP8: rings 4/4, whole P, no turns).

Semantics modelled:
* mbarrier: a phase completes after `count` arrivals; a parity wait succeeds
  while the barrier's completed-phase count has the other parity (PTX
  try_wait.parity), so a barrier that runs two phases ahead of its waiter
  blocks it, as on the hardware.
* tcgen05 MMAs from the issuing thread execute in issue order; a commit
  arrives on its mbarrier once every MMA issued before it has completed; an
  issued MMA may read or write its operands at any moment until it completes.
* TMA loads land in any order; each arrives on its stage's mbarrier.
* A named barrier completes when its thread count has arrived; a second
  arrival by the same role within one generation is an error (the hardware
  would merge it into the current generation).

Checks: no deadlock; every role finishes; an MMA reads the K/V tile, the Q tile
(rotated, for BF16) and the half of P it was issued for; no TMA load lands in a
stage an issued MMA still reads; the softmax reads S and writes P only while no
issued MMA touches that half of the buffer; O is rescaled and read only while
no PV into it is outstanding.  Planted protocol mistakes (negative controls)
must each be caught.
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
    def __init__(self, name, count, errors):
        self.name, self.count, self.errors = name, count, errors
        self.arrived, self.gen, self.who = 0, 0, set()

    def arrive(self, who, n):
        if who in self.who:
            self.errors.append(f"{who} arrives twice at {self.name} in generation {self.gen}")
        self.who.add(who)
        self.arrived += n
        if self.arrived > self.count:
            self.errors.append(f"{self.name}: {self.arrived} arrivals for a count of {self.count}")
        if self.arrived >= self.count:
            self.arrived, self.gen, self.who = 0, self.gen + 1, set()


CONFIGS = {
    "bf16_d128": dict(fp8=False, NK=3, NV=2),
    "bf16_d64": dict(fp8=False, NK=4, NV=4),
    "fp8_d128": dict(fp8=True, NK=4, NV=4),
}


def simulate(fp8, NK, NV, nkv, seed, mistake=None):
    """Run one random interleaving; returns (errors, finished)."""
    rng = random.Random(seed)
    split = pingpong = not fp8
    errors = []
    q_full = [MBar(1), MBar(1)]
    q_ready = [MBar(1), MBar(1)]  # 128 arrivals in the kernel: one per softmax thread, modelled as one
    k_full = [MBar(1) for _ in range(NK)]
    k_empty = [MBar(1 if mistake == "k_empty_single_release" else 2) for _ in range(NK)]
    v_full = [MBar(1) for _ in range(NV)]
    v_empty = [MBar(2) for _ in range(NV)]
    s_full = [MBar(1), MBar(1)]
    pv_done = [MBar(1), MBar(1)]
    p_ready = [Named(f"PReady{i}", 160, errors) for i in range(2)]
    p_half = [Named(f"PHalf{i}", 160, errors) for i in range(2)]
    turn = [Named(f"Turn{i}", 256, errors) for i in range(2)]

    qstate = ["none", "none"]
    kstage, vstage = {}, {}
    buf = [[None, None], [None, None]]  # S_i buffer halves: ("S", j) or ("P", j)
    tma = []                            # loads in flight: (kind, slot, tile)
    queue, issued, completed = [], [0], [0]
    commits = []                        # (MMAs that must have completed, barrier)

    def fire_commits():
        while commits and commits[0][0] <= completed[0]:
            commits.pop(0)[1].arrive()

    def commit(bar):
        commits.append((issued[0], bar))
        fire_commits()

    def issue(kind, i, tile, stage, halves):
        queue.append(dict(kind=kind, i=i, tile=tile, stage=stage, halves=halves))
        issued[0] += 1

    def touching(i, half):
        return [m for m in queue if m["i"] == i and (m["kind"] == "S" or half in m["halves"])]

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
            for h in m["halves"]:
                if buf[i][h] != ("P", j):
                    errors.append(f"PV{i}({j}) read half {h} holding {buf[i][h]}")
        completed[0] += 1
        fire_commits()

    def land(load):
        tma.remove(load)
        kind, slot, tile = load
        if kind == "Q":
            qstate[slot] = "loaded"
            q_full[slot].arrive()
            return
        stages, bars = (kstage, k_full) if kind == "K" else (vstage, v_full)
        mk = "S" if kind == "K" else "PV"
        if any(m["kind"] == mk and m["stage"] == slot for m in queue):
            errors.append(f"{kind} tile {tile} lands in stage {slot} while an issued MMA reads it")
        stages[slot] = tile
        bars[slot].arrive()

    # ------------------------------------------------------------------ roles
    def producer():
        for i in range(2):
            tma.append(("Q", i, 0))
        for j in range(nkv):
            sk, sv = j % NK, j % NV
            if j >= NK:
                par = ((j // NK) & 1) if mistake == "producer_parity_without_xor" else ((j // NK) & 1) ^ 1
                yield lambda sk=sk, par=par: k_empty[sk].done(par)
            tma.append(("K", sk, j))
            if j >= NV:
                yield lambda sv=sv, j=j: v_empty[sv].done(((j // NV) & 1) ^ 1)
            tma.append(("V", sv, j))

    def named_sync(bar, who, n):
        g = bar.gen
        bar.arrive(who, n)
        return lambda: bar.gen > g

    def mma():
        q_in = q_full if (fp8 or mistake == "mma_waits_unrotated_q") else q_ready
        halves_all = (0, 1)
        yield lambda: q_in[0].done(0) and k_full[0].done(0)
        issue("S", 0, 0, 0, halves_all)
        commit(s_full[0])
        commit(k_empty[0])
        yield lambda: q_in[1].done(0)
        issue("S", 1, 0, 0, halves_all)
        commit(s_full[1])
        commit(k_empty[0])
        for j in range(1, nkv + 1):
            jj, sv, sk = j - 1, (j - 1) % NV, j % NK
            yield lambda sv=sv, jj=jj: v_full[sv].done((jj // NV) & 1)
            if j < nkv:
                yield lambda sk=sk, j=j: k_full[sk].done((j // NK) & 1)
            for i in range(2):
                early_s = mistake == "s_before_pv" and j < nkv
                if early_s:
                    issue("S", i, j, sk, halves_all)
                if split:
                    yield named_sync(p_half[i], "mma", 32)
                    issue("PV", i, jj, sv, (0,))
                yield named_sync(p_ready[i], "mma", 32)
                issue("PV", i, jj, sv, (1,) if split else halves_all)
                commit(pv_done[i])
                commit(v_empty[sv])
                if j < nkv and not early_s:
                    issue("S", i, j, sk, halves_all)
                if j < nkv:
                    commit(s_full[i])
                    commit(k_empty[sk])

    def softmax(i):
        who = f"softmax{i}"
        if not fp8:
            yield lambda: q_full[i].done(0)
            if touching(i, 0):
                errors.append(f"Q{i} rotated while an MMA reads it")
            qstate[i] = "rotated"
            q_ready[i].arrive()
        for j in range(nkv):
            yield lambda j=j: s_full[i].done(j & 1)
            if any(m["kind"] == "S" and m["i"] == i for m in queue) or buf[i] != [("S", j), ("S", j)]:
                errors.append(f"softmax{i}({j}) reads S holding {buf[i]} with MMAs {len(queue)} in flight")
            grow = j > 0 and rng.random() < 0.5
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
                    if grow and mistake != "rescale_after_release":
                        if any(m["kind"] == "PV" and m["i"] == i for m in queue):
                            errors.append(f"softmax{i}({j}) rescales O while a PV writes it")
                    p_half[i].arrive(who, 128)
                    yield lambda: True  # the MMA warp may run between the halves
            if pingpong:
                if i == 0:
                    turn[1].arrive(who, 128)
                elif j + 1 < nkv and mistake != "softmax0_skips_turn":
                    turn[0].arrive(who, 128)
            if not split and grow and mistake != "rescale_after_release":
                if any(m["kind"] == "PV" and m["i"] == i for m in queue):
                    errors.append(f"softmax{i}({j}) rescales O while a PV writes it")
            p_ready[i].arrive(who, 128)
            if grow and mistake == "rescale_after_release":
                yield lambda: True
                if any(m["kind"] == "PV" and m["i"] == i for m in queue):
                    errors.append(f"softmax{i}({j}) rescales O while a PV writes it")
        yield lambda: pv_done[i].done((nkv - 1) & 1)
        if any(m["kind"] == "PV" and m["i"] == i for m in queue):
            errors.append(f"softmax{i} reads O while a PV writes it")

    roles = {"producer": producer(), "mma": mma(), "softmax0": softmax(0), "softmax1": softmax(1)}
    waiting = {name: (lambda: True) for name in roles}
    finished = set()
    for _ in range(100000):
        if errors:
            break
        options = [("role", n) for n in roles if n not in finished and waiting[n]()]
        options += [("tma", ld) for ld in tma]
        if queue:
            options.append(("mma", None))
        if not options:
            if len(finished) < len(roles):
                errors.append("deadlock: " + ", ".join(sorted(set(roles) - finished)) + " blocked")
            break
        kind, what = rng.choice(options)
        if kind == "tma":
            land(what)
        elif kind == "mma":
            complete_mma()
        else:
            try:
                waiting[what] = next(roles[what])
            except StopIteration:
                finished.add(what)
    return errors, len(finished) == len(roles)


@pytest.mark.parametrize("name", sorted(CONFIGS))
@pytest.mark.parametrize("nkv", [1, 2, 3, 4, 5, 9])
def test_protocol_completes_without_hazards(name, nkv):
    cfg = CONFIGS[name]
    for seed in range(400):
        errors, finished = simulate(nkv=nkv, seed=seed, **cfg)
        assert not errors and finished, (name, nkv, seed, errors[:3])


PLANTED = [
    ("k_empty_single_release", "bf16_d128"),      # K stage freed after S0 alone
    ("producer_parity_without_xor", "fp8_d128"),  # waits for the wrong phase: hangs
    ("s_before_pv", "bf16_d128"),                 # next S overwrites P before PV read it
    ("s_before_pv", "fp8_d128"),
    ("mma_waits_unrotated_q", "bf16_d128"),       # S reads Q before its rotation
    ("rescale_after_release", "fp8_d128"),        # O rescaled after P was handed over
    ("rescale_after_release", "bf16_d64"),
    ("softmax0_skips_turn", "bf16_d128"),         # a second arrival at Turn1 within one generation
]


@pytest.mark.parametrize("mistake,name", PLANTED)
def test_planted_protocol_mistakes_are_caught(mistake, name):
    cfg = CONFIGS[name]
    for seed in range(400):
        errors, finished = simulate(nkv=7, seed=seed, mistake=mistake, **cfg)
        if errors or not finished:
            return
    pytest.fail(f"{mistake} not caught in 400 interleavings")
