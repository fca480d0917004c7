"""Host model of the decode kernel's barrier protocol (csrc/decode_sm100.cu).

Every warp role of the two CTAs of an engine is a generator that waits on
mbarrier phases (parity waits, as the kernel's) and arrives on barriers with
the kernel's counts; a scheduler runs the roles in random interleavings over
many segment patterns and random rescale flags.  The test fails on a
deadlock (no role can move and some have not finished), on a barrier
receiving more arrivals than its count, and on a waiter that falls two or
more phases behind a barrier (where a parity wait can no longer tell the
phases apart).  Tensor-core commits and TMA loads complete at once in the
model; completing later cannot create a cycle that the model misses, since
no role waits on anything but barrier phases.

The model is a transcription: a change to the kernel's waits, arrivals,
ring sizes or barrier counts must be made here too.
"""
import random

import pytest

K_SLOTS, N_S, N_REC, V_SLOTS, PASS = 3, 2, 3, 5, 3


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.done = name, count, count, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, f"{self.name}: more arrivals than its count"
        if self.pending == 0:
            self.done += 1
            self.pending = self.count

    def passes(self, parity, phase):
        ok = (self.done & 1) != parity
        if ok and phase is not None:
            assert self.done <= phase + 2, f"{self.name}: waiter for phase {phase} lapped ({self.done} done)"
        return ok


def roles(segs, rescale, k_slots, n_rec):
    B = {}

    def bar(name, count):
        B[name] = Bar(name, count)

    for i in range(k_slots):
        bar(f"k_full{i}", 1); bar(f"k_empty{i}", 1)
    for i in range(N_S):
        bar(f"s_full{i}", 1); bar(f"s_empty{i}", 128)
    bar("q_ready", 128); bar("q_free", 1)
    for i in range(n_rec):
        bar(f"stage_full{i}", 128); bar(f"stage_empty{i}", 64)   # score CTA staging
        bar(f"p_full{i}", 64); bar(f"p_empty{i}", 5)             # value CTA record / its release
    for i in range(V_SLOTS):
        bar(f"v_full{i}", 1); bar(f"v_empty{i}", 1); bar(f"v_fixed{i}", 1)
    bar("pv_prev", 1); bar("corr_done", 128); bar("o_ready", 1); bar("o_free", 128)

    def wait(name, parity, phase=None):
        return ("wait", name, parity, phase)

    def score_tma():
        cit = 0
        for lo, hi in segs:
            for _ in range(lo, hi, PASS):
                for _ch in range(9):
                    s = cit % k_slots
                    yield wait(f"k_empty{s}", ((cit // k_slots) & 1) ^ 1, cit // k_slots - 1)
                    B[f"k_full{s}"].arrive()
                    cit += 1

    def score_mma():
        cit = pit = 0
        for seg, (lo, hi) in enumerate(segs):
            yield wait("q_ready", seg & 1, seg)
            for _ in range(lo, hi, PASS):
                sb = pit % N_S
                yield wait(f"s_empty{sb}", ((pit // N_S) & 1) ^ 1, pit // N_S - 1)
                for _ch in range(9):
                    s = cit % k_slots
                    yield wait(f"k_full{s}", (cit // k_slots) & 1, cit // k_slots)
                    B[f"k_empty{s}"].arrive()
                    cit += 1
                B[f"s_full{sb}"].arrive()
                pit += 1
            B["q_free"].arrive()

    def softmax():
        it = pit = 0
        for seg, (lo, hi) in enumerate(segs):
            if seg > 0:
                yield wait("q_free", (seg - 1) & 1, seg - 1)
            B["q_ready"].arrive(128)
            for j in range(lo, hi):
                k = (j - lo) % PASS
                sb = pit % N_S
                if k == 0:
                    yield wait(f"s_full{sb}", (pit // N_S) & 1, pit // N_S)
                if k == PASS - 1 or j + 1 == hi:
                    B[f"s_empty{sb}"].arrive(128)
                    pit += 1
                r = it % n_rec
                yield wait(f"stage_empty{r}", ((it // n_rec) & 1) ^ 1, it // n_rec - 1)
                B[f"stage_full{r}"].arrive(128)
                it += 1

    def sender():
        it = 0
        for lo, hi in segs:
            for _ in range(lo, hi):
                r = it % n_rec
                yield wait(f"stage_full{r}", (it // n_rec) & 1, it // n_rec)
                yield wait(f"p_empty{r}", ((it // n_rec) & 1) ^ 1, it // n_rec - 1)
                B[f"p_full{r}"].arrive(64)        # st.async bytes land with the arrivals
                B[f"stage_empty{r}"].arrive(64)
                it += 1
        for k in range(max(0, it - n_rec), it):  # drain: every record released
            yield wait(f"p_empty{k % n_rec}", (k // n_rec) & 1, k // n_rec)

    def value_tma():
        vit = 0
        for lo, hi in segs:
            for _ in range(lo, hi):
                for _n in range(2):
                    s = vit % V_SLOTS
                    yield wait(f"v_empty{s}", ((vit // V_SLOTS) & 1) ^ 1, vit // V_SLOTS - 1)
                    B[f"v_full{s}"].arrive()
                    vit += 1

    def fixup():
        vit = 0
        for lo, hi in segs:
            for _ in range(lo, hi):
                for _n in range(2):
                    s = vit % V_SLOTS
                    yield wait(f"v_full{s}", (vit // V_SLOTS) & 1, vit // V_SLOTS)
                    B[f"v_fixed{s}"].arrive()
                    vit += 1

    def value_mma():
        it = vit = ncorr = 0
        for seg, (lo, hi) in enumerate(segs):
            if seg > 0:
                yield wait("o_free", (seg - 1) & 1, seg - 1)
            for j in range(lo, hi):
                r = it % n_rec
                yield wait(f"p_full{r}", (it // n_rec) & 1, it // n_rec)
                if rescale[it] and j != lo:
                    B["pv_prev"].arrive()
                    yield wait("corr_done", ncorr & 1, ncorr)
                    ncorr += 1
                for _n in range(2):
                    s = vit % V_SLOTS
                    yield wait(f"v_full{s}", (vit // V_SLOTS) & 1, vit // V_SLOTS)
                    yield wait(f"v_fixed{s}", (vit // V_SLOTS) & 1, vit // V_SLOTS)
                    B[f"v_empty{s}"].arrive()
                    vit += 1
                B[f"p_empty{r}"].arrive()          # commit multicast to the score CTA
                if j == hi - 1:
                    B["o_ready"].arrive()
                it += 1

    def epilogue():
        it = ncorr = 0
        for seg, (lo, hi) in enumerate(segs):
            for j in range(lo, hi):
                r = it % n_rec
                yield wait(f"p_full{r}", (it // n_rec) & 1, it // n_rec)
                B[f"p_empty{r}"].arrive(4)              # remote, one per warp
                if rescale[it] and j != lo:
                    yield wait("pv_prev", ncorr & 1, ncorr)
                    ncorr += 1
                    B["corr_done"].arrive(128)
                if j == hi - 1:
                    yield wait("o_ready", seg & 1, seg)
                    B["o_free"].arrive(128)
                it += 1

    procs = dict(score_tma=score_tma(), score_mma=score_mma(), softmax=softmax(),
                 sender=sender(), value_tma=value_tma(), fixup=fixup(),
                 value_mma=value_mma(), epilogue=epilogue())
    return B, procs


def simulate(segs, seed, k_slots=K_SLOTS, n_rec=N_REC):
    """True when every role finishes; else the blocked roles' waits."""
    rng = random.Random(seed)
    nblk = sum(hi - lo for lo, hi in segs)
    rescale = [rng.random() < 0.3 for _ in range(nblk)]
    B, procs = roles(segs, rescale, k_slots, n_rec)
    pending = {name: None for name in procs}
    alive = set(procs)

    def step(name):
        g, req, moved = procs[name], pending[name], False
        while True:
            send = None
            if req is not None:
                if req[0] == "wait":
                    if not B[req[1]].passes(req[2], req[3]):
                        pending[name] = req
                        return moved
                else:
                    send = (B[req[1]].done & 1) != req[2]
            moved = True
            try:
                req = g.send(send) if req is not None else next(g)
            except StopIteration:
                alive.discard(name)
                return True
            if rng.random() < 0.3:
                pending[name] = req
                return True

    while alive:
        order = sorted(alive)
        rng.shuffle(order)
        if not any([step(n) for n in order if n in alive]):
            return {n: pending[n] for n in alive}
    return True


def _patterns():
    pats = [[(0, 1)], [(0, 3)], [(0, 4)], [(0, 64)], [(5, 7), (0, 9)], [(0, 1)] * 3,
            [(0, 2), (0, 5), (0, 1), (0, 7)], [(3, 4), (0, 64), (0, 10)]]
    rng = random.Random(1)
    pats += [[(0, rng.randint(1, 20)) for _ in range(rng.randint(1, 5))] for _ in range(24)]
    return pats


@pytest.mark.parametrize("k_slots", [3])
def test_protocol_finishes_in_every_interleaving(k_slots):
    for i, segs in enumerate(_patterns()):
        for seed in range(12):
            res = simulate(segs, 1000 * seed + i, k_slots=k_slots)
            assert res is True, f"segments {segs}, seed {seed}: blocked {res}"


def test_model_finds_a_planted_deadlock():
    """Planted fault: the value CTA's MMA releases records only after the
    epilogue's arrivals would need a fifth arrival that never comes (a
    record count of 6 instead of 5): the sender then waits for good."""
    orig = Bar.__init__

    def planted(self, name, count):
        orig(self, name, 6 if name.startswith("p_empty") else count)

    Bar.__init__ = planted
    try:
        blocked = [simulate([(0, 9)], seed) for seed in range(4)]
    finally:
        Bar.__init__ = orig
    assert all(b is not True for b in blocked)
