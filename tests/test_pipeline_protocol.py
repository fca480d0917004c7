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
ring sizes or barrier counts must be made here too.  Rescale flags are drawn
per block (the kernel raises them only on a pass's first block; the protocol
is the same).
"""
import random

import pytest

K_SLOTS, FILLS, N_REC, V_SLOTS, PASS = 3, 5, 5, 4, 4


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


def _passes(lo, hi):
    j = lo
    while j < hi:
        nb = min(PASS, hi - j)
        yield j, nb
        j += nb


def roles(segs, rescale, k_slots, n_rec):
    """The kernel's roles as generators: score CTA (TMA, QK MMA, the two
    softmax halves of 128 threads), value CTA (TMA, fixup warp, PV MMA, the
    eight epilogue warps)."""
    B = {}

    def bar(name, count):
        B[name] = Bar(name, count)

    for i in range(k_slots):
        bar(f"k_full{i}", 1); bar(f"k_empty{i}", 1)
    bar("s_full", 1); bar("s_empty", 256)
    bar("q_ready", 256); bar("q_free", 1)
    bar("q_full", 1); bar("qstage_free", 8)          # each segment's query staged in K slots 1-2
    bar("xchg", 2)                                   # one quadrant's two warps, one per half
    for i in range(n_rec):
        bar(f"p_full{i}", 4)                         # the four warps of the writing half
        bar(f"p_empty{i}", 1)                        # PV commit, or the epilogue at a segment end
    for i in range(V_SLOTS):
        bar(f"v_full{i}", 1); bar(f"v_empty{i}", 1); bar(f"v_fixed{i}", 1)
    bar("epi_req", 2); bar("corr_done", 256); bar("o_free", 256); bar("meta_done", 8)

    def wait(name, parity, phase=None):
        return ("wait", name, parity, phase)

    def score_tma():
        fit = 0
        for seg, (lo, hi) in enumerate(segs):
            if fit > 0:                              # the ring drained: the last fill consumed
                k = fit - 1
                yield wait(f"k_empty{k % k_slots}", (k // k_slots) & 1, k // k_slots)
            B["q_full"].arrive()                     # the segment's query tile lands in slots 1-2
            staged = True
            for _j, _nb in _passes(lo, hi):
                for _f in range(FILLS):
                    s = fit % k_slots
                    yield wait(f"k_empty{s}", ((fit // k_slots) & 1) ^ 1, fit // k_slots - 1)
                    if staged and s != 0:            # slots 1-2 free once the tile moved to TMEM
                        yield wait("qstage_free", seg & 1, seg)
                        staged = False
                    B[f"k_full{s}"].arrive()
                    fit += 1

    def score_mma():
        fit = pit = 0
        for seg, (lo, hi) in enumerate(segs):
            yield wait("q_ready", seg & 1, seg)
            for _j, _nb in _passes(lo, hi):
                yield wait("s_empty", (pit & 1) ^ 1, pit - 1)
                for _f in range(FILLS):
                    s = fit % k_slots
                    yield wait(f"k_full{s}", (fit // k_slots) & 1, fit // k_slots)
                    B[f"k_empty{s}"].arrive()
                    fit += 1
                B["s_full"].arrive()
                pit += 1
            B["q_free"].arrive()

    def softmax(half):
        it = pit = xit = 0
        for seg, (lo, hi) in enumerate(segs):
            if seg > 0:
                yield wait("q_free", (seg - 1) & 1, seg - 1)
            yield wait("q_full", seg & 1, seg)
            B["qstage_free"].arrive(4)               # lane 0 of each of the half's four warps
            B["q_ready"].arrive(128)
            for j0, nb in _passes(lo, hi):
                yield wait("s_full", pit & 1, pit)
                B["s_empty"].arrive(128)
                pit += 1
                B["xchg"].arrive()
                yield wait("xchg", xit & 1, xit)
                xit += 1
                last_pass = j0 + PASS >= hi
                final = None
                for k in range(2):
                    kb = half + 2 * k                # blocks half and half + 2
                    if kb >= nb:
                        continue
                    ib = it + kb
                    r = ib % n_rec
                    yield wait(f"p_empty{r}", ((ib // n_rec) & 1) ^ 1, ib // n_rec - 1)
                    if last_pass and kb == nb - 1:
                        final = r                    # its factors wait for the sums
                    else:
                        B[f"p_full{r}"].arrive(4)    # a record is full once its bytes landed
                if last_pass:                        # last pass: the sums are exchanged
                    B["xchg"].arrive()
                    yield wait("xchg", xit & 1, xit)
                    xit += 1
                if final is not None:
                    B[f"p_full{final}"].arrive(4)
                it += nb
        for k in range(max(0, it - n_rec), it):      # drain: every record released
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
                    B["epi_req"].arrive(2)           # request posted + commit
                    yield wait("corr_done", ncorr & 1, ncorr)
                    ncorr += 1
                for _n in range(2):
                    s = vit % V_SLOTS
                    yield wait(f"v_fixed{s}", (vit // V_SLOTS) & 1, vit // V_SLOTS)
                    B[f"v_empty{s}"].arrive()
                    vit += 1
                if j == hi - 1:
                    B["epi_req"].arrive(2)           # final request; the epilogue releases r
                else:
                    B[f"p_empty{r}"].arrive()        # commit multicast to the score CTA
                it += 1

    def epilogue():
        it = nreq = nfinal = 0
        for seg, (lo, hi) in enumerate(segs):
            for j in range(lo, hi):
                r = it % n_rec
                if rescale[it] and j != lo:
                    yield wait("epi_req", nreq & 1, nreq)
                    nreq += 1
                    B["corr_done"].arrive(256)
                if j == hi - 1:
                    yield wait("epi_req", nreq & 1, nreq)
                    nreq += 1
                    B["meta_done"].arrive(8)
                    yield wait("meta_done", nfinal & 1, nfinal)
                    nfinal += 1
                    B[f"p_empty{r}"].arrive()        # remote, by one warp
                    B["o_free"].arrive(256)
                it += 1

    procs = dict(score_tma=score_tma(), score_mma=score_mma(), softmax0=softmax(0),
                 softmax1=softmax(1), value_tma=value_tma(), fixup=fixup(),
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
    """Planted fault: the record-release barrier expects two arrivals where
    the value CTA gives one: the softmax then waits for good."""
    orig = Bar.__init__

    def planted(self, name, count):
        orig(self, name, 2 if name.startswith("p_empty") else count)

    Bar.__init__ = planted
    try:
        blocked = [simulate([(0, 9)], seed) for seed in range(4)]
    finally:
        Bar.__init__ = orig
    assert all(b is not True for b in blocked)


def _with_planted_count(name_prefix, count):
    orig = Bar.__init__

    def planted(self, name, c):
        orig(self, name, count if name.startswith(name_prefix) else c)
    return orig, planted


def test_model_finds_a_planted_query_staging_fault():
    """Planted fault: the query-staging release expects nine warp arrivals
    where the eight softmax warps give eight: the TMA warp then never refills
    K slots 1-2 and the pipeline stops, on the first segment and on later
    ones."""
    orig, planted = _with_planted_count("qstage_free", 9)
    Bar.__init__ = planted
    try:
        blocked = [simulate(segs, seed) for segs in ([(0, 9)], [(0, 3), (3, 11)]) for seed in range(3)]
    finally:
        Bar.__init__ = orig
    assert all(b is not True for b in blocked)
