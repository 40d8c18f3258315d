"""A model check of the hand-offs of the tcgen05 chunked-prefill kernel (prefill_tc_kernel in
paged_kv_cache_470_b200/csrc/prefill.cu), on the CPU.

The model follows the kernel's actors and barriers: the producer warp (TMA loads of K and V into
two-stage rings, K two tiles ahead), the MMA thread (S = Q K^T into one of two S buffers, P V into
O, tcgen05.commit arrivals), four softmax warps (32 rows each: read S, maybe rescale O, write P
over S, zero the V rows of the last tile, hand P over) and the epilogue. Barriers behave like
mbarriers: an arrival count per phase, and a wait by parity that succeeds while the current phase
differs in parity from the one asked for (so it cannot tell phases two apart). Loads land and MMAs
complete late, MMAs and their commits in issue order. A random scheduler runs many interleavings
and checks that every read sees the data of its own tile (K, V, S, every warp's P, O after all
P V) and that no run deadlocks. The two hand-off mistakes the kernel once had (one P-ready barrier
for both tile parities; the epilogue waiting for the last P V by the parity of the P-V barrier)
are planted in the model and must be caught, as must a producer that refills a stage without
waiting for it to come free (which shows that the stage checks have teeth).
"""
import random

import pytest

WARPS = 4
STAGES = 2


class Violation(AssertionError):
    pass


class MBar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        """mbarrier.try_wait.parity: true while the current phase's parity differs."""
        return (self.phase & 1) != parity


class Model:
    def __init__(self, ntiles, one_p_barrier=False, epilogue_by_pv_parity=False, loads_ignore_empty=False,
                 seed=0):
        self.n = ntiles
        self.rng = random.Random(seed)
        self.one_p = one_p_barrier
        self.epi_parity = epilogue_by_pv_parity
        self.no_empty = loads_ignore_empty
        self.fullK = [MBar(1) for _ in range(STAGES)]
        self.emptyK = [MBar(1) for _ in range(STAGES)]
        self.fullV = [MBar(1) for _ in range(STAGES)]
        self.emptyV = [MBar(1) for _ in range(STAGES)]
        self.s_full = [MBar(1), MBar(1)]
        self.p_full = [MBar(WARPS * 32), MBar(WARPS * 32)]
        self.pv_done = MBar(1)
        self.o_done = MBar(1)
        # contents: which tile each stage / buffer holds (None: nothing yet)
        self.k_stage = [None] * STAGES
        self.v_stage = [None] * STAGES
        self.s_buf = [None, None]                       # the tile whose S each buffer holds
        self.p_rows = [[None] * WARPS for _ in range(2)]  # tile whose P each warp wrote in a buffer
        self.o_tiles = 0                                # P V done
        self.v_zeroed = set()
        self.inflight = []                              # (landing step, action)
        self.tc_queue = []                              # tensor-core ops in issue order
        self.reads = {}                                 # stage readers still in flight
        self.step = 0

    # ---- asynchronous units ----
    def land(self, kind, t):
        s = t % STAGES
        stage = self.k_stage if kind == "K" else self.v_stage
        # the load overwrites the stage: its previous tile's MMA must be done
        if self.reads.get((kind, s)):
            raise Violation(f"{kind}({t}) lands while an MMA still reads tile {stage[s]}'s stage")
        stage[s] = t
        (self.fullK if kind == "K" else self.fullV)[s].arrive()

    def run_tc_op(self, op):
        kind = op[0]
        if kind == "S":
            t = op[1]
            if self.k_stage[t % STAGES] != t:
                raise Violation(f"S({t}) reads K stage holding tile {self.k_stage[t % STAGES]}")
            self.s_buf[t & 1] = t
            self.p_rows[t & 1] = [None] * WARPS
            self.reads[("K", t % STAGES)] = False
        elif kind == "PV":
            t = op[1]
            if self.v_stage[t % STAGES] != t:
                raise Violation(f"PV({t}) reads V stage holding tile {self.v_stage[t % STAGES]}")
            if any(w != t for w in self.p_rows[t & 1]):
                raise Violation(f"PV({t}) reads P rows {self.p_rows[t & 1]} (not all of tile {t})")
            if t == self.n - 1 and t not in self.v_zeroed:
                raise Violation(f"PV({t}) reads the last tile's V before its tail rows are zeroed")
            if self.o_tiles != t:
                raise Violation("P V out of order")
            self.o_tiles = t + 1
            self.reads[("V", t % STAGES)] = False
        elif kind == "commit":
            op[1].arrive()

    # ---- actors (generators yielding wait conditions) ----
    def producer(self):
        order = [("K", t) for t in range(min(STAGES, self.n))]
        for t in range(self.n):
            order.append(("V", t))
            if t + STAGES < self.n:
                order.append(("K", t + STAGES))
        for kind, t in order:
            s = t % STAGES
            empty = (self.emptyK if kind == "K" else self.emptyV)[s]
            if self.no_empty:
                yield lambda: True
            else:
                yield lambda e=empty, p=((t // STAGES) & 1) ^ 1: e.done(p)
            self.inflight.append((self.step + self.rng.randint(1, 40), ("land", kind, t)))

    def mma(self):
        def issue_s(j):
            self.reads[("K", j % STAGES)] = True
            self.tc_queue.append(("S", j))
            self.tc_queue.append(("commit", self.s_full[j & 1]))
            if j + STAGES < self.n:
                self.tc_queue.append(("commit", self.emptyK[j % STAGES]))
        yield lambda: self.fullK[0].done(0)
        issue_s(0)
        for j in range(self.n):
            if j + 1 < self.n:
                if j >= 1:
                    yield lambda p=(j - 1) & 1: self.pv_done.done(p)
                yield lambda s=(j + 1) % STAGES, p=((j + 1) // STAGES) & 1: self.fullK[s].done(p)
                issue_s(j + 1)
            pf = self.p_full[0] if self.one_p else self.p_full[j & 1]
            pp = (j & 1) if self.one_p else ((j >> 1) & 1)
            yield lambda b=pf, p=pp: b.done(p)
            yield lambda s=j % STAGES, p=(j // STAGES) & 1: self.fullV[s].done(p)
            self.reads[("V", j % STAGES)] = True
            self.tc_queue.append(("PV", j))
            self.tc_queue.append(("commit", self.pv_done))
            if j + STAGES < self.n:
                self.tc_queue.append(("commit", self.emptyV[j % STAGES]))
        self.tc_queue.append(("commit", self.o_done))
        yield lambda: self.o_done.done(0)

    def softmax(self, w):
        for j in range(self.n):
            yield lambda b=self.s_full[j & 1], p=(j >> 1) & 1: b.done(p)
            if self.s_buf[j & 1] != j:
                raise Violation(f"warp {w} reads S buffer holding {self.s_buf[j & 1]} at tile {j}")
            if j > 0 and self.rng.random() < 0.3:          # the row maximum grew: rescale O
                yield lambda p=(j - 1) & 1: self.pv_done.done(p)
                if self.o_tiles != j:
                    raise Violation(f"warp {w} rescales O with {self.o_tiles} of {j} P V done")
            for _ in range(self.rng.randint(0, 3)):        # the softmax takes a while
                yield lambda: True
            self.p_rows[j & 1][w] = j
            if j == self.n - 1:                            # zero the last tile's tail V rows
                yield lambda s=j % STAGES, p=(j // STAGES) & 1: self.fullV[s].done(p)
                if self.v_stage[j % STAGES] != j:
                    raise Violation(f"warp {w} zeroes rows of V stage holding {self.v_stage[j % STAGES]}")
                self.v_zeroed.add(j)
            bar = self.p_full[0] if self.one_p else self.p_full[j & 1]
            for _ in range(32):
                bar.arrive()
        if self.epi_parity:
            yield lambda p=(self.n - 1) & 1: self.pv_done.done(p)
        else:
            yield lambda: self.o_done.done(0)
        if self.o_tiles != self.n:
            raise Violation(f"warp {w} reads O with {self.o_tiles} of {self.n} P V done")

    # ---- scheduler ----
    def run(self, max_steps=200000):
        actors = {"producer": self.producer(), "mma": self.mma()}
        for w in range(WARPS):
            actors[f"softmax{w}"] = self.softmax(w)
        waits = {name: (lambda: True) for name in actors}
        while actors or self.inflight or self.tc_queue:
            self.step += 1
            if self.step > max_steps:
                raise Violation("no progress")
            choices = [name for name in actors if waits[name]()]
            if self.tc_queue:
                choices.append("tc")
            due = [x for x in self.inflight if x[0] <= self.step]
            if due:
                choices.append("land")
            if not choices:
                if self.inflight:
                    continue                          # time passes until a load lands
                raise Violation(f"deadlock: {sorted(actors)} wait, nothing in flight")
            pick = self.rng.choice(choices)
            if pick == "tc":
                self.run_tc_op(self.tc_queue.pop(0))
            elif pick == "land":
                x = min(due)
                self.inflight.remove(x)
                self.land(x[1][1], x[1][2])
            else:
                try:
                    waits[pick] = next(actors[pick])
                except StopIteration:
                    del actors[pick]
        return True


@pytest.mark.parametrize("ntiles", [1, 2, 3, 4, 7])
def test_kernel_hand_offs_hold_under_random_schedules(ntiles):
    for seed in range(150):
        Model(ntiles, seed=seed).run()


@pytest.mark.parametrize("bug", ["one_p_barrier", "epilogue_by_pv_parity", "loads_ignore_empty"])
def test_the_model_catches_the_hand_off_mistakes(bug):
    caught = 0
    for seed in range(300):
        try:
            Model(5, seed=seed, **{bug: True}).run()
        except Violation:
            caught += 1
    assert caught > 0, f"{bug} never showed up in 300 schedules"
