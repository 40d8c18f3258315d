"""A model check of the hand-offs of the tcgen05 chunked-prefill kernel (prefill_tc_kernel in
paged_kv_cache_470_b200/csrc/prefill.cu), on the CPU.

The model follows the kernel's actors and barriers: the producer warp (TMA loads of K and V into
their own rings, K issued ahead of V), the MMA thread (S = Q K^T into one of SB S buffers, P V into
O, tcgen05.commit arrivals), four softmax warps (32 rows each: read S, maybe rescale O, write P
over S, zero the V rows of the last tile, hand P over) and the epilogue. The kernel has SB = 2 S
buffers at D = 128 and SB = 3 (with three K and three V stages) at D = 64, where tensor memory has room: S of
tile j + SB - 1 is issued once the P V of tile j - 1 is done, and the S-full, P-ready and P-V-done
barriers are one per S buffer. Barriers behave like mbarriers: an arrival count per phase, and a wait
by parity that succeeds while the current phase differs in parity from the one asked for (so it
cannot tell phases two apart). Loads land and MMAs complete late, MMAs and their commits in issue
order. A random scheduler runs many interleavings and checks that every read sees the data of its
own tile (K, V, S, every warp's P, O after all P V) and that no run deadlocks. Mistakes are planted
in the model and must be caught: the two the kernel once had (one P-ready barrier for both tile
parities; the epilogue waiting for the last P V by the parity of one P-V barrier), the two a third
buffer invites (P-ready barriers by tile parity; one P-V barrier waited by parity), and a producer
that refills a stage without waiting for it to come free (which shows that the stage checks have
teeth).
"""
import random

import pytest

WARPS = 4


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
    def __init__(self, ntiles, sbufs=2, kstages=2, vstages=2, one_p_barrier=False, epilogue_by_pv_parity=False,
                 loads_ignore_empty=False, p_by_parity=False, one_pv_barrier=False, seed=0):
        self.n = ntiles
        self.sb, self.ks, self.vs = sbufs, kstages, vstages
        self.rng = random.Random(seed)
        self.one_p = one_p_barrier
        self.p_parity = p_by_parity
        self.one_pv = one_pv_barrier
        self.epi_parity = epilogue_by_pv_parity
        self.no_empty = loads_ignore_empty
        self.fullK = [MBar(1) for _ in range(kstages)]
        self.emptyK = [MBar(1) for _ in range(kstages)]
        self.fullV = [MBar(1) for _ in range(vstages)]
        self.emptyV = [MBar(1) for _ in range(vstages)]
        self.s_full = [MBar(1) for _ in range(sbufs)]
        self.p_full = [MBar(WARPS * 32) for _ in range(sbufs)]
        self.pv_done = [MBar(1) for _ in range(sbufs)]
        self.pv_all = MBar(1)        # one barrier committed after every P V: only the planted mistakes use it
        self.o_done = MBar(1)
        # contents: which tile each stage / buffer holds (None: nothing yet)
        self.k_stage = [None] * kstages
        self.v_stage = [None] * vstages
        self.s_buf = [None] * sbufs                            # the tile whose S each buffer holds
        self.p_rows = [[None] * WARPS for _ in range(sbufs)]   # tile whose P each warp wrote in a buffer
        self.o_tiles = 0                                       # P V done
        self.v_zeroed = set()
        self.inflight = []                                     # (landing step, action)
        self.tc_queue = []                                     # tensor-core ops in issue order
        self.reads = {}                                        # stage readers still in flight
        self.step = 0

    # barrier and parity of P-ready (and of the P-V-done wait) for tile j, as the kernel (or a mistake) picks
    def p_bar(self, j):
        if self.one_p:
            return self.p_full[0], j & 1
        if self.p_parity:
            return self.p_full[j & 1], (j >> 1) & 1
        return self.p_full[j % self.sb], (j // self.sb) & 1

    def pv_wait(self, j):
        """(barrier, parity) of a wait for P V(j) to be done."""
        if self.one_pv:
            return self.pv_all, j & 1
        return self.pv_done[j % self.sb], (j // self.sb) & 1

    # ---- asynchronous units ----
    def land(self, kind, t):
        ns = self.ks if kind == "K" else self.vs
        s = t % ns
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
            if self.k_stage[t % self.ks] != t:
                raise Violation(f"S({t}) reads K stage holding tile {self.k_stage[t % self.ks]}")
            b = t % self.sb
            if self.s_buf[b] is not None and self.o_tiles <= self.s_buf[b]:
                raise Violation(f"S({t}) overwrites the P of tile {self.s_buf[b]} before its P V")
            self.s_buf[b] = t
            self.p_rows[b] = [None] * WARPS
            self.reads[("K", t % self.ks)] = False
        elif kind == "PV":
            t = op[1]
            b = t % self.sb
            if self.v_stage[t % self.vs] != t:
                raise Violation(f"PV({t}) reads V stage holding tile {self.v_stage[t % self.vs]}")
            if self.s_buf[b] != t or any(w != t for w in self.p_rows[b]):
                raise Violation(f"PV({t}) reads P rows {self.p_rows[b]} (not all of tile {t})")
            if t == self.n - 1 and t not in self.v_zeroed:
                raise Violation(f"PV({t}) reads the last tile's V before its tail rows are zeroed")
            if self.o_tiles != t:
                raise Violation("P V out of order")
            self.o_tiles = t + 1
            self.reads[("V", t % self.vs)] = False
        elif kind == "commit":
            for bar in op[1:]:
                bar.arrive()

    # ---- actors (generators yielding wait conditions) ----
    def producer(self):
        order = [("K", t) for t in range(min(self.ks, self.n))]
        for t in range(self.n):
            order.append(("V", t))
            if t + self.ks < self.n:
                order.append(("K", t + self.ks))
        for kind, t in order:
            ns = self.ks if kind == "K" else self.vs
            s = t % ns
            empty = (self.emptyK if kind == "K" else self.emptyV)[s]
            if self.no_empty:
                yield lambda: True
            else:
                yield lambda e=empty, p=((t // ns) & 1) ^ 1: e.done(p)
            self.inflight.append((self.step + self.rng.randint(1, 40), ("land", kind, t)))

    def mma(self):
        def issue_s(j):
            self.reads[("K", j % self.ks)] = True
            self.tc_queue.append(("S", j))
            self.tc_queue.append(("commit", self.s_full[j % self.sb]))
            if j + self.ks < self.n:
                self.tc_queue.append(("commit", self.emptyK[j % self.ks]))
        for j in range(min(self.sb - 1, self.n)):                 # S of the first SB - 1 tiles
            yield lambda s=j % self.ks, p=(j // self.ks) & 1: self.fullK[s].done(p)
            issue_s(j)
        for j in range(self.n):
            t = j + self.sb - 1
            if t < self.n:
                if t >= self.sb:                                  # its S buffer's previous P V
                    yield lambda bp=self.pv_wait(t - self.sb): bp[0].done(bp[1])
                yield lambda s=t % self.ks, p=(t // self.ks) & 1: self.fullK[s].done(p)
                issue_s(t)
            yield lambda bp=self.p_bar(j): bp[0].done(bp[1])
            yield lambda s=j % self.vs, p=(j // self.vs) & 1: self.fullV[s].done(p)
            self.reads[("V", j % self.vs)] = True
            self.tc_queue.append(("PV", j))
            self.tc_queue.append(("commit", self.pv_done[j % self.sb], self.pv_all))
            if j + self.vs < self.n:
                self.tc_queue.append(("commit", self.emptyV[j % self.vs]))
        self.tc_queue.append(("commit", self.o_done))
        yield lambda: self.o_done.done(0)

    def softmax(self, w):
        for j in range(self.n):
            b = j % self.sb
            yield lambda bar=self.s_full[b], p=(j // self.sb) & 1: bar.done(p)
            if self.s_buf[b] != j:
                raise Violation(f"warp {w} reads S buffer holding {self.s_buf[b]} at tile {j}")
            if j > 0 and self.rng.random() < 0.3:          # the row maximum grew: rescale O
                yield lambda bp=self.pv_wait(j - 1): bp[0].done(bp[1])
                if self.o_tiles != j:
                    raise Violation(f"warp {w} rescales O with {self.o_tiles} of {j} P V done")
            for _ in range(self.rng.randint(0, 3)):        # the softmax takes a while
                yield lambda: True
            if self.s_buf[b] != j:
                raise Violation(f"warp {w} writes P over S buffer holding {self.s_buf[b]} at tile {j}")
            self.p_rows[b][w] = j
            if j == self.n - 1:                            # zero the last tile's tail V rows
                yield lambda s=j % self.vs, p=(j // self.vs) & 1: self.fullV[s].done(p)
                if self.v_stage[j % self.vs] != j:
                    raise Violation(f"warp {w} zeroes rows of V stage holding {self.v_stage[j % self.vs]}")
                self.v_zeroed.add(j)
            bar = self.p_bar(j)[0]
            for _ in range(32):
                bar.arrive()
        if self.epi_parity:
            yield lambda p=(self.n - 1) & 1: self.pv_all.done(p)
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


GEOMETRIES = {"D128": dict(sbufs=2, kstages=2, vstages=2), "D64": dict(sbufs=3, kstages=3, vstages=3)}


@pytest.mark.parametrize("geo", sorted(GEOMETRIES))
@pytest.mark.parametrize("ntiles", [1, 2, 3, 4, 7])
def test_kernel_hand_offs_hold_under_random_schedules(ntiles, geo):
    for seed in range(150):
        Model(ntiles, seed=seed, **GEOMETRIES[geo]).run()


@pytest.mark.parametrize("geo,bug", [("D128", "one_p_barrier"), ("D128", "epilogue_by_pv_parity"),
                                     ("D128", "loads_ignore_empty"), ("D64", "p_by_parity"),
                                     ("D64", "one_pv_barrier"), ("D64", "loads_ignore_empty"),
                                     ("D64", "epilogue_by_pv_parity"), ("D64", "two_v_stages")])
def test_the_model_catches_the_hand_off_mistakes(geo, bug):
    caught = 0
    geometry = dict(GEOMETRIES[geo])
    if bug == "two_v_stages":       # three S buffers run far enough ahead to wrap a two-stage V ring
        geometry["vstages"] = 2
        planted = {}
    else:
        planted = {bug: True}
    for seed in range(300):
        try:
            Model(7, seed=seed, **geometry, **planted).run()
        except Violation:
            caught += 1
    assert caught > 0, f"{bug} never showed up in 300 schedules"
