"""A model check of the hand-offs of the two-tile tcgen05 chunked-prefill kernel (prefill_pair_kernel in
paged_kv_cache_470_b200/csrc/prefill.cu), on the CPU.

The kernel's CTA takes two query tiles that share every K/V tile. The model follows its actors and
barriers: the producer warp (K and V of each KV tile into their own rings), the MMA thread (S_t = Q_t K^T
and O_t += P_t V for tiles t = 0, 1; a K or V stage is released by a commit after both tiles' MMAs have
read it), four softmax warps per tile (read S, maybe rescale O, write P, hand P over; tile 0's warps also
zero the last KV tile's V rows past the context) and the epilogue. Two layouts: P written over S
(D = 128), where the next S waits for the P V and the MMAs go in a fixed order (per KV tile, tile 0's then
tile 1's), and P in columns of its own (D = 64), where the next S only waits until the softmax has read S,
the softmax waits for the last P V before it writes P again, and the MMA thread issues whichever tile's
next S or P V is ready (the model picks among the ready ones at random; the commit that releases a stage
follows the second of the two MMAs that read it, and tile 1's P V of the last KV tile waits for tile 0's). Barriers behave like mbarriers (an arrival count per
phase; a wait by parity cannot tell phases two apart); loads land and MMAs complete late, MMAs and their
commits in issue order; an MMA may run before an earlier one into another accumulator (tcgen05.mma
orders only MMAs with the same accumulator and shape), and a commit arrives once every MMA before it is
done, which is why an S written where a P V still reads must wait for that P V's commit. A random
scheduler runs many interleavings and checks that every read sees the data of its own tile and that no
run deadlocks. Mistakes are planted and must be caught.
"""
import random

import pytest

WARPS = 4  # softmax warps per query tile


class Violation(AssertionError):
    pass


class MBar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self, n=1):
        for _ in range(n):
            self.pending -= 1
            assert self.pending >= 0
            if self.pending == 0:
                self.phase += 1
                self.pending = self.count

    def done(self, parity):
        """mbarrier.try_wait.parity: true while the current phase's parity differs."""
        return (self.phase & 1) != parity


class PairModel:
    def __init__(self, ntiles, sep_p, kstages, vstages, seed=0, bug=None):
        self.n, self.sep_p, self.ks, self.vs, self.bug = ntiles, sep_p, kstages, vstages, bug
        self.rng = random.Random(seed)
        self.fullK = [MBar(1) for _ in range(kstages)]
        self.emptyK = [MBar(1) for _ in range(kstages)]
        self.fullV = [MBar(1) for _ in range(vstages)]
        self.emptyV = [MBar(1) for _ in range(vstages)]
        self.s_full = [MBar(1) for _ in range(2)]
        self.s_read = [MBar(WARPS * 32) for _ in range(2)]
        self.p_full = [MBar(WARPS * 32) for _ in range(2)]
        self.pv_done = [MBar(1) for _ in range(2)]
        self.o_done = MBar(1)
        self.k_stage = [None] * kstages
        self.v_stage = [None] * vstages
        self.readers = {}                               # (kind, stage) -> MMAs still to read it
        self.s_buf = [None, None]                       # the KV tile whose S each query tile's S holds
        self.s_read_by = [[None] * WARPS for _ in range(2)]  # last KV tile whose S each warp has read
        self.p_rows = [[None] * WARPS for _ in range(2)]     # KV tile whose P each warp wrote
        self.o_tiles = [0, 0]                           # P V done per query tile
        self.v_zeroed = set()
        self.inflight = []
        self.tc_queue = []
        self.step = 0

    @staticmethod
    def accumulator(op):
        return ("S" if op[0] == "S" else "O", op[2])

    # ---- asynchronous units ----
    def land(self, kind, j):
        ns = self.ks if kind == "K" else self.vs
        s = j % ns
        if self.readers.get((kind, s), 0):
            held = (self.k_stage if kind == "K" else self.v_stage)[s]
            raise Violation(f"{kind}({j}) lands while an MMA still reads tile {held}'s stage")
        (self.k_stage if kind == "K" else self.v_stage)[s] = j
        (self.fullK if kind == "K" else self.fullV)[s].arrive()

    def run_tc_op(self, op):
        kind = op[0]
        if kind == "S":
            j, t = op[1], op[2]
            if self.k_stage[j % self.ks] != j:
                raise Violation(f"S({j},{t}) reads K stage holding tile {self.k_stage[j % self.ks]}")
            prev = self.s_buf[t]
            if prev is not None:
                if any(r != prev for r in self.s_read_by[t]):
                    raise Violation(f"S({j},{t}) overwrites S of tile {prev} before every warp read it")
                if not self.sep_p and self.o_tiles[t] <= prev:
                    raise Violation(f"S({j},{t}) overwrites P of tile {prev} before its P V")
            self.s_buf[t] = j
            if not self.sep_p:
                self.p_rows[t] = [None] * WARPS
            self.readers[("K", j % self.ks)] -= 1
        elif kind == "PV":
            j, t = op[1], op[2]
            if self.v_stage[j % self.vs] != j:
                raise Violation(f"PV({j},{t}) reads V stage holding tile {self.v_stage[j % self.vs]}")
            if any(w != j for w in self.p_rows[t]):
                raise Violation(f"PV({j},{t}) reads P rows {self.p_rows[t]} (not all of tile {j})")
            if j == self.n - 1 and j not in self.v_zeroed:
                raise Violation(f"PV({j},{t}) reads the last tile's V before its tail rows are zeroed")
            if self.o_tiles[t] != j:
                raise Violation("P V out of order")
            self.o_tiles[t] = j + 1
            self.readers[("V", j % self.vs)] -= 1
        elif kind == "commit":
            for bar in op[1:]:
                bar.arrive()

    # ---- actors (generators yielding wait conditions) ----
    def producer(self):
        for j in range(self.n):
            for kind in ("K", "V"):
                ns = self.ks if kind == "K" else self.vs
                s = j % ns
                empty = (self.emptyK if kind == "K" else self.emptyV)[s]
                if self.bug == "loads_ignore_empty":
                    yield lambda: True
                else:
                    yield lambda e=empty, p=((j // ns) & 1) ^ 1: e.done(p)
                self.inflight.append((self.step + self.rng.randint(1, 40), ("land", kind, j)))

    def mma(self):
        def issue_s(j, t):
            self.readers[("K", j % self.ks)] = self.readers.get(("K", j % self.ks), 0) + 1
            self.tc_queue.append(("S", j, t))
            self.tc_queue.append(("commit", self.s_full[t]))
            release = 0 if self.bug == "release_k_after_one" else 1
            if t == release and j + self.ks < self.n:
                self.tc_queue.append(("commit", self.emptyK[j % self.ks]))

        def issue_pv(j, t):
            self.readers[("V", j % self.vs)] = self.readers.get(("V", j % self.vs), 0) + 1
            self.tc_queue.append(("PV", j, t))
            self.tc_queue.append(("commit", self.pv_done[t]))
            release = 0 if self.bug == "release_v_after_one" else 1
            if t == release and j + self.vs < self.n:
                self.tc_queue.append(("commit", self.emptyV[j % self.vs]))

        yield lambda: self.fullK[0].done(0)
        issue_s(0, 0)
        issue_s(0, 1)
        if self.sep_p:
            yield from self.mma_ready_first()
            return
        for j in range(self.n):
            more = j + 1 < self.n
            kn, kp = (j + 1) % self.ks, ((j + 1) // self.ks) & 1
            order = (1, 0) if self.bug == "tile1_first" else (0, 1)
            for t in order:
                if self.sep_p and more:
                    if self.bug != "s_without_read_wait":
                        yield lambda t=t, p=j & 1: self.s_read[t].done(p)
                    if t == order[0]:
                        yield lambda s=kn, p=kp: self.fullK[s].done(p)
                    issue_s(j + 1, t)
                yield lambda t=t, p=j & 1: self.p_full[t].done(p)
                if t == order[0]:
                    yield lambda s=j % self.vs, p=(j // self.vs) & 1: self.fullV[s].done(p)
                issue_pv(j, t)
                if not self.sep_p and more:
                    if t == order[0]:
                        yield lambda s=kn, p=kp: self.fullK[s].done(p)
                    if self.bug != "s_without_pv_wait":
                        yield lambda t=t, p=j & 1: self.pv_done[t].done(p)
                    issue_s(j + 1, t)
        self.tc_queue.append(("commit", self.o_done))
        yield lambda: self.o_done.done(0)

    def mma_ready_first(self):
        n, ks, vs = self.n, self.ks, self.vs
        ns, np_ = [1, 1], [0, 0]

        def ready():
            ops = []
            for t in (0, 1):
                j = ns[t]
                if (j < n and (self.bug == "s_without_read_wait" or self.s_read[t].done((j - 1) & 1))
                        and self.fullK[j % ks].done((j // ks) & 1)):
                    ops.append(("S", t))
                j = np_[t]
                last_waits = t == 1 and j == n - 1 and np_[0] < n and self.bug != "last_pv_before_zeroing"
                if (j < n and not last_waits and self.p_full[t].done(j & 1)
                        and self.fullV[j % vs].done((j // vs) & 1)):
                    ops.append(("PV", t))
            return ops

        while np_[0] < n or np_[1] < n:
            yield lambda: bool(ready())
            kind, t = self.rng.choice(ready())
            if kind == "S":
                j = ns[t]
                self.readers[("K", j % ks)] = self.readers.get(("K", j % ks), 0) + 1
                self.tc_queue.append(("S", j, t))
                self.tc_queue.append(("commit", self.s_full[t]))
                second = ns[1 - t] > j
                if (second != (self.bug == "release_k_after_one")) and j + ks < n:
                    self.tc_queue.append(("commit", self.emptyK[j % ks]))
                ns[t] = j + 1
            else:
                j = np_[t]
                self.readers[("V", j % vs)] = self.readers.get(("V", j % vs), 0) + 1
                self.tc_queue.append(("PV", j, t))
                self.tc_queue.append(("commit", self.pv_done[t]))
                second = np_[1 - t] > j
                if (second != (self.bug == "release_v_after_one")) and j + vs < n:
                    self.tc_queue.append(("commit", self.emptyV[j % vs]))
                np_[t] = j + 1
        self.tc_queue.append(("commit", self.o_done))
        yield lambda: self.o_done.done(0)

    def softmax(self, t, w):
        for j in range(self.n):
            yield lambda t=t, p=j & 1: self.s_full[t].done(p)
            if self.s_buf[t] != j:
                raise Violation(f"tile {t} warp {w} reads S holding {self.s_buf[t]} at KV tile {j}")
            self.s_read_by[t][w] = j
            if self.sep_p:
                self.s_read[t].arrive(32)
            rescale = j > 0 and self.rng.random() < 0.3     # the row maximum grew
            if j > 0 and (rescale or (self.sep_p and self.bug != "p_without_pv_wait")):
                yield lambda t=t, p=(j - 1) & 1: self.pv_done[t].done(p)
            if rescale and self.o_tiles[t] != j:
                raise Violation(f"tile {t} warp {w} rescales O with {self.o_tiles[t]} of {j} P V done")
            for _ in range(self.rng.randint(0, 3)):         # the softmax takes a while
                yield lambda: True
            if not self.sep_p and self.s_buf[t] != j:
                raise Violation(f"tile {t} warp {w} writes P over S holding {self.s_buf[t]} at {j}")
            if self.sep_p and self.p_rows[t][w] is not None and self.o_tiles[t] <= self.p_rows[t][w]:
                raise Violation(f"tile {t} warp {w} overwrites P of tile {self.p_rows[t][w]} before its P V")
            self.p_rows[t][w] = j
            if t == 0 and j == self.n - 1:                  # zero the last tile's V rows past the context
                yield lambda s=j % self.vs, p=(j // self.vs) & 1: self.fullV[s].done(p)
                if self.v_stage[j % self.vs] != j:
                    raise Violation(f"warp {w} zeroes rows of V stage holding {self.v_stage[j % self.vs]}")
                self.v_zeroed.add(j)
            self.p_full[t].arrive(32)
        if self.bug == "epilogue_by_pv_parity":
            yield lambda t=t, p=(self.n - 1) & 1: self.pv_done[t].done(p)
        else:
            yield lambda: self.o_done.done(0)
        if self.o_tiles[t] != self.n:
            raise Violation(f"tile {t} warp {w} reads O with {self.o_tiles[t]} of {self.n} P V done")

    # ---- scheduler ----
    def run(self, max_steps=200000):
        actors = {"producer": self.producer(), "mma": self.mma()}
        for t in range(2):
            for w in range(WARPS):
                actors[f"softmax{t}.{w}"] = self.softmax(t, w)
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
                    continue
                raise Violation(f"deadlock: {sorted(actors)} wait, nothing in flight")
            pick = self.rng.choice(choices)
            if pick == "tc":
                # any MMA whose accumulator has no earlier MMA pending, or the first commit once every MMA
                # before it is done
                q, ready = self.tc_queue, []
                for i, op in enumerate(q):
                    earlier = q[:i]
                    if op[0] == "commit":
                        if not any(e[0] in ("S", "PV") for e in earlier) and not any(e[0] == "commit" for e in earlier):
                            ready.append(i)
                    elif not any(e[0] in ("S", "PV") and self.accumulator(e) == self.accumulator(op) for e in earlier):
                        ready.append(i)
                self.run_tc_op(q.pop(self.rng.choice(ready)))
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


# the kernel's two layouts: P over S with two K and two V stages (D = 128); P apart with three each (D = 64)
LAYOUTS = {"P_over_S": dict(sep_p=False, kstages=2, vstages=2), "P_apart": dict(sep_p=True, kstages=3, vstages=3)}


@pytest.mark.parametrize("layout", sorted(LAYOUTS))
@pytest.mark.parametrize("ntiles", [1, 2, 3, 5, 8])
def test_pair_kernel_hand_offs_hold_under_random_schedules(ntiles, layout):
    for seed in range(120):
        PairModel(ntiles, seed=seed, **LAYOUTS[layout]).run()


# (An epilogue that waits for the last P V by the parity of its tile's P-V barrier, the mistake the one-tile
# kernel once had, is no mistake here: a softmax warp reaches the epilogue only after the P V of the KV tile
# before the last is done, so that wait is never two phases behind.)
@pytest.mark.parametrize("layout,bug", [
    ("P_over_S", "release_k_after_one"), ("P_over_S", "release_v_after_one"),
    ("P_over_S", "s_without_pv_wait"), ("P_over_S", "tile1_first"),
    ("P_over_S", "loads_ignore_empty"),
    ("P_apart", "release_k_after_one"), ("P_apart", "release_v_after_one"),
    ("P_apart", "s_without_read_wait"), ("P_apart", "p_without_pv_wait"),
    ("P_apart", "last_pv_before_zeroing"), ("P_apart", "loads_ignore_empty")])
def test_the_pair_model_catches_the_hand_off_mistakes(layout, bug):
    caught = 0
    for seed in range(300):
        try:
            PairModel(6, seed=seed, bug=bug, **LAYOUTS[layout]).run()
        except Violation:
            caught += 1
    assert caught > 0, f"{bug} never showed up in 300 schedules"
