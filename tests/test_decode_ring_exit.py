"""A model check, on the CPU, of how the decode kernel's producer warp (decode_kernel in
paged_kv_cache_470_b200/csrc/decode.cu) leaves its shared-memory ring when a wait gives up.

The ring has S stages; the CTA's work unit uu goes to stage uu % S, and its loads may be issued only
once the consumers released unit uu - S (the stage's empty mbarrier). NL producer lanes issue the
units in rounds of NL consecutive units; a round never crosses the end of a 32-unit batch of block
ids or of a work item's run. The first `pre` units may go out before the loop (early loads, one per
stage); the loop's rounds pass over them. Consumer stream j releases its units (uu % NS == j) in
order. When the consumers give up (a wait ran out), a lane whose stage is still occupied fails its
wait and the producer stops after that round, possibly with some of the round's lanes having issued
their loads.

Before the CTA exits, the producer must wait (bounded) for every load that may still land: every
issued unit the consumers have not released. A wait on a stage is by the parity of its full
mbarrier, which cannot tell phases two apart, so it must not target a unit whose stage was refilled
since (it would miss and run out its time limit), nor a unit that was never issued. The kernel's
rule: wait for units [issued - S, issued), where `issued` counts the units of the rounds that went
through in full, except those whose stage a unit of the stopped round refilled, and for the units
the stopped round issued. Checked under random runs, lane counts, stream counts, early loads and
moments of giving up; two wrong rules are planted and must be caught: the window alone (it misses
the stopped round's loads) and the window moved past the stopped round's last issued unit (it drops
a stage whose load may still be in flight).
"""
import random

import pytest


def rounds_of(count, runs, NL):
    """The producer's rounds: consecutive units, NL at a time, cut at each run's 32-unit batches."""
    u = 0
    for run in runs:
        for bi in range(0, run, 32):
            m = min(32, run - bi)
            for i0 in range(0, m, NL):
                yield list(range(u + bi + i0, u + bi + min(i0 + NL, m)))
        u += run
    assert u == count


def exit_waits(issued, went, S, NL, rule):
    if rule == "kernel":
        waits = {v for v in range(max(0, issued - S), issued)
                 if not (v + S - issued < NL and (v + S - issued) in went)}
        return waits | {issued + l for l in went}
    if rule == "window_only":
        return set(range(max(0, issued - S), issued))
    if rule == "window_moved":
        top = issued + max(went) + 1 if went else issued
        return set(range(max(0, top - S), top))
    raise ValueError(rule)


def simulate(rng, S, NL, NS, count, runs, pre, p_abort, rule):
    """One CTA's producer until it finishes or stops; returns the violations of the exit rule."""
    issued_set = set(range(pre))          # early loads
    released = set()
    stream_next = list(range(NS))
    aborted = False

    def release_one():
        ready = [j for j in range(NS) if stream_next[j] < count and stream_next[j] in issued_set]
        if not ready:
            return False
        j = rng.choice(ready)
        released.add(stream_next[j])
        stream_next[j] += NS
        return True

    def free(uu):
        return uu < S or (uu - S) in released

    issued, went = 0, set()
    for rnd in rounds_of(count, runs, NL):
        for _ in range(rng.randrange(3)):      # consumers make progress between rounds
            if not aborted:
                release_one()
        while not aborted and not all(uu < pre or free(uu) for uu in rnd):
            if rng.random() < p_abort:
                aborted = True                 # the consumers gave up: occupied stages stay occupied
            elif not release_one():
                raise AssertionError("no progress possible")
        ok = [uu < pre or free(uu) for uu in rnd]
        for uu, good in zip(rnd, ok):
            if good and uu >= pre:
                assert uu not in issued_set
                issued_set.add(uu)
        if not all(ok):
            went = {l for l, good in enumerate(ok) if good}
            break
        issued = rnd[-1] + 1
    waits = exit_waits(issued, went, S, NL, rule)
    problems = []
    for uu in sorted(issued_set - released):
        if uu not in waits:
            problems.append(f"unit {uu} may still land and is not waited for")
    for uu in sorted(waits):
        if uu not in issued_set:
            problems.append(f"wait for unit {uu}, never issued")
        elif uu + S in issued_set:
            problems.append(f"wait for unit {uu}, whose stage unit {uu + S} refilled")
    return problems, bool(went) or aborted


def random_case(rng):
    NL = rng.choice([1, 2, 4, 8])
    NS = rng.choice([1, 2, 4, 8])
    unit_of = max(NL, NS)
    S = rng.choice([s for s in (6, 12, 24, 48) if s % unit_of == 0 and s >= unit_of] or [unit_of])
    count = rng.randrange(1, 260)
    runs, left = [], count
    while left:
        r = rng.randrange(1, min(left, 90) + 1)
        runs.append(r)
        left -= r
    pre = rng.choice([0, min(S, runs[0], 32)])
    return S, NL, NS, count, runs, pre


@pytest.mark.parametrize("seed", range(6))
def test_the_exit_waits_cover_every_load_in_flight(seed):
    rng = random.Random(seed)
    stopped = 0
    for _ in range(400):
        S, NL, NS, count, runs, pre = random_case(rng)
        problems, stop = simulate(rng, S, NL, NS, count, runs, pre, rng.choice([0.0, 0.05, 0.3]), "kernel")
        assert not problems, (S, NL, NS, count, runs, pre, problems[:3])
        stopped += stop
    assert stopped > 50          # the stopped-round path was exercised


@pytest.mark.parametrize("rule", ["window_only", "window_moved"])
def test_planted_exit_rules_are_caught(rule):
    rng = random.Random(99)
    caught = 0
    for _ in range(2000):
        S, NL, NS, count, runs, pre = random_case(rng)
        state = rng.getstate()
        problems, _ = simulate(rng, S, NL, NS, count, runs, pre, 0.3, rule)
        rng.setstate(state)
        good, _ = simulate(rng, S, NL, NS, count, runs, pre, 0.3, "kernel")
        assert not good
        caught += bool(problems)
    assert caught > 0, rule


# ---------------------------------------------------------------------------------------------------------
# Why the ring's stage count is a multiple of the consumer streams. Consumer stream j takes units j, j + NS,
# ...; with S a multiple of NS, every stage then has a single consuming stream. A stage's full mbarrier is
# waited on by parity, which cannot tell phases two apart: were S not a multiple of NS, two streams would
# share a stage, and one that reached the stage's next phase while the other still held the current one
# would pass its wait on stale data. The model runs a producer, loads landing late and the streams under
# random schedules, and catches exactly that when S is odd.
# ---------------------------------------------------------------------------------------------------------
class StageBar:
    def __init__(self):
        self.phase = 0

    def arrive(self):  # one arrival completes a phase (the model counts whole releases and landings)
        self.phase += 1

    def done(self, parity):
        return (self.phase & 1) != parity


def run_streams(rng, S, NS, count):
    """Returns the first read of a stage that holds another unit's data, or None."""
    full, empty = [StageBar() for _ in range(S)], [StageBar() for _ in range(S)]
    stage = [None] * S
    nxt = list(range(NS))                  # each stream's next unit
    issued, inflight = 0, []
    for _ in range(50 * count + 100):
        acts = []
        if issued < count and empty[issued % S].done(((issued // S) & 1) ^ 1):
            acts.append("issue")
        if inflight:
            acts.append("land")
        acts += [j for j in range(NS) if nxt[j] < count and full[nxt[j] % S].done((nxt[j] // S) & 1)]
        if not acts:
            break
        a = rng.choice(acts)
        if a == "issue":
            inflight.append(issued)
            issued += 1
        elif a == "land":
            uu = inflight.pop(rng.randrange(len(inflight)))
            stage[uu % S] = uu
            full[uu % S].arrive()
        else:
            uu = nxt[a]
            if stage[uu % S] != uu:
                return f"stream {a} passed its wait for unit {uu} with stage {uu % S} holding {stage[uu % S]}"
            nxt[a] += NS
            empty[uu % S].arrive()
    assert all(n >= count for n in nxt), "the schedule stopped before every unit was read"
    return None


@pytest.mark.parametrize("S,NS", [(6, 2), (12, 4), (24, 8), (12, 2), (48, 8)])
def test_a_stage_count_the_streams_divide_keeps_every_read_fresh(S, NS):
    rng = random.Random(S * 100 + NS)
    for _ in range(60):
        assert run_streams(rng, S, NS, rng.randrange(1, 4 * S + 7)) is None


def test_an_odd_stage_count_is_caught():
    rng = random.Random(5)
    assert sum(run_streams(rng, 13, 2, 80) is not None for _ in range(200)) > 0


@pytest.mark.parametrize("S,NS", [(12, 2), (6, 2), (12, 4), (24, 8), (48, 8), (2, 2)])
def test_stepped_stage_and_phase_match_the_unit_index(S, NS):
    """Each consumer stream steps its units' stage and phase (stage + NS, wrapping with a phase flip) instead of
    dividing the unit index: from any item start u and for every stream, the stepped values equal uu % S and
    (uu / S) & 1 for each unit uu = u + i, u + i + NS, ... the stream takes."""
    for u in range(0, 3 * S + 5):
        for stream in range(NS):
            i = (stream - u) % NS
            s, ph = (u + i) % S, ((u + i) // S) & 1
            for _ in range(4 * S):
                uu = u + i
                assert (s, ph) == (uu % S, (uu // S) & 1), (S, NS, u, stream, uu)
                i += NS
                s += NS
                if s >= S:
                    s -= S
                    ph ^= 1
