"""A model check, on the CPU, of how the decode kernel (decode_kernel in
paged_kv_cache_470_b200/csrc/decode.cu) divides work between CTAs and merges split items.

Plan. A launch may cover L layers, whose work positions follow one another (tables and lengths are
shared, so every layer has the same positions). Every non-empty sequence has items_per_seq items (kv-head group x query-head chunk); each
item is preceded by item_cost work positions and then has one position per KV block (unit). CTAs
take equal ranges of `chunk` positions. A CTA locates its first unit (sequence, item, block
offset, position of the item's first unit) and its unit count from a scan over the sequences, as
the kernel does; a range that starts or ends inside an item's cost positions starts or ends at
that item's first unit. An item's pieces belong to CTAs pos // chunk .. (pos + n - 1) // chunk.

Merge. A piece of a split item either finds every other piece already counted (the counter read
by the checker lane, relaxed, while its last unit runs) and merges them ("solo", no count), or
stores its partial and counts itself in with a fetch-add; the fetch-add that completes the count
merges. Earlier pieces of a CTA are counted by its helper warp, the last by the CTA itself. The
merger resets the counter, which the next launch needs at zero.

Checked over random lengths, item counts, item costs, grid sizes and layer counts: the CTAs' unit
ranges tile all units in order; the cursors point at those units; each item's first and last CTA
are the CTAs that hold its first and last unit; the workspace slots of split pieces (CTA index +
item index) never collide and stay inside the workspace; and, under random interleavings of the CTAs and their helpers,
every item is merged exactly once, only after all of its pieces are in, and every counter is back
at zero. A solo merge that forgets the reset, an off-by-one solo test, and a locating scan that
stops at the range's end (right for one layer, wrong for several) are planted and caught.
"""
import random

import pytest

BLOCK = 16


def plan(lens, ips, w, G, min_chunk, L=1, stop_at_end=False):
    """Per CTA: None (no work) or (cursor (layer, b, k, off, pos), count); and chunk.

    Layers: every layer has the same positions (tables and lengths are shared) and layer l's follow
    layer l - 1's. The kernel finds the layer of each end of a CTA's range by division and the
    position within the layer by one scan over the sequences, which must run until both ends are
    found (stop_at_end plants the single-layer rule, stopping once the end is found)."""
    nblk = [-(-max(c, 0) // BLOCK) for c in lens]
    val = [ips * (n + w) if n > 0 else 0 for n in nblk]
    per_layer = sum(val)
    nonempty = sum(1 for n in nblk if n > 0)
    units_layer = per_layer - w * ips * nonempty
    total = L * per_layer
    chunk = max(-(-total // G), min_chunk) if total else min_chunk
    out = []
    for cta in range(G):
        start, end = cta * chunk, min(cta * chunk + chunk, total)
        if start >= total:
            out.append(None)
            continue
        ls, ss = divmod(start, per_layer)
        le, se = divmod(end - 1, per_layer)
        lo, nonempty_before, cur, start_u, end_u = 0, 0, None, None, None
        for b, n in enumerate(nblk):
            v = val[b]
            hi = lo + v
            units_before = lo - w * ips * nonempty_before
            if n > 0 and lo <= ss < hi:
                r = ss - lo
                k, rr = divmod(r, n + w)
                cur = (ls, b, k, max(0, rr - w), ls * per_layer + lo + k * (n + w) + w)
                start_u = ls * units_layer + units_before + k * n + max(0, rr - w)
            if n > 0 and lo <= se < hi:
                r = se - lo
                k, rr = divmod(r, n + w)
                end_u = le * units_layer + units_before + k * n + max(0, rr - w) + (1 if rr >= w else 0)
            lo = hi
            nonempty_before += 1 if n > 0 else 0
            if end_u is not None and (stop_at_end or cur is not None):
                break
        if cur is None:          # the start was never located: the CTA would work from a stale cursor
            cur, start_u = (0, 0, 0, 0, 0), 0
        count = end_u - start_u
        out.append((cur, count) if count > 0 else None)
    return out, chunk, nblk


def next_item(cur, ips, w, nblk, L=1):
    layer, b, k, off, pos = cur
    pos += nblk[b] + w
    k += 1
    if k == ips:
        k = 0
        while True:
            b += 1
            if b == len(nblk):
                if layer + 1 == L:
                    break
                layer, b = layer + 1, 0
            if nblk[b] > 0:
                break
    return (layer, b, k, 0, pos)


def pieces_of(lens, ips, w, G, min_chunk, L=1, stop_at_end=False):
    """Each CTA's pieces in order: (item (layer, b, k), first unit, units, first_cta, last_cta)."""
    ctas, chunk, nblk = plan(lens, ips, w, G, min_chunk, L, stop_at_end)
    out = []
    for entry in ctas:
        mine = []
        if entry is not None:
            cur, count = entry
            u = 0
            while u < count:
                layer, b, k, off, pos = cur
                n = nblk[b]
                run = min(n - off, count - u)
                mine.append(((layer, b, k), off, run, pos // chunk, (pos + n - 1) // chunk))
                u += run
                if u < count:
                    cur = next_item(cur, ips, w, nblk, L)
        out.append(mine)
    return out, chunk, nblk


def random_case(rng):
    B = rng.randint(1, 40)
    lens = [rng.choice([0, rng.randint(1, 40), rng.randint(1, 700)]) for _ in range(B)]
    return lens, rng.choice([1, 2, 4]), rng.choice([0, 1, 3, 6]), rng.choice([1, 2, 3, 7, 16, 148]), \
        rng.choice([1, 4]), rng.choice([1, 1, 2, 3, 5])


def tiling_errors(lens, ips, w, G, mc, L, **plant):
    """What is wrong with the CTAs' pieces (empty list: nothing)."""
    per_cta, chunk, nblk = pieces_of(lens, ips, w, G, mc, L, **plant)
    errors = []
    # every unit (layer, sequence, item, block) in order, each held by exactly one CTA
    expected = [(l, b, k, o) for l in range(L) for b, n in enumerate(nblk) for k in range(ips) for o in range(n)]
    held, owner = [], {}
    for cta, pieces in enumerate(per_cta):
        for item, off, run, first, last in pieces:
            if not (run > 0 and off + run <= nblk[item[1]]):
                errors.append(f"CTA {cta}: bad piece {item} {off} {run}")
            for o in range(off, off + run):
                held.append(item + (o,))
                owner[item + (o,)] = cta
    if held != expected:
        errors.append("units not tiled exactly once in order")
        return errors
    # the pieces of an item agree on its first and last CTA, which hold its first and last unit
    B = len(lens)
    slots = {}
    for cta, pieces in enumerate(per_cta):
        for item, off, run, first, last in pieces:
            n = nblk[item[1]]
            if first != owner[item + (0,)] or last != owner[item + (n - 1,)] or not first <= cta <= last:
                errors.append(f"CTA {cta}: item {item} owners {first}..{last}")
            # the workspace slot of a split piece: CTA index + the item's index in the launch
            idx = (item[0] * B + item[1]) * ips + item[2]
            if first != last:
                slot = cta + idx
                if slot in slots and slots[slot] != (cta, item):
                    errors.append(f"slot {slot} shared by {slots[slot]} and {(cta, item)}")
                slots[slot] = (cta, item)
                if slot >= G + L * B * ips:
                    errors.append(f"slot {slot} beyond the workspace's {G + L * B * ips}")
    return errors


@pytest.mark.parametrize("seed", range(8))
def test_ctas_tile_every_unit_and_agree_on_item_owners(seed):
    rng = random.Random(seed)
    for _ in range(250):
        lens, ips, w, G, mc, L = random_case(rng)
        assert tiling_errors(lens, ips, w, G, mc, L) == [], (lens, ips, w, G, mc, L)


def test_a_scan_that_stops_at_the_end_is_caught():
    """With several layers a CTA's range can end at an earlier position of a later layer than the one it
    starts at; a scan that stops once the end is found then misses the start."""
    rng = random.Random(3)
    caught = 0
    for _ in range(300):
        lens, ips, w, G, mc, L = random_case(rng)
        if tiling_errors(lens, ips, w, G, mc, L, stop_at_end=True):
            caught += 1
    assert caught > 0


class Violation(AssertionError):
    pass


def run_merges(per_cta, rng, forget_reset=False, solo_off_by_one=False):
    counters, written, merged = {}, set(), {}
    pieces_of_item = {}
    for cta, pieces in enumerate(per_cta):
        for item, off, run, first, last in pieces:
            pieces_of_item.setdefault(item, set()).add(cta)

    def merge(item, first, last, me, own_in_smem):
        for c in range(first, last + 1):
            if c == me and own_in_smem:
                continue
            if (item, c) not in written:
                raise Violation(f"item {item} merged before the piece of CTA {c} is in")
        merged[item] = merged.get(item, 0) + 1
        if not forget_reset:
            counters[item] = 0

    def fetch_add(item):
        old = counters.get(item, 0)
        counters[item] = old + 1
        return old

    def cta_actor(cta, pieces, queue):
        for i, (item, off, run, first, last) in enumerate(pieces):
            final = i == len(pieces) - 1
            k = last - first
            if first == last:
                for _ in range(rng.randint(1, 3)):
                    yield
                merged[item] = merged.get(item, 0) + 1
                continue
            for _ in range(rng.randint(0, 3)):               # units before the checker's last one
                yield
            seen = counters.get(item, 0)                     # the checker's relaxed read
            for _ in range(rng.randint(1, 3)):               # its last unit
                yield
            solo = seen >= k - 1 if solo_off_by_one else seen == k
            if solo:
                merge(item, first, last, cta, True)
                continue
            written.add((item, cta))                        # the partial, then the count
            yield
            if not final:
                queue.append((item, first, last))
            else:
                if fetch_add(item) == k:
                    merge(item, first, last, cta, False)
        queue.append(None)

    def helper_actor(cta, queue):
        while True:
            while not queue:
                yield
            entry = queue.pop(0)
            if entry is None:
                return
            item, first, last = entry
            yield
            if fetch_add(item) == last - first:
                merge(item, first, last, cta, False)

    actors = []
    for cta, pieces in enumerate(per_cta):
        q = []
        actors.append(cta_actor(cta, pieces, q))
        actors.append(helper_actor(cta, q))
    while actors:
        a = rng.choice(actors)
        try:
            next(a)
        except StopIteration:
            actors.remove(a)
    for item in pieces_of_item:
        if merged.get(item, 0) != 1:
            raise Violation(f"item {item} merged {merged.get(item, 0)} times")
    if any(v != 0 for v in counters.values()):
        raise Violation("a counter is not back at zero for the next launch")


@pytest.mark.parametrize("seed", range(8))
def test_every_split_item_is_merged_once_and_counters_reset(seed):
    rng = random.Random(100 + seed)
    for _ in range(120):
        lens, ips, w, G, mc, L = random_case(rng)
        per_cta, _, _ = pieces_of(lens, ips, w, G, mc, L)
        for _ in range(3):
            run_merges(per_cta, rng)


@pytest.mark.parametrize("bug", ["forget_reset", "solo_off_by_one"])
def test_planted_merge_mistakes_are_caught(bug):
    rng = random.Random(7)
    caught = 0
    for _ in range(200):
        lens, ips, w, G, mc, L = random_case(rng)
        per_cta, _, _ = pieces_of(lens, ips, w, G, mc, L)
        try:
            run_merges(per_cta, rng, **{bug: True})
        except Violation:
            caught += 1
    assert caught > 0
