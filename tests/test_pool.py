"""Host block pool (C++ in libpagedkv.so) against the page's rules and the oracle's pool model."""
import random

import pytest
import torch


def test_alloc_free_incref_basics(pkv):
    p = pkv.BlockPool(8)
    assert p.num_free() == 8 and p.num_blocks() == 8
    a = p.alloc(3)
    assert len(set(a)) == 3 and all(0 <= i < 8 for i in a)
    assert all(p.refcount(i) == 1 for i in a)
    p.incref(a[:2])
    assert [p.refcount(i) for i in a] == [2, 2, 1]
    p.free(a)
    assert [p.refcount(i) for i in a] == [1, 1, 0]
    assert p.num_free() == 6
    p.free(a[:2])
    assert p.num_free() == 8
    assert p.refcount(-1) == -1 and p.refcount(8) == -1


def test_oom_is_all_or_nothing(pkv):
    p = pkv.BlockPool(5)
    p.alloc(4)
    with pytest.raises(pkv.KVError) as e:
        p.alloc(2)
    assert e.value.status == pkv.KV_ERR_OOM
    assert p.num_free() == 1


def test_underflow_and_bad_ids_change_nothing(pkv):
    p = pkv.BlockPool(4)
    a = p.alloc(2)
    with pytest.raises(pkv.KVError) as e:
        p.free([a[0], a[0]])            # refcount 1, two drops requested
    assert e.value.status == pkv.KV_ERR_STATE
    assert p.refcount(a[0]) == 1
    with pytest.raises(pkv.KVError):
        p.free([a[1], 7])               # out of range id
    assert p.refcount(a[1]) == 1
    free_id = next(i for i in range(4) if p.refcount(i) == 0)
    with pytest.raises(pkv.KVError):
        p.incref([a[0], free_id])       # a free block cannot be shared
    assert p.refcount(a[0]) == 1


def test_random_ops_match_reference_model(pkv, oracle_mod):
    rng = random.Random(470)
    p, ref = pkv.BlockPool(64), oracle_mod.RefBlockPool(64)
    live = []
    for _ in range(3000):
        op = rng.random()
        if op < 0.4:
            n = rng.randint(0, 6)
            want_ok = ref.alloc(n) is not None
            try:
                ids = p.alloc(n)
                ok = True
            except pkv.KVError:
                ok = False
            assert ok == want_ok
            if ok:
                ref.take(ids)
                live += ids
        elif op < 0.6 and live:
            ids = rng.sample(live, min(len(live), rng.randint(1, 3)))
            ok_ref = ref.incref(ids)
            try:
                p.incref(ids)
                ok = True
            except pkv.KVError:
                ok = False
            assert ok == ok_ref
            if ok:
                live += ids
        elif live:
            k = rng.randint(1, 3)
            ids = [rng.choice(live) for _ in range(k)]
            if rng.random() < 0.1:
                ids.append(rng.randrange(64))        # sometimes a block that may be free
            ok_ref = ref.free(ids)
            try:
                p.free(ids)
                ok = True
            except pkv.KVError:
                ok = False
            assert ok == ok_ref
            if ok:
                for i in ids:
                    live.remove(i)
        assert p.num_free() == ref.num_free()
    assert all(p.refcount(i) == ref.refcount[i] for i in range(64))
    # conservation: the sum of refcounts equals the live table references
    assert sum(p.refcount(i) for i in range(64)) == len(live)


def _grow(pkv, p, lens0, W, steps):
    B = len(lens0)
    tables = torch.full((B, W), -1, dtype=torch.int32)
    lens = torch.zeros(B, dtype=torch.int32)
    slots = torch.zeros(B, dtype=torch.int64)
    for _ in range(steps):
        p.append_slots(tables, lens, slots)
    return tables, lens, slots


def test_append_slots_waste_invariant(pkv, oracle_mod):
    # "unused space is at most one partly filled block per request" (Module 23: Serving, Exercise (extend))
    p = pkv.BlockPool(200)
    B, W = 5, 12
    tables = torch.full((B, W), -1, dtype=torch.int32)
    lens = torch.zeros(B, dtype=torch.int32)
    slots = torch.zeros(B, dtype=torch.int64)
    seen = set()
    for step in range(150):
        before = lens.clone()
        p.append_slots(tables, lens, slots)
        assert torch.equal(lens, before + 1)
        for b in range(B):
            c = int(lens[b])
            nb = oracle_mod.blocks_needed(c)
            assert (tables[b, :nb] >= 0).all() and (tables[b, nb:] == -1).all()
            pos = c - 1
            assert int(slots[b]) == int(tables[b, pos // 16]) * 16 + pos % 16
            assert int(slots[b]) not in seen
            seen.add(int(slots[b]))
        assert p.num_free() == 200 - sum(oracle_mod.blocks_needed(int(c)) for c in lens)


def test_append_slots_errors_leave_state_unchanged(pkv):
    p = pkv.BlockPool(3)
    B, W = 2, 2
    tables = torch.full((B, W), -1, dtype=torch.int32)
    lens = torch.zeros(B, dtype=torch.int32)
    slots = torch.zeros(B, dtype=torch.int64)
    p.append_slots(tables, lens, slots)            # 2 blocks used
    lens[:] = 16                                   # both need a new block, only 1 free
    t0, l0 = tables.clone(), lens.clone()
    with pytest.raises(pkv.KVError) as e:
        p.append_slots(tables, lens, slots)
    assert e.value.status == pkv.KV_ERR_OOM
    assert torch.equal(tables, t0) and torch.equal(lens, l0) and p.num_free() == 1
    lens[:] = 32                                   # would exceed W = 2 blocks
    with pytest.raises(pkv.KVError) as e:
        p.append_slots(tables, lens, slots)
    assert e.value.status == pkv.KV_ERR_ARG


def test_append_into_shared_block_is_refused(pkv):
    p = pkv.BlockPool(4)
    tables = torch.full((2, 2), -1, dtype=torch.int32)
    blk = p.alloc(1)[0]
    p.incref([blk])                                # two sequences share a partly filled block
    tables[:, 0] = blk
    lens = torch.tensor([5, 5], dtype=torch.int32)
    slots = torch.zeros(2, dtype=torch.int64)
    with pytest.raises(pkv.KVError) as e:
        p.append_slots(tables, lens, slots)
    assert e.value.status == pkv.KV_ERR_STATE
    assert lens.tolist() == [5, 5]


def test_reservation_admits_four_paging_admits_eight(pkv):
    """96 blocks, 8 requests: reserving each maximum admits 4, paging runs all 8
    ("Module 23: Serving", 23.4, figure paged-attention). The maximum per request
    is read as 96 / 4 = 24 blocks (384 tokens); final lengths are drawn below it."""
    rng = random.Random(195)
    final = [rng.randint(40, 180) for _ in range(8)]
    assert sum(-(-c // 16) for c in final) <= 96
    # reservation: each request takes its maximum (24 blocks) up front
    p = pkv.BlockPool(96)
    admitted = 0
    for _ in range(8):
        try:
            p.alloc(24)
            admitted += 1
        except pkv.KVError:
            break
    assert admitted == 4
    # paging: blocks are handed out token by token as each request grows
    p = pkv.BlockPool(96)
    W = 24
    tables = torch.full((8, W), -1, dtype=torch.int32)
    lens = torch.zeros(8, dtype=torch.int32)
    slots = torch.zeros(8, dtype=torch.int64)
    done = [False] * 8
    while not all(done):
        active = [b for b in range(8) if not done[b]]
        sub_t = tables[active].clone()
        sub_l = lens[active].clone()
        sub_s = torch.zeros(len(active), dtype=torch.int64)
        p.append_slots(sub_t, sub_l, sub_s)
        tables[active], lens[active] = sub_t, sub_l
        for b in active:
            done[b] = int(lens[b]) >= final[b]
    assert lens.tolist() == final
    assert 96 - p.num_free() == sum(-(-c // 16) for c in final)


def test_continuous_batch_redraw_keeps_refcounts(pkv):
    """The 70B-style mix: half the sequences share a 64-block prefix; 10% are re-drawn each step."""
    from paged_kv_cache_470_b200 import workloads
    from paged_kv_cache_470_b200.batch import ContinuousBatch
    cfg = workloads.small_config(5, batch=40)
    layout = workloads.draw_layout(cfg)
    cb = ContinuousBatch(cfg, int(layout.num_blocks * 1.3))
    cb.check()
    assert len(cb.prefix) == 64
    assert all(cb.pool.refcount(i) == 1 + int(cb.shares.sum()) for i in cb.prefix)
    for _ in range(10):
        rows = cb.redraw()
        assert len(rows) == 4
        cb.check()
        for b in range(cfg.batch):
            c = int(cb.context_lens[b])
            assert 1 <= c <= cfg.W * 16
            if cb.shares[b]:
                assert c >= 1025 and cb.block_tables[b, :64].tolist() == cb.prefix
        slots = cb.slot_mapping()
        assert len(set(slots.tolist())) == cfg.batch        # every new token has its own slot
        for b in range(cfg.batch):                          # ... in a block no other sequence uses
            assert cb.pool.refcount(int(slots[b]) // 16) == 1


# ---------------------------------------------------------------------------
# fork and copy-on-write ("Designing an LLM serving system", section "Paged attention")
# ---------------------------------------------------------------------------
def test_fork_shares_every_block(pkv):
    p = pkv.BlockPool(6)
    parent = p.alloc(3)
    child = p.fork(parent)
    assert child == parent and all(p.refcount(i) == 2 for i in parent)
    free_id = next(i for i in range(6) if p.refcount(i) == 0)
    with pytest.raises(pkv.KVError) as e:
        p.fork([parent[0], free_id])               # a free block cannot be forked
    assert e.value.status == pkv.KV_ERR_STATE
    assert all(p.refcount(i) == 2 for i in parent)
    assert p.fork([]) == []


def test_copy_on_write_keeps_every_sequence_view(pkv, oracle_mod):
    from cow_cases import ForkScenario, OracleBackend
    for seed in (0, 1, 2):
        sc = ForkScenario(pkv, seed=seed)
        sc.run(oracle_mod, OracleBackend(oracle_mod, sc), n_random_steps=60)
        assert sc.copies_total >= 3


def test_copy_on_write_without_sharing_matches_append_slots(pkv):
    """With no shared tail, the copy-on-write variant does exactly what append_slots does."""
    a, b = pkv.BlockPool(40), pkv.BlockPool(40)
    B, W = 4, 8
    ta, tb = torch.full((B, W), -1, dtype=torch.int32), torch.full((B, W), -1, dtype=torch.int32)
    la, lb = torch.zeros(B, dtype=torch.int32), torch.zeros(B, dtype=torch.int32)
    sa, sb = torch.zeros(B, dtype=torch.int64), torch.zeros(B, dtype=torch.int64)
    for _ in range(70):
        a.append_slots(ta, la, sa)
        src, dst = b.append_slots_cow(tb, lb, sb)
        assert src == [] and dst == []
        assert torch.equal(ta, tb) and torch.equal(la, lb) and torch.equal(sa, sb)


def test_copy_on_write_errors_leave_state_unchanged(pkv):
    p = pkv.BlockPool(3)
    tables = torch.full((3, 2), -1, dtype=torch.int32)
    blk = p.alloc(1)[0]
    p.fork([blk])
    p.fork([blk])                                  # three sequences on one 5-token block
    tables[:, 0] = blk
    p.alloc(1)                                     # one block left free
    lens = torch.tensor([5, 5, 5], dtype=torch.int32)
    slots = torch.zeros(3, dtype=torch.int64)
    t0, l0 = tables.clone(), lens.clone()
    with pytest.raises(pkv.KVError) as e:          # all three append: two copies, one free block
        p.append_slots_cow(tables, lens, slots)
    assert e.value.status == pkv.KV_ERR_OOM
    assert torch.equal(tables, t0) and torch.equal(lens, l0)
    assert p.refcount(blk) == 3 and p.num_free() == 1
    sub_t, sub_l, sub_s = tables[:2].clone(), lens[:2].clone(), slots[:2].clone()
    with pytest.raises(pkv.KVError):               # two of three append: still two copies
        p.append_slots_cow(sub_t, sub_l, sub_s)
    assert p.refcount(blk) == 3 and p.num_free() == 1
    sub_t, sub_l, sub_s = tables[:1].clone(), lens[:1].clone(), slots[:1].clone()
    src, dst = p.append_slots_cow(sub_t, sub_l, sub_s)   # one appends: one copy
    assert src == [blk] and dst == [int(sub_t[0, 0])] and dst[0] != blk
    assert int(sub_s[0]) == dst[0] * 16 + 5 and int(sub_l[0]) == 6
    assert p.refcount(blk) == 2 and p.refcount(dst[0]) == 1 and p.num_free() == 0
    p.free([dst[0]])
    bad = tables[:1].clone()
    bad[0, 0] = dst[0]                              # a free block as the tail
    with pytest.raises(pkv.KVError) as e:
        p.append_slots_cow(bad, lens[:1].clone(), slots[:1].clone())
    assert e.value.status == pkv.KV_ERR_STATE and p.num_free() == 1


# ---------------------------------------------------------------------------
# chunked-prefill layouts (host side of the prefill workloads)
# ---------------------------------------------------------------------------
def test_prefill_layout_places_each_chunk_at_the_end_of_its_context(oracle_mod):
    from paged_kv_cache_470_b200 import workloads
    cfg = workloads.PrefillConfig("t", 8, 2, 64, 5, 0, 0, 0, 16)
    chunk, prior = [37, 1, 16, 0, 40], [0, 250, 15, 33, 7]
    lay = workloads.draw_prefill_layout(cfg, chunk_lens=chunk, prior_lens=prior, seed=9)
    assert lay.context_lens.tolist() == [c + p for c, p in zip(chunk, prior)]
    assert lay.query_start.tolist() == [0, 37, 38, 54, 54, 94]
    slots = lay.slot_mapping().tolist()
    assert len(slots) == sum(chunk) and len(set(slots)) == len(slots)
    k = 0
    for b in range(5):
        c = int(lay.context_lens[b])
        nblk = oracle_mod.blocks_needed(c)
        row = lay.block_tables[b]
        assert (row[:nblk] >= 0).all() and (row[nblk:] == -1).all()
        for pos in range(c - chunk[b], c):      # the chunk is the last chunk[b] positions
            assert slots[k] == int(row[pos // 16]) * 16 + pos % 16
            k += 1
    used = [int(x) for x in lay.block_tables.flatten().tolist() if x >= 0]
    assert len(set(used)) == len(used) and max(used) < lay.num_blocks
