"""Pins for the float64 oracle, checked against what the pages and mathematics fix.

None of these compares the oracle with itself: each check uses a closed form,
a value printed on the pages, a library routine on unpaged data, an invariant
or a brute-force restatement, chosen so that a plausible mistake in the oracle
(wrong kv-head map, swapped block/offset, dropped scale, wrong softmax shift,
V gathered from K, over-read past the context) fails at least one of them.
The last test plants such mistakes in a copy of the oracle and checks that the
pins catch every one.
"""
import ctypes
import json
import math
import os
import subprocess

import numpy as np
import pytest
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_cache_sizes.json")
NAN_BF16 = np.uint16(0x7FC0)


# ---------------------------------------------------------------------------
# helpers: dense data, and the test's own placement of it into a paged pool
# ---------------------------------------------------------------------------
def bf16_round(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def make_dense_case(seed, lens, Hq, Hkv, D, scale_data=1.0):
    g = torch.Generator().manual_seed(seed)
    q = bf16_round(torch.randn(len(lens), Hq, D, generator=g) * scale_data)
    K = [bf16_round(torch.randn(c, Hkv, D, generator=g) * scale_data) for c in lens]
    V = [bf16_round(torch.randn(c, Hkv, D, generator=g)) for c in lens]
    return q, K, V


def paginate(K, V, lens, Hkv, D, num_blocks, W, seed, fill=NAN_BF16):
    """Place token t of sequence b at pool[ids_b[t // 16], t % 16]; every other row holds `fill`."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(num_blocks)
    kpool = np.full((num_blocks, 16, Hkv, D), fill, dtype=np.uint16)
    vpool = np.full((num_blocks, 16, Hkv, D), fill, dtype=np.uint16)
    tables = np.full((len(lens), W), -1, dtype=np.int32)
    cur = 0
    for b, c in enumerate(lens):
        nb = -(-c // 16)
        ids = perm[cur:cur + nb]
        cur += nb
        tables[b, :nb] = ids
        kb, vb = bits(K[b]), bits(V[b])
        for t in range(c):
            kpool[ids[t // 16], t % 16] = kb[t]
            vpool[ids[t // 16], t % 16] = vb[t]
    return kpool, vpool, tables


def dense_reference(q, K, V, lens, Hq, Hkv, scale):
    """torch SDPA in float64 on unpaged K/V, kv head h // (Hq // Hkv) via repeat_interleave."""
    g = Hq // Hkv
    outs = []
    for b, c in enumerate(lens):
        if c == 0:
            outs.append(torch.zeros(Hq, q.shape[-1], dtype=torch.float64))
            continue
        qb = q[b].to(torch.float64)[:, None, :]                              # [Hq, 1, D]
        kb = K[b].to(torch.float64).permute(1, 0, 2).repeat_interleave(g, 0)  # [Hq, c, D]
        vb = V[b].to(torch.float64).permute(1, 0, 2).repeat_interleave(g, 0)
        outs.append(F.scaled_dot_product_attention(qb, kb, vb, scale=scale)[:, 0, :])
    return torch.stack(outs).numpy()


TINY_LENS = [1, 15, 16, 17, 33, 40, 2, 32]


def run_tiny(oracle_mod, lens=TINY_LENS, Hq=4, Hkv=2, D=8, seed=0, scale=None, num_blocks=None, W=3):
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    q, K, V = make_dense_case(seed, lens, Hq, Hkv, D)
    nb = num_blocks or sum(-(-c // 16) for c in lens) + 5
    kp, vp, tab = paginate(K, V, lens, Hkv, D, nb, W, seed + 1)
    out, wsum = oracle_mod.paged_attention_decode(bits(q), kp, vp, tab, np.array(lens, np.int32), scale,
                                                  return_weight_sums=True)
    return q, K, V, kp, vp, tab, out, wsum, scale


# ---------------------------------------------------------------------------
# closed form and the pages' printed values
# ---------------------------------------------------------------------------
def test_closed_form_matches_printed_values(oracle_mod):
    spec = json.load(open(GOLDEN))
    units = {"B": 1, "KiB": 1024, "MB": 1e6, "GB": 1e9, "GiB": 2 ** 30}
    for e in spec["entries"]:
        got = oracle_mod.kv_cache_bytes(e["n_layers"], e["n_kv_heads"], e["d_head"], e["L"], e["B"], e["n_bytes"])
        want = e["printed"] * units[e["unit"]]
        if e["rounding"] == "exact":
            assert got == want, e["what"]
        elif e["rounding"] == "1 decimal":
            assert round(got / units[e["unit"]], 1) == e["printed"], e["what"]
        elif e["rounding"].startswith("about (within 1 MB)"):
            assert abs(got - want) <= 1e6, e["what"]
        else:
            assert abs(got - want) <= 0.05 * want, e["what"]


def test_closed_form_figure_points(oracle_mod):
    fig = json.load(open(GOLDEN))["figure"]
    for heads, tokens, gb in fig["points"]:
        got = oracle_mod.kv_cache_bytes(fig["n_layers"], heads, fig["d_head"], tokens, 1, fig["n_bytes"])
        assert round(got / 1e9, 2) == pytest.approx(gb, abs=1e-9), (heads, tokens)


def test_closed_form_each_factor_is_linear(oracle_mod):
    # "doubling any one factor doubles the total" (Module 23: Serving, 23.1, kv-cache-calculator)
    base = (32, 8, 128, 8192, 1, 2)
    b0 = oracle_mod.kv_cache_bytes(*base)
    for i in range(6):
        args = list(base)
        args[i] *= 2
        assert oracle_mod.kv_cache_bytes(*args) == 2 * b0


# ---------------------------------------------------------------------------
# attention against an unpaged library routine
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("Hq,Hkv,D", [(4, 2, 8), (4, 4, 8), (6, 1, 16), (8, 2, 64)])
def test_matches_dense_sdpa(oracle_mod, Hq, Hkv, D):
    q, K, V, kp, vp, tab, out, _, scale = run_tiny(oracle_mod, Hq=Hq, Hkv=Hkv, D=D, seed=Hq * 7 + D)
    ref = dense_reference(q, K, V, TINY_LENS, Hq, Hkv, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_matches_dense_sdpa_with_other_scale(oracle_mod):
    q, K, V, kp, vp, tab, out, _, scale = run_tiny(oracle_mod, scale=0.37, seed=11)
    np.testing.assert_allclose(out, dense_reference(q, K, V, TINY_LENS, 4, 2, 0.37), rtol=1e-12, atol=1e-12)


def test_softmax_weights_sum_to_one(oracle_mod):
    *_, out, wsum, _ = run_tiny(oracle_mod, seed=3)
    np.testing.assert_allclose(wsum, 1.0, atol=1e-12)


def test_permuting_physical_blocks_is_bit_identical(oracle_mod):
    q, K, V, kp, vp, tab, out, _, scale = run_tiny(oracle_mod, seed=5)
    nb = kp.shape[0]
    perm = np.random.default_rng(9).permutation(nb)
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp                # block i moves to perm[i]
    tab2 = np.where(tab >= 0, perm[np.maximum(tab, 0)], -1).astype(np.int32)
    out2 = oracle_mod.paged_attention_decode(bits(q), kp2, vp2, tab2, np.array(TINY_LENS, np.int32), scale)
    assert np.array_equal(out, out2)


# ---------------------------------------------------------------------------
# special cases with exact answers
# ---------------------------------------------------------------------------
def test_single_token_returns_v_exactly(oracle_mod):
    q, K, V, kp, vp, tab, out, _, _ = run_tiny(oracle_mod, lens=[1, 1, 1], seed=21)
    for b in range(3):
        for h in range(4):
            assert np.array_equal(out[b, h], V[b][0, h // 2].to(torch.float64).numpy())


def test_zero_query_averages_v(oracle_mod):
    lens = [5, 16, 37]
    q, K, V = make_dense_case(4, lens, 4, 2, 8)
    q = torch.zeros_like(q)
    kp, vp, tab = paginate(K, V, lens, 2, 8, 10, 3, 4)
    out = oracle_mod.paged_attention_decode(bits(q), kp, vp, tab, np.array(lens, np.int32), 0.3)
    for b, c in enumerate(lens):
        for h in range(4):
            np.testing.assert_allclose(out[b, h], V[b][:, h // 2].to(torch.float64).mean(0).numpy(), atol=1e-12)


def test_constant_v_rows_return_that_row(oracle_mod):
    lens = [9, 30]
    q, K, V = make_dense_case(6, lens, 4, 2, 8)
    row = bf16_round(torch.randn(2, 8, generator=torch.Generator().manual_seed(1)))
    V = [row.expand(c, 2, 8).clone() for c in lens]
    kp, vp, tab = paginate(K, V, lens, 2, 8, 8, 2, 6)
    out = oracle_mod.paged_attention_decode(bits(q), kp, vp, tab, np.array(lens, np.int32), 0.35)
    for b in range(2):
        for h in range(4):
            np.testing.assert_allclose(out[b, h], row[h // 2].to(torch.float64).numpy(), atol=1e-12)


def test_duplicated_keys_give_uniform_weights(oracle_mod):
    lens = [23]
    q, K, V = make_dense_case(8, lens, 4, 2, 8)
    K = [K[0][:1].expand(23, 2, 8).clone()]
    kp, vp, tab = paginate(K, V, lens, 2, 8, 4, 2, 8)
    out = oracle_mod.paged_attention_decode(bits(q), kp, vp, tab, np.array(lens, np.int32), 0.35)
    for h in range(4):
        np.testing.assert_allclose(out[0, h], V[0][:, h // 2].to(torch.float64).mean(0).numpy(), atol=1e-12)


def test_brute_force_without_max_shift(oracle_mod):
    lens = [3, 11, 20]
    q, K, V, kp, vp, tab, out, _, scale = run_tiny(oracle_mod, lens=lens, seed=13, W=2)
    for b, c in enumerate(lens):
        for h in range(4):
            qh = q[b, h].to(torch.float64).numpy()
            z = np.array([scale * sum(qh[d] * float(K[b][t, h // 2, d]) for d in range(8)) for t in range(c)])
            e = np.exp(z)
            ref = sum((e[t] / e.sum()) * V[b][t, h // 2].to(torch.float64).numpy() for t in range(c))
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-12, atol=1e-12)


def test_large_logits_stay_finite_and_pick_the_argmax(oracle_mod):
    # scale 1e4 pushes exp(z) far past float64 range without the max shift
    lens = [19]
    q, K, V, kp, vp, tab, out, _, scale = run_tiny(oracle_mod, lens=lens, seed=17, scale=1e4, W=2)
    assert np.isfinite(out).all()
    for h in range(4):
        z = (K[0][:, h // 2].to(torch.float64) @ q[0, h].to(torch.float64))
        np.testing.assert_allclose(out[0, h], V[0][int(torch.argmax(z)), h // 2].to(torch.float64).numpy(),
                                   atol=1e-9)


def test_empty_context_gives_zeros_and_reads_nothing(oracle_mod):
    lens = [0, 7]
    q, K, V = make_dense_case(2, lens, 4, 2, 8)
    kp, vp, tab = paginate(K, V, lens, 2, 8, 3, 2, 2)
    tab[0, :] = 123456  # never read for an empty sequence
    out = oracle_mod.paged_attention_decode(bits(q), kp, vp, tab, np.array(lens, np.int32), 0.35)
    assert np.array_equal(out[0], np.zeros((4, 8)))
    assert np.isfinite(out[1]).all()


def test_rejects_bad_block_ids_and_lengths(oracle_mod):
    q, K, V, kp, vp, tab, *_ = run_tiny(oracle_mod, lens=[20], seed=1, W=2)
    bad = tab.copy()
    bad[0, 1] = kp.shape[0]
    with pytest.raises(ValueError):
        oracle_mod.paged_attention_decode(bits(q), kp, vp, bad, np.array([20], np.int32), 0.3)
    with pytest.raises(ValueError):
        oracle_mod.paged_attention_decode(bits(q), kp, vp, tab, np.array([33], np.int32), 0.3)


# ---------------------------------------------------------------------------
# append oracle
# ---------------------------------------------------------------------------
def test_append_writes_exactly_the_targeted_rows(oracle_mod):
    rng = np.random.default_rng(0)
    nb, Hkv, D, T = 6, 3, 8, 7
    kc = rng.integers(0, 2 ** 16, size=(nb, 16, Hkv, D), dtype=np.uint16)
    vc = rng.integers(0, 2 ** 16, size=(nb, 16, Hkv, D), dtype=np.uint16)
    kn = rng.integers(0, 2 ** 16, size=(T, Hkv, D), dtype=np.uint16)
    vn = rng.integers(0, 2 ** 16, size=(T, Hkv, D), dtype=np.uint16)
    slots = np.array([5, -1, 17, 95, 0, -7, 48], dtype=np.int64)
    k2, v2 = oracle_mod.kv_cache_append(kc, vc, kn, vn, slots)
    # expected: the flat [nb*16] row view written at the non-negative slots
    ek, ev = kc.reshape(nb * 16, Hkv, D).copy(), vc.reshape(nb * 16, Hkv, D).copy()
    for i, s in enumerate(slots):
        if s >= 0:
            ek[s], ev[s] = kn[i], vn[i]
    assert np.array_equal(k2.reshape(nb * 16, Hkv, D), ek)
    assert np.array_equal(v2.reshape(nb * 16, Hkv, D), ev)
    untouched = np.setdiff1d(np.arange(nb * 16), slots[slots >= 0])
    assert np.array_equal(k2.reshape(nb * 16, Hkv, D)[untouched], kc.reshape(nb * 16, Hkv, D)[untouched])


def test_append_rejects_slot_past_the_pool(oracle_mod):
    z = np.zeros((2, 16, 1, 8), np.uint16)
    n = np.zeros((1, 1, 8), np.uint16)
    with pytest.raises(ValueError):
        oracle_mod.kv_cache_append(z, z, n, n, np.array([32], np.int64))


def test_append_then_attend_sees_the_new_token(oracle_mod):
    # context length counts the appended token: a 1-token sequence attends only to it
    nb, Hkv, D = 4, 2, 8
    kc = np.full((nb, 16, Hkv, D), NAN_BF16, np.uint16)
    vc = np.full((nb, 16, Hkv, D), NAN_BF16, np.uint16)
    kn = bits(bf16_round(torch.randn(1, Hkv, D)))
    vn = bits(bf16_round(torch.randn(1, Hkv, D)))
    k2, v2 = oracle_mod.kv_cache_append(kc, vc, kn, vn, np.array([2 * 16], np.int64))
    q = bits(bf16_round(torch.randn(1, 4, D)))
    out = oracle_mod.paged_attention_decode(q, k2, v2, np.array([[2]], np.int32), np.array([1], np.int32), 0.35)
    for h in range(4):
        assert np.array_equal(out[0, h], oracle_mod.bf16_bits_to_float64(vn[0, h // 2]))


# ---------------------------------------------------------------------------
# block-pool model
# ---------------------------------------------------------------------------
def test_ref_pool_semantics(oracle_mod):
    p = oracle_mod.RefBlockPool(4)
    ids = p.alloc(3)
    p.take(ids)
    assert p.num_free() == 1
    assert p.alloc(2) is None                     # all or nothing
    assert p.incref(ids[:1]) and p.refcount[ids[0]] == 2
    assert p.free(ids[:1]) and p.refcount[ids[0]] == 1
    assert not p.free([ids[1], ids[1]])           # would go below zero: no change
    assert p.refcount[ids[1]] == 1
    assert p.free(ids) and p.num_free() == 4
    assert not p.incref([0])                      # free blocks cannot be shared
    assert [oracle_mod.blocks_needed(c) for c in (0, 1, 16, 17, 32)] == [0, 1, 1, 2, 2]


# ---------------------------------------------------------------------------
# fp16 inputs ("Module 23: Serving", section 23.1: 2 bytes per number, fp16 or bf16)
# ---------------------------------------------------------------------------
def test_widening_matches_libraries_for_every_code(oracle_mod):
    codes = np.arange(65536, dtype=np.uint16)
    for kind, ref in (("fp16", codes.view(np.float16).astype(np.float64)),
                      ("bf16", torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).double().numpy())):
        got = np.array([oracle_mod.widen(kind, c) for c in codes])
        same = (got == ref) | (np.isnan(got) & np.isnan(ref))
        assert same.all(), f"{kind}: first mismatch at code {int(np.argmin(same)):#06x}"
        assert (np.signbit(got) == np.signbit(ref))[~np.isnan(ref)].all()


def test_fp16_decode_matches_dense_attention(oracle_mod):
    lens, Hq, Hkv, D = TINY_LENS, 4, 2, 8
    g = torch.Generator().manual_seed(21)
    q = torch.randn(len(lens), Hq, D, generator=g).half()
    K = [torch.randn(c, Hkv, D, generator=g).half() for c in lens]
    V = [torch.randn(c, Hkv, D, generator=g).half() for c in lens]
    nb = sum(-(-c // 16) for c in lens) + 5
    kp, vp, tab = paginate(K, V, lens, Hkv, D, nb, 3, 22, fill=np.uint16(0x7E00))   # fp16 NaN filler
    scale = 1.0 / math.sqrt(D)
    out = oracle_mod.paged_attention_decode(q, kp, vp, tab, np.array(lens, np.int32), scale, dtype="fp16")
    ref = dense_reference(q, K, V, lens, Hq, Hkv, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    # the same bit patterns read as bf16 give a different answer: the dtype is honoured
    other = oracle_mod.paged_attention_decode(bits(q), kp, vp, tab, np.array(lens, np.int32), scale)
    assert not np.allclose(np.nan_to_num(other), ref)


# ---------------------------------------------------------------------------
# chunked prefill ("Module 23: Serving", 23.2; "Designing an LLM serving system",
# Scheduling: when prefill meets decode)
# ---------------------------------------------------------------------------
def dense_causal_reference(q, K, V, lens, nq, qs, Hq, Hkv, scale):
    """torch SDPA in float64 with an explicit boolean mask: query i of sequence b sees tokens < c - n + i + 1."""
    g = Hq // Hkv
    outs = []
    for b, c in enumerate(lens):
        n = nq[b]
        if n == 0:
            continue
        qb = q[qs[b]:qs[b + 1]].to(torch.float64).permute(1, 0, 2)
        kb = K[b].to(torch.float64).permute(1, 0, 2).repeat_interleave(g, 0)
        vb = V[b].to(torch.float64).permute(1, 0, 2).repeat_interleave(g, 0)
        mask = torch.zeros(n, c, dtype=torch.bool)
        for i in range(n):
            mask[i, :c - n + i + 1] = True
        outs.append(F.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask, scale=scale).permute(1, 0, 2))
    return torch.cat(outs).numpy()


@pytest.mark.parametrize("Hq,Hkv,D", [(4, 2, 8), (6, 6, 16), (8, 1, 8)])
def test_prefill_matches_dense_causal_attention(oracle_mod, Hq, Hkv, D):
    lens = [5, 20, 33, 16, 40]
    nq = [5, 7, 1, 0, 40]            # whole prompts, a chunk, one token (a decode step), none, whole
    g = torch.Generator().manual_seed(Hq * 100 + D)
    K = [bf16_round(torch.randn(c, Hkv, D, generator=g)) for c in lens]
    V = [bf16_round(torch.randn(c, Hkv, D, generator=g)) for c in lens]
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    q = bf16_round(torch.randn(int(qs[-1]), Hq, D, generator=g))
    nb = sum(-(-c // 16) for c in lens) + 4
    kp, vp, tab = paginate(K, V, lens, Hkv, D, nb, 3, 5)
    scale = 1.0 / math.sqrt(D)
    out = oracle_mod.paged_attention_prefill(bits(q), kp, vp, tab, np.array(lens, np.int32), qs, scale)
    ref = dense_causal_reference(q, K, V, lens, nq, qs, Hq, Hkv, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    # the last query of a chunk sees the whole context: it equals the decode step at that length
    dec = oracle_mod.paged_attention_decode(bits(q[qs[2] - 1:qs[2]]), kp, vp, tab[1:2], np.array([20], np.int32), scale)
    np.testing.assert_array_equal(out[qs[2] - 1], dec[0])


def test_prefill_rejects_bad_chunks(oracle_mod):
    lens = [4]
    kp = np.zeros((2, 16, 1, 8), np.uint16)
    tab = np.array([[0, 1]], np.int32)
    with pytest.raises(ValueError):   # a chunk longer than its context
        oracle_mod.paged_attention_prefill(np.zeros((5, 1, 8), np.uint16), kp, kp, tab, np.array(lens, np.int32),
                                           np.array([0, 5]), 1.0)
    with pytest.raises(ValueError):   # offsets that do not cover q
        oracle_mod.paged_attention_prefill(np.zeros((3, 1, 8), np.uint16), kp, kp, tab, np.array(lens, np.int32),
                                           np.array([0, 2]), 1.0)


# ---------------------------------------------------------------------------
# reading through the table, and whole-block moves
# ---------------------------------------------------------------------------
def test_sequence_tokens_recovers_the_dense_sequence(oracle_mod):
    """paginate() places each dense sequence in shuffled blocks with its own loop; reading
    back through the table gives the dense rows, and never a filler row."""
    lens = [1, 15, 16, 17, 40]
    q, K, V = make_dense_case(5, lens, 4, 2, 8)
    kp, vp, tab = paginate(K, V, lens, 2, 8, 20, 3, 6)
    for b, c in enumerate(lens):
        np.testing.assert_array_equal(oracle_mod.sequence_tokens(kp, tab[b], c), bits(K[b]))
        np.testing.assert_array_equal(oracle_mod.sequence_tokens(vp, tab[b], c), bits(V[b]))


def test_block_moves(oracle_mod):
    rng = np.random.default_rng(7)
    cache = rng.integers(0, 2 ** 16, size=(12, 16, 2, 8), dtype=np.uint16)
    src, dst = [3, 3, 9], [0, 5, 11]
    out = oracle_mod.copy_blocks(cache, src, dst)
    for s_, d_ in zip(src, dst):
        np.testing.assert_array_equal(out[d_], cache[s_])
    untouched = [i for i in range(12) if i not in dst]
    np.testing.assert_array_equal(out[untouched], cache[untouched])
    # a swap: every source read before any write
    sw = oracle_mod.copy_blocks(cache, [1, 2], [2, 1])
    np.testing.assert_array_equal(sw[1], cache[2])
    np.testing.assert_array_equal(sw[2], cache[1])
    # gather then scatter into other blocks moves the rows; gathering those gives them back
    ids, new_ids = [7, 2, 10], [4, 8, 6]
    packed = oracle_mod.gather_blocks(cache, ids)
    assert packed.shape == (3, 16, 2, 8)
    for k, i in enumerate(ids):
        assert int(packed[k].astype(np.uint64).sum()) == int(cache[i].astype(np.uint64).sum())
    back = oracle_mod.scatter_blocks(np.zeros_like(cache), packed, new_ids)
    np.testing.assert_array_equal(oracle_mod.gather_blocks(back, new_ids), packed)
    assert not back[[i for i in range(12) if i not in new_ids]].any()
    assert oracle_mod.gather_blocks(cache, []).shape == (0, 16, 2, 8)


# ---------------------------------------------------------------------------
# the pins catch planted mistakes
# ---------------------------------------------------------------------------
MUTANTS = {
    "head map h % group": ("const int j = h / group;", "const int j = h % group;"),
    "block and offset swapped": ("block_tables[(size_t)b * W + t / ORACLE_BLOCK_TOKENS]",
                                 "block_tables[(size_t)b * W + t % ORACLE_BLOCK_TOKENS]"),
    "scale dropped": ("z[t] = scale * dot;", "z[t] = dot;"),
    "shift sign flipped": ("z[t] = exp(z[t] - zmax);", "z[t] = exp(z[t] + zmax - 2.0 * zmax * (t == 0));"),
    "V gathered from K": ("const uint16_t *vt = v_cache +", "const uint16_t *vt = k_cache +"),
    "reads one token too many": ("for (int t = 0; t < c; ++t) {\n            const double w",
                                 "for (int t = 0; t <= c && t < 16 * W; ++t) {\n            const double w"),
}


MUTANT_RUNNER = r"""
import ctypes, math, sys
import numpy as np
sys.path.insert(0, sys.argv[2])
from test_oracle import make_dense_case, paginate, bits, dense_reference
lib = ctypes.CDLL(sys.argv[1])
P, I = ctypes.c_void_p, ctypes.c_int
lib.oracle_paged_attention_decode.argtypes = [P, P, P, P, P, P, I, P, I, I, I, I, I, ctypes.c_double]
lib.oracle_paged_attention_decode.restype = I
lens = [1, 15, 16, 17, 33, 40]
Hq, Hkv, D = 4, 2, 8
q, K, V = make_dense_case(99, lens, Hq, Hkv, D)
kp, vp, tab = paginate(K, V, lens, Hkv, D, 16, 3, 98)
qb = bits(q)
lens_a = np.array(lens, np.int32)
out = np.zeros((len(lens), Hq, D))
ws = np.zeros((len(lens), Hq))
ptr = lambda a: a.ctypes.data_as(P)
rc = lib.oracle_paged_attention_decode(ptr(out), ptr(ws), ptr(qb), ptr(kp), ptr(vp), ptr(tab), tab.shape[1],
                                       ptr(lens_a), len(lens), 16, Hq, Hkv, D, 1.0 / math.sqrt(D))
ref = dense_reference(q, K, V, lens, Hq, Hkv, 1.0 / math.sqrt(D))
agree = rc == 0 and np.allclose(out, ref, rtol=1e-12, atol=1e-12, equal_nan=False)
print("AGREE" if agree else "DIFFER")
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(oracle_mod, tmp_path, name):
    """Compile a mutated copy of the oracle and run the dense pin on it in a child process
    (a mutant that reads outside its arrays may crash, which also counts as caught)."""
    import sys
    src = open(os.path.join(os.path.dirname(oracle_mod.__file__), "pagedkv_oracle.c")).read()
    old, new = MUTANTS[name]
    assert old in src, f"mutation anchor not found for {name}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(path), "-lm"])
    runner = tmp_path / "run_mutant.py"
    runner.write_text(MUTANT_RUNNER)
    r = subprocess.run([sys.executable, str(runner), str(so), os.path.dirname(__file__)], capture_output=True,
                       text=True, timeout=300)
    caught = r.returncode != 0 or "DIFFER" in r.stdout
    assert "AGREE" in r.stdout or "DIFFER" in r.stdout or r.returncode != 0, r.stderr
    assert caught, f"the dense-attention pin missed the mutant '{name}'"
