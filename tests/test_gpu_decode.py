"""GPU parity: append (bit-exact) and decode attention (within 5e-3 + 1e-2|ref|) against the oracle.

Every call goes through the C ABI of libpagedkv.so via the ctypes binding.
"""
import random

import numpy as np
import pytest
import torch

from paged_kv_cache_470_b200 import workloads
from gpu_cases import Case, bf16_bits_np, compare, gpu_step, oracle_step

pytestmark = pytest.mark.gpu

PATHS = {"tensor_cores": 1, "cuda_cores": 2}


@pytest.fixture(autouse=True)
def _default_options(pkv):
    yield
    for key in (pkv.KV_OPT_COMPUTE, pkv.KV_OPT_COMBINE, pkv.KV_OPT_GRID, pkv.KV_OPT_MIN_CHUNK,
                pkv.KV_OPT_PRODUCER_LANES, pkv.KV_OPT_HEAD_GROUP, pkv.KV_OPT_ITEM_COST, pkv.KV_OPT_EARLY_LOADS):
        pkv.set_option(key, 0)


def run_and_check(pkv, oracle_mod, case, layers=None, what="", fused=None):
    """Every listed layer against the oracle; `fused` None alternates separate and fused append."""
    cfg = case.cfg
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    for n, layer in enumerate(range(case.n_layers) if layers is None else layers):
        host = case.host_inputs(layer)
        f = (n % 2 == 1) if fused is None else fused
        out = gpu_step(pkv, case, layer, ws, fused=f)
        torch.cuda.synchronize()
        k2, v2, ref = oracle_step(oracle_mod, case, layer, host)
        assert np.array_equal(bf16_bits_np(case.k[layer]), k2), f"{what} layer {layer}: K append not bit-exact"
        assert np.array_equal(bf16_bits_np(case.v[layer]), v2), f"{what} layer {layer}: V append not bit-exact"
        compare(out, ref, f"{what} layer {layer}{' (fused append)' if f else ''}")
    assert pkv.read_status(ws) == 0


# ---------------------------------------------------------------------------
# the tiny workload, every path and combine mode
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("combine", [0, 1])
def test_tiny_workload(pkv, oracle_mod, cuda_device, path, combine, fused):
    pkv.set_option(pkv.KV_OPT_COMPUTE, PATHS[path])
    pkv.set_option(pkv.KV_OPT_COMBINE, combine)
    case = Case(workloads.WORKLOADS[1], cuda_device)
    run_and_check(pkv, oracle_mod, case, what=f"tiny/{path}/combine{combine}", fused=fused)


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("D,Hq,Hkv", [(64, 20, 4), (128, 32, 8), (128, 8, 8), (64, 16, 2), (128, 64, 8),
                                      (128, 32, 2), (64, 12, 1), (64, 18, 6), (128, 7, 7), (128, 32, 32)])
def test_ragged_lengths_and_head_groups(pkv, oracle_mod, cuda_device, path, D, Hq, Hkv):
    """Lengths at and around block edges, the table's maximum, 1 and 0; groups 1..16."""
    pkv.set_option(pkv.KV_OPT_COMPUTE, PATHS[path])
    lens = [1, 15, 16, 17, 31, 32, 33, 255, 256, 0, 100, 2]
    cfg = workloads.small_config(1, Hq=Hq, Hkv=Hkv, D=D, batch=len(lens), pool_blocks=0, n_layers=2)
    case = Case(cfg, cuda_device, lens=lens, n_layers=2)
    run_and_check(pkv, oracle_mod, case, what=f"ragged D{D} {Hq}/{Hkv} {path}")


@pytest.mark.parametrize("cid", [2, 3])
@pytest.mark.parametrize("grid,min_chunk", [(1, 1), (3, 1), (7, 2), (296, 1), (0, 1)])
def test_many_split_pieces(pkv, oracle_mod, cuda_device, cid, grid, min_chunk):
    """Items cut into many split-K pieces; few CTAs, each wrapping its stage ring many times."""
    pkv.set_option(pkv.KV_OPT_GRID, grid)
    pkv.set_option(pkv.KV_OPT_MIN_CHUNK, min_chunk)
    cfg = workloads.small_config(cid, batch=6, ctx_lo=1, ctx_hi=1500, W=96, n_layers=1)
    case = Case(cfg, cuda_device)
    run_and_check(pkv, oracle_mod, case, what=f"config {cid} shape, grid {grid} min_chunk {min_chunk}")


@pytest.mark.parametrize("cost", [-1, 1, 7, 64])
@pytest.mark.parametrize("cid", [2, 5])
def test_item_cost_changes_only_the_split(pkv, oracle_mod, cuda_device, cid, cost):
    """Charging items more or less (so CTAs get different ranges) gives the same answers."""
    pkv.set_option(pkv.KV_OPT_ITEM_COST, cost)
    pkv.set_option(pkv.KV_OPT_GRID, 37)
    cfg = workloads.small_config(cid, batch=11, ctx_lo=1, ctx_hi=1200, W=80, n_layers=1, shared_fraction=0.0,
                                 lognormal_mean=600.0)
    case = Case(cfg, cuda_device)
    run_and_check(pkv, oracle_mod, case, what=f"config {cid} shape, item cost {cost}")


@pytest.mark.parametrize("early", [0, 1])
@pytest.mark.parametrize("grid", [0, 5])
@pytest.mark.parametrize("cid", [2, 3])
def test_back_to_back_layers(pkv, oracle_mod, cuda_device, cid, grid, early):
    """Fused launches of several layers back to back on one stream and one workspace, no
    synchronisation between them: each launch's prologue overlaps the previous launch. With early loads,
    each launch's first tiles are read while the previous layer's launch still runs (it writes only its own
    layer's cache, so the promise holds)."""
    pkv.set_option(pkv.KV_OPT_GRID, grid)
    pkv.set_option(pkv.KV_OPT_EARLY_LOADS, early)
    cfg = workloads.small_config(cid, batch=7, ctx_lo=1, ctx_hi=1300, W=96, n_layers=4)
    case = Case(cfg, cuda_device, n_layers=4)
    hosts = [case.host_inputs(layer) for layer in range(4)]
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    outs = [gpu_step(pkv, case, layer, ws, fused=True) for layer in range(4)]
    torch.cuda.synchronize()
    for layer in range(4):
        k2, v2, ref = oracle_step(oracle_mod, case, layer, hosts[layer])
        assert np.array_equal(bf16_bits_np(case.k[layer]), k2)
        compare(outs[layer], ref, f"back to back, config {cid} shape, layer {layer}")
    assert pkv.read_status(ws) == 0


@pytest.mark.parametrize("hg", [1, 2, 4])
def test_forced_head_groups(pkv, oracle_mod, cuda_device, hg):
    """Work units of 1, 2 or 4 kv heads give the same answers."""
    pkv.set_option(pkv.KV_OPT_HEAD_GROUP, hg)
    cfg = workloads.small_config(2, batch=9, ctx_lo=1, ctx_hi=900, W=64, n_layers=2)
    case = Case(cfg, cuda_device, n_layers=2)
    run_and_check(pkv, oracle_mod, case, what=f"{hg} kv heads per unit")


@pytest.mark.parametrize("lanes", [1, 2, 4, 8])
@pytest.mark.parametrize("Hkv", [1, 4])
def test_producer_lanes(pkv, oracle_mod, cuda_device, lanes, Hkv):
    """Tile loads issued from 1..8 producer lanes (units of 1 or 4 kv heads)."""
    pkv.set_option(pkv.KV_OPT_PRODUCER_LANES, lanes)
    cfg = workloads.small_config(2, Hq=4 * Hkv, Hkv=Hkv, batch=5, ctx_lo=1, ctx_hi=900, W=64, n_layers=1)
    case = Case(cfg, cuda_device)
    run_and_check(pkv, oracle_mod, case, what=f"{lanes} producer lanes, Hkv {Hkv}")


# ---------------------------------------------------------------------------
# exact special cases and invariances
# ---------------------------------------------------------------------------
def test_single_token_context_returns_v_exactly(pkv, oracle_mod, cuda_device):
    cfg = workloads.small_config(1, batch=8)
    case = Case(cfg, cuda_device, lens=[1] * 8)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    out = gpu_step(pkv, case, 0, ws)
    g = cfg.Hq // cfg.Hkv
    expect = case.v_new[0].repeat_interleave(g, dim=1)   # the only token is the appended one
    assert torch.equal(out, expect)


def test_empty_context_gives_zeros(pkv, cuda_device):
    cfg = workloads.small_config(1, batch=3)
    case = Case(cfg, cuda_device, lens=[0, 5, 0])
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    out = torch.full_like(case.q[0], 7.0)
    gpu_step(pkv, case, 0, ws, out)
    torch.cuda.synchronize()
    assert (out[0] == 0).all() and (out[2] == 0).all() and torch.isfinite(out[1].float()).all()


def test_physical_permutation_is_bit_identical(pkv, cuda_device):
    cfg = workloads.small_config(2, batch=16, n_layers=1)
    case = Case(cfg, cuda_device)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    out1 = gpu_step(pkv, case, 0, ws).clone()
    nb = case.layout.num_blocks
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(3)).to(cuda_device)
    k2, v2 = torch.empty_like(case.k[0]), torch.empty_like(case.v[0])
    k2[perm], v2[perm] = case.k[0], case.v[0]
    tables2 = torch.where(case.tables >= 0, perm[case.tables.clamp(min=0).long()].int(), case.tables)
    out2 = torch.empty_like(out1)
    pkv.paged_attention_decode(out2, case.q[0], k2, v2, tables2, case.lens, cfg.scale, ws)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)


def test_repeat_is_bit_identical(pkv, cuda_device):
    cfg = workloads.small_config(3, batch=8, n_layers=1)
    case = Case(cfg, cuda_device)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    out1 = gpu_step(pkv, case, 0, ws).clone()
    out2 = torch.empty_like(out1)
    for _ in range(3):
        pkv.paged_attention_decode(out2, case.q[0], case.k[0], case.v[0], case.tables, case.lens, cfg.scale, ws)
        torch.cuda.synchronize()
        assert torch.equal(out1, out2)


def test_bad_block_id_and_length_are_flagged_not_faulted(pkv, cuda_device):
    cfg = workloads.small_config(1, batch=4)
    case = Case(cfg, cuda_device, lens=[40, 40, 40, 40])
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    out = torch.empty_like(case.q[0])
    tables = case.tables.clone()
    tables[1, 1] = case.layout.num_blocks + 1000
    pkv.paged_attention_decode(out, case.q[0], case.k[0], case.v[0], tables, case.lens, cfg.scale, ws)
    assert pkv.read_status(ws) & pkv.KV_STATUS_BAD_BLOCK_ID
    lens = case.lens.clone()
    lens[2] = cfg.W * 16 + 5
    pkv.paged_attention_decode(out, case.q[0], case.k[0], case.v[0], case.tables, lens, cfg.scale, ws)
    assert pkv.read_status(ws) & pkv.KV_STATUS_BAD_CONTEXT
    # a clean call afterwards is clean
    pkv.paged_attention_decode(out, case.q[0], case.k[0], case.v[0], case.tables, case.lens, cfg.scale, ws)
    assert pkv.read_status(ws) == 0


def test_append_bit_exact_with_padding_and_bad_slots(pkv, oracle_mod, cuda_device):
    g = torch.Generator(device=cuda_device).manual_seed(5)
    nb, Hkv, D, T = 37, 8, 128, 50
    kc = torch.randn(nb, 16, Hkv, D, generator=g, device=cuda_device).to(torch.bfloat16)
    vc = torch.randn(nb, 16, Hkv, D, generator=g, device=cuda_device).to(torch.bfloat16)
    kn = torch.randn(T, Hkv, D, generator=g, device=cuda_device).to(torch.bfloat16)
    vn = torch.randn(T, Hkv, D, generator=g, device=cuda_device).to(torch.bfloat16)
    slots = torch.randperm(nb * 16, generator=torch.Generator().manual_seed(1))[:T].to(torch.int64)
    slots[::7] = -1
    k_host, v_host = kc.cpu(), vc.cpu()
    ek, ev = oracle_mod.kv_cache_append(k_host, v_host, kn.cpu(), vn.cpu(), slots.numpy())
    flag = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pkv.kv_cache_append(kn, vn, kc, vc, slots.to(cuda_device), flag)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits_np(kc), ek) and np.array_equal(bf16_bits_np(vc), ev)
    assert int(flag) == 0
    bad = slots.clone()
    bad[3] = nb * 16          # one past the pool: skipped and flagged
    before_k, before_v = kc.clone(), vc.clone()
    pkv.kv_cache_append(kn, vn, kc, vc, bad.to(cuda_device), flag)
    torch.cuda.synchronize()
    assert int(flag) & pkv.KV_STATUS_BAD_SLOT
    # the other rows were rewritten with the same bytes; nothing else changed
    assert torch.equal(kc, before_k) and torch.equal(vc, before_v)


# ---------------------------------------------------------------------------
# full-size workloads, in the launch configuration the bench times
# ---------------------------------------------------------------------------
def _full_size(pkv, oracle_mod, cuda_device, cid, n_alloc):
    cfg = workloads.WORKLOADS[cid]
    case = Case(cfg, cuda_device, n_layers=n_alloc)
    layers = sorted({0, n_alloc - 1, random.Random(cid).randrange(n_alloc)})
    run_and_check(pkv, oracle_mod, case, layers=layers, what=f"config {cid}")


def test_full_size_05b_gqa(pkv, oracle_mod, cuda_device):
    _full_size(pkv, oracle_mod, cuda_device, 2, 24)


def test_full_size_llama3_8b_shape(pkv, oracle_mod, cuda_device):
    _full_size(pkv, oracle_mod, cuda_device, 3, 3)


def test_full_size_llama2_7b_mha(pkv, oracle_mod, cuda_device):
    _full_size(pkv, oracle_mod, cuda_device, 4, 2)


def test_full_size_70b_mix_with_shared_prefix(pkv, oracle_mod, cuda_device):
    _full_size(pkv, oracle_mod, cuda_device, 5, 2)


def test_full_size_70b_mix_after_redraws(pkv, oracle_mod, cuda_device):
    """The 70B-style mix after two steps of re-drawing 10% of the batch through the block pool."""
    from paged_kv_cache_470_b200.batch import ContinuousBatch
    cfg = workloads.WORKLOADS[5]
    cb = ContinuousBatch(cfg, int(workloads.draw_layout(cfg).num_blocks * 1.25))
    cb.redraw()
    cb.redraw()
    cb.check()
    case = Case(cfg, cuda_device, n_layers=2, layout=cb)
    run_and_check(pkv, oracle_mod, case, what="70B mix after re-draws")


def test_fused_append_rejects_a_slot_that_is_not_the_last_token(pkv, oracle_mod, cuda_device):
    cfg = workloads.small_config(1, batch=4)
    case = Case(cfg, cuda_device, lens=[40, 17, 1, 33])
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    bad = case.slots.clone()
    bad[1] -= 1                              # one row before sequence 1's last token
    before_k, before_v = case.k[0].clone(), case.v[0].clone()
    out = torch.empty_like(case.q[0])
    pkv.paged_attention_decode_append(out, case.q[0], case.k_new[0], case.v_new[0], case.k[0], case.v[0], bad,
                                      case.tables, case.lens, cfg.scale, ws)
    assert pkv.read_status(ws) & pkv.KV_STATUS_BAD_SLOT
    # sequences 0, 2, 3 were appended exactly; sequence 1's rows are untouched
    host_k, host_v = before_k.cpu(), before_v.cpu()
    slots = bad.clone()
    slots[1] = -1
    ek, ev = oracle_mod.kv_cache_append(host_k, host_v, case.k_new[0].cpu(), case.v_new[0].cpu(), slots.cpu().numpy())
    assert np.array_equal(bf16_bits_np(case.k[0]), ek) and np.array_equal(bf16_bits_np(case.v[0]), ev)
    # a negative slot appends nothing and is not an error
    slots_none = torch.full_like(case.slots, -1)
    pkv.paged_attention_decode_append(out, case.q[0], case.k_new[0], case.v_new[0], case.k[0], case.v[0],
                                      slots_none, case.tables, case.lens, cfg.scale, ws)
    assert pkv.read_status(ws) == 0


# ---------------------------------------------------------------------------
# several layers in one launch (paged_attention_decode_layers)
# ---------------------------------------------------------------------------
def run_layers_and_check(pkv, oracle_mod, case, layers=None, append=True, what=""):
    """One multi-layer launch over all of the case's layers; the listed layers against the oracle (append
    bit-exact, attention within tolerance)."""
    cfg, L = case.cfg, case.n_layers
    check = list(range(L)) if layers is None else layers
    host = {layer: case.host_inputs(layer) for layer in check}
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D, num_layers=L)
    out = torch.full_like(case.q, float("nan"))
    kw = dict(k_new=case.k_new, v_new=case.v_new, slot_mapping=case.slots) if append else {}
    pkv.paged_attention_decode_layers(out, case.q, case.k_all, case.v_all, case.tables, case.lens, cfg.scale, ws,
                                      **kw)
    torch.cuda.synchronize()
    assert pkv.read_status(ws) == 0
    for layer in check:
        q, k, v, kn, vn = host[layer]
        if append:
            k2, v2, ref = oracle_step(oracle_mod, case, layer, host[layer])
            assert np.array_equal(bf16_bits_np(case.k[layer]), k2), f"{what} layer {layer}: K append not bit-exact"
            assert np.array_equal(bf16_bits_np(case.v[layer]), v2), f"{what} layer {layer}: V append not bit-exact"
        else:
            assert torch.equal(case.k[layer].cpu(), k) and torch.equal(case.v[layer].cpu(), v)
            ref = oracle_mod.paged_attention_decode(q, k, v, case.layout.block_tables.numpy(),
                                                    case.layout.context_lens.numpy(), cfg.scale, dtype=cfg.elem)
        compare(out[layer], ref, f"{what} layer {layer} (one launch for {L} layers)")
    return out


@pytest.mark.parametrize("append", [True, False])
@pytest.mark.parametrize("path", sorted(PATHS))
def test_layers_in_one_launch(pkv, oracle_mod, cuda_device, path, append):
    pkv.set_option(pkv.KV_OPT_COMPUTE, PATHS[path])
    cfg = workloads.small_config(2, batch=9, ctx_lo=1, ctx_hi=700, W=48)
    case = Case(cfg, cuda_device, n_layers=5)
    run_layers_and_check(pkv, oracle_mod, case, append=append, what=f"layers/{path}")


@pytest.mark.parametrize("cid", [2, 3])
@pytest.mark.parametrize("grid,min_chunk,combine", [(1, 1, 0), (3, 1, 0), (7, 2, 1), (296, 1, 0), (0, 1, 1)])
def test_layers_split_everywhere(pkv, oracle_mod, cuda_device, cid, grid, min_chunk, combine):
    """Grids from one CTA (one piece per item, every layer in it) to twice the SMs; CTA ranges start and end in
    different layers; the merge in the last CTA or in the combine kernel."""
    pkv.set_option(pkv.KV_OPT_GRID, grid)
    pkv.set_option(pkv.KV_OPT_MIN_CHUNK, min_chunk)
    pkv.set_option(pkv.KV_OPT_COMBINE, combine)
    cfg = workloads.small_config(cid, batch=6, ctx_lo=1, ctx_hi=900, W=64)
    case = Case(cfg, cuda_device, n_layers=4)
    run_layers_and_check(pkv, oracle_mod, case, what=f"layers cfg{cid} grid {grid} combine {combine}")


def test_layers_with_a_stride_larger_than_a_pool_and_empty_sequences(pkv, oracle_mod, cuda_device):
    cfg = workloads.small_config(3, batch=7, W=40)
    case = Case(cfg, cuda_device, n_layers=3, lens=[0, 1, 16, 17, 0, 640, 33], spare_blocks=5)
    assert case.k_all.stride(0) > case.k_all[0].numel()
    run_layers_and_check(pkv, oracle_mod, case, what="layers, strided pools")


def test_layers_one_layer_equals_the_per_layer_call(pkv, cuda_device):
    """num_layers = 1 is the per-layer call: the same grid and split, so the same bits."""
    cfg = workloads.small_config(2, batch=20, ctx_lo=1, ctx_hi=2000)
    case = Case(cfg, cuda_device, n_layers=1)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    a = torch.empty_like(case.q[:1])
    pkv.paged_attention_decode_layers(a, case.q[:1], case.k_all, case.v_all, case.tables, case.lens, cfg.scale, ws)
    b = torch.empty_like(case.q[0])
    pkv.paged_attention_decode(b, case.q[0], case.k[0], case.v[0], case.tables, case.lens, cfg.scale, ws)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b)


def test_layers_workspace_too_small_is_refused(pkv, cuda_device):
    cfg = workloads.small_config(2, batch=8, ctx_lo=1, ctx_hi=300, W=32)
    case = Case(cfg, cuda_device, n_layers=3)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D, num_layers=2)
    out = torch.empty_like(case.q)
    with pytest.raises(pkv.KVError):
        pkv.paged_attention_decode_layers(out, case.q, case.k_all, case.v_all, case.tables, case.lens, cfg.scale, ws)


@pytest.mark.parametrize("cid", [2, 3, 4, 5])
def test_full_size_layers_in_one_launch(pkv, oracle_mod, cuda_device, cid):
    """The bench's multi-layer step at full size: every layer of the 0.5B and 70B-mix workloads in one launch,
    four layers of the larger ones (memory of the oracle's host copies); first, last and one random layer
    checked."""
    cfg = workloads.WORKLOADS[cid]
    L = cfg.n_layers if cid in (2, 5) else 4
    case = Case(cfg, cuda_device, n_layers=L)
    layers = sorted({0, L - 1, random.Random(cid).randrange(L)})
    run_layers_and_check(pkv, oracle_mod, case, layers=layers, what=f"config {cid}")


@pytest.mark.parametrize("layers", [1, 3])
@pytest.mark.parametrize("policy", [1, 2, 3])
def test_l2_priorities_and_early_loads_keep_the_result(pkv, oracle_mod, cuda_device, policy, layers):
    """Every L2 priority of the tile loads, with and without early loads (whose promise holds here: the
    launch before each is the previous one over other layers' caches, or none), gives the oracle's result."""
    pkv.set_option(pkv.KV_OPT_L2_POLICY, policy)
    try:
        for early in (0, 1):
            pkv.set_option(pkv.KV_OPT_EARLY_LOADS, early)
            cfg = workloads.small_config(2, batch=10, ctx_lo=1, ctx_hi=900, W=64)
            case = Case(cfg, cuda_device, n_layers=layers, seed=policy * 10 + early)
            if layers == 1:
                run_and_check(pkv, oracle_mod, case, what=f"L2 policy {policy}, early {early}", fused=True)
            else:
                run_layers_and_check(pkv, oracle_mod, case, what=f"L2 policy {policy}, early {early}")
    finally:
        pkv.set_option(pkv.KV_OPT_L2_POLICY, 0)
        pkv.set_option(pkv.KV_OPT_EARLY_LOADS, 0)
