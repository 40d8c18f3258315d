"""GPU parity of chunked-prefill attention (paged_attention_prefill) against the
oracle, which states a query at position p as a decode over p + 1 tokens:
within |gpu - ref| <= 5e-3 + 1e-2 |ref| elementwise. The chunk's K/V are
appended with kv_cache_append first, and that append is checked bit-exactly.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_470_b200 import workloads
from gpu_cases import compare

pytestmark = pytest.mark.gpu

PREFILL_PATHS = {"tcgen05": 1, "mma_sync": 2, "tcgen05_pair": 3}


@pytest.fixture(autouse=True)
def _default_path(pkv):
    yield
    pkv.set_option(pkv.KV_OPT_PREFILL_PATH, 0)


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


class PrefillCase:
    def __init__(self, cfg, device, chunk_lens=None, prior_lens=None, seed=None):
        self.cfg = cfg
        self.layout = workloads.draw_prefill_layout(cfg, chunk_lens=chunk_lens, prior_lens=prior_lens, seed=seed)
        gen = workloads.device_generator(cfg.seed if seed is None else seed, device)
        dt = cfg.torch_dtype
        self.k, self.v = workloads.make_layer_cache(self.layout.num_blocks, cfg.Hkv, cfg.D, gen, device, dt)
        T = int(self.layout.query_start[-1])
        self.q = workloads.random_bf16((T, cfg.Hq, cfg.D), gen, device, dt)
        self.k_new = workloads.random_bf16((T, cfg.Hkv, cfg.D), gen, device, dt)
        self.v_new = workloads.random_bf16((T, cfg.Hkv, cfg.D), gen, device, dt)
        self.tables = self.layout.block_tables.to(device)
        self.lens = self.layout.context_lens.to(device)
        self.qs = self.layout.query_start.to(device)
        self.slots = self.layout.slot_mapping().to(device)
        self.max_q = int(self.layout.chunk_lens.max()) if self.layout.chunk_lens.numel() else 0


def run_case(pkv, oracle_mod, case, what, rows=None):
    cfg = case.cfg
    k_host, v_host = case.k.cpu(), case.v.cpu()
    flag = torch.zeros(1, dtype=torch.int32, device=case.q.device)
    pkv.kv_cache_append(case.k_new, case.v_new, case.k, case.v, case.slots, flag)
    out = torch.full_like(case.q, float("nan"))
    pkv.paged_attention_prefill(out, case.q, case.k, case.v, case.tables, case.lens, case.qs, case.max_q, cfg.scale,
                                flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    k2, v2 = oracle_mod.kv_cache_append(k_host, v_host, case.k_new.cpu(), case.v_new.cpu(),
                                        case.layout.slot_mapping().numpy())
    assert np.array_equal(bits(case.k), k2) and np.array_equal(bits(case.v), v2), f"{what}: append not bit-exact"
    seqs = range(cfg.batch) if rows is None else rows
    qs = case.layout.query_start.numpy()
    for b in seqs:
        lo, hi = int(qs[b]), int(qs[b + 1])
        if hi == lo:
            continue
        ref = oracle_mod.paged_attention_prefill(bits(case.q[lo:hi]), k2, v2, case.layout.block_tables.numpy()[b:b + 1],
                                                 case.layout.context_lens.numpy()[b:b + 1], np.array([0, hi - lo]),
                                                 cfg.scale, dtype=cfg.elem)
        compare(out[lo:hi], ref, f"{what}, sequence {b}", small_abs=False)
    return out


@pytest.mark.parametrize("path", sorted(PREFILL_PATHS))
@pytest.mark.parametrize("elem", ["bf16", "fp16"])
@pytest.mark.parametrize("Hq,Hkv,D", [(20, 4, 64), (32, 8, 128), (8, 8, 128), (12, 1, 64), (16, 2, 128), (6, 6, 64)])
def test_prefill_chunks(pkv, oracle_mod, cuda_device, Hq, Hkv, D, elem, path):
    """Whole prompts, chunks over a cached prefix, single tokens and empty chunks; lengths at and
    around block edges."""
    pkv.set_option(pkv.KV_OPT_PREFILL_PATH, PREFILL_PATHS[path])
    chunk = [37, 1, 16, 100, 0, 64, 17, 5]
    prior = [0, 250, 15, 33, 40, 0, 111, 1]
    cfg = workloads.PrefillConfig("test", Hq, Hkv, D, len(chunk), 0, 0, 0, 16, seed=Hq * 7 + D, elem=elem)
    case = PrefillCase(cfg, cuda_device, chunk_lens=chunk, prior_lens=prior)
    run_case(pkv, oracle_mod, case, f"prefill {Hq}/{Hkv} D{D} {elem} {path}")


def test_single_token_chunk_matches_the_decode(pkv, cuda_device):
    """A one-token chunk is a decode step: both kernels agree to within rounding."""
    cfg = workloads.PrefillConfig("test", 32, 8, 128, 4, 1, 100, 700, 64, seed=3)
    case = PrefillCase(cfg, cuda_device)
    pkv.kv_cache_append(case.k_new, case.v_new, case.k, case.v, case.slots)
    out_p = torch.empty_like(case.q)
    pkv.paged_attention_prefill(out_p, case.q, case.k, case.v, case.tables, case.lens, case.qs, 1, cfg.scale)
    out_d = torch.empty_like(case.q)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    pkv.paged_attention_decode(out_d, case.q, case.k, case.v, case.tables, case.lens, cfg.scale, ws)
    torch.cuda.synchronize()
    d = (out_p.float() - out_d.float()).abs()
    assert float(d.max()) <= 2e-2, float(d.max())


@pytest.mark.parametrize("path", sorted(PREFILL_PATHS))
@pytest.mark.parametrize("key,elem", [("llama3_8b", "bf16"), ("llama3_8b", "fp16"), ("0p5b", "bf16")])
def test_full_size_prefill_workload(pkv, oracle_mod, cuda_device, path, key, elem):
    """The bench's prefill workloads (LLaMA-3-8B and 0.5B shapes), three sequences of each against the oracle."""
    from dataclasses import replace
    pkv.set_option(pkv.KV_OPT_PREFILL_PATH, PREFILL_PATHS[path])
    cfg = replace(workloads.PREFILL_CONFIGS[key], elem=elem)
    case = PrefillCase(cfg, cuda_device)
    run_case(pkv, oracle_mod, case, f"full-size prefill {key} {elem} {path}", rows=[0, 7, 15])


@pytest.mark.parametrize("path", sorted(PREFILL_PATHS))
def test_bad_chunks_are_flagged(pkv, cuda_device, path):
    pkv.set_option(pkv.KV_OPT_PREFILL_PATH, PREFILL_PATHS[path])
    cfg = workloads.PrefillConfig("test", 8, 2, 64, 3, 10, 20, 40, 8, seed=5)
    case = PrefillCase(cfg, cuda_device)
    out = torch.zeros_like(case.q)
    flag = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    lens = case.lens.clone()
    lens[1] = 5                                   # shorter than its 10-token chunk
    pkv.paged_attention_prefill(out, case.q, case.k, case.v, case.tables, lens, case.qs, case.max_q, cfg.scale, flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & pkv.KV_STATUS_BAD_CONTEXT
    assert not out[10:20].any()                   # that sequence's rows are not written
    flag.zero_()
    tables = case.tables.clone()
    tables[0, 0] = 10 ** 6                        # outside the pool
    pkv.paged_attention_prefill(out, case.q, case.k, case.v, tables, case.lens, case.qs, case.max_q, cfg.scale, flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & pkv.KV_STATUS_BAD_BLOCK_ID


@pytest.mark.parametrize("path", sorted(PREFILL_PATHS))
@pytest.mark.parametrize("D", [64, 128])
def test_stale_shared_memory_stays_out(pkv, oracle_mod, cuda_device, D, path):
    """A launch over a cache of NaNs first leaves NaNs in every SM's tile stages; a CTA whose rows end
    before its sequence does, and whose last tile has blocks it does not load, must not let those
    stale rows (or the pool's rows past the context) into its output."""
    pkv.set_option(pkv.KV_OPT_PREFILL_PATH, PREFILL_PATHS[path])
    Hq, Hkv = (16, 4) if D == 128 else (20, 4)
    poison = workloads.PrefillConfig("test", Hq, Hkv, D, 64, 256, 0, 1024, 80, seed=11)
    pc = PrefillCase(poison, cuda_device)
    pc.k.view(torch.int16).fill_(0x7fc0)            # bf16 and fp16 NaN patterns alike
    pc.v.view(torch.int16).fill_(0x7fc0)
    junk = torch.empty_like(pc.q)
    pkv.paged_attention_prefill(junk, pc.q, pc.k, pc.v, pc.tables, pc.lens, pc.qs, pc.max_q, poison.scale)
    torch.cuda.synchronize()
    chunk = [100, 37, 130, 9]
    prior = [33, 3, 70, 200]
    cfg = workloads.PrefillConfig("test", Hq, Hkv, D, len(chunk), 0, 0, 0, 32, seed=12)
    case = PrefillCase(cfg, cuda_device, chunk_lens=chunk, prior_lens=prior)
    run_case(pkv, oracle_mod, case, f"after a NaN launch, D{D} {path}")


@pytest.mark.parametrize("path", ["tcgen05", "tcgen05_pair"])
@pytest.mark.parametrize("D", [64, 128])
def test_slow_softmax_warp_keeps_the_result(pkv, oracle_mod, cuda_device, D, path):
    """The first softmax warp of every CTA hands over its first P ~30 us late, so the other warps run a
    tile ahead of it: the P V of a tile must still wait for all of that tile's P."""
    pkv.set_option(pkv.KV_OPT_PREFILL_PATH, PREFILL_PATHS[path])
    pkv.set_option(pkv.KV_OPT_TEST_SLOW_SOFTMAX, 1)
    try:
        Hq, Hkv = (32, 8) if D == 128 else (20, 4)
        chunk = [37, 100, 64, 17, 300, 5]
        prior = [0, 33, 200, 111, 40, 700]
        cfg = workloads.PrefillConfig("test", Hq, Hkv, D, len(chunk), 0, 0, 0, 48, seed=21 + D)
        case = PrefillCase(cfg, cuda_device, chunk_lens=chunk, prior_lens=prior)
        run_case(pkv, oracle_mod, case, f"slow first softmax warp, D{D} {path}")
    finally:
        pkv.set_option(pkv.KV_OPT_TEST_SLOW_SOFTMAX, 0)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("B,equal", [(40, True), (300, False)])
def test_launch_order_covers_every_sequence_once(pkv, oracle_mod, cuda_device, D, B, equal):
    """The default kernel launches its CTAs longest sequence first: each CTA ranks the batch's context lengths
    (ties by index) for batches of up to 256 sequences and takes them in order beyond. With every length equal
    (all ties) and with more sequences than are ranked, every sequence's rows are written, and right."""
    chunk = [3 + (i % 5) for i in range(B)]
    prior = [40 - chunk[i] + 3 for i in range(B)] if equal else [(i * 37) % 97 for i in range(B)]
    if equal:
        assert len({c + p for c, p in zip(chunk, prior)}) == 1
    cfg = workloads.PrefillConfig("test", 16, 4, D, B, 0, 0, 0, 8, seed=31 + D + B)
    case = PrefillCase(cfg, cuda_device, chunk_lens=chunk, prior_lens=prior)
    out = run_case(pkv, oracle_mod, case, f"launch order, B={B}, D{D}")
    assert torch.isfinite(out.float()).all(), "rows left unwritten"
