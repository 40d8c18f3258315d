"""GPU parity of the fp16 variant (q, K, V, out all IEEE binary16; 2 bytes per
number like bf16: "Module 23: Serving", section 23.1) against the oracle's fp16
entry point: append bit-exact, attention within 5e-3 + 1e-2|ref|.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_470_b200 import workloads
from gpu_cases import Case
from test_gpu_decode import PATHS, run_and_check

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _default_options(pkv):
    yield
    for key in (pkv.KV_OPT_COMPUTE, pkv.KV_OPT_COMBINE, pkv.KV_OPT_GRID, pkv.KV_OPT_MIN_CHUNK):
        pkv.set_option(key, 0)


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("combine", [0, 1])
def test_tiny_workload_fp16(pkv, oracle_mod, cuda_device, path, combine, fused):
    pkv.set_option(pkv.KV_OPT_COMPUTE, PATHS[path])
    pkv.set_option(pkv.KV_OPT_COMBINE, combine)
    case = Case(workloads.small_config(1, elem="fp16"), cuda_device)
    assert case.k[0].dtype == torch.float16
    run_and_check(pkv, oracle_mod, case, what=f"fp16 tiny/{path}/combine{combine}", fused=fused)


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("D,Hq,Hkv", [(64, 20, 4), (128, 32, 8), (128, 8, 8), (64, 12, 1), (128, 64, 8)])
def test_ragged_lengths_fp16(pkv, oracle_mod, cuda_device, path, D, Hq, Hkv):
    pkv.set_option(pkv.KV_OPT_COMPUTE, PATHS[path])
    lens = [1, 15, 16, 17, 31, 32, 33, 255, 256, 0, 100, 2]
    cfg = workloads.small_config(1, Hq=Hq, Hkv=Hkv, D=D, batch=len(lens), pool_blocks=0, n_layers=2, elem="fp16")
    case = Case(cfg, cuda_device, lens=lens, n_layers=2)
    run_and_check(pkv, oracle_mod, case, what=f"fp16 ragged D{D} {Hq}/{Hkv} {path}")


@pytest.mark.parametrize("grid", [3, 7, 0])
def test_split_pieces_fp16(pkv, oracle_mod, cuda_device, grid):
    pkv.set_option(pkv.KV_OPT_GRID, grid)
    pkv.set_option(pkv.KV_OPT_MIN_CHUNK, 1)
    cfg = workloads.small_config(3, batch=6, ctx_lo=1, ctx_hi=1500, W=96, n_layers=1, elem="fp16")
    run_and_check(pkv, oracle_mod, Case(cfg, cuda_device), what=f"fp16 config 3 shape, grid {grid}")


def test_single_token_context_returns_v_exactly_fp16(pkv, cuda_device):
    cfg = workloads.small_config(1, batch=3, elem="fp16")
    case = Case(cfg, cuda_device, lens=[1, 1, 1])
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    out = torch.empty_like(case.q[0])
    pkv.paged_attention_decode_append(out, case.q[0], case.k_new[0], case.v_new[0], case.k[0], case.v[0],
                                      case.slots, case.tables, case.lens, cfg.scale, ws)
    torch.cuda.synchronize()
    want = case.v_new[0].repeat_interleave(cfg.group, dim=1)
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))
    assert pkv.read_status(ws) == 0


def test_large_values_stay_finite_fp16(pkv, oracle_mod, cuda_device):
    """Inputs near +-200 (logits ~ 4e5 before the scale): fp32 inside, no fp16 overflow."""
    cfg = workloads.small_config(3, batch=4, ctx_lo=30, ctx_hi=400, W=32, n_layers=1, elem="fp16")
    case = Case(cfg, cuda_device)
    for t in (case.q, case.k[0], case.v[0], case.k_new, case.v_new):
        t.mul_(200.0)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    out = torch.empty_like(case.q[0])
    host = case.host_inputs(0)
    pkv.paged_attention_decode_append(out, case.q[0], case.k_new[0], case.v_new[0], case.k[0], case.v[0],
                                      case.slots, case.tables, case.lens, cfg.scale, ws)
    torch.cuda.synchronize()
    k2, v2 = oracle_mod.kv_cache_append(host[1], host[2], host[3], host[4], case.layout.slot_mapping().numpy())
    ref = oracle_mod.paged_attention_decode(host[0], k2, v2, case.layout.block_tables.numpy(),
                                            case.layout.context_lens.numpy(), cfg.scale, dtype="fp16")
    assert np.isfinite(ref).all()
    # outputs are ~200 in size: the bf16/fp16-scale absolute tolerance applies relative to that
    g = out.double().cpu().numpy()
    assert np.isfinite(g).all()
    err = np.abs(g - ref)
    assert (err <= 5e-3 * 200 + 1e-2 * np.abs(ref)).all(), float(err.max())
    assert pkv.read_status(ws) == 0


def test_full_size_llama2_7b_mha_fp16(pkv, oracle_mod, cuda_device):
    """The LLaMA-2-7B-shaped MHA workload in fp16, as the pages' worked example has it."""
    cfg = workloads.small_config(4, elem="fp16")
    case = Case(cfg, cuda_device, n_layers=2)
    run_and_check(pkv, oracle_mod, case, layers=[0, 1], what="fp16 config 4")


def test_dtype_mismatch_is_refused(pkv, cuda_device):
    cfg = workloads.small_config(1, elem="fp16")
    case = Case(cfg, cuda_device)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    with pytest.raises(ValueError):
        pkv.paged_attention_decode(torch.empty_like(case.q[0]), case.q[0].to(torch.bfloat16), case.k[0], case.v[0],
                                   case.tables, case.lens, cfg.scale, ws)
    with pytest.raises(ValueError):
        pkv.paged_attention_decode(torch.empty_like(case.q[0]), case.q[0].float(), case.k[0].float(),
                                   case.v[0].float(), case.tables, case.lens, cfg.scale, ws)


@pytest.mark.parametrize("path", sorted(PATHS))
def test_layers_in_one_launch_fp16(pkv, oracle_mod, cuda_device, path):
    """The multi-layer launch on the fp16 LLaMA-2-7B shape (32 kv heads, D = 128): three full-size layers."""
    from test_gpu_decode import run_layers_and_check
    pkv.set_option(pkv.KV_OPT_COMPUTE, PATHS[path])
    cfg = workloads.small_config(4, elem="fp16", batch=8, pool_blocks=2048)
    case = Case(cfg, cuda_device, n_layers=3)
    assert case.k_all.dtype == torch.float16
    run_layers_and_check(pkv, oracle_mod, case, what=f"fp16 layers/{path}")
