"""The stated error bounds, asserted outright: with KV_OPT_OUT_F32 the kernels write their normalised fp32
result before any rounding to 16 bits, and it must agree with the float64 oracle to max abs error <= 5e-3 and
max relative error <= 1e-2 (relative error over the elements with |ref| >= 1e-2), on all five workloads at full
size, for both arithmetic paths, the separate and the fused append, the per-layer and the multi-layer calls.

(The 16-bit outputs of the other tests cannot meet the relative bound near zero by themselves: rounding to bf16
moves a number by up to 2^-9 of itself. They are held to |gpu - ref| <= 5e-3 + 1e-2 |ref| and to max abs <= 5e-3
where |ref| < 1.)
"""
import random

import numpy as np
import pytest
import torch

from paged_kv_cache_470_b200 import workloads
from gpu_cases import Case, bf16_bits_np, compare_strict, oracle_step

pytestmark = pytest.mark.gpu

PATHS = {"tensor_cores": 1, "cuda_cores": 2}


@pytest.fixture(autouse=True)
def _fp32_out(pkv):
    pkv.set_option(pkv.KV_OPT_OUT_F32, 1)
    yield
    for key in (pkv.KV_OPT_OUT_F32, pkv.KV_OPT_COMPUTE, pkv.KV_OPT_PREFILL_PATH):
        pkv.set_option(key, 0)


def _f32_like(t):
    return torch.full(t.shape, float("nan"), dtype=torch.float32, device=t.device)


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("cid", [1, 2, 3, 4, 5])
def test_decode_meets_the_stated_bounds(pkv, oracle_mod, cuda_device, cid, path):
    pkv.set_option(pkv.KV_OPT_COMPUTE, PATHS[path])
    cfg = workloads.WORKLOADS[cid]
    L = min(2, cfg.n_layers)
    case = Case(cfg, cuda_device, n_layers=L)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    worst = [0.0, 0.0]
    # the separate append on the first layer, the fused one on the last (the same layer again when there
    # is one: rewriting this step's token is idempotent, and the oracle appends it again as well)
    for layer, fused in ((0, False), (L - 1, True)):
        host = case.host_inputs(layer)
        out = _f32_like(case.q[layer])
        if fused:
            pkv.paged_attention_decode_append(out, case.q[layer], case.k_new[layer], case.v_new[layer],
                                              case.k[layer], case.v[layer], case.slots, case.tables, case.lens,
                                              cfg.scale, ws)
        else:
            pkv.kv_cache_append(case.k_new[layer], case.v_new[layer], case.k[layer], case.v[layer], case.slots)
            pkv.paged_attention_decode(out, case.q[layer], case.k[layer], case.v[layer], case.tables, case.lens,
                                       cfg.scale, ws)
        torch.cuda.synchronize()
        k2, v2, ref = oracle_step(oracle_mod, case, layer, host)
        assert np.array_equal(bf16_bits_np(case.k[layer]), k2) and np.array_equal(bf16_bits_np(case.v[layer]), v2)
        mx, rel = compare_strict(out, ref, f"config {cid}/{path} layer {layer}{' fused' if fused else ''}")
        worst = [max(worst[0], mx), max(worst[1], rel)]
    assert pkv.read_status(ws) == 0
    print(f"config {cid} {path}: max abs {worst[0]:.3e}, max rel {worst[1]:.3e}")


@pytest.mark.parametrize("cid", [2, 3, 5])
def test_multi_layer_launch_meets_the_stated_bounds(pkv, oracle_mod, cuda_device, cid):
    cfg = workloads.WORKLOADS[cid]
    L = min(cfg.n_layers, 8)
    case = Case(cfg, cuda_device, n_layers=L)
    check = sorted({0, L - 1, random.Random(cid).randrange(L)})
    host = {layer: case.host_inputs(layer) for layer in check}
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D, num_layers=L)
    out = _f32_like(case.q)
    pkv.paged_attention_decode_layers(out, case.q, case.k_all, case.v_all, case.tables, case.lens, cfg.scale, ws,
                                      k_new=case.k_new, v_new=case.v_new, slot_mapping=case.slots)
    torch.cuda.synchronize()
    assert pkv.read_status(ws) == 0
    for layer in check:
        _, _, ref = oracle_step(oracle_mod, case, layer, host[layer])
        compare_strict(out[layer], ref, f"config {cid} layer {layer} of a {L}-layer launch")


@pytest.mark.parametrize("prefill_path", [1, 2, 3])
@pytest.mark.parametrize("key", sorted(workloads.PREFILL_CONFIGS))
def test_prefill_fp32_output(pkv, oracle_mod, cuda_device, key, prefill_path):
    """The chunked prefill's fp32 result: max abs <= 5e-3 outright. Its probabilities are rounded to the element
    type before they multiply V (a tensor-core operand), so its relative error near small outputs is that
    rounding's (up to 2^-9 of each weight), not the decode's; it is reported, and held to 2^-9 * sum_t w_t |V_t|
    per output by construction, not asserted against 1e-2."""
    pkv.set_option(pkv.KV_OPT_PREFILL_PATH, prefill_path)
    cfg = workloads.PREFILL_CONFIGS[key]
    layout = workloads.draw_prefill_layout(cfg)
    gen = workloads.device_generator(cfg.seed, cuda_device)
    k, v = workloads.make_layer_cache(layout.num_blocks, cfg.Hkv, cfg.D, gen, cuda_device, cfg.torch_dtype)
    T = int(layout.query_start[-1])
    q = workloads.random_bf16((T, cfg.Hq, cfg.D), gen, cuda_device, cfg.torch_dtype)
    out = _f32_like(q)
    flag = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    pkv.paged_attention_prefill(out, q, k, v, layout.block_tables.to(cuda_device), layout.context_lens.to(cuda_device),
                                layout.query_start.to(cuda_device), cfg.chunk, cfg.scale, flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    ref = oracle_mod.paged_attention_prefill(q.cpu(), k.cpu(), v.cpu(), layout.block_tables.numpy(),
                                             layout.context_lens.numpy(), layout.query_start.numpy(), cfg.scale)
    g = out.cpu().double().numpy()
    assert np.isfinite(g).all()
    err = np.abs(g - ref)
    big = np.abs(ref) >= 1e-2
    print(f"prefill {key} path {prefill_path}: max abs {err.max():.3e}, "
          f"max rel (|ref|>=1e-2) {(err[big] / np.abs(ref[big])).max():.3e}")
    assert err.max() <= 5e-3
