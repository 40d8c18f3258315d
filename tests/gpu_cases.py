"""Shared helpers for the GPU parity tests: seeded cases, and the oracle comparison.

Inputs come from paged_kv_cache_470_b200.workloads (seeded, shared with the
oracle side); expected values come only from the oracle, fed with the same
pre-step inputs copied to the host.
"""
import numpy as np
import torch

from paged_kv_cache_470_b200 import workloads

ATOL, RTOL = 5e-3, 1e-2   # |gpu - ref| <= ATOL + RTOL * |ref|, elementwise (16-bit outputs)
# The stated bounds, asserted outright on fp32 outputs (KV_OPT_OUT_F32): max |gpu - ref| <= MAX_ABS over all
# elements, and max |gpu - ref| / |ref| <= MAX_REL over the elements with |ref| >= REL_FLOOR.
MAX_ABS, MAX_REL, REL_FLOOR = 5e-3, 1e-2, 1e-2


class Case:
    """One decode step over `n_layers` layers of a workload, resident on the GPU.

    The layers' caches are views of two stacked tensors (k_all, v_all: [n_layers, num_blocks, 16, Hkv, D]), so
    one case serves the per-layer calls and the multi-layer one; spare_blocks puts zero blocks after each layer's
    pool, making the layers' stride larger than a pool."""

    def __init__(self, cfg, device, n_layers=1, lens=None, seed=None, layout=None, spare_blocks=0):
        self.cfg = cfg
        self.layout = layout if layout is not None else workloads.draw_layout(cfg, context_lens=lens, seed=seed)
        gen = workloads.device_generator(cfg.seed if seed is None else seed, device)
        self.k_all, self.v_all = workloads.make_stacked_caches(n_layers, self.layout.num_blocks, cfg.Hkv, cfg.D, gen,
                                                               device, cfg.torch_dtype, spare_blocks)
        self.k, self.v = list(self.k_all.unbind(0)), list(self.v_all.unbind(0))
        self.q, self.k_new, self.v_new = workloads.make_step_inputs(cfg, gen, device, n_layers)
        self.tables = self.layout.block_tables.to(device)
        self.lens = self.layout.context_lens.to(device)
        self.slots = self.layout.slot_mapping().to(device)
        self.n_layers = n_layers
        self.device = device

    def host_inputs(self, layer):
        """Pre-step inputs of one layer, on the host, for the oracle."""
        return (self.q[layer].cpu(), self.k[layer].cpu(), self.v[layer].cpu(), self.k_new[layer].cpu(),
                self.v_new[layer].cpu())


def oracle_step(oracle_mod, case, layer, host=None):
    """Oracle append then oracle attention for one layer; returns (k_after, v_after, out64)."""
    q, k, v, kn, vn = host if host is not None else case.host_inputs(layer)
    k2, v2 = oracle_mod.kv_cache_append(k, v, kn, vn, case.layout.slot_mapping().numpy())
    out = oracle_mod.paged_attention_decode(q, k2, v2, case.layout.block_tables.numpy(),
                                            case.layout.context_lens.numpy(), case.cfg.scale, dtype=case.cfg.elem)
    return k2, v2, out


def gpu_step(pkv, case, layer, workspace, out=None, fused=False):
    """Append this step's token and attend: two kernels, or one with the append fused in."""
    if out is None:
        out = torch.empty_like(case.q[layer])
    if fused:
        pkv.paged_attention_decode_append(out, case.q[layer], case.k_new[layer], case.v_new[layer], case.k[layer],
                                          case.v[layer], case.slots, case.tables, case.lens, case.cfg.scale,
                                          workspace)
    else:
        pkv.kv_cache_append(case.k_new[layer], case.v_new[layer], case.k[layer], case.v[layer], case.slots)
        pkv.paged_attention_decode(out, case.q[layer], case.k[layer], case.v[layer], case.tables, case.lens,
                                   case.cfg.scale, workspace)
    return out


def bf16_bits_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def compare(gpu_out: torch.Tensor, ref: np.ndarray, what: str, small_abs: bool = True):
    """A 16-bit output: elementwise |gpu - ref| <= ATOL + RTOL |ref|, and (small_abs) outright max abs <= MAX_ABS
    over the elements with |ref| < 1 (where rounding to bf16 alone moves a number by at most 2^-9).

    The chunked prefill passes small_abs=False: it rounds its probabilities to the element type before they
    multiply V, which moves a weight by up to 2^-9 of itself, so before the output's own rounding its error is
    bounded by 2^-9 sum_t w_t |V_t - out| rather than by the decode's arithmetic; its fp32 output is held to
    max abs <= MAX_ABS in tests/test_gpu_strict.py."""
    g = gpu_out.detach().float().cpu().double().numpy()
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    big = np.abs(ref) >= REL_FLOOR
    rel = (err[big] / np.abs(ref[big])).max() if big.any() else 0.0
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; "
                           f"max abs err {err.max():.3e}, max rel err (|ref|>=1e-2) {rel:.3e}")
    small = np.abs(ref) < 1.0
    if small_abs and small.any():
        assert err[small].max() <= MAX_ABS, f"{what}: max abs err {err[small].max():.3e} where |ref| < 1"
    return float(err.max()), float(rel)


def compare_strict(gpu_out: torch.Tensor, ref: np.ndarray, what: str):
    """An fp32 output (KV_OPT_OUT_F32): max abs error <= MAX_ABS and max relative error <= MAX_REL (over
    |ref| >= REL_FLOOR), both outright. Returns (max abs, max rel)."""
    assert gpu_out.dtype == torch.float32, f"{what}: expected an fp32 output"
    g = gpu_out.detach().cpu().double().numpy()
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref)
    big = np.abs(ref) >= REL_FLOOR
    rel = float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    mx = float(err.max()) if err.size else 0.0
    assert mx <= MAX_ABS, f"{what}: max abs err {mx:.3e} > {MAX_ABS}"
    assert rel <= MAX_REL, f"{what}: max rel err {rel:.3e} > {MAX_REL} (over |ref| >= {REL_FLOOR})"
    return mx, rel
