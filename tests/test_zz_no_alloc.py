"""The decode entry point that allocates nothing, checked against the one that takes a workspace.

paged_attention_decode_noalloc serves callers that cannot allocate device
memory (a plugin inside a program that owns all device allocations, or code
that must avoid cudaMalloc's implicit synchronisation): its split-K scratch is
a fixed array inside the library. This file is collected last, so a run that
stops at the first failure has run every other test before it.
"""
import ctypes

import pytest
import torch

from paged_kv_cache_470_b200 import workloads
from gpu_cases import ATOL, RTOL, Case

pytestmark = pytest.mark.gpu


def _noalloc(pkv):
    lib = ctypes.CDLL(pkv.LIB_PATH)
    f = lib.paged_attention_decode_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, P, I, P, I, I, I, I, I, ctypes.c_float, I, P]
    f.restype = I
    return f


def _call(f, out, case, layer=0):
    cfg = case.cfg
    return f(out.data_ptr(), case.q[layer].data_ptr(), case.k[layer].data_ptr(), case.v[layer].data_ptr(),
             case.tables.data_ptr(), case.tables.shape[1], case.lens.data_ptr(), cfg.batch,
             case.layout.num_blocks, cfg.Hq, cfg.Hkv, cfg.D, cfg.scale, 0,
             torch.cuda.current_stream().cuda_stream or None)


@pytest.mark.parametrize("cid", [2, 3])
def test_noalloc_matches_workspace_entry_point(pkv, cuda_device, cid):
    f = _noalloc(pkv)
    cfg = workloads.small_config(cid, batch=12, ctx_lo=1, ctx_hi=1500, W=96, n_layers=1)
    case = Case(cfg, cuda_device)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    ref = torch.empty_like(case.q[0])
    pkv.paged_attention_decode(ref, case.q[0], case.k[0], case.v[0], case.tables, case.lens, cfg.scale, ws)
    for call in range(2):                       # two calls in a row share the fixed scratch
        out = torch.full_like(case.q[0], float("nan"))
        assert _call(f, out, case) == pkv.KV_OK
        torch.cuda.synchronize()
        err = (out.float() - ref.float()).abs()
        assert torch.isfinite(out.float()).all(), f"call {call}: non-finite output"
        assert (err <= ATOL + RTOL * ref.float().abs()).all(), f"call {call}: max abs diff {err.max().item()}"


def test_noalloc_rejects_sizes_beyond_its_scratch(pkv, cuda_device):
    f = _noalloc(pkv)
    # 4096 sequences x 32 kv heads x D=128 needs far more than the fixed 16 MiB of scratch
    B, Hq, Hkv, D = 4096, 32, 32, 128
    assert pkv.workspace_size(B, Hq, Hkv, D) > (16 << 20)
    dummy = torch.zeros(16, dtype=torch.bfloat16, device=cuda_device)
    rc = f(dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), 1,
           dummy.data_ptr(), B, 1, Hq, Hkv, D, 0.1, 0, None)
    assert rc == pkv.KV_ERR_ARG
