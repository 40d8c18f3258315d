"""The decode entry point that allocates nothing, checked against the one that takes a workspace.

paged_attention_decode_noalloc serves callers that cannot allocate device
memory (a plugin inside a program that owns all device allocations, or code
that must avoid cudaMalloc's implicit synchronisation): its split-K scratch is
a fixed array inside the library. It runs the same kernel on the same grid as
paged_attention_decode, so its output must be bitwise the same. This file is
collected last, so a run that stops at the first failure has run every other
test before it.
"""
import ctypes

import pytest
import torch

from paged_kv_cache_470_b200 import workloads
from gpu_cases import Case, compare

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20   # KV_NOALLOC_SCRATCH_BYTES


def _noalloc(pkv):
    """The entry point through its C declaration (ctypes), not through the package's wrapper."""
    lib = ctypes.CDLL(pkv.LIB_PATH)
    f = lib.paged_attention_decode_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, P, I, P, I, I, I, I, I, ctypes.c_float, I, P]
    f.restype = I
    return f


def _call(f, out, case, layer=0, stream=None):
    cfg = case.cfg
    s = stream if stream is not None else torch.cuda.current_stream()
    return f(out.data_ptr(), case.q[layer].data_ptr(), case.k[layer].data_ptr(), case.v[layer].data_ptr(),
             case.tables.data_ptr(), case.tables.shape[1], case.lens.data_ptr(), cfg.batch,
             case.layout.num_blocks, cfg.Hq, cfg.Hkv, cfg.D, cfg.scale, 0, s.cuda_stream or None)


def _with_workspace(pkv, case, layer=0):
    cfg = case.cfg
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    ref = torch.empty_like(case.q[layer])
    pkv.paged_attention_decode(ref, case.q[layer], case.k[layer], case.v[layer], case.tables, case.lens, cfg.scale,
                               ws)
    assert pkv.read_status(ws) == 0          # the same kernel on the same data: no data error to report
    return ref


@pytest.mark.parametrize("cid", [2, 3])
def test_noalloc_matches_workspace_entry_point(pkv, oracle_mod, cuda_device, cid):
    f = _noalloc(pkv)
    cfg = workloads.small_config(cid, batch=12, ctx_lo=1, ctx_hi=1500, W=96, n_layers=1)
    case = Case(cfg, cuda_device)
    ref = _with_workspace(pkv, case)
    oracle = oracle_mod.paged_attention_decode(case.q[0].cpu(), case.k[0].cpu(), case.v[0].cpu(),
                                               case.layout.block_tables.numpy(), case.layout.context_lens.numpy(),
                                               cfg.scale)
    for call in range(2):                       # two calls in a row share the fixed scratch
        out = torch.full_like(case.q[0], float("nan"))
        assert _call(f, out, case) == pkv.KV_OK
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"call {call}: differs from paged_attention_decode"
        compare(out, oracle, f"no-alloc call {call}")


def test_noalloc_back_to_back_on_one_stream(pkv, cuda_device):
    """Two calls queued on one stream with no synchronisation between them: the second clears and reuses the
    scratch only after the first has finished with it."""
    f = _noalloc(pkv)
    cfg = workloads.small_config(2, batch=40, ctx_lo=1, ctx_hi=2000, n_layers=2)
    case = Case(cfg, cuda_device, n_layers=2)
    refs = [_with_workspace(pkv, case, layer) for layer in range(2)]
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    outs = [torch.full_like(case.q[layer], float("nan")) for layer in range(2)]
    with torch.cuda.stream(stream):
        for layer in range(2):
            assert _call(f, outs[layer], case, layer, stream) == pkv.KV_OK
    stream.synchronize()
    for layer in range(2):
        assert torch.equal(outs[layer], refs[layer]), f"layer {layer}"


@pytest.mark.parametrize("cid", [1, 2, 3, 4, 5])
def test_every_workload_shape_fits_the_scratch(pkv, cuda_device, cid):
    """Each workload's full batch and heads fit the fixed array and give the workspace call's bits."""
    cfg = workloads.WORKLOADS[cid]
    assert pkv.workspace_size(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D) <= SCRATCH_BYTES
    f = _noalloc(pkv)
    case = Case(cfg, cuda_device, n_layers=1)
    ref = _with_workspace(pkv, case)
    out = torch.full_like(case.q[0], float("nan"))
    assert _call(f, out, case) == pkv.KV_OK
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_the_python_wrapper(pkv, cuda_device):
    cfg = workloads.small_config(3, batch=5, ctx_lo=1, ctx_hi=800, W=64, n_layers=1)
    case = Case(cfg, cuda_device)
    ref = _with_workspace(pkv, case)
    out = torch.full_like(case.q[0], float("nan"))
    assert pkv.paged_attention_decode_noalloc(out, case.q[0], case.k[0], case.v[0], case.tables, case.lens,
                                              cfg.scale) is out
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    with pytest.raises(ValueError):
        pkv.paged_attention_decode_noalloc(out[:1], case.q[0], case.k[0], case.v[0], case.tables, case.lens,
                                           cfg.scale)


def test_noalloc_rejects_sizes_beyond_its_scratch(pkv, cuda_device):
    f = _noalloc(pkv)
    # 4096 sequences x 32 kv heads x D=128 needs far more than the fixed 16 MiB of scratch
    B, Hq, Hkv, D = 4096, 32, 32, 128
    assert pkv.workspace_size(B, Hq, Hkv, D) > SCRATCH_BYTES
    dummy = torch.zeros(16, dtype=torch.bfloat16, device=cuda_device)
    rc = f(dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), 1,
           dummy.data_ptr(), B, 1, Hq, Hkv, D, 0.1, 0, None)
    assert rc == pkv.KV_ERR_ARG
