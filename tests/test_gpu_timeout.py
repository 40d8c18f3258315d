"""The timeout path of the decode kernel, on the GPU, without a fault: a test
hook keeps one tile load from ever being issued, so the bounded wait for it runs
out (about a second). The call must come back with KV_STATUS_WAIT_TIMEOUT in the
status word, and the same context must then decode correctly.
"""
import time

import numpy as np
import pytest
import torch

from paged_kv_cache_470_b200 import workloads
from gpu_cases import Case, compare, gpu_step, oracle_step

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fused", [False, True])
def test_wait_runs_out_and_the_context_survives(pkv, oracle_mod, cuda_device, fused):
    cfg = workloads.small_config(2, batch=8, ctx_lo=200, ctx_hi=900, W=64, n_layers=1)
    case = Case(cfg, cuda_device)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)
    host = case.host_inputs(0)
    try:
        pkv.set_option(pkv.KV_OPT_TEST_DROP_LOAD, 1)     # the CTA with the first unit never loads it
        t0 = time.perf_counter()
        gpu_step(pkv, case, 0, ws, fused=fused)
        status = pkv.read_status(ws)                    # synchronises
        waited = time.perf_counter() - t0
    finally:
        pkv.set_option(pkv.KV_OPT_TEST_DROP_LOAD, 0)
    assert status & pkv.KV_STATUS_WAIT_TIMEOUT, status
    assert 0.5 < waited < 30.0, waited
    # the context is usable: with the workspace re-initialised (a timed-out call may leave split-K
    # counts behind), a clean call on fresh inputs matches the oracle
    pkv.workspace_init(ws)
    case2 = Case(cfg, cuda_device, seed=cfg.seed + 1)
    host2 = case2.host_inputs(0)
    out = gpu_step(pkv, case2, 0, ws, fused=fused)
    torch.cuda.synchronize()
    _, _, ref = oracle_step(oracle_mod, case2, 0, host2)
    compare(out, ref, "decode after a timed-out call")
    assert pkv.read_status(ws) == 0
    assert host[0].shape == (cfg.batch, cfg.Hq, cfg.D)
