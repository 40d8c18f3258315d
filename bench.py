"""Benchmark: one decode step (append + paged attention over every layer) on one or more B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2] [--impl ours|reference]

A step is the whole hot path over one batch: for each layer, scatter the new
token's K/V into its slot, then decode attention over every sequence's paged
cache (with the split-K merge). Inputs are synthetic and seeded, shaped like
the pages' models (see paged_kv_cache_470_b200/workloads.py); the default is
the 0.5B GQA model's decode step (24 layers, Hq=20, Hkv=4, D=64, batch 64,
context U[128,2048]).

Reported (one JSON line on rank 0):
  value      achieved HBM GB/s = algorithmic bytes of the step / step time,
             summed over GPUs (inputs resident in HBM, CUDA-graph replay)
  e2e        the same metric through the C ABI with host buffers: pinned-host
             -> device copies of the step's inputs and a device -> host copy of
             its outputs inside the timed region
  roofline   the decode kernel alone: its algorithmic bytes per launch over its
             CUDA-event duration, against the measured HBM copy bandwidth
  cpu_baseline  the float64 oracle on this host's cores, on a bounded sample

With --gpus N > 1 (under torchrun) each rank runs an independent replica of
the workload on its own GPU (the path needs no exchange between GPUs); the
step time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import random
import re
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_470_b200 import workloads  # noqa: E402  (no CUDA library needed)

NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
PROFILE_DIR = os.path.join(ROOT, "profiles")
DECODE_SRC = os.path.join(ROOT, "paged_kv_cache_470_b200", "csrc", "decode.cu")


# ---------------------------------------------------------------------------
# algorithmic bytes (what one decode step must move at least once)
# ---------------------------------------------------------------------------
def layer_bytes(cfg, lens, shares_prefix=None, unique_prefix=False):
    """Bytes one layer's append + attention must move, from the drawn lengths.

    KV read: 2 (K and V) x c x Hkv x D x 2 per sequence; q read and out write:
    2 x Hq x D x 2 per sequence; table entries 4 x ceil(c/16) and the length
    (4); append: the new K/V rows read and written (4 x Hkv x D x 2) and the
    slot (8). With unique_prefix, a shared prefix's blocks count once.
    """
    B = len(lens)
    kv = 0
    for b, c in enumerate(lens):
        own = c
        if unique_prefix and shares_prefix is not None and shares_prefix[b]:
            own = c - cfg.shared_prefix_tokens
        kv += 2 * own * cfg.Hkv * cfg.D * 2
    if unique_prefix and shares_prefix is not None and any(shares_prefix):
        kv += 2 * cfg.shared_prefix_tokens * cfg.Hkv * cfg.D * 2
    qo = 2 * B * cfg.Hq * cfg.D * 2
    tables = sum(4 * -(-c // 16) + 4 for c in lens)
    append = B * (4 * cfg.Hkv * cfg.D * 2 + 8)
    return {"kv": kv, "q_out": qo, "tables": tables, "append": append,
            "decode_kernel": kv + qo + tables, "total": kv + qo + tables + append}


def prefill_pairs(context_lens, chunk_lens):
    """(query, visible token) pairs of a chunked prefill: chunk token i of a sequence with c tokens
    (its n-token chunk included) sits at position c - n + i and sees positions 0 .. c - n + i."""
    return sum(sum(int(c) - int(n) + i + 1 for i in range(int(n))) for c, n in zip(context_lens, chunk_lens))


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor throughput of this machine's B200s (a kernel timed alone: the burst figure)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured cuBLAS bf16 GEMM (burst)"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def profiled_traffic(cfg):
    """DRAM bytes per decode launch from a committed ncu summary of this workload and element type,
    if one matches the current kernel source (else None)."""
    try:
        src_hash = hashlib.sha256(open(DECODE_SRC, "rb").read()).hexdigest()[:16]
        for name in sorted(os.listdir(PROFILE_DIR)):
            if not name.endswith(".txt"):
                continue
            text = open(os.path.join(PROFILE_DIR, name)).read()
            m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
            h = re.search(r"decode\.cu sha256\[:16\]:\s*([0-9a-f]+)", text)
            c = re.search(r"^config_id:\s*(\d+)", text, re.M)
            e = re.search(r"^elem:\s*(\w+)", text, re.M)
            if m and h and c and e and h.group(1) == src_hash and int(c.group(1)) == cfg.cid \
                    and e.group(1) == cfg.elem:
                return float(m.group(1))
    except OSError:
        pass
    return None


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x1: "gpu_idle"}

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._period = period_s
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = getattr(props, "pci_bus_id", None)
            if bus is not None:
                dom = getattr(props, "pci_domain_id", 0)
                dev = getattr(props, "pci_device_id", 0)
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{dev:02x}.0".encode())
            else:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report what is missing
            self.error = str(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nvml.nvmlDeviceGetClockInfo(self._h, self._nvml.NVML_CLOCK_SM))
                mask = self._nvml.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._h is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t.is_alive():
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0, "note": getattr(self, "error", "no samples")}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ---------------------------------------------------------------------------
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if (torch.cuda.is_available() and args.impl == "ours") else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def dist_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def dist_done(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
class Workload:
    def __init__(self, cfg, device, rank=0):
        import paged_kv_cache_470_b200 as pkv
        self.pkv = pkv
        self.cfg = cfg
        self.layout = workloads.draw_layout(cfg)
        if cfg.redraw_fraction > 0:
            # the batch is re-formed every step through the block pool (shared-prefix refcounts)
            from paged_kv_cache_470_b200.batch import ContinuousBatch
            self.layout = ContinuousBatch(cfg, int(self.layout.num_blocks * 1.25), seed=cfg.seed + 1000 * rank)
        gen = workloads.device_generator(cfg.seed + 1000 * rank, device)
        self.k, self.v = [], []
        for _ in range(cfg.n_layers):
            k, v = workloads.make_layer_cache(self.layout.num_blocks, cfg.Hkv, cfg.D, gen, device, cfg.torch_dtype)
            self.k.append(k)
            self.v.append(v)
        self.q, self.k_new, self.v_new = workloads.make_step_inputs(cfg, gen, device)
        self.tables = self.layout.block_tables.to(device)
        self.lens = self.layout.context_lens.to(device)
        self.slots = self.layout.slot_mapping().to(device)
        self.out = torch.empty_like(self.q)
        self.ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D, device)
        self.fused = True

    def redraw(self):
        """Re-form the batch (host bookkeeping) and upload the new tables; not timed."""
        self.layout.redraw()
        self.tables.copy_(self.layout.block_tables)
        self.lens.copy_(self.layout.context_lens)
        self.slots.copy_(self.layout.slot_mapping())

    def layer(self, layer, stream=None):
        """One layer: append this step's token and attend (one fused launch, or two kernels)."""
        pkv, cfg = self.pkv, self.cfg
        if self.fused:
            pkv.paged_attention_decode_append(self.out[layer], self.q[layer], self.k_new[layer],
                                              self.v_new[layer], self.k[layer], self.v[layer], self.slots,
                                              self.tables, self.lens, cfg.scale, self.ws, stream=stream)
        else:
            pkv.kv_cache_append(self.k_new[layer], self.v_new[layer], self.k[layer], self.v[layer], self.slots,
                                stream=stream)
            pkv.paged_attention_decode(self.out[layer], self.q[layer], self.k[layer], self.v[layer],
                                       self.tables, self.lens, cfg.scale, self.ws, stream=stream)

    def step(self, stream=None):
        """Every layer, in order."""
        for layer in range(self.cfg.n_layers):
            self.layer(layer, stream)


def capture(fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm up outside the graph once (library set-up)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_replays(graph, steps, world):
    dist_barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        graph.replay()
    end.record()
    torch.cuda.synchronize()
    dist_barrier(world)
    return start.elapsed_time(end) / steps


def time_replays_redraw(graph, wl, steps, world):
    """Per-step device time of the graph, with an untimed batch re-draw before each step.

    Returns (mean ms per step, total algorithmic bytes over the timed steps).
    """
    cfg = wl.cfg
    total_ms, total_bytes = 0.0, 0
    dist_barrier(world)
    for _ in range(steps):
        wl.redraw()
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        graph.replay()
        end.record()
        torch.cuda.synchronize()
        total_ms += start.elapsed_time(end)
        lens = [int(c) for c in wl.layout.context_lens]
        total_bytes += layer_bytes(cfg, lens, wl.layout.shares_prefix.tolist(), unique_prefix=True)["total"] * cfg.n_layers
    dist_barrier(world)
    return total_ms / steps, total_bytes


def decode_kernel_duration_ms(wl, reps=5):
    """Average duration of one decode launch (with the fused append when the step uses it), by CUDA events on
    its stream, cycling through the layers."""
    pkv, cfg = wl.pkv, wl.cfg
    stream = torch.cuda.current_stream()
    evs = []
    for _ in range(reps):
        for layer in range(cfg.n_layers):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            if wl.fused:  # rewriting this step's token is idempotent
                pkv.paged_attention_decode_append(wl.out[layer], wl.q[layer], wl.k_new[layer], wl.v_new[layer],
                                                  wl.k[layer], wl.v[layer], wl.slots, wl.tables, wl.lens,
                                                  cfg.scale, wl.ws, stream=stream)
            else:
                pkv.paged_attention_decode(wl.out[layer], wl.q[layer], wl.k[layer], wl.v[layer], wl.tables,
                                           wl.lens, cfg.scale, wl.ws, stream=stream)
            b.record(stream)
            evs.append((a, b))
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) for a, b in evs]
    return sum(times) / len(times), len(times)


def block_moves_measure(wl, peak, reps=10):
    """Whole-block moves over every layer's K and V cache, one launch per call: swap-out staging (gather) and
    swap-in (scatter) of the blocks of a tenth of the batch's sequences, and copy-on-write copies of as many of
    them into free blocks. Algorithmic bytes = every moved block read once and written once. Not part of the
    timed step; the scatter writes back the bytes the gather read, the copies land in blocks no table uses."""
    pkv, cfg, layout = wl.pkv, wl.cfg, wl.layout
    rng = random.Random(cfg.seed)
    lens = layout.context_lens.tolist()
    tables = layout.block_tables
    victims = rng.sample(range(cfg.batch), max(1, cfg.batch // 10))
    ids = [int(x) for b in victims for x in tables[b, :-(-lens[b] // 16)].tolist()]
    used = set(int(x) for x in tables.flatten().tolist() if x >= 0)
    free = [i for i in range(layout.num_blocks) if i not in used]
    caches = [t for layer in range(cfg.n_layers) for t in (wl.k[layer], wl.v[layer])]
    dev = wl.q.device
    blk_bytes = 16 * cfg.Hkv * cfg.D * wl.k[0].element_size()
    ids_d = torch.tensor(ids, dtype=torch.int32, device=dev)
    n_copy = min(len(ids), len(free))
    src_d = ids_d[:n_copy].contiguous()
    dst_d = torch.tensor(free[:n_copy], dtype=torch.int32, device=dev)
    staged = torch.empty((len(caches), len(ids), 16, cfg.Hkv, cfg.D), dtype=wl.k[0].dtype, device=dev)
    flag = torch.zeros(1, dtype=torch.int32, device=dev)
    ops = {"gather": (lambda: pkv.kv_cache_gather_blocks(staged, caches, ids_d, error_flag=flag), len(ids)),
           "scatter": (lambda: pkv.kv_cache_scatter_blocks(caches, staged, ids_d, error_flag=flag), len(ids)),
           "copy": (lambda: pkv.kv_cache_copy_blocks(caches, src_d, dst_d, error_flag=flag), n_copy)}
    res = {"blocks_swapped": len(ids), "blocks_copied": n_copy, "tensors": len(caches), "bytes_per_block": blk_bytes,
           "timing": "CUDA events, mean of %d launches after 2 warm-up launches" % reps}
    stream = torch.cuda.current_stream()
    for name, (fn, n) in ops.items():
        if n == 0:
            continue
        for _ in range(2):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / reps
        gbs = 2 * n * len(caches) * blk_bytes / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 5), "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4)}
    res["status"] = int(flag.item())
    del staged
    return res


def prefill_measure(pkv, device, elem, reps=20, keys=("llama3_8b", "0p5b")):
    """The chunked-prefill workloads: one layer's paged_attention_prefill each, timed with CUDA events.
    Algorithmic flops = 4 * Hq * D per (query, visible token) pair (Q K^T and P V, a multiply-add = 2)."""
    from dataclasses import replace
    peak, kind = measured_tensor_peak()
    res = {}
    for key in keys:
        cfg = replace(workloads.PREFILL_CONFIGS[key], elem=elem)
        layout = workloads.draw_prefill_layout(cfg)
        gen = workloads.device_generator(cfg.seed, device)
        k, v = workloads.make_layer_cache(layout.num_blocks, cfg.Hkv, cfg.D, gen, device, cfg.torch_dtype)
        T = int(layout.query_start[-1])
        q = workloads.random_bf16((T, cfg.Hq, cfg.D), gen, device, cfg.torch_dtype)
        out = torch.empty_like(q)
        tables, lens, qs = (layout.block_tables.to(device), layout.context_lens.to(device),
                            layout.query_start.to(device))
        flag = torch.zeros(1, dtype=torch.int32, device=device)
        pairs = prefill_pairs(layout.context_lens.tolist(), layout.chunk_lens.tolist())
        flops = 4.0 * cfg.Hq * cfg.D * pairs
        stream = torch.cuda.current_stream()

        def one():
            pkv.paged_attention_prefill(out, q, k, v, tables, lens, qs, cfg.chunk, cfg.scale, flag, stream=stream)
        for _ in range(3):
            one()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            one()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / reps
        tf = flops / (ms * 1e-3) / 1e12
        res[key] = {"workload": cfg.name, "bound": "tensor", "achieved": round(tf, 1), "unit": "TFLOP/s",
                    "peak": peak, "peak_kind": kind, "frac": round(tf / peak, 4), "ms": round(ms, 4),
                    "flops_per_launch": flops, "status": int(flag.item()),
                    "arithmetic": (f"mma.sync m16n8k16 {elem} in, fp32 accumulate"
                                   if pkv.get_option(pkv.KV_OPT_PREFILL_PATH) == 2 else
                                   f"tcgen05.mma kind::f16 M=128 {elem} in, fp32 accumulate in tensor memory"),
                    "timing": f"CUDA events, mean of {reps} back-to-back launches after 3 warm-up launches; "
                              f"KV {2 * k.numel() * k.element_size() / 1e6:.0f} MB + q "
                              f"{q.numel() * q.element_size() / 1e6:.0f} MB per launch (L2 126 MB)"}
        del k, v, q, out
    return res


def gpu_local_cpus(device_index: int):
    """The host CPUs nearest the GPU (NVML's CPU affinity), or None."""
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
        words = pynvml.nvmlDeviceGetCpuAffinity(h, (os.cpu_count() + 63) // 64)
        cpus = {w * 64 + bit for w, mask in enumerate(words) for bit in range(64) if (int(mask) >> bit) & 1}
        cpus &= os.sched_getaffinity(0)
        return cpus or None
    except Exception:
        return None


def pinned_near(tensors, device_index: int):
    """Pinned host copies of the tensors, first touched from the CPUs nearest the GPU (NUMA-local pages)."""
    old = os.sched_getaffinity(0)
    near = gpu_local_cpus(device_index)
    try:
        if near:
            os.sched_setaffinity(0, near)
        return [t.cpu().pin_memory() for t in tensors]
    finally:
        if near:
            os.sched_setaffinity(0, old)


def e2e_measure(wl, steps, warmup, world, chunks=4):
    """The same step through the C ABI with host buffers: every step copies its inputs from pinned host
    memory and its outputs back. The copies run on two side streams, pipelined with the layers: the tables,
    lengths and slots, then q, k_new and v_new in `chunks` groups of layers, each ahead of its first launch;
    each layer's output is copied back while later layers run -- as a serving loop would. One CUDA graph.
    The host buffers are pinned pages on the GPU's NUMA node."""
    cfg = wl.cfg
    L = cfg.n_layers
    dev_index = wl.q.device.index or 0
    step_in = {"tables": wl.tables, "lens": wl.lens, "slots": wl.slots}
    layer_in = {"q": wl.q, "k_new": wl.k_new, "v_new": wl.v_new}
    names = list(step_in) + list(layer_in)
    pinned = pinned_near([step_in.get(k, layer_in.get(k)) for k in names] + [wl.out], dev_index)
    host = dict(zip(names, pinned[:-1]))
    host_out = pinned[-1]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = host_out.numel() * host_out.element_size()
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
    per = -(-L // chunks)
    ev_in = [torch.cuda.Event() for _ in range(chunks)]
    ev_done = [torch.cuda.Event() for _ in range(L)]

    def one():
        main = torch.cuda.current_stream()
        h2d_stream.wait_stream(main)
        d2h_stream.wait_stream(main)
        with torch.cuda.stream(h2d_stream):
            for k in step_in:
                step_in[k].copy_(host[k], non_blocking=True)
            for c in range(chunks):
                lo, hi = c * per, min(L, (c + 1) * per)
                for k in layer_in:
                    layer_in[k][lo:hi].copy_(host[k][lo:hi], non_blocking=True)
                ev_in[c].record(h2d_stream)
        for layer in range(L):
            if layer % per == 0:
                main.wait_event(ev_in[layer // per])
            wl.layer(layer)
            ev_done[layer].record(main)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(ev_done[layer])
                host_out[layer].copy_(wl.out[layer], non_blocking=True)
        main.wait_stream(h2d_stream)
        main.wait_stream(d2h_stream)

    g = capture(one)
    for _ in range(warmup):
        g.replay()
    ms = time_replays(g, steps, world)
    return ms, h2d, d2h


class OracleSampler:
    """The float64 oracle on whole layers of the workload (append + attention), on this host's cores."""

    def __init__(self, cfg, layout):
        import oracle
        self.oracle, self.cfg, self.layout = oracle, cfg, layout
        gen = workloads.device_generator(cfg.seed, "cpu")
        self.k, self.v = workloads.make_layer_cache(layout.num_blocks, cfg.Hkv, cfg.D, gen, "cpu", cfg.torch_dtype)
        q, kn, vn = workloads.make_step_inputs(cfg, gen, "cpu", n_layers=1)
        self.q, self.kn, self.vn = q[0], kn[0], vn[0]
        self.slots = layout.slot_mapping().numpy()
        self.tables = layout.block_tables.numpy()
        self.lens = layout.context_lens.numpy()
        lens = [int(c) for c in self.lens]
        self.layer_bytes = layer_bytes(cfg, lens, layout.shares_prefix.tolist(), unique_prefix=True)["total"]
        self.cores = oracle.num_threads()

    def run(self, seconds: float):
        """Whole layers until `seconds` have passed (at least one). Returns (bytes, seconds, seq-layers)."""
        done_bytes, done_layers, t0 = 0, 0, time.perf_counter()
        while True:
            k2, v2 = self.oracle.kv_cache_append(self.k, self.v, self.kn, self.vn, self.slots)
            self.oracle.paged_attention_decode(self.q, k2, v2, self.tables, self.lens, self.cfg.scale,
                                               dtype=self.cfg.elem)
            done_bytes += self.layer_bytes
            done_layers += 1
            if time.perf_counter() - t0 >= seconds:
                break
        return done_bytes, time.perf_counter() - t0, done_layers * self.cfg.batch


def run_profile_step(args, cfg, device):
    """Only the step's graph replays (for ncu): no e2e, no per-kernel timing, no CPU baseline."""
    import paged_kv_cache_470_b200 as pkv
    wl = Workload(cfg, device)
    wl.fused = not args.separate_append
    graph = capture(wl.step)
    for _ in range(args.warmup + args.steps):
        graph.replay()
    torch.cuda.synchronize()
    print(json.dumps({"profile_step": cfg.name, "layers": cfg.n_layers, "replays": args.warmup + args.steps,
                      "status": pkv.read_status(wl.ws)}), flush=True)


def pick_config(args):
    """The workload named by --config, with --layers and --dtype applied."""
    over = {"elem": args.dtype}
    if args.layers:
        over["n_layers"] = args.layers
    return workloads.small_config(args.config, **over)


def run_ours(args, world, rank, local):
    import paged_kv_cache_470_b200 as pkv
    cfg = pick_config(args)
    device = torch.device("cuda", local if world > 1 else 0)
    if args.compute:
        pkv.set_option(pkv.KV_OPT_COMPUTE, {"tensor": 1, "cuda": 2}[args.compute])
    if args.grid:
        pkv.set_option(pkv.KV_OPT_GRID, args.grid)
    if args.combine_kernel:
        pkv.set_option(pkv.KV_OPT_COMBINE, 1)
    if args.head_group:
        pkv.set_option(pkv.KV_OPT_HEAD_GROUP, args.head_group)
    if args.item_cost:
        pkv.set_option(pkv.KV_OPT_ITEM_COST, args.item_cost)
    if args.profile_step:
        return run_profile_step(args, cfg, device)
    if args.profile_prefill:
        r = prefill_measure(pkv, device, cfg.elem, reps=args.steps, keys=(args.profile_prefill,))
        print(json.dumps(r), flush=True)
        return
    wl = Workload(cfg, device, rank)
    wl.fused = not args.separate_append
    lens = [int(c) for c in wl.layout.context_lens]
    share = wl.layout.shares_prefix.tolist()
    lb_logical = layer_bytes(cfg, lens, share, unique_prefix=False)
    lb_unique = layer_bytes(cfg, lens, share, unique_prefix=True)
    step_bytes = lb_unique["total"] * cfg.n_layers

    graph = capture(wl.step)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    redraw = cfg.redraw_fraction > 0
    with ClockSampler(device.index or 0) as clk:
        if redraw:
            ms, timed_bytes = time_replays_redraw(graph, wl, args.steps, world)
            step_bytes = timed_bytes // args.steps
        else:
            ms = time_replays(graph, args.steps, world)
    ms = dist_max(ms, world)
    status = pkv.read_status(wl.ws)

    # the decode kernel alone, for the roofline (on the batch as it stands now)
    lens = [int(c) for c in wl.layout.context_lens]
    lb_unique = layer_bytes(cfg, lens, wl.layout.shares_prefix.tolist(), unique_prefix=True)
    lb_logical = layer_bytes(cfg, lens, wl.layout.shares_prefix.tolist(), unique_prefix=False)
    iso_ms, n_launch = decode_kernel_duration_ms(wl)
    iso_ms = dist_max(iso_ms, world)
    peak, peak_kind = measured_peak()
    kern_bytes = lb_unique["decode_kernel"] + (lb_unique["append"] if wl.fused else 0)
    if wl.fused and not args.combine_kernel:
        # the timed step is nothing but n_layers launches of the decode kernel
        kern_ms = ms / cfg.n_layers
        kern_bytes = step_bytes / cfg.n_layers
        kern_how = "timed step / launches per step (the step holds only this kernel)"
    else:
        kern_ms = iso_ms
        kern_how = "CUDA events around single launches, layers cycled"
    achieved = kern_bytes / (kern_ms * 1e-3) / 1e9
    traffic = profiled_traffic(cfg)

    e2e_ms, h2d, d2h = e2e_measure(wl, max(args.steps // 4, 3), args.warmup, world)
    moves = block_moves_measure(wl, peak)
    prefill = prefill_measure(pkv, device, cfg.elem)
    e2e_ms = dist_max(e2e_ms, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sampler = OracleSampler(cfg, wl.layout)
        b, s, nsl = sampler.run(args.cpu_seconds)
        cpu = {"value": round(b / s / 1e9, 4), "unit": "GB/s", "cores": sampler.cores, "kind": "oracle",
               "seq_layers_per_s": round(nsl / s, 2),
               "sample": f"{nsl // cfg.batch} layer(s) of this workload (all {cfg.batch} sequences, append + "
                         f"attention) in float64 on the host, {s:.1f} s"}

    value = step_bytes * world / (ms * 1e-3) / 1e9
    line = {
        "metric": "decode-attention achieved HBM GB/s (% of B200 peak); seq·layers/sec per step",
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.elem,
        "data": "synthetic",
        "seq_layers_per_s": round(cfg.batch * cfg.n_layers * world / (ms * 1e-3), 1),
        "pct_of_nominal_8TBs": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        "pct_of_measured_hbm": round(100 * value / world / peak, 2),
        "config": {"workload": cfg.name, "config_id": cfg.cid, "elem": cfg.elem, "layers": cfg.n_layers, "batch": cfg.batch,
                   "Hq": cfg.Hq, "Hkv": cfg.Hkv, "D": cfg.D, "block_tokens": 16,
                   "mean_context": round(sum(lens) / len(lens), 1),
                   "kv_bytes_per_step": lb_unique["kv"] * cfg.n_layers,
                   "kv_bytes_per_step_logical": lb_logical["kv"] * cfg.n_layers,
                   "algorithmic_bytes_per_step": step_bytes,
                   "l2": "inputs larger than L2: every step reads all layers' distinct caches "
                         f"({lb_unique['kv'] * cfg.n_layers / 1e9:.2f} GB of KV vs 126 MB L2)",
                   "timing": "CUDA-graph replay of the whole step, CUDA events, max over ranks"
                             + ("; 10% of the batch re-drawn through the block pool before each step (untimed)"
                                if redraw else ""),
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "algorithmic_bytes_per_launch": kern_bytes, "kernel_ms": round(kern_ms, 5),
                     "kernel_ms_how": kern_how,
                     "kernel_ms_single_launch": round(iso_ms, 5), "single_launches_timed": n_launch,
                     "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "frac_of_nominal_8TBs": round(achieved / NOMINAL_HBM_GBS, 4)},
        "e2e": {"value": round(step_bytes * world / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": ("paged_attention_decode_append" if wl.fused else "kv_cache_append + paged_attention_decode")
                       + " per layer; inputs copied host-to-device on a side stream in 4 groups of layers ahead "
                         "of their launches, each layer's output copied back on another behind it, all in one "
                         "CUDA graph; pinned host buffers on the GPU's NUMA node"},
        "gpu_launches": ((1 if wl.fused else 2) + (pkv.get_option(pkv.KV_OPT_COMBINE) == 1))
                        * cfg.n_layers * args.steps,
        "clocks": clk.summary(),
        "device_status": status,
        "cpu_baseline": cpu,
        "block_moves": moves,
        "prefill": prefill,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args, world, rank):
    """The oracle on the host cores, on bounded samples of the same workload."""
    if rank != 0:
        return
    cfg = pick_config(args)
    layout = workloads.draw_layout(cfg)
    total_steps = args.steps + args.warmup
    per_step = max(0.05, min(2.0, args.reference_budget / max(total_steps, 1)))
    sampler = OracleSampler(cfg, layout)
    cores = sampler.cores
    for _ in range(args.warmup):
        sampler.run(0.0)
    b_all = s_all = n_all = 0
    for _ in range(args.steps):
        b, s, n = sampler.run(per_step)
        b_all, s_all, n_all = b_all + b, s_all + s, n_all + n
    value = b_all / s_all / 1e9
    sample = (f"each step: whole layers of this workload (append + attention, all {cfg.batch} sequences) "
              f"for about {per_step:.2f} s")
    line = {"impl": "reference", "metric": "decode-attention achieved HBM GB/s (% of B200 peak); seq·layers/sec per step",
            "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * s_all / args.steps, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "seq_layers_per_s": round(n_all / s_all, 2),
            "config": {"workload": cfg.name, "config_id": cfg.cid, "elem": cfg.elem},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=2, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--compute", choices=["tensor", "cuda"], default=None)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-budget", type=float, default=120.0)
    ap.add_argument("--layers", type=int, default=0, help="use only this many layers (profiling a smaller case)")
    ap.add_argument("--profile-step", action="store_true", help="only replay the step graph (for ncu)")
    ap.add_argument("--profile-prefill", choices=sorted(workloads.PREFILL_CONFIGS), default=None,
                    help="only run the chunked-prefill workload: 3 warm-up and --steps timed launches (for ncu)")
    ap.add_argument("--grid", type=int, default=0, help="decode CTAs per launch (0: one per SM)")
    ap.add_argument("--combine-kernel", action="store_true", help="split-K merge in a separate kernel")
    ap.add_argument("--head-group", type=int, default=0, help="kv heads per work unit (0: auto)")
    ap.add_argument("--item-cost", type=int, default=0,
                    help="work positions charged per work item when dividing work between CTAs (0 auto, -1 none)")
    ap.add_argument("--dtype", choices=["bf16", "fp16"], default="bf16", help="element type of q, K, V and out")
    ap.add_argument("--separate-append", action="store_true",
                    help="append with kv_cache_append, then paged_attention_decode (two launches per layer)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        dist_done(world)


if __name__ == "__main__":
    main()
