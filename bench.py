"""Benchmark: one decode step (append + paged attention over every layer) on one or more B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4] [--impl ours|reference]

A step is the whole hot path over one batch: for each layer, scatter the new
token's K/V into its slot, then decode attention over every sequence's paged
cache (with the split-K merge). Inputs are synthetic and seeded, shaped like
the pages' models (see paged_kv_cache_470_b200/workloads.py). The headline
workload is the largest one that fits one GPU: the LLaMA-2-7B-shaped MHA step
(32 layers, Hq = Hkv = 32, D = 128, batch 32, every context 4096: 64 GiB of
KV). The other workloads are measured in the same run under `per_config`.

The step runs as the library's multi-layer call (paged_attention_decode_layers
with the append fused: one launch for all layers, inputs all present). Beside
it, `per_layer` times the same step as one fused append + decode launch per
layer, which is what a transformer forward pays (its layer l + 1 query comes
from layer l's output).

Reported (one JSON line on rank 0):
  value      achieved HBM GB/s = algorithmic bytes of the step / step time,
             summed over GPUs (inputs resident in HBM, CUDA-graph replay)
  e2e        the same metric through the C ABI with host buffers: pinned-host
             -> device copies of the step's inputs and a device -> host copy of
             its outputs inside the timed region
  roofline   the step's kernel: its algorithmic bytes per launch over its
             CUDA-event duration, against the measured HBM copy bandwidth
  per_config the other workloads, each with its own step time, roofline,
             per-layer figures and clock record
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
from dataclasses import replace

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


def profiled_traffic(cfg, launch="layers"):
    """DRAM bytes per launch from a committed ncu summary of this workload, element type and kind of launch
    ("layers": the multi-layer launch, whose summary gives bytes per layer, scaled here to the workload's layer
    count; "per_layer": one layer's launch), if one matches the current kernel source (else None)."""
    try:
        src_hash = hashlib.sha256(open(DECODE_SRC, "rb").read()).hexdigest()[:16]
        for name in sorted(os.listdir(PROFILE_DIR)):
            if not name.endswith(".txt"):
                continue
            text = open(os.path.join(PROFILE_DIR, name)).read()
            h = re.search(r"decode\.cu sha256\[:16\]:\s*([0-9a-f]+)", text)
            c = re.search(r"^config_id:\s*(\d+)", text, re.M)
            e = re.search(r"^elem:\s*(\w+)", text, re.M)
            k = re.search(r"^launch:\s*(\w+)", text, re.M)
            if not (h and c and e and k) or h.group(1) != src_hash or int(c.group(1)) != cfg.cid \
                    or e.group(1) != cfg.elem or k.group(1) != launch:
                continue
            if launch == "layers":
                m = re.search(r"dram_bytes_per_layer:\s*([0-9.eE+]+)", text)
                if m:
                    return float(m.group(1)) * cfg.n_layers
            else:
                m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
                if m:
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
    """One workload resident on the GPU: every layer's K and V pools (two stacked tensors, one view per layer),
    this step's q and new K/V rows of every layer, the tables, lengths and slots, and the outputs."""

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
        self.k_all, self.v_all = workloads.make_stacked_caches(cfg.n_layers, self.layout.num_blocks, cfg.Hkv, cfg.D,
                                                               gen, device, cfg.torch_dtype)
        self.k, self.v = list(self.k_all.unbind(0)), list(self.v_all.unbind(0))
        self.q, self.k_new, self.v_new = workloads.make_step_inputs(cfg, gen, device)
        self.tables = self.layout.block_tables.to(device)
        self.lens = self.layout.context_lens.to(device)
        self.slots = self.layout.slot_mapping().to(device)
        self.out = torch.empty_like(self.q)
        self.ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D, device)                  # per-layer calls
        self.ws_all = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D, device, cfg.n_layers)  # one launch
        self.fused = True

    def redraw(self):
        """Re-form the batch (host bookkeeping) and upload the new tables; not timed."""
        self.layout.redraw()
        self.tables.copy_(self.layout.block_tables)
        self.lens.copy_(self.layout.context_lens)
        self.slots.copy_(self.layout.slot_mapping())

    def layers_call(self, lo=0, hi=None, stream=None, ws=None):
        """Layers lo .. hi - 1 in one launch, the append fused (paged_attention_decode_layers)."""
        hi = self.cfg.n_layers if hi is None else hi
        self.pkv.paged_attention_decode_layers(self.out[lo:hi], self.q[lo:hi], self.k_all[lo:hi], self.v_all[lo:hi],
                                               self.tables, self.lens, self.cfg.scale,
                                               self.ws_all if ws is None else ws, k_new=self.k_new[lo:hi],
                                               v_new=self.v_new[lo:hi], slot_mapping=self.slots, stream=stream)

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
        """The step as the library runs it for inputs that are all present: every layer in one launch."""
        self.layers_call(stream=stream)

    def step_per_layer(self, stream=None):
        """The step as a transformer forward runs it: one launch per layer, in order."""
        for layer in range(self.cfg.n_layers):
            self.layer(layer, stream)

    def free(self):
        for name in ("k_all", "v_all", "k", "v", "q", "k_new", "v_new", "out", "ws", "ws_all"):
            setattr(self, name, None)


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
    res = {"workload": cfg.name, "blocks_swapped": len(ids), "blocks_copied": n_copy, "tensors": len(caches),
           "bytes_per_block": blk_bytes, "timing": "CUDA events, mean of %d launches after 2 warm-up launches" % reps}
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


def prefill_arithmetic(path: int, elem: str) -> str:
    """What the chunked-prefill kernel of KV_OPT_PREFILL_PATH computes with (0 is the default kernel)."""
    if path == 2:
        return f"mma.sync m16n8k16 {elem} in, fp32 accumulate"
    if path == 1:
        return f"tcgen05.mma kind::f16 M=128 N=64 {elem} in, fp32 accumulate in tensor memory; one query tile per CTA"
    return (f"tcgen05.mma kind::f16 M=128 N=128 {elem} in, fp32 accumulate in tensor memory; two query tiles per "
            f"CTA sharing each 128-token K/V tile")


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
                    "arithmetic": prefill_arithmetic(pkv.get_option(pkv.KV_OPT_PREFILL_PATH), elem),
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


def e2e_groups(L: int, cap: int = 8) -> list[tuple[int, int]]:
    """Layer groups for the end-to-end step: sizes 1, 2, 4, ... (below `cap`) at the start and the same
    back down at the end, the layers between in even groups of at most `cap`. Only the first group's inputs
    and the last group's outputs cross to or from the host with no launch to overlap, so those groups are
    one layer each; every group is one launch, so the middle ones are large."""
    cap = max(1, min(cap, L // 2))
    up, nxt = [], 1
    while nxt < cap and 2 * (sum(up) + nxt) <= L - cap:
        up.append(nxt)
        nxt *= 2
    rest = L - 2 * sum(up)
    n_mid = -(-rest // cap)
    sizes = up + [rest // n_mid + (1 if i < rest % n_mid else 0) for i in range(n_mid)] + up[::-1]
    bounds, lo = [], 0
    for sz in sizes:
        bounds.append((lo, lo + sz))
        lo += sz
    assert lo == L and all(hi > lo_ for lo_, hi in bounds)
    return bounds


def e2e_measure(wl, steps, warmup, world):
    """The same step through the C ABI with host buffers: every step copies its inputs from pinned host
    memory and its outputs back. The layers go in groups (e2e_groups: small first and last), each one
    multi-layer launch: the copies run on two side streams, pipelined with the groups (the tables, lengths
    and slots, then q, k_new and v_new of each group ahead of its launch; each group's output copied back
    while later groups run). One CUDA graph. The host buffers are pinned pages on the GPU's NUMA node."""
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
    groups = e2e_groups(L)
    ev_in = [torch.cuda.Event() for _ in groups]
    ev_done = [torch.cuda.Event() for _ in groups]

    def one():
        main = torch.cuda.current_stream()
        h2d_stream.wait_stream(main)
        d2h_stream.wait_stream(main)
        with torch.cuda.stream(h2d_stream):
            for k in step_in:
                step_in[k].copy_(host[k], non_blocking=True)
            for g, (lo, hi) in enumerate(groups):
                for k in layer_in:
                    layer_in[k][lo:hi].copy_(host[k][lo:hi], non_blocking=True)
                ev_in[g].record(h2d_stream)
        for g, (lo, hi) in enumerate(groups):
            main.wait_event(ev_in[g])
            wl.layers_call(lo, hi)
            ev_done[g].record(main)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(ev_done[g])
                host_out[lo:hi].copy_(wl.out[lo:hi], non_blocking=True)
        main.wait_stream(h2d_stream)
        main.wait_stream(d2h_stream)

    g = capture(one)
    for _ in range(warmup):
        g.replay()
    ms = time_replays(g, steps, world)
    del g
    return ms, h2d, d2h, len(groups)


class OracleSampler:
    """The float64 oracle on whole layers (append + attention) of a bounded sample of the workload, on this
    host's cores: all sequences of one layer when that layer's KV is at most `max_layer_bytes`, else the first
    few sequences of a batch drawn with the workload's length law, block placement and shapes."""

    def __init__(self, cfg, layout=None, max_layer_bytes=400e6):
        import oracle
        self.oracle, self.cfg = oracle, cfg
        if layout is None:
            layout = workloads.draw_layout(cfg)
        lens = [int(c) for c in layout.context_lens]
        full_kv = layer_bytes(cfg, lens, layout.shares_prefix.tolist(), unique_prefix=True)["kv"]
        if full_kv > max_layer_bytes:
            nb = max(1, int(cfg.batch * max_layer_bytes / full_kv))
            layout = workloads.draw_layout(replace(cfg, batch=nb, pool_blocks=0))
            self.what = f"{nb} of the {cfg.batch} sequences (a batch of {nb} drawn with the workload's shapes and " \
                        f"length law)"
        else:
            self.what = f"all {cfg.batch} sequences"
        self.layout = layout
        self.batch = len(layout.context_lens)
        gen = workloads.device_generator(cfg.seed, "cpu")
        self.k, self.v = workloads.make_layer_cache(layout.num_blocks, cfg.Hkv, cfg.D, gen, "cpu", cfg.torch_dtype)
        sub = replace(cfg, batch=self.batch)
        q, kn, vn = workloads.make_step_inputs(sub, gen, "cpu", n_layers=1)
        self.q, self.kn, self.vn = q[0], kn[0], vn[0]
        self.slots = layout.slot_mapping().numpy()
        self.tables = layout.block_tables.numpy()
        self.lens = layout.context_lens.numpy()
        lens = [int(c) for c in self.lens]
        self.layer_bytes = layer_bytes(sub, lens, layout.shares_prefix.tolist(), unique_prefix=True)["total"]
        self.cores = oracle.num_threads()

    def run(self, seconds: float):
        """Whole layers until `seconds` have passed (at least one). Returns (bytes, seconds, seq-layers, layers)."""
        done_bytes, done_layers, t0 = 0, 0, time.perf_counter()
        while True:
            k2, v2 = self.oracle.kv_cache_append(self.k, self.v, self.kn, self.vn, self.slots)
            self.oracle.paged_attention_decode(self.q, k2, v2, self.tables, self.lens, self.cfg.scale,
                                               dtype=self.cfg.elem)
            done_bytes += self.layer_bytes
            done_layers += 1
            if time.perf_counter() - t0 >= seconds:
                break
        return done_bytes, time.perf_counter() - t0, done_layers * self.batch, done_layers


def config_record(cfg, layout, world):
    """The `config` object of both arms' lines: the workload's shapes and the bytes of its first step."""
    lens = [int(c) for c in layout.context_lens]
    share = layout.shares_prefix.tolist()
    lb_logical = layer_bytes(cfg, lens, share, unique_prefix=False)
    lb_unique = layer_bytes(cfg, lens, share, unique_prefix=True)
    return {"workload": cfg.name, "config_id": cfg.cid, "elem": cfg.elem, "layers": cfg.n_layers,
            "batch": cfg.batch, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "D": cfg.D, "block_tokens": 16,
            "mean_context": round(sum(lens) / len(lens), 1),
            "kv_bytes_per_step": lb_unique["kv"] * cfg.n_layers,
            "kv_bytes_per_step_logical": lb_logical["kv"] * cfg.n_layers,
            "algorithmic_bytes_per_step": lb_unique["total"] * cfg.n_layers,
            "l2": "inputs larger than L2: every step reads all layers' distinct caches "
                  f"({lb_unique['kv'] * cfg.n_layers / 1e9:.2f} GB of KV vs 126 MB L2)",
            "parallelism": f"replicas x{world}"}


def run_profile_step(args, cfg, device):
    """Only the step's graph replays (for ncu): no e2e, no per-kernel timing, no CPU baseline."""
    import paged_kv_cache_470_b200 as pkv
    wl = Workload(cfg, device)
    wl.fused = not args.separate_append
    graph = capture(wl.step_per_layer if args.per_layer else wl.step)
    for _ in range(args.warmup + args.steps):
        graph.replay()
    torch.cuda.synchronize()
    ws = wl.ws if args.per_layer else wl.ws_all
    print(json.dumps({"profile_step": cfg.name, "layers": cfg.n_layers, "replays": args.warmup + args.steps,
                      "per_layer": bool(args.per_layer), "status": pkv.read_status(ws)}), flush=True)


def pick_config(args, cid=None):
    """The workload named by --config (or cid), with --layers and --dtype applied."""
    over = {"elem": args.dtype}
    if args.layers:
        over["n_layers"] = args.layers
    return workloads.small_config(args.config if cid is None else cid, **over)


def timed_windows(graph, wl, steps, world, min_seconds):
    """Time `steps` replays of the step's graph (the measurement), then repeat windows of the same length until
    about `min_seconds` of replays have run, so that the clock sampler sees the kernels at work. Every rank runs
    the same number of windows (the largest any rank needs). Returns (first window's ms per step, all windows'
    ms per step, bytes per step of the first window or None)."""
    redraw = wl.cfg.redraw_fraction > 0

    def window():
        if redraw:
            ms, tb = time_replays_redraw(graph, wl, steps, world)
            return ms, tb // steps
        return time_replays(graph, steps, world), None

    first, step_bytes = window()
    more = max(0, math.ceil(min_seconds * 1e3 / max(first * steps, 1e-3)) - 1)
    more = min(199, int(dist_max(float(more), world)))
    windows = [first] + [window()[0] for _ in range(more)]
    return first, windows, step_bytes


def roofline(step_bytes, ms, launches, peak, peak_kind, traffic, how):
    kern_ms = ms / launches
    achieved = step_bytes / launches / (kern_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "algorithmic_bytes_per_launch": step_bytes / launches, "kernel_ms": round(kern_ms, 5),
            "kernel_ms_how": how, "peak_kind": f"{peak_kind} HBM copy bandwidth",
            "frac_of_nominal_8TBs": round(achieved / NOMINAL_HBM_GBS, 4)}


def measure_config(args, cfg, device, world, rank, headline):
    """One workload: the multi-layer step (the line's figures) and the per-layer step beside it, each a CUDA
    graph timed over --steps replays with CUDA events; clocks sampled while they run. With `headline`, also the
    e2e figure, the block moves and the workload object handed back for the CPU baseline."""
    import paged_kv_cache_470_b200 as pkv
    wl = Workload(cfg, device, rank)
    wl.fused = not args.separate_append
    peak, peak_kind = measured_peak()
    cfg_rec = config_record(cfg, wl.layout, world)
    step_bytes0 = cfg_rec["algorithmic_bytes_per_step"]
    combine = pkv.get_option(pkv.KV_OPT_COMBINE) == 1
    res = {}
    early_default = pkv.get_option(pkv.KV_OPT_EARLY_LOADS)
    for name, fn, launches in (("layers", wl.step, 1 + combine),
                               ("per_layer", wl.step_per_layer,
                                cfg.n_layers * ((1 if wl.fused else 2) + combine))):
        # Per layer, the launch before layer l's is layer l-1's (its own cache) or, for layer 0, the previous
        # step's last layer: none writes the caches that the launch reads, so the per-layer step may start its
        # first tile loads early. The multi-layer launch follows the previous step's launch over the same caches
        # (it appended rows to them), so it may not.
        pkv.set_option(pkv.KV_OPT_EARLY_LOADS, 1 if (name == "per_layer" and wl.fused) else early_default)
        graph = capture(fn)
        pkv.set_option(pkv.KV_OPT_EARLY_LOADS, early_default)
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        with ClockSampler(device.index or 0, period_s=0.002) as clk:
            ms, windows, tb = timed_windows(graph, wl, args.steps, world, args.clock_window_s)
        ms = dist_max(ms, world)
        step_bytes = tb if tb is not None else step_bytes0
        status = pkv.read_status(wl.ws_all if name == "layers" else wl.ws)
        del graph
        res[name] = {"ms": ms, "windows": windows, "step_bytes": step_bytes, "clocks": clk.summary(),
                     "status": status, "launches": launches}
    ml, pl = res["layers"], res["per_layer"]
    traffic = profiled_traffic(cfg)
    kernel_of_step = (combine == 0)
    how_ml = ("timed step / 1 (the step is one launch of the multi-layer kernel)" if kernel_of_step else
              "timed step / launches (decode and combine kernels)")
    rec = {
        "ms_per_step": round(ml["ms"], 5),
        "value": round(ml["step_bytes"] * world / (ml["ms"] * 1e-3) / 1e9, 2),
        "unit": "GB/s",
        "seq_layers_per_s": round(cfg.batch * cfg.n_layers * world / (ml["ms"] * 1e-3), 1),
        "pct_of_nominal_8TBs": round(100 * ml["step_bytes"] / (ml["ms"] * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 2),
        "pct_of_measured_hbm": round(100 * ml["step_bytes"] / (ml["ms"] * 1e-3) / 1e9 / peak, 2),
        "config": cfg_rec,
        "roofline": roofline(ml["step_bytes"], ml["ms"], ml["launches"], peak, peak_kind, traffic, how_ml),
        "windows_ms_per_step": {"n": len(ml["windows"]), "median": round(statistics.median(ml["windows"]), 5),
                                "min": round(min(ml["windows"]), 5), "max": round(max(ml["windows"]), 5)},
        "clocks": ml["clocks"],
        "device_status": ml["status"],
        "per_layer": {
            "api": ("paged_attention_decode_append per layer with KV_OPT_EARLY_LOADS (the launch before each "
                    "reads no cache it writes)" if wl.fused else "kv_cache_append + paged_attention_decode per layer")
                   + ", in a CUDA graph with programmatic dependent launch",
            "ms_per_step": round(pl["ms"], 5),
            "value": round(pl["step_bytes"] * world / (pl["ms"] * 1e-3) / 1e9, 2),
            "pct_of_nominal_8TBs": round(100 * pl["step_bytes"] / (pl["ms"] * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 2),
            "roofline": roofline(pl["step_bytes"], pl["ms"], pl["launches"], peak, peak_kind,
                                 profiled_traffic(cfg, "per_layer") if wl.fused and not combine else None,
                                 "timed step / launches per step (the step holds only these launches)"),
            "windows_ms_per_step": {"n": len(pl["windows"]), "median": round(statistics.median(pl["windows"]), 5)},
            "clocks": pl["clocks"],
            "device_status": pl["status"],
        },
        "gpu_launches": ml["launches"] * args.steps,
    }
    if cfg.redraw_fraction > 0:
        rec["timing_note"] = "10% of the batch re-drawn through the block pool before each step (untimed)"
    if headline:
        e2e_ms, h2d, d2h, groups = e2e_measure(wl, max(args.steps // 4, 3), args.warmup, world)
        e2e_ms = dist_max(e2e_ms, world)
        rec["e2e"] = {"value": round(ml["step_bytes"] * world / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                      "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "api": f"paged_attention_decode_layers over {groups} groups of layers; inputs copied "
                             "host-to-device on a side stream ahead of each group's launch, each group's output "
                             "copied back on another behind it, all in one CUDA graph; pinned host buffers on "
                             "the GPU's NUMA node"}
        rec["block_moves"] = block_moves_measure(wl, peak)
    wl.free()
    del wl
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def run_ours(args, world, rank, local):
    import paged_kv_cache_470_b200 as pkv
    cfg = pick_config(args)
    device = torch.device("cuda", local if world > 1 else 0)
    if args.compute:
        pkv.set_option(pkv.KV_OPT_COMPUTE, {"tensor": 1, "cuda": 2}[args.compute])
    if args.grid:
        pkv.set_option(pkv.KV_OPT_GRID, args.grid)
    if args.prefill_path:
        pkv.set_option(pkv.KV_OPT_PREFILL_PATH, args.prefill_path)
    if args.combine_kernel:
        pkv.set_option(pkv.KV_OPT_COMBINE, 1)
    if args.head_group:
        pkv.set_option(pkv.KV_OPT_HEAD_GROUP, args.head_group)
    if args.item_cost:
        pkv.set_option(pkv.KV_OPT_ITEM_COST, args.item_cost)
    if args.producer_lanes:
        pkv.set_option(pkv.KV_OPT_PRODUCER_LANES, args.producer_lanes)
    if args.early_loads:
        pkv.set_option(pkv.KV_OPT_EARLY_LOADS, 1)
    if args.l2_policy:
        pkv.set_option(pkv.KV_OPT_L2_POLICY, {"first": 1, "normal": 2, "last": 3}[args.l2_policy])
    if args.profile_step:
        return run_profile_step(args, cfg, device)
    if args.profile_prefill:
        r = prefill_measure(pkv, device, cfg.elem, reps=args.steps, keys=(args.profile_prefill,))
        print(json.dumps(r), flush=True)
        return
    if args.profile_blocks:
        r = block_moves_measure(Workload(cfg, device), measured_peak()[0], reps=args.steps)
        print(json.dumps(r), flush=True)
        return
    torch.cuda.nvtx.range_push(f"workload {cfg.cid}")
    head = measure_config(args, cfg, device, world, rank, headline=True)
    torch.cuda.nvtx.range_pop()
    per_config = {}
    others = [] if args.no_per_config else [int(c) for c in args.per_config.split(",") if c.strip()]
    for cid in others:
        if cid == cfg.cid:
            continue
        torch.cuda.nvtx.range_push(f"workload {cid}")
        per_config[str(cid)] = measure_config(args, pick_config(args, cid), device, world, rank, headline=False)
        torch.cuda.nvtx.range_pop()
    prefill = prefill_measure(pkv, device, cfg.elem) if not args.no_prefill else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sampler = OracleSampler(cfg)
        b, s, nsl, layers = sampler.run(args.cpu_seconds)
        cpu = {"value": round(b / s / 1e9, 4), "unit": "GB/s", "cores": sampler.cores, "kind": "oracle",
               "seq_layers_per_s": round(nsl / s, 2),
               "sample": f"{layers} layer(s) of this workload, each {sampler.what}, append + attention, in "
                         f"float64 on the host, {s:.1f} s"}

    line = {
        "metric": "decode-attention achieved HBM GB/s (% of B200 peak); seq·layers/sec per step",
        "value": head["value"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.elem,
        "data": "synthetic",
        "seq_layers_per_s": head["seq_layers_per_s"],
        "pct_of_nominal_8TBs": head["pct_of_nominal_8TBs"],
        "pct_of_measured_hbm": head["pct_of_measured_hbm"],
        "config": head["config"],
        "timing": "CUDA-graph replay of the whole step (one multi-layer launch), CUDA events, max over ranks; "
                  "the first window of --steps replays; further windows of the same length only to give the "
                  "clock sampler time (their spread is windows_ms_per_step)"
                  + ("; " + head["timing_note"] if "timing_note" in head else ""),
        "roofline": head["roofline"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "windows_ms_per_step": head["windows_ms_per_step"],
        "device_status": head["device_status"],
        "per_layer": head["per_layer"],
        "per_config": per_config,
        "cpu_baseline": cpu,
        "block_moves": head["block_moves"],
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
        b, s, n, _ = sampler.run(per_step)
        b_all, s_all, n_all = b_all + b, s_all + s, n_all + n
    value = b_all / s_all / 1e9
    sample = (f"each step: whole layers of this workload ({sampler.what}, append + attention) for about "
              f"{per_step:.2f} s")
    line = {"impl": "reference", "metric": "decode-attention achieved HBM GB/s (% of B200 peak); seq·layers/sec per step",
            "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * s_all / args.steps, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "seq_layers_per_s": round(n_all / s_all, 2),
            "config": config_record(cfg, layout, world),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=4, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--per-config", default="2,3,5",
                    help="the other workloads measured in the same run (comma-separated ids)")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--clock-window-s", type=float, default=0.25,
                    help="repeat the timed window until this many seconds of replays ran (clock samples)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--compute", choices=["tensor", "cuda"], default=None)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-budget", type=float, default=120.0)
    ap.add_argument("--layers", type=int, default=0, help="use only this many layers (profiling a smaller case)")
    ap.add_argument("--profile-step", action="store_true", help="only replay the step graph (for ncu)")
    ap.add_argument("--per-layer", action="store_true", help="with --profile-step: the per-layer step")
    ap.add_argument("--profile-prefill", choices=sorted(workloads.PREFILL_CONFIGS), default=None,
                    help="only run the chunked-prefill workload: 3 warm-up and --steps timed launches (for ncu)")
    ap.add_argument("--profile-blocks", action="store_true",
                    help="only run the block moves of --config (swap-out gather, swap-in scatter, copies): 2 warm-up "
                         "and --steps timed launches of each (for ncu)")
    ap.add_argument("--grid", type=int, default=0, help="decode CTAs per launch (0: one per SM)")
    ap.add_argument("--prefill-path", type=int, default=0, choices=[0, 1, 2, 3],
                    help="chunked prefill kernel: 0 auto, 1 tcgen05 one query tile per CTA, 2 mma.sync, "
                         "3 tcgen05 two query tiles per CTA")
    ap.add_argument("--combine-kernel", action="store_true", help="split-K merge in a separate kernel")
    ap.add_argument("--head-group", type=int, default=0, help="kv heads per work unit (0: auto)")
    ap.add_argument("--item-cost", type=int, default=0,
                    help="work positions charged per work item when dividing work between CTAs (0 auto, -1 none)")
    ap.add_argument("--producer-lanes", type=int, default=0, choices=[0, 1, 2, 4, 8],
                    help="lanes of the decode producer warp that issue tile loads (0: the library's choice)")
    ap.add_argument("--early-loads", action="store_true",
                    help="KV_OPT_EARLY_LOADS for every call (valid for the per-layer step only)")
    ap.add_argument("--l2-policy", choices=["first", "normal", "last"], default=None,
                    help="L2 priority of the decode kernels' K/V tile loads (default: the library's)")
    ap.add_argument("--dtype", choices=["bf16", "fp16"], default="bf16", help="element type of q, K, V and out")
    ap.add_argument("--separate-append", action="store_true",
                    help="per-layer step: append with kv_cache_append, then paged_attention_decode")
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
