"""Seeded synthetic inputs for paged decode attention.

This module only draws inputs: context lengths, a placement of each sequence's
blocks in a shuffled physical pool, random q/K/V, and the slot each new token
goes to. It holds none of the attention arithmetic and imports neither the
CUDA library nor the oracle, so both sides can be fed from it.

The five workloads follow the shapes of the pages' models:

1. tiny: 1 layer, Hq=20, Hkv=4, D=64, batch 4, context U[1,256], a 128-block
   shuffled pool (the 0.5B model of "Scaling LLM serving", section "The KV
   cache").
2. 0.5B GQA decode step: 24 layers, Hq=20, Hkv=4, D=64 (24 KB of KV per token,
   same section), batch 64, context U[128,2048].
3. LLaMA-3-8B shape: 32 layers, Hq=32, Hkv=8, D=128, batch 32, context
   U[1024,8192] ("Module 23: Serving", section 23.1, worked example).
4. LLaMA-2-7B shape: 32 layers, Hq=Hkv=32, D=128, batch 32, every context 4096
   (64 GiB of KV; "Module 23: Serving", section 23.1 and Exercises).
5. 70B-style continuous-batching mix: 8 layers, Hq=64, Hkv=8, D=128, batch 256,
   lognormal contexts with mean 2000 capped at 8192, half the sequences sharing
   the physical blocks of one 1024-token prefix ("Designing an LLM serving
   system", sections "What it must do" and "Paged attention").

Context length counts the cached tokens after this step's append: the new token
sits at position c - 1 and attention covers positions 0 .. c - 1.

Random numbers: integers (lengths, block placement, re-draws) come from a CPU
``torch.Generator`` seeded with ``470 + config id``; float data (q, K, V, new
K/V) from a generator on the device the tensors live on, seeded the same way
plus a per-tensor offset. Values are N(0, 1) in fp32, rounded to bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

BLOCK_TOKENS = 16


@dataclass(frozen=True)
class DecodeConfig:
    cid: int
    name: str
    n_layers: int
    Hq: int
    Hkv: int
    D: int
    batch: int
    ctx_kind: str                 # "uniform", "fixed" or "lognormal"
    ctx_lo: int
    ctx_hi: int
    W: int                        # table width (max blocks per sequence)
    pool_blocks: int = 0          # 0: just enough blocks plus slack
    shared_prefix_tokens: int = 0
    shared_fraction: float = 0.0
    redraw_fraction: float = 0.0
    lognormal_mean: float = 0.0
    lognormal_sigma: float = 0.0
    elem: str = "bf16"            # element type of q, K, V and out: "bf16" or "fp16"

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float16 if self.elem == "fp16" else torch.bfloat16

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def seed(self) -> int:
        return 470 + self.cid


WORKLOADS = {
    1: DecodeConfig(1, "tiny paged decode (1 layer, Hq=20, Hkv=4, D=64, batch 4, ctx U[1,256], 128-block pool)",
                    1, 20, 4, 64, 4, "uniform", 1, 256, 16, pool_blocks=128),
    2: DecodeConfig(2, "0.5B GQA decode step (24 layers, Hq=20, Hkv=4, D=64, batch 64, ctx U[128,2048])",
                    24, 20, 4, 64, 64, "uniform", 128, 2048, 128),
    3: DecodeConfig(3, "LLaMA-3-8B-shaped decode (32 layers, Hq=32, Hkv=8, D=128, batch 32, ctx U[1024,8192])",
                    32, 32, 8, 128, 32, "uniform", 1024, 8192, 512),
    4: DecodeConfig(4, "LLaMA-2-7B-shaped MHA decode (32 layers, Hq=Hkv=32, D=128, batch 32, ctx 4096)",
                    32, 32, 32, 128, 32, "fixed", 4096, 4096, 256, pool_blocks=8192),
    5: DecodeConfig(5, "70B-style continuous-batching mix (8 layers, Hq=64, Hkv=8, D=128, batch 256, "
                       "lognormal ctx mean 2000 cap 8192, half share a 1024-token prefix, 10% re-drawn per step)",
                    8, 64, 8, 128, 256, "lognormal", 1, 8192, 512,
                    shared_prefix_tokens=1024, shared_fraction=0.5, redraw_fraction=0.1,
                    lognormal_mean=2000.0, lognormal_sigma=0.8),
}


def cpu_generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def device_generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def draw_one_length(cfg: DecodeConfig, gen: torch.Generator, shares_prefix: bool) -> int:
    if cfg.ctx_kind == "fixed":
        c = cfg.ctx_lo
    elif cfg.ctx_kind == "uniform":
        c = int(torch.randint(cfg.ctx_lo, cfg.ctx_hi + 1, (1,), generator=gen).item())
    elif cfg.ctx_kind == "lognormal":
        s = cfg.lognormal_sigma
        mu = math.log(cfg.lognormal_mean) - s * s / 2.0
        x = torch.empty(1, dtype=torch.float64).log_normal_(mu, s, generator=gen).item()
        c = int(min(max(round(x), cfg.ctx_lo), cfg.ctx_hi))
    else:
        raise ValueError(cfg.ctx_kind)
    if shares_prefix:
        # the prefix plus at least one token of its own, so the new token lands in a private block
        c = max(c, cfg.shared_prefix_tokens + 1)
    return c


@dataclass
class BatchLayout:
    """Where every sequence's tokens live in the physical pool (shared by all layers)."""
    cfg: DecodeConfig
    num_blocks: int
    context_lens: torch.Tensor           # [B] int32, CPU
    block_tables: torch.Tensor           # [B, W] int32, CPU; unused entries are -1
    shares_prefix: torch.Tensor          # [B] bool, CPU
    prefix_blocks: list = field(default_factory=list)
    free_blocks: list = field(default_factory=list)   # physical ids not referenced by any table

    def slot_mapping(self) -> torch.Tensor:
        """Slot of each sequence's new token (position c - 1); -1 for an empty sequence."""
        lens = self.context_lens.to(torch.int64)
        pos = (lens - 1).clamp(min=0)
        blk = torch.gather(self.block_tables.to(torch.int64), 1, (pos // BLOCK_TOKENS).unsqueeze(1)).squeeze(1)
        slots = blk * BLOCK_TOKENS + pos % BLOCK_TOKENS
        return torch.where(lens > 0, slots, torch.full_like(slots, -1))

    def blocks_in_use(self) -> int:
        n = sum(-(-int(c) // BLOCK_TOKENS) for c in self.context_lens.tolist())
        if self.prefix_blocks:
            n -= (int(self.shares_prefix.sum()) - 1) * len(self.prefix_blocks) if int(self.shares_prefix.sum()) else 0
        return n


def draw_layout(cfg: DecodeConfig, context_lens=None, seed=None) -> BatchLayout:
    """Draw context lengths and scatter each sequence's blocks over a shuffled pool."""
    gen = cpu_generator(cfg.seed if seed is None else seed)
    B = cfg.batch
    n_share = int(round(B * cfg.shared_fraction)) if cfg.shared_prefix_tokens else 0
    share = torch.zeros(B, dtype=torch.bool)
    if n_share:
        share[torch.randperm(B, generator=gen)[:n_share]] = True
    if context_lens is None:
        lens = [draw_one_length(cfg, gen, bool(share[b])) for b in range(B)]
    else:
        lens = [int(c) for c in context_lens]
    n_prefix = cfg.shared_prefix_tokens // BLOCK_TOKENS if n_share else 0
    need = 0
    for b in range(B):
        nb = -(-lens[b] // BLOCK_TOKENS)
        if nb > cfg.W:
            raise ValueError(f"context {lens[b]} exceeds the table width {cfg.W} blocks")
        need += nb - (n_prefix if share[b] else 0)
    need += n_prefix
    num_blocks = cfg.pool_blocks if cfg.pool_blocks else int(math.ceil(need * 1.08)) + 16
    if need > num_blocks:
        raise ValueError(f"pool of {num_blocks} blocks cannot hold {need}")
    order = torch.randperm(num_blocks, generator=gen).tolist()
    prefix = order[:n_prefix]
    cursor = n_prefix
    tables = torch.full((B, cfg.W), -1, dtype=torch.int32)
    for b in range(B):
        nb = -(-lens[b] // BLOCK_TOKENS)
        own = 0
        if share[b]:
            tables[b, :n_prefix] = torch.tensor(prefix, dtype=torch.int32)
            own = n_prefix
        k = nb - own
        if k > 0:
            tables[b, own:nb] = torch.tensor(order[cursor:cursor + k], dtype=torch.int32)
            cursor += k
    return BatchLayout(cfg, num_blocks, torch.tensor(lens, dtype=torch.int32), tables, share,
                       prefix, order[cursor:])


def random_bf16(shape, gen: torch.Generator, device, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, 1) drawn in fp32 on ``device`` and rounded to bf16 (or to ``dtype``)."""
    x = torch.empty(shape, dtype=torch.float32, device=device)
    x.normal_(0.0, 1.0, generator=gen)
    return x.to(dtype)


def make_layer_cache(num_blocks: int, Hkv: int, D: int, gen: torch.Generator, device, dtype=torch.bfloat16):
    """One layer's K and V pools, [num_blocks, 16, Hkv, D] bf16 (or dtype) each, every byte random."""
    k = random_bf16((num_blocks, BLOCK_TOKENS, Hkv, D), gen, device, dtype)
    v = random_bf16((num_blocks, BLOCK_TOKENS, Hkv, D), gen, device, dtype)
    return k, v


def make_stacked_caches(n_layers: int, num_blocks: int, Hkv: int, D: int, gen: torch.Generator, device,
                        dtype=torch.bfloat16, spare_blocks: int = 0):
    """Every layer's K and V pools in two tensors [n_layers, num_blocks + spare_blocks, 16, Hkv, D], drawn in the
    order of n_layers calls of make_layer_cache (the same values); the spare blocks, if any, hold zeros and sit
    after each layer's pool, so layer l's [:num_blocks] views lie a larger stride apart."""
    shape = (n_layers, num_blocks + spare_blocks, BLOCK_TOKENS, Hkv, D)
    k = torch.zeros(shape, dtype=dtype, device=device)
    v = torch.zeros(shape, dtype=dtype, device=device)
    for layer in range(n_layers):
        kl, vl = make_layer_cache(num_blocks, Hkv, D, gen, device, dtype)
        k[layer, :num_blocks].copy_(kl)
        v[layer, :num_blocks].copy_(vl)
        del kl, vl
    return k[:, :num_blocks], v[:, :num_blocks]


def make_step_inputs(cfg: DecodeConfig, gen: torch.Generator, device, n_layers=None):
    """Per-layer q [B,Hq,D] and new-token K/V [B,Hkv,D], all of the config's element type."""
    L = cfg.n_layers if n_layers is None else n_layers
    dt = cfg.torch_dtype
    q = random_bf16((L, cfg.batch, cfg.Hq, cfg.D), gen, device, dt)
    k_new = random_bf16((L, cfg.batch, cfg.Hkv, cfg.D), gen, device, dt)
    v_new = random_bf16((L, cfg.batch, cfg.Hkv, cfg.D), gen, device, dt)
    return q, k_new, v_new


def small_config(cid: int = 1, **overrides) -> DecodeConfig:
    """A copy of one workload with some fields changed (edge-case and CPU-sized tests)."""
    return replace(WORKLOADS[cid], **overrides)


# ---------------------------------------------------------------------------
# Chunked prefill ("Module 23: Serving", section 23.2; "Designing an LLM serving
# system", section "Scheduling: when prefill meets decode"): each sequence adds a
# chunk of new tokens on top of what it already holds in the cache.
# ---------------------------------------------------------------------------
@dataclass(frozen=True)
class PrefillConfig:
    name: str
    Hq: int
    Hkv: int
    D: int
    batch: int
    chunk: int                    # new tokens per sequence
    prior_lo: int                 # tokens already cached before the chunk: U[prior_lo, prior_hi]
    prior_hi: int
    W: int
    seed: int = 4700
    elem: str = "bf16"

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float16 if self.elem == "fp16" else torch.bfloat16


PREFILL_CONFIGS = {
    "llama3_8b": PrefillConfig("chunked prefill, LLaMA-3-8B shape (Hq=32, Hkv=8, D=128): 16 sequences, "
                               "512-token chunks on U[0,3584] cached tokens, one layer", 32, 8, 128, 16, 512, 0,
                               3584, 256),
    "0p5b": PrefillConfig("chunked prefill, 0.5B GQA shape (Hq=20, Hkv=4, D=64): 16 sequences, "
                          "512-token chunks on U[0,3584] cached tokens, one layer", 20, 4, 64, 16, 512, 0, 3584, 256,
                          seed=4701),
}


@dataclass
class PrefillLayout:
    num_blocks: int
    context_lens: torch.Tensor    # [B] int32, chunk included
    chunk_lens: torch.Tensor      # [B] int32
    query_start: torch.Tensor     # [B+1] int32
    block_tables: torch.Tensor    # [B, W] int32, -1 past each sequence's blocks

    def slot_mapping(self) -> torch.Tensor:
        """int64 slot of every chunk token, in q's row order (for kv_cache_append)."""
        out = []
        for b in range(self.block_tables.shape[0]):
            c, n = int(self.context_lens[b]), int(self.chunk_lens[b])
            for p in range(c - n, c):
                out.append(int(self.block_tables[b, p // BLOCK_TOKENS]) * BLOCK_TOKENS + p % BLOCK_TOKENS)
        return torch.tensor(out, dtype=torch.int64)


def draw_prefill_layout(cfg: PrefillConfig, chunk_lens=None, prior_lens=None, seed=None) -> PrefillLayout:
    """Chunk and prior lengths, and the sequences' blocks scattered over a shuffled pool."""
    gen = cpu_generator(cfg.seed if seed is None else seed)
    B = cfg.batch
    if prior_lens is None:
        prior_lens = torch.randint(cfg.prior_lo, cfg.prior_hi + 1, (B,), generator=gen).tolist()
    if chunk_lens is None:
        chunk_lens = [cfg.chunk] * B
    lens = [int(p) + int(n) for p, n in zip(prior_lens, chunk_lens)]
    need = sum(-(-c // BLOCK_TOKENS) for c in lens)
    num_blocks = max(1, int(need * 1.08) + 16)
    perm = torch.randperm(num_blocks, generator=gen).tolist()
    tables = torch.full((B, cfg.W), -1, dtype=torch.int32)
    cur = 0
    for b, c in enumerate(lens):
        nb = -(-c // BLOCK_TOKENS)
        if nb > cfg.W:
            raise ValueError("context longer than the table")
        tables[b, :nb] = torch.tensor(perm[cur:cur + nb], dtype=torch.int32)
        cur += nb
    qs = [0]
    for n in chunk_lens:
        qs.append(qs[-1] + int(n))
    return PrefillLayout(num_blocks, torch.tensor(lens, dtype=torch.int32),
                         torch.tensor([int(n) for n in chunk_lens], dtype=torch.int32),
                         torch.tensor(qs, dtype=torch.int32), tables)
