"""A batch of sequences living in a paged KV pool, kept by the C++ block pool.

Host bookkeeping only (no kernels): which physical blocks each sequence owns,
reference counts for a prefix that several sequences share ("Designing an LLM
serving system", sections "Paged attention" and "Caching and shortcuts":
sequences sharing a prompt point at the same physical blocks), and a per-step
re-draw of the batch in which some sequences finish and new ones take their
place ("Module 23: Serving", section 23.3: the batch is re-formed every step).

The tables this class writes are what `paged_attention_decode` reads; their
content, not the class, is the interface.
"""
from __future__ import annotations

import torch

from . import BlockPool
from .workloads import BLOCK_TOKENS, DecodeConfig, cpu_generator, draw_one_length


class ContinuousBatch:
    """B sequences in a pool of `num_blocks` blocks, optionally sharing one prefix.

    Sequence b caches context_lens[b] tokens (this step's token included) in
    blocks block_tables[b, :ceil(c/16)]; a sequence that shares the prefix has
    the prefix's blocks first, each referenced once per sharing sequence plus
    once by the batch itself (so the prefix outlives any one sequence).
    """

    def __init__(self, cfg: DecodeConfig, num_blocks: int, seed: int | None = None):
        self.cfg = cfg
        self.gen = cpu_generator(cfg.seed if seed is None else seed)
        self.pool = BlockPool(num_blocks)
        # hand blocks out in a shuffled physical order
        everything = self.pool.alloc(num_blocks)
        order = torch.randperm(num_blocks, generator=self.gen).tolist()
        self.pool.free([everything[i] for i in order])
        self.block_tables = torch.full((cfg.batch, cfg.W), -1, dtype=torch.int32)
        self.context_lens = torch.zeros(cfg.batch, dtype=torch.int32)
        self.shares = torch.zeros(cfg.batch, dtype=torch.bool)
        self.prefix: list[int] = []
        n_prefix = cfg.shared_prefix_tokens // BLOCK_TOKENS if cfg.shared_prefix_tokens else 0
        if n_prefix:
            self.prefix = self.pool.alloc(n_prefix)      # the batch's own reference
        for b in range(cfg.batch):
            self._admit(b)

    # ------------------------------------------------------------------
    def _draw_share(self) -> bool:
        if not self.prefix:
            return False
        return bool(torch.rand(1, generator=self.gen).item() < self.cfg.shared_fraction)

    def _admit(self, b: int) -> None:
        share = self._draw_share()
        c = draw_one_length(self.cfg, self.gen, share)
        nb = -(-c // BLOCK_TOKENS)
        row = []
        if share:
            self.pool.incref(self.prefix)
            row += self.prefix
        row += self.pool.alloc(nb - len(row))
        self.block_tables[b] = -1
        self.block_tables[b, :nb] = torch.tensor(row, dtype=torch.int32)
        self.context_lens[b] = c
        self.shares[b] = share

    def _release(self, b: int) -> None:
        nb = -(-int(self.context_lens[b]) // BLOCK_TOKENS)
        self.pool.free(self.block_tables[b, :nb].tolist())
        self.block_tables[b] = -1
        self.context_lens[b] = 0

    def redraw(self, fraction: float | None = None) -> list[int]:
        """Free a random `fraction` of the sequences and admit new ones in their rows."""
        frac = self.cfg.redraw_fraction if fraction is None else fraction
        k = int(round(frac * self.cfg.batch))
        rows = torch.randperm(self.cfg.batch, generator=self.gen)[:k].tolist()
        for b in rows:
            self._release(b)
        for b in rows:
            self._admit(b)
        return rows

    # ------------------------------------------------------------------
    @property
    def num_blocks(self) -> int:
        return self.pool.num_blocks()

    @property
    def shares_prefix(self) -> torch.Tensor:
        return self.shares

    def slot_mapping(self) -> torch.Tensor:
        """Slot of each sequence's newest token (position c - 1)."""
        lens = self.context_lens.to(torch.int64)
        pos = lens - 1
        blk = torch.gather(self.block_tables.to(torch.int64), 1, (pos // BLOCK_TOKENS).unsqueeze(1)).squeeze(1)
        return blk * BLOCK_TOKENS + pos % BLOCK_TOKENS

    def unique_blocks(self) -> int:
        return self.pool.num_blocks() - self.pool.num_free()

    def check(self) -> None:
        """Pool invariants: refcount of every block == references from the batch."""
        refs = {}
        for b in range(self.cfg.batch):
            nb = -(-int(self.context_lens[b]) // BLOCK_TOKENS)
            for i in self.block_tables[b, :nb].tolist():
                refs[i] = refs.get(i, 0) + 1
        for i in self.prefix:
            refs[i] = refs.get(i, 0) + 1
        for i in range(self.pool.num_blocks()):
            assert self.pool.refcount(i) == refs.get(i, 0), (i, self.pool.refcount(i), refs.get(i, 0))
