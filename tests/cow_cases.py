"""Forked sequences that share blocks and diverge: drives the pool's fork and
copy-on-write bookkeeping, with the cache writes done by a pluggable backend
(the oracle's numpy moves on the CPU, the library's kernels on the GPU).

What must hold after every step, whatever the backend ("Designing an LLM
serving system", section "Paged attention": shared blocks, copied on write
when sequences diverge):

* every sequence, read through its own table, holds exactly the tokens it
  was given (its prompt, inherited at the fork, then its own);
* each block's reference count equals the number of table entries that
  point at it, and the free count is the rest of the pool;
* a shared partly filled tail with r references, k of which append in this
  step, costs min(k, r - 1) copies (the last appender keeps the block).
"""
from __future__ import annotations

import numpy as np
import torch


def random_bf16_bits(rng: np.random.Generator, shape) -> np.ndarray:
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16)
    return x.view(torch.int16).numpy().view(np.uint16).copy()


class ForkScenario:
    def __init__(self, pkv, n_seqs=5, num_blocks=96, W=10, n_layers=2, Hkv=2, D=8, seed=0):
        self.pool = pkv.BlockPool(num_blocks)
        self.num_blocks, self.W, self.n_layers, self.Hkv, self.D = num_blocks, W, n_layers, Hkv, D
        self.rng = np.random.default_rng(seed)
        self.tables = torch.full((n_seqs, W), -1, dtype=torch.int32)
        self.lens = torch.zeros(n_seqs, dtype=torch.int32)
        self.live = [False] * n_seqs
        # model[layer][kind][seq] = list of token rows [Hkv, D] (uint16 bf16 bits); kind 0 = K, 1 = V
        self.model = [[[[] for _ in range(n_seqs)] for _ in range(2)] for _ in range(n_layers)]
        self.copies_total = 0

    # ---------------------------------------------------------------- steps
    def step(self, active, backend) -> tuple[list[int], list[int]]:
        """One decode step of bookkeeping and cache writes for the sequences in `active`."""
        active = list(active)
        idx = torch.tensor(active, dtype=torch.long)
        sub_t, sub_l = self.tables[idx].clone(), self.lens[idx].clone()
        slots = torch.zeros(len(active), dtype=torch.int64)
        expected = self._expected_copies(active)
        src, dst = self.pool.append_slots_cow(sub_t, sub_l, slots)
        assert len(src) == expected, (len(src), expected)
        self.tables[idx], self.lens[idx] = sub_t, sub_l
        for a in active:
            self.live[a] = True
        if src:
            backend.copy(src, dst)
            self.copies_total += len(src)
        for layer in range(self.n_layers):
            k_new = random_bf16_bits(self.rng, (len(active), self.Hkv, self.D))
            v_new = random_bf16_bits(self.rng, (len(active), self.Hkv, self.D))
            backend.append(layer, slots.numpy(), k_new, v_new)
            for i, a in enumerate(active):
                self.model[layer][0][a].append(k_new[i])
                self.model[layer][1][a].append(v_new[i])
        return src, dst

    def fork(self, parent: int, child: int) -> None:
        assert self.live[parent] and not self.live[child]
        n = -(-int(self.lens[parent]) // 16)
        self.tables[child, :n] = torch.tensor(self.pool.fork(self.tables[parent, :n].tolist()), dtype=torch.int32)
        self.lens[child] = self.lens[parent]
        self.live[child] = True
        for layer in range(self.n_layers):
            for kind in range(2):
                self.model[layer][kind][child] = list(self.model[layer][kind][parent])

    def finish(self, seq: int) -> None:
        n = -(-int(self.lens[seq]) // 16)
        self.pool.free(self.tables[seq, :n].tolist())
        self.tables[seq] = -1
        self.lens[seq] = 0
        self.live[seq] = False
        for layer in range(self.n_layers):
            for kind in range(2):
                self.model[layer][kind][seq] = []

    def _expected_copies(self, active) -> int:
        appenders: dict[int, int] = {}
        for a in active:
            c = int(self.lens[a])
            if c % 16:
                blk = int(self.tables[a, c // 16])
                appenders[blk] = appenders.get(blk, 0) + 1
        return sum(min(k, self.pool.refcount(blk) - 1) for blk, k in appenders.items())

    # --------------------------------------------------------------- checks
    def check(self, oracle_mod, caches) -> None:
        """caches[layer][kind] as uint16 arrays [num_blocks,16,Hkv,D]."""
        refs: dict[int, int] = {}
        for s, live in enumerate(self.live):
            c = int(self.lens[s])
            if not live:
                assert c == 0
                continue
            n = -(-c // 16)
            row = self.tables[s]
            assert (row[:n] >= 0).all() and (row[n:] == -1).all()
            for blk in row[:n].tolist():
                refs[blk] = refs.get(blk, 0) + 1
            for layer in range(self.n_layers):
                for kind in range(2):
                    got = oracle_mod.sequence_tokens(caches[layer][kind], row.numpy(), c)
                    want = np.stack(self.model[layer][kind][s])
                    np.testing.assert_array_equal(got, want, err_msg=f"seq {s} layer {layer} kind {kind}")
        for blk in range(self.num_blocks):
            assert self.pool.refcount(blk) == refs.get(blk, 0), blk
        assert self.pool.num_free() == self.num_blocks - len(refs)

    # ------------------------------------------------------------- schedule
    def run(self, oracle_mod, backend, n_random_steps=40, check_every=1, on_step=None) -> None:
        """A fixed opening (prompt, a 4-way fork inside a partly filled block, partial and full
        divergence), then random steps with forks and finishes."""
        n_seqs = len(self.live)
        for _ in range(37):                        # prompt of sequence 0: 2 full blocks + 5 tokens
            self.step([0], backend)
        for child in (1, 2, 3):
            self.fork(0, child)                    # the 5-token tail block now has 4 references
        self.check(oracle_mod, backend.caches())
        src, _ = self.step([1, 2], backend)        # two diverge: two copies
        assert len(src) == 2
        src, _ = self.step([0, 3], backend)        # the last two on the block: one copy, one keeps it
        assert len(src) == 1
        self.check(oracle_mod, backend.caches())
        for it in range(n_random_steps):
            live = [s for s in range(n_seqs) if self.live[s]]
            r = self.rng.random()
            if r < 0.12 and len(live) < n_seqs:
                child = next(s for s in range(n_seqs) if not self.live[s])
                self.fork(int(self.rng.choice(live)), child)
            elif r < 0.2 and len(live) > 2:
                self.finish(int(self.rng.choice(live)))
            live = [s for s in range(n_seqs) if self.live[s]]
            k = int(self.rng.integers(1, len(live) + 1))
            active = sorted(self.rng.choice(live, size=k, replace=False).tolist())
            self.step(active, backend)
            if on_step is not None:
                on_step(self)
            if (it + 1) % check_every == 0:
                self.check(oracle_mod, backend.caches())
        self.check(oracle_mod, backend.caches())


class OracleBackend:
    """Cache writes by the oracle's numpy block moves and its append."""

    def __init__(self, oracle_mod, scenario: ForkScenario, fill=0x7FC0):
        self.o = oracle_mod
        shape = (scenario.num_blocks, 16, scenario.Hkv, scenario.D)
        self.c = [[np.full(shape, fill, np.uint16) for _ in range(2)] for _ in range(scenario.n_layers)]

    def copy(self, src, dst):
        for layer in self.c:
            for kind in range(2):
                layer[kind] = self.o.copy_blocks(layer[kind], src, dst)

    def append(self, layer, slots, k_new, v_new):
        self.c[layer][0], self.c[layer][1] = self.o.kv_cache_append(self.c[layer][0], self.c[layer][1], k_new, v_new,
                                                                    slots)

    def caches(self):
        return self.c
