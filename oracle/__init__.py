"""Float64 CPU oracle for paged decode attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product library
(``paged_kv_cache_470_b200``) never imports it, and this package imports
nothing from the product: the two share no code.

Contents, each citing the passage it follows:

* :func:`kv_cache_bytes` -- the KV-size closed form of "Module 23: Serving",
  section 23.1 (The Memory Wall), equation Memory_KV, which is also the
  per-token formula of "Scaling LLM serving", section "The KV cache".
* :func:`paged_attention_decode` -- softmax(scale * q K^T) V per query head,
  gathering K/V through the block table ("Module 23: Serving", section 23.4;
  "Designing an LLM serving system", section "Paged attention"), with query
  head h reading kv head h // (Hq // Hkv) ("Scaling LLM serving", section
  "The KV cache", Share key/value heads). Implemented in plain C, float64,
  in ``pagedkv_oracle.c``.
  With ``dtype="fp16"`` the inputs are IEEE binary16 instead of bf16 (2 bytes
  per number for fp16 or bf16: "Module 23: Serving", section 23.1).
* :func:`kv_cache_append` -- the byte-exact scatter of new tokens into their
  block slots, slot = block * 16 + offset ("Module 23: Serving", section 23.4:
  blocks are allocated as the sequence grows).
* :func:`paged_attention_prefill` -- a chunk of new query tokens per
  sequence attending causally over the paged cache ("Module 23: Serving",
  section 23.2, Prefill and Decode; "Designing an LLM serving system",
  section "Scheduling: when prefill meets decode": chunked prefill). A query
  at position p sees tokens 0..p, so it is a decode step over a context of
  p + 1 tokens: the oracle is written as exactly that.
* :func:`sequence_tokens` -- the logical token rows of one sequence, read
  through its block table (step 1 of the attention definition above).
* :func:`copy_blocks`, :func:`gather_blocks`, :func:`scatter_blocks` --
  whole-block moves: the copy of a shared block when sequences diverge
  ("Designing an LLM serving system", section "Paged attention": copy on
  write) and swapping a preempted sequence's blocks out and back in (same
  page, section "Scheduling: when prefill meets decode").
* :class:`RefBlockPool` -- a dictionary model of block allocation with
  reference counts for shared prefixes ("Designing an LLM serving system",
  section "Paged attention": blocks can be shared; "Module 23: Serving",
  Exercise (extend): waste is at most one partly filled block per request).

Parity status: every function here is pinned by ``tests/test_oracle.py``
against closed forms, the pages' printed values, a dense-attention library
routine and invariants. No function is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

BLOCK_TOKENS = 16  # "say 16 tokens" -- Module 23: Serving, section 23.4

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pagedkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2, OpenMP, strict IEEE: no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.oracle_paged_attention_decode.argtypes = [P, P, P, P, P, P, I, P, I, I, I, I, I,
                                                          ctypes.c_double]
            lib.oracle_paged_attention_decode.restype = I
            lib.oracle_paged_attention_decode_fp16.argtypes = lib.oracle_paged_attention_decode.argtypes
            lib.oracle_paged_attention_decode_fp16.restype = I
            lib.oracle_widen.argtypes = [I, ctypes.c_uint16]
            lib.oracle_widen.restype = ctypes.c_double
            lib.oracle_kv_cache_append.argtypes = [P, P, P, P, P, I, I, I, I]
            lib.oracle_kv_cache_append.restype = I
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = I
            _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the oracle's OpenMP loop uses on this host."""
    return int(_load().oracle_num_threads())


def bf16_bits(x) -> np.ndarray:
    """Raw bf16 bit patterns (uint16, C-contiguous) of a CPU bf16 tensor or a uint16 array."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("expected bf16 bit patterns as uint16")
        return np.ascontiguousarray(x)
    import torch  # only for unpacking a bf16 tensor's bits
    if x.dtype != torch.bfloat16:
        raise TypeError(f"expected a bf16 tensor, got {x.dtype}")
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def fp16_bits(x) -> np.ndarray:
    """Raw IEEE binary16 bit patterns (uint16) of a CPU float16 tensor or a uint16 array."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("expected fp16 bit patterns as uint16")
        return np.ascontiguousarray(x)
    import torch
    if x.dtype != torch.float16:
        raise TypeError(f"expected a float16 tensor, got {x.dtype}")
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def widen(kind: str, bits: int) -> float:
    """The C oracle's exact widening of one 16-bit pattern ("bf16" or "fp16") to float64."""
    return float(_load().oracle_widen(1 if kind == "fp16" else 0, int(bits)))


def bf16_bits_to_float64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64 (bf16 is the top half of binary32)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------------------
# Closed form: Module 23: Serving, section 23.1, equation Memory_KV.
# ---------------------------------------------------------------------------
def kv_cache_bytes(n_layers: int, n_kv_heads: int, d_head: int, context_len: int,
                   batch: int, n_bytes: int) -> int:
    """Memory_KV = 2 x n_layers x n_kv_heads x d_head x L x B x n_bytes.

    The leading 2 counts keys and values; L is the context length in tokens and
    B the batch size (Module 23: Serving, section 23.1).
    """
    return 2 * n_layers * n_kv_heads * d_head * context_len * batch * n_bytes


# ---------------------------------------------------------------------------
# Attention oracle (C, float64).
# ---------------------------------------------------------------------------
def paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                           return_weight_sums: bool = False, dtype: str = "bf16"):
    """Reference decode attention in float64.

    q [B,Hq,D], k_cache/v_cache [num_blocks,16,Hkv,D] as bf16 (or, with
    dtype="fp16", float16) tensors or uint16 bit arrays; block_tables [B,W]
    int32; context_lens [B] int32.
    Returns out [B,Hq,D] float64 (and the per-(b,h) softmax weight sums).
    """
    if dtype not in ("bf16", "fp16"):
        raise ValueError("dtype must be 'bf16' or 'fp16'")
    unpack = fp16_bits if dtype == "fp16" else bf16_bits
    qb, kb, vb = unpack(q), unpack(k_cache), unpack(v_cache)
    tables = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
    lens = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    B, Hq, D = qb.shape
    num_blocks, blk, Hkv, Dk = kb.shape
    if blk != BLOCK_TOKENS or Dk != D or vb.shape != kb.shape:
        raise ValueError("cache must be [num_blocks,16,Hkv,D] for both K and V")
    if tables.ndim != 2 or tables.shape[0] != B or lens.shape != (B,):
        raise ValueError("block_tables must be [B,W] and context_lens [B]")
    W = tables.shape[1]
    out = np.empty((B, Hq, D), dtype=np.float64)
    wsum = np.empty((B, Hq), dtype=np.float64)
    fn = _load().oracle_paged_attention_decode_fp16 if dtype == "fp16" else _load().oracle_paged_attention_decode
    rc = fn(_ptr(out), _ptr(wsum), _ptr(qb), _ptr(kb), _ptr(vb),
                                               _ptr(tables), W, _ptr(lens), B, num_blocks,
                                               Hq, Hkv, D, float(scale))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (status {rc})")
    return (out, wsum) if return_weight_sums else out


def _is_fp16(x) -> bool:
    return not isinstance(x, np.ndarray) and str(x.dtype) == "torch.float16"


def paged_attention_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, scale: float,
                            dtype: str = "bf16"):
    """Reference chunked-prefill attention in float64.

    q [T,Hq,D] holds, for sequence b, query_start[b+1] - query_start[b] = n_b
    new tokens (rows query_start[b] ..), at positions c_b - n_b .. c_b - 1 of
    its context (c_b = context_lens[b], the chunk included and already in the
    cache). Token i of the chunk attends to cache positions 0 .. c_b - n_b + i.
    Returns out [T,Hq,D] float64.
    """
    unpack = fp16_bits if dtype == "fp16" else bf16_bits
    qb = unpack(q)
    tables = np.asarray(block_tables, dtype=np.int32)
    lens = np.asarray(context_lens, dtype=np.int64)
    qs = np.asarray(query_start, dtype=np.int64)
    B = tables.shape[0]
    if qs.shape != (B + 1,) or qs[0] != 0 or qs[-1] != qb.shape[0] or (np.diff(qs) < 0).any():
        raise ValueError("query_start must be [B+1], starting at 0, non-decreasing, ending at T")
    rows, ctx = [], []
    for b in range(B):
        n = int(qs[b + 1] - qs[b])
        if n > lens[b]:
            raise ValueError("a chunk longer than its context")
        for i in range(n):
            rows.append(b)
            ctx.append(int(lens[b]) - n + i + 1)   # the query's own position, plus one
    if not rows:
        return np.zeros(qb.shape, dtype=np.float64)
    per_query_tables = np.ascontiguousarray(tables[np.array(rows)])
    return paged_attention_decode(qb, k_cache, v_cache, per_query_tables, np.array(ctx, np.int32), scale,
                                  dtype=dtype)


def kv_cache_append(k_cache, v_cache, k_new, v_new, slot_mapping):
    """Reference append: returns new (k_cache, v_cache) uint16 bit arrays.

    For every i with slot_mapping[i] >= 0, cache[slot // 16][slot % 16] = new[i]
    for all heads, byte for byte; every other byte is unchanged.
    """
    unpack = fp16_bits if _is_fp16(k_cache) else bf16_bits
    kc, vc = unpack(k_cache).copy(), unpack(v_cache).copy()
    kn, vn = unpack(k_new), unpack(v_new)
    slots = np.ascontiguousarray(np.asarray(slot_mapping, dtype=np.int64))
    num_blocks, _, Hkv, D = kc.shape
    T = slots.shape[0]
    if kn.shape != (T, Hkv, D) or vn.shape != (T, Hkv, D):
        raise ValueError("k_new/v_new must be [T,Hkv,D]")
    rc = _load().oracle_kv_cache_append(_ptr(kc), _ptr(vc), _ptr(kn), _ptr(vn), _ptr(slots),
                                        T, num_blocks, Hkv, D)
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (status {rc})")
    return kc, vc


# ---------------------------------------------------------------------------
# Reading a sequence through its table, and whole-block moves (numpy).
# ---------------------------------------------------------------------------
def sequence_tokens(cache: np.ndarray, table_row, context_len: int) -> np.ndarray:
    """Rows [c, ...] of one sequence: token t is cache[table_row[t // 16]][t % 16].

    "Designing an LLM serving system", section "Paged attention": logical
    positions map to physical blocks through the sequence's page table.
    """
    out = np.empty((context_len,) + cache.shape[2:], dtype=cache.dtype)
    for t in range(context_len):
        out[t] = cache[int(table_row[t // BLOCK_TOKENS])][t % BLOCK_TOKENS]
    return out


def copy_blocks(cache: np.ndarray, src_ids, dst_ids) -> np.ndarray:
    """A new cache with block dst_ids[i] replaced by block src_ids[i] (all read before any write)."""
    src_ids, dst_ids = list(src_ids), list(dst_ids)
    if len(src_ids) != len(dst_ids):
        raise ValueError("src_ids and dst_ids differ in length")
    out = cache.copy()
    for s, d in zip(src_ids, dst_ids):
        out[d] = cache[s]
    return out


def gather_blocks(cache: np.ndarray, ids) -> np.ndarray:
    """Blocks ids[0], ids[1], ... stacked in that order (swap-out staging)."""
    return np.stack([cache[i] for i in ids]) if len(ids) else np.empty((0,) + cache.shape[1:], cache.dtype)


def scatter_blocks(cache: np.ndarray, data: np.ndarray, ids) -> np.ndarray:
    """A new cache with block ids[i] replaced by data[i] (swap-in)."""
    out = cache.copy()
    for i, b in enumerate(ids):
        out[b] = data[i]
    return out


# ---------------------------------------------------------------------------
# Block-pool model (host bookkeeping), a plain dictionary state machine.
# ---------------------------------------------------------------------------
class RefBlockPool:
    """Blocks with reference counts.

    * alloc(n): n fresh blocks, each with refcount 1, or nothing at all if fewer
      than n are free (allocation as the sequence grows, Module 23: Serving,
      section 23.4).
    * incref(ids): one more sequence points at these blocks (shared prefix,
      Designing an LLM serving system, section "Paged attention").
    * free(ids): one fewer; a block returns to the free set at refcount 0.
      Decrementing a free block is an error.
    """

    def __init__(self, num_blocks: int):
        self.num_blocks = num_blocks
        self.refcount = {i: 0 for i in range(num_blocks)}

    def num_free(self) -> int:
        return sum(1 for r in self.refcount.values() if r == 0)

    def alloc(self, n: int):
        free = [i for i, r in self.refcount.items() if r == 0]
        if n < 0:
            raise ValueError("negative count")
        if n > len(free):
            return None
        return free[:n]

    def take(self, ids):
        """Mark ids (chosen by the pool under test) as allocated; they must be free."""
        for i in ids:
            if self.refcount[i] != 0:
                raise AssertionError(f"block {i} handed out twice")
            self.refcount[i] = 1

    def incref(self, ids) -> bool:
        if any(self.refcount.get(i, 0) <= 0 for i in ids):
            return False
        for i in ids:
            self.refcount[i] += 1
        return True

    def free(self, ids) -> bool:
        need = {}
        for i in ids:
            need[i] = need.get(i, 0) + 1
        if any(i not in self.refcount or self.refcount[i] < k for i, k in need.items()):
            return False
        for i in ids:
            self.refcount[i] -= 1
        return True


def blocks_needed(context_len: int) -> int:
    """Blocks a sequence of this many tokens occupies: ceil(c / 16).

    "Module 23: Serving", Exercise (extend): unused space is at most one partly
    filled block per request.
    """
    return -(-context_len // BLOCK_TOKENS)
