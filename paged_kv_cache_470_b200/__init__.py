"""Python binding of libpagedkv.so (the C ABI declared in include/pagedkv.h).

Argument marshalling only: every step of a decode (append, attention, split-K
merge) runs in the library's CUDA kernels, and the block pool runs in its C++
code. PyTorch supplies device memory and the stream. There is no fallback: the
library is loaded by the first call that needs it (or by ``load()``), and if
the shared library is missing that call raises ImportError. Importing the
package alone maps no library, so that its seeded input generator
(``workloads``) can serve code that must not load it.

Build it with ``python paged_kv_cache_470_b200/build.py``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

KV_OK, KV_ERR_ARG, KV_ERR_OOM, KV_ERR_STATE, KV_ERR_CUDA = 0, -1, -2, -3, -4
KV_DTYPE_BF16, KV_DTYPE_FP16 = 0, 1
BLOCK_TOKENS = 16
KV_STATUS_BAD_BLOCK_ID, KV_STATUS_BAD_CONTEXT, KV_STATUS_WAIT_TIMEOUT, KV_STATUS_BAD_SLOT = 1, 2, 4, 8
KV_OPT_COMPUTE, KV_OPT_COMBINE, KV_OPT_GRID, KV_OPT_MIN_CHUNK, KV_OPT_PRODUCER_LANES, KV_OPT_HEAD_GROUP = (
    1, 2, 3, 4, 5, 6)
KV_OPT_ITEM_COST, KV_OPT_PREFILL_PATH, KV_OPT_TEST_DROP_LOAD = 7, 8, 9
KV_OPT_TEST_SLOW_SOFTMAX = 10
KV_OPT_OUT_F32 = 11
KV_OPT_L2_POLICY = 12
KV_OPT_EARLY_LOADS = 13
COMPUTE_AUTO, COMPUTE_TENSOR_CORES, COMPUTE_CUDA_CORES = 0, 1, 2

_P, _I, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_sig = {
    "kv_cache_append": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "paged_attention_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "paged_attention_workspace_init": (_I, [_P, _SZ, _P]),
    "paged_attention_decode": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P, _SZ,
                                    _P]),
    "paged_attention_decode_append": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, ctypes.c_float,
                                           _I, _P, _SZ, _P]),
    "paged_attention_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, ctypes.c_float, _I,
                                            _P]),
    "paged_attention_workspace_size_layers": (_SZ, [_I, _I, _I, _I, _I]),
    "paged_attention_decode_layers": (_I, [_P, _P, _P, _P, _P, _P, _SZ, _I, _P, _P, _I, _P, _I, _I, _I, _I, _I,
                                           ctypes.c_float, _I, _P, _SZ, _P]),
    "paged_attention_read_status": (_I, [_P, _P, _I, _P]),
    "paged_attention_prefill": (_I, [_P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P,
                                     _P]),
    "kv_decode_set_option": (_I, [_I, _I]),
    "kv_decode_get_option": (_I, [_I]),
    "kv_pool_create": (_I, [_I, ctypes.POINTER(ctypes.c_void_p)]),
    "kv_pool_destroy": (None, [_P]),
    "kv_pool_alloc": (_I, [_P, _I, _P]),
    "kv_pool_incref": (_I, [_P, _P, _I]),
    "kv_pool_free": (_I, [_P, _P, _I]),
    "kv_pool_num_free": (_I, [_P]),
    "kv_pool_num_blocks": (_I, [_P]),
    "kv_pool_refcount": (_I, [_P, ctypes.c_int32]),
    "kv_pool_append_slots": (_I, [_P, _P, _I, _P, _I, _P]),
    "kv_pool_fork": (_I, [_P, _P, _I, _P]),
    "kv_pool_append_slots_cow": (_I, [_P, _P, _I, _P, _I, _P, _P, _P, ctypes.POINTER(ctypes.c_int)]),
    "kv_cache_copy_blocks": (_I, [_P, _I, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    "kv_cache_gather_blocks": (_I, [_P, _P, _I, _P, _I, _I, _I, _I, _I, _P, _P]),
    "kv_cache_scatter_blocks": (_I, [_P, _I, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
}
EXPORTED = tuple(_sig)
_handle = None


def load() -> ctypes.CDLL:
    """The library, loaded on first use with every call's signature set; ImportError if it is missing."""
    global _handle
    if _handle is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python paged_kv_cache_470_b200/build.py`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _handle = lib
    return _handle


class _Lib:
    """Attribute access loads the library (so `_lib.call(...)` reads as a direct call)."""

    def __getattr__(self, name):
        return getattr(load(), name)


_lib = _Lib()


class KVError(RuntimeError):
    def __init__(self, call: str, status: int):
        names = {KV_ERR_ARG: "KV_ERR_ARG", KV_ERR_OOM: "KV_ERR_OOM", KV_ERR_STATE: "KV_ERR_STATE",
                 KV_ERR_CUDA: "KV_ERR_CUDA"}
        super().__init__(f"{call} failed: {names.get(status, status)}")
        self.status = status


def _check(call: str, status: int) -> None:
    if status != KV_OK:
        raise KVError(call, status)


def _stream_handle(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream or None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream or None
    return int(stream) or None


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


# ---------------------------------------------------------------------------
# kernels
# ---------------------------------------------------------------------------
def kv_cache_append(k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                    slot_mapping: torch.Tensor, error_flag: torch.Tensor | None = None, stream=None) -> None:
    """Scatter k_new/v_new [T,Hkv,D] into the caches [num_blocks,16,Hkv,D] at slot_mapping [T] (int64).

    All four tensors are bfloat16, or all float16.
    """
    T, Hkv, D = k_new.shape
    num_blocks = k_cache.shape[0]
    dt, code = k_cache.dtype, _cache_dtype(k_cache)
    ef = _dev(error_flag, "error_flag", torch.int32) if error_flag is not None else None
    _check("kv_cache_append", _lib.kv_cache_append(
        _dev(k_new, "k_new", dt), _dev(v_new, "v_new", dt),
        _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        _dev(slot_mapping, "slot_mapping", torch.int64), T, num_blocks, Hkv, D, code, ef,
        _stream_handle(stream)))


def workspace_size(B: int, Hq: int, Hkv: int, D: int) -> int:
    n = _lib.paged_attention_workspace_size(B, Hq, Hkv, D)
    if n == 0:
        raise KVError("paged_attention_workspace_size", KV_ERR_ARG)
    return int(n)


def workspace_size_layers(B: int, Hq: int, Hkv: int, D: int, num_layers: int) -> int:
    n = _lib.paged_attention_workspace_size_layers(B, Hq, Hkv, D, num_layers)
    if n == 0:
        raise KVError("paged_attention_workspace_size_layers", KV_ERR_ARG)
    return int(n)


def make_workspace(B: int, Hq: int, Hkv: int, D: int, device=None, num_layers: int = 1) -> torch.Tensor:
    """A zeroed workspace (uint8) sized for these shapes (and layers per launch) on the current device."""
    return torch.zeros(workspace_size_layers(B, Hq, Hkv, D, num_layers), dtype=torch.uint8,
                       device=device or "cuda")


def _out_dtype(dt: torch.dtype) -> torch.dtype:
    """What `out` must hold: the element type, or float32 while KV_OPT_OUT_F32 is on."""
    return torch.float32 if get_option(KV_OPT_OUT_F32) == 1 else dt


def paged_attention_decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                           block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                           workspace: torch.Tensor, stream=None) -> torch.Tensor:
    """out[B,Hq,D] = softmax(scale * q K^T) V over each sequence's paged cache.

    out, q and the caches are all bfloat16, or all float16.
    """
    B, Hq, D = q.shape
    num_blocks, _, Hkv, Dk = k_cache.shape
    if Dk != D or tuple(out.shape) != (B, Hq, D) or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("shape mismatch")
    dt, code = k_cache.dtype, _cache_dtype(k_cache)
    _check("paged_attention_decode", _lib.paged_attention_decode(
        _dev(out, "out", _out_dtype(dt)), _dev(q, "q", dt),
        _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), B, num_blocks, Hq, Hkv, D, float(scale), code,
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_handle(stream)))
    return out


def paged_attention_decode_append(out: torch.Tensor, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                                  k_cache: torch.Tensor, v_cache: torch.Tensor, slot_mapping: torch.Tensor,
                                  block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                                  workspace: torch.Tensor, stream=None) -> torch.Tensor:
    """kv_cache_append of this step's token (the last of each sequence) fused into the decode."""
    B, Hq, D = q.shape
    num_blocks, _, Hkv, Dk = k_cache.shape
    if Dk != D or tuple(out.shape) != (B, Hq, D) or tuple(k_new.shape) != (B, Hkv, D):
        raise ValueError("shape mismatch")
    dt, code = k_cache.dtype, _cache_dtype(k_cache)
    _check("paged_attention_decode_append", _lib.paged_attention_decode_append(
        _dev(out, "out", _out_dtype(dt)), _dev(q, "q", dt),
        _dev(k_new, "k_new", dt), _dev(v_new, "v_new", dt),
        _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        _dev(slot_mapping, "slot_mapping", torch.int64),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), B, num_blocks, Hq, Hkv, D, float(scale), code,
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_handle(stream)))
    return out


def paged_attention_decode_layers(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                  block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                                  workspace: torch.Tensor, k_new: torch.Tensor | None = None,
                                  v_new: torch.Tensor | None = None, slot_mapping: torch.Tensor | None = None,
                                  stream=None) -> torch.Tensor:
    """Every layer of a decode step in one launch: out[l] = decode of q[l] over layer l's caches.

    q, out [L,B,Hq,D] and k_new, v_new [L,B,Hkv,D] contiguous; k_cache, v_cache [L,num_blocks,16,Hkv,D] whose
    layers may sit any equal stride apart (each layer contiguous), e.g. views of one larger pool. With k_new,
    v_new and slot_mapping given, this step's token of every sequence is appended to every layer first (fused).
    The workspace must be sized for L layers (make_workspace(..., num_layers=L)).
    """
    L, B, Hq, D = q.shape
    Lk, num_blocks, bt, Hkv, Dk = k_cache.shape
    if (Lk != L or Dk != D or bt != BLOCK_TOKENS or tuple(out.shape) != (L, B, Hq, D)
            or tuple(v_cache.shape) != tuple(k_cache.shape) or block_tables.dim() != 2 or block_tables.shape[0] != B):
        raise ValueError("shape mismatch")
    if k_cache.stride(0) != v_cache.stride(0) or not (k_cache[0].is_contiguous() and v_cache[0].is_contiguous()):
        raise ValueError("k_cache and v_cache must be layers of contiguous pools at one common stride")
    if (k_new is None) != (v_new is None) or (k_new is None) != (slot_mapping is None):
        raise ValueError("k_new, v_new and slot_mapping come together")
    dt, code = k_cache.dtype, _cache_dtype(k_cache)
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        if not t.is_cuda or t.dtype != dt:
            raise ValueError(f"{name} must be a CUDA {dt} tensor")
    if k_new is not None:
        if tuple(k_new.shape) != (L, B, Hkv, D) or tuple(v_new.shape) != (L, B, Hkv, D):
            raise ValueError("shape mismatch")
        kn, vn = _dev(k_new, "k_new", dt), _dev(v_new, "v_new", dt)
        sm = _dev(slot_mapping, "slot_mapping", torch.int64)
    else:
        kn = vn = sm = None
    stride = k_cache.stride(0) if L > 1 else num_blocks * BLOCK_TOKENS * Hkv * D
    _check("paged_attention_decode_layers", _lib.paged_attention_decode_layers(
        _dev(out, "out", _out_dtype(dt)), _dev(q, "q", dt), kn, vn, k_cache.data_ptr(), v_cache.data_ptr(), stride, L,
        sm, _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), B, num_blocks, Hq, Hkv, D, float(scale), code,
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_handle(stream)))
    return out


def paged_attention_prefill(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                            block_tables: torch.Tensor, context_lens: torch.Tensor, query_start: torch.Tensor,
                            max_query_len: int, scale: float, error_flag: torch.Tensor | None = None,
                            stream=None) -> torch.Tensor:
    """Chunked prefill: rows q[query_start[b]:query_start[b+1]] are the last tokens of sequence b's context;
    each attends causally over the paged cache. q/out [T,Hq,D], query_start [B+1] int32."""
    T, Hq, D = q.shape
    num_blocks, _, Hkv, Dk = k_cache.shape
    B = block_tables.shape[0]
    if Dk != D or tuple(out.shape) != (T, Hq, D) or query_start.numel() != B + 1 or context_lens.numel() != B:
        raise ValueError("shape mismatch")
    dt, code = k_cache.dtype, _cache_dtype(k_cache)
    ef = _dev(error_flag, "error_flag", torch.int32) if error_flag is not None else None
    _check("paged_attention_prefill", _lib.paged_attention_prefill(
        _dev(out, "out", _out_dtype(dt)), _dev(q, "q", dt), _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), _dev(query_start, "query_start", torch.int32), B,
        int(max_query_len), num_blocks, Hq, Hkv, D, float(scale), code, ef, _stream_handle(stream)))
    return out


def _cache_dtype(cache: torch.Tensor) -> int:
    if cache.dtype == torch.bfloat16:
        return KV_DTYPE_BF16
    if cache.dtype == torch.float16:
        return KV_DTYPE_FP16
    raise ValueError(f"cache must be bfloat16 or float16, got {cache.dtype}")


def _cache_list(caches) -> tuple[ctypes.Array, int, tuple]:
    """Host pointer array for a list of same-shape, same-dtype cache tensors [num_blocks,16,Hkv,D]."""
    caches = list(caches)
    if not caches:
        raise ValueError("no caches given")
    shape, dtype = tuple(caches[0].shape), caches[0].dtype
    if len(shape) != 4 or shape[1] != BLOCK_TOKENS:
        raise ValueError("caches must be [num_blocks,16,Hkv,D]")
    for i, c in enumerate(caches):
        if tuple(c.shape) != shape or c.dtype != dtype:
            raise ValueError("caches must share shape and dtype")
        _dev(c, f"caches[{i}]")
    ptrs = (ctypes.c_void_p * len(caches))(*[c.data_ptr() for c in caches])
    return ptrs, len(caches), shape


def kv_cache_copy_blocks(caches, src_ids: torch.Tensor, dst_ids: torch.Tensor,
                         error_flag: torch.Tensor | None = None, stream=None) -> None:
    """caches[c][dst_ids[i]] = caches[c][src_ids[i]] for whole blocks of every cache (copy-on-write).

    ``caches`` is a list of cache tensors (e.g. every layer's K and V); ids are int32 on the device.
    """
    ptrs, nc, (num_blocks, _, Hkv, D) = _cache_list(caches)
    n = src_ids.numel()
    if dst_ids.numel() != n:
        raise ValueError("shape mismatch")
    ef = _dev(error_flag, "error_flag", torch.int32) if error_flag is not None else None
    _check("kv_cache_copy_blocks", _lib.kv_cache_copy_blocks(
        ptrs, nc, _dev(src_ids, "src_ids", torch.int32), _dev(dst_ids, "dst_ids", torch.int32), n,
        num_blocks, Hkv, D, _cache_dtype(caches[0]), ef, _stream_handle(stream)))


def kv_cache_gather_blocks(out: torch.Tensor, caches, block_ids: torch.Tensor,
                           error_flag: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[c,i] = caches[c][block_ids[i]]; out is [len(caches),n,16,Hkv,D] (swap-out staging)."""
    ptrs, nc, (num_blocks, bt, Hkv, D) = _cache_list(caches)
    n = block_ids.numel()
    if tuple(out.shape) != (nc, n, bt, Hkv, D) or out.dtype != caches[0].dtype:
        raise ValueError("shape mismatch")
    ef = _dev(error_flag, "error_flag", torch.int32) if error_flag is not None else None
    _check("kv_cache_gather_blocks", _lib.kv_cache_gather_blocks(
        _dev(out, "out"), ptrs, nc, _dev(block_ids, "block_ids", torch.int32), n, num_blocks, Hkv, D,
        _cache_dtype(caches[0]), ef, _stream_handle(stream)))
    return out


def kv_cache_scatter_blocks(caches, inp: torch.Tensor, block_ids: torch.Tensor,
                            error_flag: torch.Tensor | None = None, stream=None) -> None:
    """caches[c][block_ids[i]] = inp[c,i]; inp is [len(caches),n,16,Hkv,D] (swap-in)."""
    ptrs, nc, (num_blocks, bt, Hkv, D) = _cache_list(caches)
    n = block_ids.numel()
    if tuple(inp.shape) != (nc, n, bt, Hkv, D) or inp.dtype != caches[0].dtype:
        raise ValueError("shape mismatch")
    ef = _dev(error_flag, "error_flag", torch.int32) if error_flag is not None else None
    _check("kv_cache_scatter_blocks", _lib.kv_cache_scatter_blocks(
        ptrs, nc, _dev(inp, "inp"), _dev(block_ids, "block_ids", torch.int32), n, num_blocks, Hkv, D,
        _cache_dtype(caches[0]), ef, _stream_handle(stream)))


def paged_attention_decode_noalloc(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                   block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                                   stream=None) -> torch.Tensor:
    """paged_attention_decode with the library's own fixed scratch instead of a caller workspace.

    Calls that can overlap on the GPU share that scratch: serialise them (one stream, or events)."""
    B, Hq, D = q.shape
    num_blocks, _, Hkv, Dk = k_cache.shape
    if Dk != D or tuple(out.shape) != (B, Hq, D) or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("shape mismatch")
    dt, code = k_cache.dtype, _cache_dtype(k_cache)
    _check("paged_attention_decode_noalloc", _lib.paged_attention_decode_noalloc(
        _dev(out, "out", _out_dtype(dt)), _dev(q, "q", dt), _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
        _dev(context_lens, "context_lens", torch.int32), B, num_blocks, Hq, Hkv, D, float(scale), code,
        _stream_handle(stream)))
    return out


def workspace_init(workspace: torch.Tensor, stream=None) -> None:
    """Zero a workspace on the stream (before first use, and after a call reported KV_STATUS_WAIT_TIMEOUT)."""
    _check("paged_attention_workspace_init", _lib.paged_attention_workspace_init(
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_handle(stream)))


def read_status(workspace: torch.Tensor, clear: bool = True, stream=None) -> int:
    """Synchronise the stream and return (optionally clearing) the device status word."""
    v = ctypes.c_int32(0)
    _check("paged_attention_read_status", _lib.paged_attention_read_status(
        _dev(workspace, "workspace", torch.uint8), ctypes.byref(v), int(clear), _stream_handle(stream)))
    return int(v.value)


def set_option(key: int, value: int) -> None:
    _check("kv_decode_set_option", _lib.kv_decode_set_option(key, value))


def get_option(key: int) -> int:
    return int(_lib.kv_decode_get_option(key))


# ---------------------------------------------------------------------------
# host block pool
# ---------------------------------------------------------------------------
def _i32(a) -> ctypes.Array:
    return (ctypes.c_int32 * len(a))(*[int(x) for x in a])


class BlockPool:
    """Reference-counted physical block ids (host only; owns no device memory)."""

    def __init__(self, num_blocks: int):
        h = ctypes.c_void_p()
        _check("kv_pool_create", _lib.kv_pool_create(num_blocks, ctypes.byref(h)))
        self._h = h

    def close(self) -> None:
        if self._h:
            _lib.kv_pool_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    def alloc(self, n: int) -> list[int]:
        buf = (ctypes.c_int32 * max(n, 1))()
        _check("kv_pool_alloc", _lib.kv_pool_alloc(self._h, n, buf))
        return list(buf[:n])

    def incref(self, ids) -> None:
        ids = list(ids)
        _check("kv_pool_incref", _lib.kv_pool_incref(self._h, _i32(ids), len(ids)))

    def free(self, ids) -> None:
        ids = list(ids)
        _check("kv_pool_free", _lib.kv_pool_free(self._h, _i32(ids), len(ids)))

    def num_free(self) -> int:
        return int(_lib.kv_pool_num_free(self._h))

    def num_blocks(self) -> int:
        return int(_lib.kv_pool_num_blocks(self._h))

    def refcount(self, block_id: int) -> int:
        return int(_lib.kv_pool_refcount(self._h, block_id))

    def append_slots(self, block_tables: torch.Tensor, context_lens: torch.Tensor, slot_mapping: torch.Tensor) -> None:
        """One decode step of bookkeeping on host tensors (int32 [B,W], int32 [B], int64 [B]), in place."""
        for t, name, dt in ((block_tables, "block_tables", torch.int32), (context_lens, "context_lens", torch.int32),
                            (slot_mapping, "slot_mapping", torch.int64)):
            if t.is_cuda or not t.is_contiguous() or t.dtype != dt:
                raise ValueError(f"{name} must be a contiguous host {dt} tensor")
        B, W = block_tables.shape
        _check("kv_pool_append_slots", _lib.kv_pool_append_slots(
            self._h, block_tables.data_ptr(), W, context_lens.data_ptr(), B, slot_mapping.data_ptr()))

    def fork(self, parent_ids) -> list[int]:
        """A child's block ids: the parent's, each with one more reference."""
        ids = list(parent_ids)
        child = (ctypes.c_int32 * max(len(ids), 1))()
        _check("kv_pool_fork", _lib.kv_pool_fork(self._h, _i32(ids), len(ids), child))
        return list(child[:len(ids)])

    def append_slots_cow(self, block_tables: torch.Tensor, context_lens: torch.Tensor,
                         slot_mapping: torch.Tensor) -> tuple[list[int], list[int]]:
        """append_slots that copies a shared partly filled tail block instead of refusing it.

        Returns (src, dst): the blocks to copy, in every layer's caches, before this step's append.
        """
        for t, name, dt in ((block_tables, "block_tables", torch.int32), (context_lens, "context_lens", torch.int32),
                            (slot_mapping, "slot_mapping", torch.int64)):
            if t.is_cuda or not t.is_contiguous() or t.dtype != dt:
                raise ValueError(f"{name} must be a contiguous host {dt} tensor")
        B, W = block_tables.shape
        src = (ctypes.c_int32 * max(B, 1))()
        dst = (ctypes.c_int32 * max(B, 1))()
        n = ctypes.c_int(0)
        _check("kv_pool_append_slots_cow", _lib.kv_pool_append_slots_cow(
            self._h, block_tables.data_ptr(), W, context_lens.data_ptr(), B, slot_mapping.data_ptr(), src, dst,
            ctypes.byref(n)))
        return list(src[:n.value]), list(dst[:n.value])


# ---------------------------------------------------------------------------
# the C ABI's names: each call of include/pagedkv.h under its own name, bound to the marshalling above
# (a pool is a BlockPool, whose handle the kv_pool_* calls take)
# ---------------------------------------------------------------------------
paged_attention_workspace_size = workspace_size
paged_attention_workspace_size_layers = workspace_size_layers
paged_attention_workspace_init = workspace_init
paged_attention_read_status = read_status
kv_decode_set_option = set_option
kv_decode_get_option = get_option
kv_pool_create = BlockPool
kv_pool_destroy = BlockPool.close
kv_pool_alloc = BlockPool.alloc
kv_pool_incref = BlockPool.incref
kv_pool_free = BlockPool.free
kv_pool_num_free = BlockPool.num_free
kv_pool_num_blocks = BlockPool.num_blocks
kv_pool_refcount = BlockPool.refcount
kv_pool_append_slots = BlockPool.append_slots
kv_pool_fork = BlockPool.fork
kv_pool_append_slots_cow = BlockPool.append_slots_cow
