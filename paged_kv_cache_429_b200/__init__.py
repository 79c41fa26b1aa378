"""B200 paged-KV-cache decode attention: Python binding of libpa.so.

Argument marshalling only. Every step of the path runs in the CUDA kernels
of libpa.so; PyTorch is used for device memory, streams and dtypes. The
functions carry the names of the C entry points (include/pa.h):

    pa_decode               decode-step attention through block tables
    pa_decode_append        the same with the step's new tokens written to their slots in-kernel
    pa_prefill              chunked causal prefill attention through block tables
    pa_reshape_and_cache    scatter new K/V into cache slots (bf16 / fp8)
    pa_copy_blocks          copy-on-write block copies
    pa_swap_blocks          block copies between the GPU cache and pinned host memory
    pa_decode_no_alloc      split-context decode with the library's fixed scratch
    pa_decode_workspace_size, pa_get_device_error, pa_status_string
    BlockPool               host block pool (pa_pool_*), incl. swap_out / swap_in

Cache layout: [num_blocks][num_kv_heads][16][head_dim], bf16 or
float8_e4m3fn (uint8 is accepted for fp8 bytes).
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

from . import _lib
from ._lib import STATUS_NAMES, LibraryNotBuilt

__all__ = [
    "PA_KV_BF16", "PA_KV_FP8_E4M3", "BLOCK_SIZE", "PagedAttentionError",
    "LibraryNotBuilt", "pa_decode", "pa_decode_append", "pa_decode_no_alloc", "pa_prefill", "pa_reshape_and_cache", "pa_copy_blocks",
    "pa_swap_blocks", "pa_decode_workspace_size", "pa_get_device_error",
    "pa_status_string",
    "BlockPool", "kv_dtype_of",
]

PA_KV_BF16 = 0
PA_KV_FP8_E4M3 = 1
BLOCK_SIZE = 16


class PagedAttentionError(RuntimeError):
    """A non-OK status from libpa.so."""

    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


def _ok(status: int, what: str) -> None:
    if status != 0:
        raise PagedAttentionError(status, what)


def pa_status_string(status: int) -> str:
    return _lib.lib().pa_status_string(status).decode()


def kv_dtype_of(cache: torch.Tensor) -> int:
    if cache.dtype == torch.bfloat16:
        return PA_KV_BF16
    if cache.dtype in (torch.float8_e4m3fn, torch.uint8):
        return PA_KV_FP8_E4M3
    raise TypeError(f"unsupported KV cache dtype {cache.dtype}")


def _stream_ptr(stream: Optional[torch.cuda.Stream], device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _device_of(*tensors: torch.Tensor) -> torch.device:
    """The one CUDA device all CUDA tensors of a call live on.

    The library launches on the calling thread's current device and looks up
    per-device state (the no-alloc scratch, kernel attributes) there, so each
    launching call makes this device current for its duration."""
    devs = {t.device for t in tensors if t.is_cuda}
    if len(devs) != 1:
        raise ValueError(f"the call's CUDA tensors must share one device, got {sorted(map(str, devs))}")
    return devs.pop()


def _need(t: torch.Tensor, name: str, dtypes, ndim: int, cuda: bool = True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")


def pa_decode_workspace_size(num_seqs: int, num_q_heads: int, head_dim: int,
                             max_context_len: int, partition_size: int = -1) -> int:
    return int(_lib.lib().pa_decode_workspace_size(
        num_seqs, num_q_heads, head_dim, max_context_len, partition_size))


def pa_decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
              v_cache: torch.Tensor, block_tables: torch.Tensor,
              context_lens: torch.Tensor, max_context_len: int, sm_scale: float,
              *, k_scale: float = 1.0, v_scale: float = 1.0,
              partition_size: int = -1,
              workspace: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Decode attention (see pa.h): out[S][Hq][D] fp32 is written in place.

    When the split-context path may run and no workspace is given, one is
    allocated with torch for this call.
    """
    _need(out, "out", (torch.float32,), 3)
    _need(q, "q", (torch.bfloat16,), 3)
    _need(k_cache, "k_cache", (torch.bfloat16, torch.float8_e4m3fn, torch.uint8), 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(block_tables, "block_tables", (torch.int32,), 2)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    S, Hq, D = q.shape
    NB, Hkv, B, Dc = k_cache.shape
    if tuple(out.shape) != (S, Hq, D) or Dc != D or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between out, q and the caches")
    if block_tables.shape[0] != S or context_lens.shape[0] != S:
        raise ValueError("block_tables / context_lens must have num_seqs rows")
    if workspace is None and partition_size != 0:
        nbytes = pa_decode_workspace_size(S, Hq, D, max_context_len, partition_size)
        if nbytes:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    ws = () if workspace is None else (workspace,)
    with torch.cuda.device(_device_of(out, q, k_cache, v_cache, block_tables, context_lens, *ws)):
        rc = _lib.lib().pa_decode(
            out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
            kv_dtype_of(k_cache), float(k_scale), float(v_scale),
            block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(),
            int(max_context_len), S, Hq, Hkv, D, B, NB, float(sm_scale),
            int(partition_size), ws_ptr, ws_bytes, _stream_ptr(stream, q.device))
    _ok(rc, "pa_decode")
    return out


def pa_decode_append(out: torch.Tensor, q: torch.Tensor, key: torch.Tensor,
                     value: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                     block_tables: torch.Tensor, context_lens: torch.Tensor,
                     max_context_len: int, sm_scale: float, *, k_scale: float = 1.0,
                     v_scale: float = 1.0, partition_size: int = -1,
                     workspace: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Decode step with the new tokens' cache write fused in (see pa.h):
    key / value bf16 [S][Hkv][D] go to slot L - 1 of each sequence, then the
    decode runs; out[S][Hq][D] fp32 is written in place."""
    _need(out, "out", (torch.float32,), 3)
    _need(q, "q", (torch.bfloat16,), 3)
    _need(key, "key", (torch.bfloat16,), 3)
    _need(value, "value", (torch.bfloat16,), 3)
    _need(k_cache, "k_cache", (torch.bfloat16, torch.float8_e4m3fn, torch.uint8), 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(block_tables, "block_tables", (torch.int32,), 2)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    S, Hq, D = q.shape
    NB, Hkv, B, Dc = k_cache.shape
    if tuple(out.shape) != (S, Hq, D) or Dc != D or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between out, q and the caches")
    if tuple(key.shape) != (S, Hkv, D) or tuple(value.shape) != (S, Hkv, D):
        raise ValueError("key / value must be [num_seqs][num_kv_heads][head_dim]")
    if block_tables.shape[0] != S or context_lens.shape[0] != S:
        raise ValueError("block_tables / context_lens must have num_seqs rows")
    if workspace is None and partition_size != 0:
        nbytes = pa_decode_workspace_size(S, Hq, D, max_context_len, partition_size)
        if nbytes:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    ws = () if workspace is None else (workspace,)
    with torch.cuda.device(_device_of(out, q, key, value, k_cache, v_cache, block_tables,
                                      context_lens, *ws)):
        rc = _lib.lib().pa_decode_append(
            out.data_ptr(), q.data_ptr(), key.data_ptr(), value.data_ptr(), k_cache.data_ptr(),
            v_cache.data_ptr(), kv_dtype_of(k_cache), float(k_scale), float(v_scale),
            block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(),
            int(max_context_len), S, Hq, Hkv, D, B, NB, float(sm_scale), int(partition_size),
            ws_ptr, ws_bytes, _stream_ptr(stream, q.device))
    _ok(rc, "pa_decode_append")
    return out


def pa_decode_no_alloc(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                       v_cache: torch.Tensor, block_tables: torch.Tensor,
                       context_lens: torch.Tensor, max_context_len: int, sm_scale: float,
                       *, k_scale: float = 1.0, v_scale: float = 1.0,
                       partition_size: int = 512,
                       stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Split-context decode with the library's own fixed scratch (see pa.h:
    no allocation; launches needing more than PA_NO_ALLOC_SCRATCH_BYTES are
    refused; calls overlapping on the GPU race on the scratch)."""
    _need(out, "out", (torch.float32,), 3)
    _need(q, "q", (torch.bfloat16,), 3)
    _need(k_cache, "k_cache", (torch.bfloat16, torch.float8_e4m3fn, torch.uint8), 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(block_tables, "block_tables", (torch.int32,), 2)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    S, Hq, D = q.shape
    NB, Hkv, B, Dc = k_cache.shape
    if tuple(out.shape) != (S, Hq, D) or Dc != D or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between out, q and the caches")
    if block_tables.shape[0] != S or context_lens.shape[0] != S:
        raise ValueError("block_tables / context_lens must have num_seqs rows")
    with torch.cuda.device(_device_of(out, q, k_cache, v_cache, block_tables, context_lens)):
        rc = _lib.lib().pa_decode_no_alloc(
            out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
            kv_dtype_of(k_cache), float(k_scale), float(v_scale),
            block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(),
            int(max_context_len), S, Hq, Hkv, D, B, NB, float(sm_scale),
            int(partition_size), _stream_ptr(stream, q.device))
    _ok(rc, "pa_decode_no_alloc")
    return out


def pa_prefill(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
               v_cache: torch.Tensor, block_tables: torch.Tensor,
               query_start: torch.Tensor, context_lens: torch.Tensor,
               max_query_len: int, max_context_len: int, sm_scale: float, *,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Chunked causal prefill attention (see pa.h); out [T][Hq][D] fp32."""
    _need(out, "out", (torch.float32,), 3)
    _need(q, "q", (torch.bfloat16,), 3)
    _need(k_cache, "k_cache", (torch.bfloat16, torch.float8_e4m3fn, torch.uint8), 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(block_tables, "block_tables", (torch.int32,), 2)
    _need(query_start, "query_start", (torch.int32,), 1)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    T, Hq, D = q.shape
    NB, Hkv, B, Dc = k_cache.shape
    S = context_lens.shape[0]
    if tuple(out.shape) != (T, Hq, D) or Dc != D or query_start.shape[0] != S + 1:
        raise ValueError("shape mismatch between out, q, caches and query_start")
    with torch.cuda.device(_device_of(out, q, k_cache, v_cache, block_tables, query_start,
                                      context_lens)):
        rc = _lib.lib().pa_prefill(
            out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
            kv_dtype_of(k_cache), block_tables.data_ptr(), block_tables.shape[1],
            query_start.data_ptr(), context_lens.data_ptr(), int(max_query_len),
            int(max_context_len), S, T, Hq, Hkv, D, B, NB, float(sm_scale),
            _stream_ptr(stream, q.device))
    _ok(rc, "pa_prefill")
    return out


def pa_reshape_and_cache(key: torch.Tensor, value: torch.Tensor,
                         k_cache: torch.Tensor, v_cache: torch.Tensor,
                         slot_mapping: torch.Tensor, *, k_scale: float = 1.0,
                         v_scale: float = 1.0,
                         stream: Optional[torch.cuda.Stream] = None) -> None:
    """Write key/value [T][Hkv][D] (bf16) into their slots of the caches."""
    _need(key, "key", (torch.bfloat16,), 3)
    _need(value, "value", (torch.bfloat16,), 3)
    _need(k_cache, "k_cache", (torch.bfloat16, torch.float8_e4m3fn, torch.uint8), 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(slot_mapping, "slot_mapping", (torch.int64,), 1)
    T, Hkv, D = key.shape
    NB, Hc, B, Dc = k_cache.shape
    if tuple(value.shape) != (T, Hkv, D) or (Hc, Dc) != (Hkv, D) or slot_mapping.shape[0] != T:
        raise ValueError("shape mismatch between key/value, caches and slots")
    with torch.cuda.device(_device_of(key, value, k_cache, v_cache, slot_mapping)):
        rc = _lib.lib().pa_reshape_and_cache(
            key.data_ptr(), value.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
            slot_mapping.data_ptr(), T, Hkv, D, B, NB, kv_dtype_of(k_cache),
            float(k_scale), float(v_scale), _stream_ptr(stream, key.device))
    _ok(rc, "pa_reshape_and_cache")


def pa_copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor,
                   block_pairs: torch.Tensor, *,
                   stream: Optional[torch.cuda.Stream] = None) -> None:
    """Copy-on-write copies; block_pairs is int64 [n][2] (src, dst)."""
    _need(k_cache, "k_cache", (torch.bfloat16, torch.float8_e4m3fn, torch.uint8), 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(block_pairs, "block_pairs", (torch.int64,), 2)
    n = block_pairs.shape[0]
    block_bytes = k_cache[0].numel() * k_cache.element_size()
    with torch.cuda.device(_device_of(k_cache, v_cache, block_pairs)):
        rc = _lib.lib().pa_copy_blocks(
            k_cache.data_ptr(), v_cache.data_ptr(), block_pairs.data_ptr() if n else None,
            n, block_bytes, k_cache.shape[0], _stream_ptr(stream, k_cache.device))
    _ok(rc, "pa_copy_blocks")


def pa_swap_blocks(dst_k: torch.Tensor, dst_v: torch.Tensor, src_k: torch.Tensor,
                   src_v: torch.Tensor, block_pairs: torch.Tensor, *,
                   stream: Optional[torch.cuda.Stream] = None) -> None:
    """dst[dst_id] = src[src_id] for each (src_id, dst_id) pair of
    block_pairs (int64 [n][2]); each cache is on the current CUDA device or
    in pinned host memory (torch ``pin_memory()``)."""
    for name, t in (("dst_k", dst_k), ("dst_v", dst_v), ("src_k", src_k), ("src_v", src_v)):
        _need(t, name, (torch.bfloat16, torch.float8_e4m3fn, torch.uint8), 4, cuda=False)
        if not (t.is_cuda or t.is_pinned()):
            raise ValueError(f"{name} must be on the GPU or in pinned host memory")
    _need(block_pairs, "block_pairs", (torch.int64,), 2, cuda=False)
    if src_k.shape[1:] != dst_k.shape[1:] or src_k.dtype != dst_k.dtype:
        raise ValueError("source and destination caches differ in block geometry")
    n = block_pairs.shape[0]
    block_bytes = src_k[0].numel() * src_k.element_size()
    caches = (dst_k, dst_v, src_k, src_v)
    dev = (_device_of(*caches, block_pairs) if any(t.is_cuda for t in caches)
           else torch.cuda.current_device())
    with torch.cuda.device(dev):
        rc = _lib.lib().pa_swap_blocks(
            dst_k.data_ptr(), dst_v.data_ptr(), src_k.data_ptr(), src_v.data_ptr(),
            block_pairs.data_ptr() if n else None, n, block_bytes, src_k.shape[0],
            dst_k.shape[0], _stream_ptr(stream, dev))
    _ok(rc, "pa_swap_blocks")


def pa_get_device_error() -> int:
    """Synchronise the current device; return and clear its error bits."""
    code = ctypes.c_uint32(0)
    rc = _lib.lib().pa_get_device_error(ctypes.byref(code))
    if rc not in (0, 7):
        raise PagedAttentionError(rc, "pa_get_device_error")
    return int(code.value)


class BlockPool:
    """Host block pool with refcounts and copy-on-write (pa_pool_*)."""

    def __init__(self, num_blocks: int, block_size: int = BLOCK_SIZE,
                 shuffle_seed: Optional[int] = None):
        self._lib = _lib.lib()
        self._h = self._lib.pa_pool_create(num_blocks, block_size)
        if not self._h:
            raise PagedAttentionError(1, "pa_pool_create")
        self.num_blocks = num_blocks
        self.block_size = block_size
        if shuffle_seed is not None:
            _ok(self._lib.pa_pool_shuffle_free(self._h, shuffle_seed & (2**64 - 1)),
                "pa_pool_shuffle_free")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._lib.pa_pool_destroy(h)
            self._h = None

    def add_seq(self, seq_id: int) -> None:
        _ok(self._lib.pa_pool_add_seq(self._h, seq_id), "pa_pool_add_seq")

    def fork(self, parent: int, child: int) -> None:
        _ok(self._lib.pa_pool_fork(self._h, parent, child), "pa_pool_fork")

    def append(self, seq_id: int, n_tokens: int):
        """Returns (slots int64[n_tokens], cow pair (src, dst) or None)."""
        slots = np.empty(max(n_tokens, 0), dtype=np.int64)
        pair = np.zeros(2, dtype=np.int64)
        ncow = ctypes.c_int(0)
        _ok(self._lib.pa_pool_append(self._h, seq_id, n_tokens,
                                     slots.ctypes.data if n_tokens > 0 else None,
                                     pair.ctypes.data, ctypes.byref(ncow)),
            "pa_pool_append")
        return slots, ((int(pair[0]), int(pair[1])) if ncow.value else None)

    def append_decode(self, seq_ids):
        """One token for each listed sequence. Returns (slots int64[n],
        cow pairs int64[k][2])."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        slots = np.empty(n, dtype=np.int64)
        pairs = np.empty((max(n, 1), 2), dtype=np.int64)
        ncow = ctypes.c_int(0)
        _ok(self._lib.pa_pool_append_decode(self._h, ids.ctypes.data if n else None, n,
                                            slots.ctypes.data if n else None,
                                            pairs.ctypes.data, ctypes.byref(ncow)),
            "pa_pool_append_decode")
        return slots, pairs[:ncow.value]

    def enable_prefix_caching(self, enable: bool = True) -> None:
        _ok(self._lib.pa_pool_enable_prefix_caching(self._h, int(enable)),
            "pa_pool_enable_prefix_caching")

    def append_tokens(self, seq_id: int, token_ids):
        """Append tokens with their ids (prefix caching). Returns (slots,
        cow pair or None, n_cached): slots of cached tokens are -1."""
        ids = np.ascontiguousarray(token_ids, dtype=np.int32)
        n = ids.size
        slots = np.empty(max(n, 0), dtype=np.int64)
        pair = np.zeros(2, dtype=np.int64)
        ncow, ncached = ctypes.c_int(0), ctypes.c_int(0)
        _ok(self._lib.pa_pool_append_tokens(
            self._h, seq_id, ids.ctypes.data if n else None, n,
            slots.ctypes.data if n else None, pair.ctypes.data, ctypes.byref(ncow),
            ctypes.byref(ncached)), "pa_pool_append_tokens")
        return slots, ((int(pair[0]), int(pair[1])) if ncow.value else None), ncached.value

    @property
    def num_cached(self) -> int:
        return int(self._lib.pa_pool_num_cached(self._h))

    def free_seq(self, seq_id: int) -> None:
        _ok(self._lib.pa_pool_free_seq(self._h, seq_id), "pa_pool_free_seq")

    def block_tables(self, seq_ids: Sequence[int], max_blocks_per_seq: int):
        """Returns (tables int32[n][max_blocks_per_seq], context_lens int32[n])."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        tables = np.empty((n, max_blocks_per_seq), dtype=np.int32)
        ctx = np.empty(n, dtype=np.int32)
        _ok(self._lib.pa_pool_block_tables(self._h, ids.ctypes.data, n,
                                           tables.ctypes.data, max_blocks_per_seq,
                                           ctx.ctypes.data), "pa_pool_block_tables")
        return tables, ctx

    def _move(self, fn: str, cpu_pool: "BlockPool", seq_id: int) -> np.ndarray:
        n_max = max(self.seq_num_blocks(seq_id), cpu_pool.seq_num_blocks(seq_id), 1)
        pairs = np.zeros((n_max, 2), dtype=np.int64)
        n = ctypes.c_int(0)
        _ok(getattr(self._lib, fn)(self._h, cpu_pool._h, seq_id, pairs.ctypes.data,
                                   n_max, ctypes.byref(n)), fn)
        return pairs[:n.value]

    def swap_out(self, cpu_pool: "BlockPool", seq_id: int) -> np.ndarray:
        """Move seq_id from this (GPU) pool to cpu_pool; returns the
        (gpu block, cpu block) pairs to copy with pa_swap_blocks."""
        return self._move("pa_pool_swap_out", cpu_pool, seq_id)

    def swap_in(self, cpu_pool: "BlockPool", seq_id: int) -> np.ndarray:
        """Move seq_id from cpu_pool back to this (GPU) pool; returns the
        (cpu block, gpu block) pairs to copy with pa_swap_blocks."""
        return self._move("pa_pool_swap_in", cpu_pool, seq_id)

    @property
    def num_free(self) -> int:
        return int(self._lib.pa_pool_num_free(self._h))

    def refcount(self, block_id: int) -> int:
        return int(self._lib.pa_pool_refcount(self._h, block_id))

    def seq_len(self, seq_id: int) -> int:
        return int(self._lib.pa_pool_seq_len(self._h, seq_id))

    def seq_lens(self, seq_ids) -> np.ndarray:
        """Lengths of many sequences in one call (-1 for an unknown id)."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        out = np.empty(len(ids), dtype=np.int64)
        n = len(ids)
        _ok(self._lib.pa_pool_seq_lens(self._h, ids.ctypes.data if n else None, n,
                                       out.ctypes.data if n else None), "pa_pool_seq_lens")
        return out

    def seq_num_blocks(self, seq_id: int) -> int:
        return int(self._lib.pa_pool_seq_num_blocks(self._h, seq_id))
