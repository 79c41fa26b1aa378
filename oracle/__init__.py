"""CPU oracle for paged decode attention — TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product (the CUDA library and its
Python binding) never imports, links or runs it, and it imports nothing from
the product.

The arithmetic lives in ``oracle.c`` (plain single-threaded C, fp64); this
module is argument marshalling over ctypes plus one pure-Python invariant
checker for block tables.

Sources, cited by page title and section:
  [Ch7]    "第 7 章推理框架：vLLM 与 PagedAttention" (blog.lkad.net)
  [OSPage] "vLLM 与 PagedAttention：把 GPU 显存当操作系统内存管" (alishangtian.com)
  [Day28]  "GPU 学习日报 Day 28：vLLM 与 PagedAttention：GPU Memory 管理的艺术"
           (daoyuly.cn)

Pinning: every function here is pinned by tests under ``tests/`` marked
``not gpu`` (closed forms, worked examples from the pages, library routines
and brute force); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

KV_BF16 = 0
KV_FP8_E4M3 = 1


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (no FMA contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-o", _LIB_PATH, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i32, i64, f32, f64, vp = (ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                              ctypes.c_double, ctypes.c_void_p)
    lib.oracle_kv_bytes_per_token.argtypes = [i64, i64, i64, i64]
    lib.oracle_kv_bytes_per_token.restype = i64
    lib.oracle_kv_cache_bytes.argtypes = [i64, i64, i64, i64, i64, i64]
    lib.oracle_kv_cache_bytes.restype = i64
    lib.oracle_slot.argtypes = [vp, i64, i64]
    lib.oracle_slot.restype = i64
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = f64
    lib.oracle_e4m3_encode.argtypes = [f32]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_quantize_bf16.argtypes = [ctypes.c_uint16, f32]
    lib.oracle_quantize_bf16.restype = ctypes.c_uint8
    lib.oracle_quantize_bf16_array.argtypes = [vp, i64, f32, vp]
    lib.oracle_quantize_bf16_array.restype = None
    lib.oracle_reshape_and_cache.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32,
                                             i32, i32, i32, f32, f32]
    lib.oracle_reshape_and_cache.restype = i32
    lib.oracle_copy_blocks.argtypes = [vp, vp, vp, i32, i64, i32]
    lib.oracle_copy_blocks.restype = i32
    lib.oracle_paged_prefill.argtypes = [vp, vp, vp, vp, i32, f64, f64, vp, i32, vp,
                                         vp, i32, i32, i32, i32, i32, i32, f64]
    lib.oracle_paged_prefill.restype = i32
    lib.oracle_swap_blocks.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32]
    lib.oracle_swap_blocks.restype = i32
    lib.oracle_paged_decode.argtypes = [vp, vp, vp, vp, i32, f64, f64, vp, i32,
                                        vp, i32, i32, i32, i32, i32, i32, f64,
                                        vp, i32]
    lib.oracle_paged_decode.restype = i32
    lib.oracle_paged_decode_split.argtypes = [vp, vp, vp, vp, i32, f64, f64, vp,
                                              i32, vp, i32, i32, i32, i32, i32,
                                              i32, f64, i32]
    lib.oracle_paged_decode_split.restype = i32
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (status {rc})")


# ----------------------------------------------------------------- sizes

def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int,
                       dtype_bytes: int) -> int:
    """2 x layers x KV heads x head dim x bytes ([Ch7] §7.1 formula)."""
    return int(_load().oracle_kv_bytes_per_token(layers, kv_heads, head_dim,
                                                  dtype_bytes))


def kv_cache_bytes(layers: int, kv_heads: int, head_dim: int, dtype_bytes: int,
                   tokens: int, batch: int) -> int:
    """Per-token bytes x tokens x requests ([Ch7] §KV cache 显存估算)."""
    return int(_load().oracle_kv_cache_bytes(layers, kv_heads, head_dim,
                                              dtype_bytes, tokens, batch))


def slot(block_table_row, pos: int, block_size: int) -> int:
    """Physical slot of logical position ``pos`` ([Day28] §3.1)."""
    row = np.ascontiguousarray(block_table_row, dtype=np.int32)
    return int(_load().oracle_slot(_ptr(row), pos, block_size))


# ------------------------------------------------------------------- fp8

def e4m3_decode(code: int) -> float:
    """Value of one E4M3 code (OCP E4M3, bias 7, no inf, NaN = S.1111.111)."""
    return float(_load().oracle_e4m3_decode(code))


def e4m3_encode(y: float) -> int:
    """E4M3 code of a binary32 value: RNE, finite overflow saturates to 448."""
    return int(_load().oracle_e4m3_encode(y))


def quantize_bf16(bits: int, scale: float) -> int:
    """E4M3 code of (bf16 value / scale), the division done in binary32."""
    return int(_load().oracle_quantize_bf16(bits, scale))


def quantize_bf16_array(bits: np.ndarray, scale: float) -> np.ndarray:
    """Vector form of :func:`quantize_bf16` (uint16 bf16 bits -> uint8)."""
    x = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(x.shape, dtype=np.uint8)
    _load().oracle_quantize_bf16_array(_ptr(x), x.size, scale, _ptr(out))
    return out


# ------------------------------------------------------- cache operations

def reshape_and_cache(key: np.ndarray, value: np.ndarray, k_cache: np.ndarray,
                      v_cache: np.ndarray, slot_mapping: np.ndarray,
                      kv_dtype: int, k_scale: float = 1.0,
                      v_scale: float = 1.0) -> None:
    """In-place slot scatter of key/value [T][Hkv][D] (bf16 bits as uint16)."""
    key = np.ascontiguousarray(key, dtype=np.uint16)
    value = np.ascontiguousarray(value, dtype=np.uint16)
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    T, Hkv, D = key.shape
    NB, Hc, B, Dc = k_cache.shape
    assert (Hc, Dc) == (Hkv, D) and value.shape == key.shape
    assert k_cache.dtype == (np.uint16 if kv_dtype == KV_BF16 else np.uint8)
    _check(_load().oracle_reshape_and_cache(
        _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(slots), T,
        Hkv, D, B, NB, kv_dtype, k_scale, v_scale), "reshape_and_cache")


def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray,
                pairs: np.ndarray) -> None:
    """In-place copy-on-write block copies; pairs is [n][2] (src, dst)."""
    pairs = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
    NB = k_cache.shape[0]
    block_bytes = k_cache[0].nbytes
    _check(_load().oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache),
                                      _ptr(pairs), pairs.shape[0],
                                      block_bytes, NB), "copy_blocks")


def swap_blocks(dst_k: np.ndarray, dst_v: np.ndarray, src_k: np.ndarray,
                src_v: np.ndarray, pairs: np.ndarray) -> None:
    """dst[dst_id] = src[src_id] for each (src_id, dst_id) pair, K and V."""
    pairs = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
    assert dst_k[0].nbytes == src_k[0].nbytes
    _check(_load().oracle_swap_blocks(_ptr(dst_k), _ptr(dst_v), _ptr(src_k),
                                      _ptr(src_v), _ptr(pairs), pairs.shape[0],
                                      src_k[0].nbytes, src_k.shape[0],
                                      dst_k.shape[0]), "swap_blocks")


# ---------------------------------------------------------------- decode

def paged_decode(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                 block_tables: np.ndarray, context_lens: np.ndarray,
                 sm_scale: float, kv_dtype: int = KV_BF16,
                 k_scale: float = 1.0, v_scale: float = 1.0,
                 seq_subset=None) -> np.ndarray:
    """fp64 decode attention through block tables; returns [S][Hq][D] f64.

    q is bf16 bits (uint16) [S][Hq][D]; caches are [NB][Hkv][B][D] uint16
    (bf16 bits) or uint8 (E4M3 codes). Rows of sequences outside
    ``seq_subset`` (when given) are left as NaN.
    """
    q = np.ascontiguousarray(q, dtype=np.uint16)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, Hq, D = q.shape
    NB, Hkv, B, Dc = k_cache.shape
    assert Dc == D
    # the per-tensor scales are binary32 values (the quantiser divides by them)
    k_scale, v_scale = float(np.float32(k_scale)), float(np.float32(v_scale))
    out = np.full((S, Hq, D), np.nan, dtype=np.float64)
    if seq_subset is None:
        sub, nsub = None, 0
    else:
        sub_arr = np.ascontiguousarray(seq_subset, dtype=np.int32)
        sub, nsub = _ptr(sub_arr), sub_arr.size
    _check(_load().oracle_paged_decode(
        _ptr(out), _ptr(q), _ptr(np.ascontiguousarray(k_cache)),
        _ptr(np.ascontiguousarray(v_cache)), kv_dtype, k_scale, v_scale,
        _ptr(bt), bt.shape[1], _ptr(cl), S, Hq, Hkv, D, B, NB, sm_scale, sub,
        nsub), "paged_decode")
    return out


def paged_decode_split(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                       block_tables: np.ndarray, context_lens: np.ndarray,
                       sm_scale: float, partition_size: int,
                       kv_dtype: int = KV_BF16, k_scale: float = 1.0,
                       v_scale: float = 1.0) -> np.ndarray:
    """fp64 partition + reduce form of :func:`paged_decode`."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, Hq, D = q.shape
    NB, Hkv, B, Dc = k_cache.shape
    k_scale, v_scale = float(np.float32(k_scale)), float(np.float32(v_scale))
    out = np.zeros((S, Hq, D), dtype=np.float64)
    _check(_load().oracle_paged_decode_split(
        _ptr(out), _ptr(q), _ptr(np.ascontiguousarray(k_cache)),
        _ptr(np.ascontiguousarray(v_cache)), kv_dtype, k_scale, v_scale,
        _ptr(bt), bt.shape[1], _ptr(cl), S, Hq, Hkv, D, B, NB, sm_scale,
        partition_size), "paged_decode_split")
    return out


def paged_prefill(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                  block_tables: np.ndarray, query_start: np.ndarray,
                  context_lens: np.ndarray, sm_scale: float,
                  kv_dtype: int = KV_BF16, k_scale: float = 1.0,
                  v_scale: float = 1.0) -> np.ndarray:
    """fp64 causal chunked-prefill attention; q / out are [T][Hq][D] with
    sequence s's rows query_start[s] .. query_start[s+1]-1."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    qs = np.ascontiguousarray(query_start, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    T, Hq, D = q.shape
    NB, Hkv, B, Dc = k_cache.shape
    assert Dc == D and qs.size == cl.size + 1 and qs[-1] == T
    k_scale, v_scale = float(np.float32(k_scale)), float(np.float32(v_scale))
    out = np.zeros((T, Hq, D), dtype=np.float64)
    _check(_load().oracle_paged_prefill(
        _ptr(out), _ptr(q), _ptr(np.ascontiguousarray(k_cache)),
        _ptr(np.ascontiguousarray(v_cache)), kv_dtype, k_scale, v_scale, _ptr(bt),
        bt.shape[1], _ptr(qs), _ptr(cl), cl.size, Hq, Hkv, D, B, NB, sm_scale),
        "paged_prefill")
    return out


# ------------------------------------------------------ pool invariants

def check_block_tables(block_tables, context_lens, num_blocks: int,
                       block_size: int, refcounts=None, num_free=None):
    """Return a list of violated invariants (empty when all hold).

    Invariants, from the pages:
      * each sequence holds exactly ceil(L / B) blocks, so the unused part
        of its last block is between 0 and B - 1 slots ([Day28] §4.2 and
        FAQ Q2: waste confined to the last, partly filled block);
      * every block id is a valid physical block ([Day28] §六 item 1: the
        pool is N fixed blocks);
      * a block's reference count equals the number of block-table entries
        that point at it ([Day28] §六 item 3: shared prefix, refcount 2);
      * free blocks + distinct used blocks == N (nothing leaks).
    ``block_tables`` is a list of per-sequence lists of block ids.
    """
    errors = []
    uses: dict[int, int] = {}
    for s, (row, L) in enumerate(zip(block_tables, context_lens)):
        need = -(-int(L) // block_size)
        if len(row) != need:
            errors.append(f"seq {s}: {len(row)} blocks for {L} tokens, "
                          f"expected {need}")
        waste = block_size * len(row) - int(L)
        if not 0 <= waste <= block_size - 1 and L > 0:
            errors.append(f"seq {s}: {waste} unused slots in its last block")
        for b in row:
            if not 0 <= int(b) < num_blocks:
                errors.append(f"seq {s}: block id {b} out of range")
            uses[int(b)] = uses.get(int(b), 0) + 1
    if refcounts is not None:
        for b in range(num_blocks):
            if int(refcounts[b]) != uses.get(b, 0):
                errors.append(f"block {b}: refcount {refcounts[b]} but "
                              f"{uses.get(b, 0)} table entries")
    if num_free is not None and num_free + len(uses) != num_blocks:
        errors.append(f"{num_free} free + {len(uses)} used != {num_blocks}")
    return errors


# ------------------------------------------------- utilisation (plain defs)

def paged_utilisation(context_lens, block_size: int = 16) -> float:
    """Tokens stored / token slots of the blocks held: sum L / (B sum ceil(L/B)).
    Only the last, partly filled block of each sequence wastes slots
    ([Day28] §4.2: internal fragmentation confined to the last block)."""
    lens = [int(x) for x in context_lens]
    held = sum(-(-L // block_size) for L in lens) * block_size
    return sum(lens) / held if held else 1.0


def reserved_utilisation(context_lens, reserve_tokens: int) -> float:
    """Tokens stored / slots reserved when every running request holds a
    contiguous region of its maximum length ([Ch7] §7.1, [OSPage] §服务化痛点,
    [Day28] §4.1: preallocation by max_seq_len)."""
    lens = [int(x) for x in context_lens]
    return sum(lens) / (len(lens) * reserve_tokens) if lens else 1.0


def reserved_waste_bytes(reserve_tokens: int, used_tokens: int,
                         bytes_per_token: int) -> int:
    """Bytes of a contiguous reservation that were never used ([Day28] §4.1
    worked example: 2048 reserved, 400 used)."""
    return (reserve_tokens - used_tokens) * bytes_per_token


def effective_capacity(kv_bytes: float, utilisation: float) -> float:
    """Usable KV bytes = bytes given to KV x utilisation ([Ch7] §7.3 例 7-3)."""
    return kv_bytes * utilisation
