"""Test-side helpers: rebuild a DecodeBatch's cache with the oracle and
compare. The oracle side takes only the seeded source rows (from synth, via
the batch's source tensors), q, and the host-side write log (slots and copy
pairs chosen by the block pool); it never reads a cache or an output that a
CUDA kernel produced.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

BF16_TOL = 2e-3   # max-abs vs fp64 oracle, bf16 KV, fp32 accumulation
FP8_TOL = 6e-3    # max-abs vs fp64 oracle on the same fp8 bytes


def to_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def cache_np(t: torch.Tensor) -> np.ndarray:
    return to_u8(t) if t.element_size() == 1 else to_u16(t)


def oracle_caches(batch, subset=None, include_step=True):
    """Host caches after replaying the batch's cache operations in the
    oracle, restricted to rows/pairs owned by `subset` (or shared)."""
    w = batch.w
    shape = (batch.num_blocks, w.num_kv_heads, 16, w.head_dim)
    if w.kv_fp8:
        kc = np.full(shape, synth.SENTINEL_FP8, dtype=np.uint8)
        dt = oracle.KV_FP8_E4M3
    else:
        kc = np.full(shape, synth.SENTINEL_BF16, dtype=np.uint16)
        dt = oracle.KV_BF16
    vc = kc.copy()
    keep = None if subset is None else set(int(s) for s in subset) | {-1}
    ops = batch.setup_ops + (batch.step_ops if include_step else [])
    for op in ops:
        if keep is None:
            sel = np.arange(len(op.owner))
        else:
            sel = np.array([i for i, o in enumerate(op.owner) if int(o) in keep], dtype=np.int64)
        if len(sel) == 0:
            continue
        if op.kind == "copy":
            oracle.copy_blocks(kc, vc, op.pairs[sel])
            continue
        src_k = batch.k_old if op.src == "old" else batch.k_new
        src_v = batch.v_old if op.src == "old" else batch.v_new
        rows = torch.from_numpy(sel + op.row0).to(src_k.device)
        key = to_u16(src_k.index_select(0, rows))
        val = to_u16(src_v.index_select(0, rows))
        oracle.reshape_and_cache(key, val, kc, vc, op.slots[sel], dt,
                                 batch.k_scale, batch.v_scale)
    return kc, vc


def oracle_decode(batch, kc, vc, subset=None):
    w = batch.w
    return oracle.paged_decode(
        to_u16(batch.q), kc, vc, batch.tables, batch.lens.astype(np.int32),
        w.sm_scale, kv_dtype=oracle.KV_FP8_E4M3 if w.kv_fp8 else oracle.KV_BF16,
        k_scale=batch.k_scale, v_scale=batch.v_scale, seq_subset=subset)


def used_blocks(batch, subset=None):
    seqs = range(batch.w.num_seqs) if subset is None else subset
    ids = set()
    for s in seqs:
        nb = -(-int(batch.lens[s]) // 16)
        ids.update(int(b) for b in batch.tables[s, :nb])
    return np.array(sorted(ids), dtype=np.int64)


def assert_cache_equal(batch, kc, vc, subset=None):
    """GPU cache bytes == oracle cache bytes on every block the subset uses."""
    blocks = used_blocks(batch, subset)
    idx = torch.from_numpy(blocks).to(batch.k_cache.device)
    gk = cache_np(batch.k_cache.index_select(0, idx))
    gv = cache_np(batch.v_cache.index_select(0, idx))
    np.testing.assert_array_equal(gk, kc[blocks])
    np.testing.assert_array_equal(gv, vc[blocks])


def max_abs_err(gpu_out: torch.Tensor, ref: np.ndarray, subset=None) -> float:
    g = gpu_out.detach().cpu().double().numpy()
    if subset is not None:
        g, ref = g[subset], ref[subset]
    assert np.all(np.isfinite(g)), "non-finite output"
    return float(np.max(np.abs(g - ref)))


def tolerance(batch) -> float:
    return FP8_TOL if batch.w.kv_fp8 else BF16_TOL
