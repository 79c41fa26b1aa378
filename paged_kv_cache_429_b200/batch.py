"""A decode batch built through the block pool and the cache kernels.

`DecodeBatch.build(workload, seed, device)` runs the host block pool
(allocation on demand, prefix fork, copy-on-write pairs) to get block tables
and slot mappings, fills a fresh pool-sized cache with the sentinel, and
writes every earlier token's K/V through `pa_reshape_and_cache` (with the
CoW copies through `pa_copy_blocks` where the prefix is shared). The decode
step itself (`step`) then writes the new token of each sequence, runs any
copy the step needs, and calls `pa_decode`.

Everything host-side that fed the device (slots, pairs, which source rows
went where, in which order) is kept in `setup_ops` / `step_ops`, so that a
checker can rebuild the same cache on its own from the same source rows.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

import synth

from . import (BlockPool, pa_copy_blocks, pa_decode, pa_decode_append, pa_decode_workspace_size,
               pa_reshape_and_cache)

BS = 16


@dataclasses.dataclass
class CacheOp:
    """One host-issued cache operation, in issue order.

    kind "write": rows [row0, row1) of the source tensors named by `src`
    ("old" or "new") go to `slots`; `owner[i]` is the sequence of row i (-1
    for a prefix row shared by every sequence). kind "copy": `pairs` [n][2]
    (src, dst) block copies; `owner[i]` is the sequence the copy serves.
    """
    kind: str
    src: str = ""
    row0: int = 0
    row1: int = 0
    slots: Optional[np.ndarray] = None
    pairs: Optional[np.ndarray] = None
    owner: Optional[np.ndarray] = None


class DecodeBatch:
    def __init__(self):
        self.setup_ops: List[CacheOp] = []
        self.step_ops: List[CacheOp] = []

    # ------------------------------------------------------------ building
    @classmethod
    def build(cls, w: synth.Workload, seed: int, device="cuda",
              lens: Optional[np.ndarray] = None) -> "DecodeBatch":
        b = cls()
        b.w, b.seed = w, seed
        b.device = torch.device(device)
        lens = synth.draw_lengths(w, seed) if lens is None else np.asarray(lens, np.int64)
        assert lens.shape == (w.num_seqs,) and lens.min() >= 1
        b.lens = lens
        S, Hkv, D = w.num_seqs, w.num_kv_heads, w.head_dim
        blocks = -(-lens // BS)
        if w.pool_blocks:
            nb = w.pool_blocks
        elif w.prefix_len:
            shared_full = w.prefix_len // BS
            needed = shared_full + int(np.sum(blocks - shared_full))
            nb = int(math.ceil(w.pool_factor * needed))
        else:
            nb = int(math.ceil(w.pool_factor * int(blocks.sum())))
        b.num_blocks = nb
        b.max_blocks = int(blocks.max())
        b.max_context_len = int(lens.max())
        pool = BlockPool(nb, BS, shuffle_seed=synth.stream_seed(seed, w.name, "pool"))
        b.pool = pool

        old_slots, old_owner = [], []
        setup_pairs, setup_pair_owner = [], []
        if w.prefix_len:
            pool.add_seq(0)
            pre, _ = pool.append(0, w.prefix_len)
            for s in range(1, S):
                pool.fork(0, s)
            prefix_rows = len(pre)
            for s in range(S):
                n = int(lens[s]) - w.prefix_len - 1
                sl, cow = pool.append(s, n) if n > 0 else (np.empty(0, np.int64), None)
                if cow is not None:
                    setup_pairs.append(cow)
                    setup_pair_owner.append(s)
                old_slots.append(sl)
                old_owner.append(np.full(len(sl), s, np.int64))
        else:
            pre = np.empty(0, np.int64)
            prefix_rows = 0
            for s in range(S):
                pool.add_seq(s)
                sl, cow = pool.append(s, int(lens[s]) - 1)
                assert cow is None
                old_slots.append(sl)
                old_owner.append(np.full(len(sl), s, np.int64))
        new_slots, step_pairs, step_pair_owner = [], [], []
        for s in range(S):
            sl, cow = pool.append(s, 1)
            if cow is not None:
                step_pairs.append(cow)
                step_pair_owner.append(s)
            new_slots.append(int(sl[0]))
        tables, ctx = pool.block_tables(np.arange(S), b.max_blocks)
        assert np.array_equal(ctx, lens)
        b.tables = tables

        # ---- host-side log of the cache writes, in issue order
        suffix_slots = np.concatenate(old_slots) if old_slots else np.empty(0, np.int64)
        suffix_owner = np.concatenate(old_owner) if old_owner else np.empty(0, np.int64)
        n_old = prefix_rows + len(suffix_slots)
        if prefix_rows:
            b.setup_ops.append(CacheOp("write", "old", 0, prefix_rows, pre,
                                       owner=np.full(prefix_rows, -1, np.int64)))
        if setup_pairs:
            b.setup_ops.append(CacheOp("copy", pairs=np.array(setup_pairs, np.int64),
                                       owner=np.array(setup_pair_owner, np.int64)))
        if len(suffix_slots):
            b.setup_ops.append(CacheOp("write", "old", prefix_rows, n_old, suffix_slots,
                                       owner=suffix_owner))
        if step_pairs:
            b.step_ops.append(CacheOp("copy", pairs=np.array(step_pairs, np.int64),
                                      owner=np.array(step_pair_owner, np.int64)))
        b.step_ops.append(CacheOp("write", "new", 0, S, np.array(new_slots, np.int64),
                                  owner=np.arange(S, dtype=np.int64)))

        # ---- device tensors
        dev = b.device
        Hq = w.num_q_heads
        b.q = synth.randn_bf16((S, Hq, D), seed, w.name, "q", dev)
        b.k_old = synth.randn_bf16((n_old, Hkv, D), seed, w.name, "k_old", dev)
        b.v_old = synth.randn_bf16((n_old, Hkv, D), seed, w.name, "v_old", dev)
        b.k_new = synth.randn_bf16((S, Hkv, D), seed, w.name, "k_new", dev)
        b.v_new = synth.randn_bf16((S, Hkv, D), seed, w.name, "v_new", dev)
        if w.kv_fp8:
            # one fp32 scale per tensor: amax over every token written / 448
            def scale(a, c):
                m = torch.maximum(a.abs().max().float(), c.abs().max().float())
                return float(np.float32(m.item()) / np.float32(448.0))
            b.k_scale = scale(b.k_old, b.k_new)
            b.v_scale = scale(b.v_old, b.v_new)
            b.k_cache = torch.full((nb, Hkv, BS, D), synth.SENTINEL_FP8, dtype=torch.uint8, device=dev)
        else:
            b.k_scale = b.v_scale = 1.0
            b.k_cache = torch.full((nb, Hkv, BS, D), synth.SENTINEL_BF16, dtype=torch.int16,
                                   device=dev).view(torch.bfloat16)
        b.v_cache = b.k_cache.clone()
        b.block_tables = torch.from_numpy(tables).to(dev)
        b.context_lens = torch.from_numpy(lens.astype(np.int32)).to(dev)
        b._dev_slots = {}
        b._dev_pairs = {}
        for i, op in enumerate(b.setup_ops + b.step_ops):
            if op.kind == "write":
                b._dev_slots[id(op)] = torch.from_numpy(op.slots).to(dev)
            else:
                b._dev_pairs[id(op)] = torch.from_numpy(op.pairs).to(dev)
        b.out = torch.empty((S, Hq, D), dtype=torch.float32, device=dev)
        b.run_ops(b.setup_ops)
        return b

    # ----------------------------------------------------------- execution
    def run_ops(self, ops: List[CacheOp], stream=None) -> None:
        for op in ops:
            if op.kind == "write":
                src_k = self.k_old if op.src == "old" else self.k_new
                src_v = self.v_old if op.src == "old" else self.v_new
                pa_reshape_and_cache(src_k[op.row0:op.row1], src_v[op.row0:op.row1],
                                     self.k_cache, self.v_cache, self._dev_slots[id(op)],
                                     k_scale=self.k_scale, v_scale=self.v_scale, stream=stream)
            else:
                pa_copy_blocks(self.k_cache, self.v_cache, self._dev_pairs[id(op)], stream=stream)

    def workspace(self, partition_size: int) -> Optional[torch.Tensor]:
        n = pa_decode_workspace_size(self.w.num_seqs, self.w.num_q_heads, self.w.head_dim,
                                     self.max_context_len, partition_size)
        return torch.empty(n, dtype=torch.uint8, device=self.device) if n else None

    def decode(self, out: Optional[torch.Tensor] = None, partition_size: Optional[int] = None,
               workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        out = self.out if out is None else out
        ps = self.w.partition_size if partition_size is None else partition_size
        return pa_decode(out, self.q, self.k_cache, self.v_cache, self.block_tables,
                         self.context_lens, self.max_context_len, self.w.sm_scale,
                         k_scale=self.k_scale, v_scale=self.v_scale, partition_size=ps,
                         workspace=workspace, stream=stream)

    def step(self, partition_size: Optional[int] = None,
             workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """One decode step: write the new tokens (after any CoW copy), decode."""
        self.run_ops(self.step_ops, stream=stream)
        return self.decode(partition_size=partition_size, workspace=workspace, stream=stream)

    def step_fused(self, partition_size: Optional[int] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """The same step with the new tokens' write fused into the decode
        launch (pa_decode_append): any copy-on-write copies first, then one
        decode that also writes each sequence's new token and attends to it."""
        writes = [op for op in self.step_ops if op.kind == "write"]
        assert len(writes) == 1 and writes[0].src == "new" and writes[0].row0 == 0 \
            and writes[0].row1 == self.w.num_seqs
        for op in self.step_ops:
            if op.kind == "copy":
                pa_copy_blocks(self.k_cache, self.v_cache, self._dev_pairs[id(op)], stream=stream)
        ps = self.w.partition_size if partition_size is None else partition_size
        return pa_decode_append(self.out, self.q, self.k_new, self.v_new, self.k_cache,
                                self.v_cache, self.block_tables, self.context_lens,
                                self.max_context_len, self.w.sm_scale, k_scale=self.k_scale,
                                v_scale=self.v_scale, partition_size=ps, workspace=workspace,
                                stream=stream)

    # ---------------------------------------------------------- accounting
    def algorithmic_bytes(self) -> int:
        """Bytes a decode step must move: K and V of every context token,
        q (bf16), out (fp32), the block-table entries and context lengths."""
        w = self.w
        eb = 1 if w.kv_fp8 else 2
        kv = int(self.lens.sum()) * w.num_kv_heads * w.head_dim * eb * 2
        qo = w.num_seqs * w.num_q_heads * w.head_dim * (2 + 4)
        bt = int((-(-self.lens // BS)).sum()) * 4 + 4 * w.num_seqs
        return kv + qo + bt

    def unique_kv_bytes(self) -> int:
        """K and V bytes of the distinct physical blocks the step reads (a
        block shared by several sequences counted once, with the most
        tokens any of them uses in it)."""
        w = self.w
        eb = 1 if w.kv_fp8 else 2
        used = {}
        for s in range(w.num_seqs):
            L = int(self.lens[s])
            for j in range(-(-L // BS)):
                p = int(self.tables[s][j])
                used[p] = max(used.get(p, 0), min(BS, L - BS * j))
        return sum(used.values()) * w.num_kv_heads * w.head_dim * eb * 2
