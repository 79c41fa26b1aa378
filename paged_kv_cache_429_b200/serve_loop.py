"""A multi-step decode loop with continuous batching over the paged pool.

Iteration-level scheduling as the pages describe it: at every decode step,
requests that finished leave and their blocks go back to the pool, waiting
requests join while the pool has room, and every running request generates
one token ("第 7 章推理框架：vLLM 与 PagedAttention" §7.1 Continuous Batching;
"GPU 学习日报 Day 28" §五: requests leave and blocks return at each decode
step, new ones enter at once). When a running request needs a block and the
pool is empty, the most recently admitted request is preempted by swapping
its blocks to host memory and resumed later (Day 28 §七, FAQ Q3).

There is no model: prompts' and new tokens' K/V and the queries are seeded
random bf16 values. Each step runs the library's kernels — the admitted
prompts' K/V written block-wise (pa_reshape_and_cache), the new tokens'
K/V, copies for swaps (pa_swap_blocks), and the decode (pa_decode) — and
records the KV utilisation of the paged pool against a max-length
reservation of the same running requests (Day 28 §4.1-4.2).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np
import torch

import synth

from . import (BlockPool, PagedAttentionError, pa_decode, pa_decode_workspace_size,
               pa_reshape_and_cache, pa_swap_blocks)

BS = 16


@dataclasses.dataclass
class LoopConfig:
    num_q_heads: int = 32
    num_kv_heads: int = 32
    head_dim: int = 128
    num_blocks: int = 4096          # GPU pool
    cpu_blocks: int = 4096          # swap space in pinned host memory
    max_num_seqs: int = 128
    max_model_len: int = 2048
    prompt_median: float = 300.0    # lognormal prompt / output lengths
    prompt_sigma: float = 0.8
    output_median: float = 150.0
    output_sigma: float = 0.8
    arrivals_per_step: float = 2.0  # mean new requests per step (Poisson)
    watermark_blocks: int = 16      # kept free at admission for decode growth
    seed: int = 0


@dataclasses.dataclass
class Request:
    rid: int
    prompt_len: int
    output_len: int
    generated: int = 0
    admitted_at: int = -1


class _Staging:
    """Page-locked staging for the host arrays one step sends to the GPU
    (cache slots, swap pairs, block tables, context lengths). They are
    packed into the next buffer of a small ring and sent with one
    non-blocking copy on the current stream, so the host never waits for
    the GPU to drain before an upload and its scheduling of the next step
    runs while the GPU still works on this one. A ring buffer is refilled
    only once the copy that last read it has completed (an event recorded
    behind that copy; with a ring of three it is long done)."""

    ALIGN = 256

    def __init__(self, device: torch.device, depth: int = 3, nbytes: int = 1 << 20):
        self.device = device
        self.depth = depth
        self.host = [torch.empty(nbytes, dtype=torch.uint8).pin_memory() for _ in range(depth)]
        self.dev = [torch.empty(nbytes, dtype=torch.uint8, device=device) for _ in range(depth)]
        self.events: List[Optional[torch.cuda.Event]] = [None] * depth
        self.i = 0

    def upload(self, arrays: List[np.ndarray]) -> List[torch.Tensor]:
        k = self.i % self.depth
        self.i += 1
        offs, total = [], 0
        for a in arrays:
            offs.append(total)
            total += -(-a.nbytes // self.ALIGN) * self.ALIGN
        if self.events[k] is not None:
            self.events[k].synchronize()
        if total > self.host[k].numel():
            n = max(total, 2 * self.host[k].numel())
            self.host[k] = torch.empty(n, dtype=torch.uint8).pin_memory()
            self.dev[k] = torch.empty(n, dtype=torch.uint8, device=self.device)
        hbuf = self.host[k].numpy()
        for a, o in zip(arrays, offs):
            hbuf[o:o + a.nbytes] = np.ascontiguousarray(a).view(np.uint8).reshape(-1)
        if total:
            self.dev[k][:total].copy_(self.host[k][:total], non_blocking=True)
        if self.device.type == "cuda":
            ev = torch.cuda.Event()
            ev.record()
            self.events[k] = ev
        return [self.dev[k][o:o + a.nbytes].view(_TORCH_DTYPE[a.dtype]).view(a.shape)
                for a, o in zip(arrays, offs)]


_TORCH_DTYPE = {np.dtype(np.int64): torch.int64, np.dtype(np.int32): torch.int32}


class DecodeLoop:
    def __init__(self, cfg: LoopConfig, device="cuda", record: bool = False):
        self.cfg = cfg
        self.device = torch.device(device)
        self.record = record
        self.rng = np.random.default_rng([cfg.seed, 424242])
        self.gen = torch.Generator(device=self.device)
        self.gen.manual_seed(cfg.seed * 1000003 + 17)
        self.pool = BlockPool(cfg.num_blocks, BS, shuffle_seed=cfg.seed + 1)
        self.cpu_pool = BlockPool(cfg.cpu_blocks, BS)
        shape = (cfg.num_blocks, cfg.num_kv_heads, BS, cfg.head_dim)
        self.k_cache = torch.full(shape, synth.SENTINEL_BF16, dtype=torch.int16,
                                  device=self.device).view(torch.bfloat16)
        self.v_cache = self.k_cache.clone()
        hshape = (cfg.cpu_blocks,) + shape[1:]
        self.k_host = torch.zeros(hshape, dtype=torch.bfloat16).pin_memory()
        self.v_host = torch.zeros(hshape, dtype=torch.bfloat16).pin_memory()
        self.width = -(-cfg.max_model_len // BS)
        self.sm_scale = 1.0 / math.sqrt(cfg.head_dim)
        self.waiting: List[Request] = []
        self.running: List[Request] = []
        self.swapped: List[Request] = []
        self.next_rid = 0
        self.step_no = 0
        self.finished = 0
        self.preemptions = 0
        self.stats: List[Dict] = []
        self.log: List[tuple] = []   # (op, ...) in issue order, when recording
        self.last: Optional[Dict] = None
        self.ws = torch.empty(pa_decode_workspace_size(cfg.max_num_seqs, cfg.num_q_heads,
                                                       cfg.head_dim, cfg.max_model_len, -1),
                              dtype=torch.uint8, device=self.device)
        # one output buffer for the largest batch; a step writes its first rows
        self.out_buf = torch.empty((cfg.max_num_seqs, cfg.num_q_heads, cfg.head_dim),
                                   dtype=torch.float32, device=self.device)
        self.staging = _Staging(self.device)
        self._ops: List[tuple] = []   # this step's GPU work, in issue order

    # ------------------------------------------------------------ helpers
    def _randn(self, shape) -> torch.Tensor:
        return torch.randn(shape, generator=self.gen, device=self.device,
                           dtype=torch.float32).to(torch.bfloat16)

    def _draw(self) -> Request:
        c = self.cfg
        p = int(np.clip(np.rint(np.exp(math.log(c.prompt_median) +
                                       c.prompt_sigma * self.rng.standard_normal())),
                        1, c.max_model_len - 1))
        o = int(np.clip(np.rint(np.exp(math.log(c.output_median) +
                                       c.output_sigma * self.rng.standard_normal())),
                        1, c.max_model_len - p))
        r = Request(self.next_rid, p, o)
        self.next_rid += 1
        return r

    def _write(self, k: torch.Tensor, v: torch.Tensor, slots: np.ndarray) -> None:
        """Queue a cache write (issued in order by _launch)."""
        self._ops.append(("write", k, v, slots))
        if self.record:
            self.log.append(("write", k, v, slots.copy()))

    def _swap(self, pairs: np.ndarray, out: bool) -> None:
        """Queue a swap of whole blocks (issued in order by _launch)."""
        self._ops.append(("swap_out" if out else "swap_in", pairs))
        if self.record:
            self.log.append(("swap_out" if out else "swap_in", pairs.copy()))

    def _launch(self, decode: Optional[tuple]) -> None:
        """Send every host array of this step in one staged copy, then issue
        the step's swaps and cache writes in the order they were queued, and
        the decode last."""
        arrays = [op[-1] for op in self._ops]
        if decode is not None:
            arrays += [decode[0], decode[1]]
        dev = self.staging.upload(arrays)
        for op, d in zip(self._ops, dev):
            if op[0] == "write":
                pa_reshape_and_cache(op[1], op[2], self.k_cache, self.v_cache, d)
            elif op[0] == "swap_out":
                pa_swap_blocks(self.k_host, self.v_host, self.k_cache, self.v_cache, d)
            else:
                pa_swap_blocks(self.k_cache, self.v_cache, self.k_host, self.v_host, d)
        self._ops = []
        if decode is not None:
            tables, lens, q, out = decode
            bt, cl = dev[-2], dev[-1]
            pa_decode(out, q, self.k_cache, self.v_cache, bt, cl, int(lens.max()),
                      self.sm_scale, workspace=self.ws)

    def _preempt(self, keep: Optional[Request]) -> bool:
        """Swap out the most recently admitted running request other than
        `keep`; False if there is none or no swap space."""
        for victim in reversed(self.running):
            if victim is keep:
                continue
            try:
                pairs = self.pool.swap_out(self.cpu_pool, victim.rid)
            except PagedAttentionError:
                return False
            self._swap(pairs, out=True)
            self.running.remove(victim)
            self.swapped.append(victim)
            self.preemptions += 1
            return True
        return False

    # --------------------------------------------------------------- step
    def step(self) -> Dict:
        c = self.cfg
        # 1. finished requests leave; their blocks return at once
        still = []
        for r in self.running:
            if r.generated >= r.output_len:
                self.pool.free_seq(r.rid)
                self.finished += 1
            else:
                still.append(r)
        self.running = still
        # 2. arrivals
        for _ in range(self.rng.poisson(c.arrivals_per_step)):
            self.waiting.append(self._draw())
        # 3. resume swapped requests first, then admit new ones (FIFO)
        while self.swapped and len(self.running) < c.max_num_seqs:
            r = self.swapped[0]
            need = self.cpu_pool.seq_num_blocks(r.rid)
            if self.pool.num_free < need + c.watermark_blocks:
                break
            pairs = self.pool.swap_in(self.cpu_pool, r.rid)
            self._swap(pairs, out=False)
            self.swapped.pop(0)
            self.running.append(r)
        while self.waiting and not self.swapped and len(self.running) < c.max_num_seqs:
            r = self.waiting[0]
            need = -(-(r.prompt_len + 1) // BS)
            if self.pool.num_free < need + c.watermark_blocks:
                break
            self.waiting.pop(0)
            self.pool.add_seq(r.rid)
            slots, _ = self.pool.append(r.rid, r.prompt_len)
            shape = (r.prompt_len, c.num_kv_heads, c.head_dim)
            self._write(self._randn(shape), self._randn(shape), slots)  # prefill KV
            r.admitted_at = self.step_no
            self.running.append(r)
        # 4. every running request generates one token. A token that starts
        # a new block needs one from the pool: preempt (swap out) the most
        # recently admitted requests until the pool covers them all.
        while True:
            cur = self.pool.seq_lens([r.rid for r in self.running])  # one call
            need = int(np.count_nonzero(cur % BS == 0))
            if need <= self.pool.num_free or not self.running:
                break
            if not self._preempt(keep=None):
                raise RuntimeError("out of GPU blocks and of swap space")
        # every running request gets its slot (in order) or the call raises
        batch = list(self.running)
        n = len(batch)
        if n:
            ids = np.fromiter((r.rid for r in batch), dtype=np.int64, count=n)
            slots, cow = self.pool.append_decode(ids)
            assert len(cow) == 0  # the loop never forks, so nothing is shared
        stats = {"step": self.step_no, "running": n, "waiting": len(self.waiting),
                 "swapped": len(self.swapped)}
        decode = None
        if n:
            tables, lens = self.pool.block_tables(ids, self.width)
            kv_shape = (n, c.num_kv_heads, c.head_dim)
            self._write(self._randn(kv_shape), self._randn(kv_shape), slots)
            q = self._randn((n, c.num_q_heads, c.head_dim))
            out = self.out_buf[:n]
            decode = (tables, lens, q, out)
        self._launch(decode)
        if n:
            for r in batch:
                r.generated += 1
            held = int(((lens.astype(np.int64) + BS - 1) // BS).sum())
            stats.update(tokens=int(lens.sum()), blocks_held=held,
                         paged_util=float(lens.sum()) / (BS * held),
                         reserved_util=float(lens.sum()) / (n * c.max_model_len),
                         lens=lens.copy())
            self.last = {"q": q, "out": out, "tables": tables, "lens": lens}
        self.stats.append(stats)
        self.step_no += 1
        return stats

    def run(self, steps: int) -> List[Dict]:
        return [self.step() for _ in range(steps)]
