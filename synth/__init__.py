"""Seeded synthetic inputs for paged decode attention.

This module only draws numbers: workload shapes, context lengths, and
normal random values rounded to bf16. It holds none of the method's
arithmetic (no slots, no block tables, no attention) and imports neither the
CUDA library nor the oracle, so both sides of a parity test can use it.

The five workloads (decode batches shaped like the pages' examples):
  tiny     4 seqs, 8/8 heads, d64, bf16, L ~ U[1,256], pool of 80 blocks
  llama7b  64 seqs, 32/32 heads, d128, bf16, L ~ U[512,2048]
           (Llama-7B-shaped layer, "GPU 学习日报 Day 28" §一)
  prefix   256 seqs, 40/40 heads, d128, bf16, a shared 1000-token prefix plus
           private suffixes ~ round(exp(ln 300 + N(0,1))) clipped to
           [1, 3072] (example 7-1's 40 KV heads, d128, "第 7 章推理框架" §7.2;
           the 1000-token shared prefix of Day 28 §六)
  gqa_fp8  128 seqs, 32/8 heads, d128, fp8 E4M3 cache with per-tensor
           scales amax/448, L ~ U[4096,8192]
  long     8 seqs, 64/8 heads, d128, bf16, L ~ U[65536,131072], split into
           512-token partitions
Context lengths count the token written in the decode step itself.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

# Sentinels written into every cache slot before any real K/V: bf16 quiet
# NaN and the E4M3 NaN code. Slots no sequence owns keep them.
SENTINEL_BF16 = 0x7FC0
SENTINEL_FP8 = 0x7F


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    kv_fp8: bool
    len_lo: int = 0            # uniform lengths in [len_lo, len_hi]
    len_hi: int = 0
    prefix_len: int = 0        # shared prefix (prefix workload)
    suffix_median: float = 0.0
    suffix_sigma: float = 0.0
    suffix_clip: tuple = (1, 1)
    pool_blocks: int = 0       # fixed pool size, else pool_factor x needed
    pool_factor: float = 1.2
    partition_size: int = -1   # -1 automatic, 0 single-pass, >0 split

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


WORKLOADS = {
    "tiny": Workload("tiny", 4, 8, 8, 64, False, 1, 256, pool_blocks=80),
    "llama7b": Workload("llama7b", 64, 32, 32, 128, False, 512, 2048),
    "prefix": Workload("prefix", 256, 40, 40, 128, False, prefix_len=1000,
                       suffix_median=300.0, suffix_sigma=1.0,
                       suffix_clip=(1, 3072)),
    "gqa_fp8": Workload("gqa_fp8", 128, 32, 8, 128, True, 4096, 8192),
    "long": Workload("long", 8, 64, 8, 128, False, 65536, 131072,
                     partition_size=512),
}

_STREAM_IDS = {"lengths": 1, "q": 2, "k_old": 3, "v_old": 4, "k_new": 5,
               "v_new": 6, "pool": 7, "q_prefill": 8}


def rng(seed: int, workload: str, what: str) -> np.random.Generator:
    """Independent numpy stream per (seed, workload, purpose)."""
    key = sum(ord(c) * 131 ** i for i, c in enumerate(workload)) % (2**31)
    return np.random.default_rng([seed, key, _STREAM_IDS[what]])


def stream_seed(seed: int, workload: str, what: str) -> int:
    """A 63-bit integer seed for torch generators and the block pool."""
    return int(rng(seed, workload, what).integers(0, 2**63 - 1))


def draw_lengths(w: Workload, seed: int) -> np.ndarray:
    """Context lengths (int64), including the decode step's own token."""
    g = rng(seed, w.name, "lengths")
    if w.prefix_len:
        z = g.standard_normal(w.num_seqs)
        suf = np.rint(np.exp(math.log(w.suffix_median) + w.suffix_sigma * z))
        suf = np.clip(suf, w.suffix_clip[0], w.suffix_clip[1]).astype(np.int64)
        return w.prefix_len + suf
    return g.integers(w.len_lo, w.len_hi + 1, size=w.num_seqs).astype(np.int64)


def randn_bf16(shape, seed: int, workload: str, what: str,
               device="cpu") -> torch.Tensor:
    """N(0, 1) values drawn in fp32 by torch's generator, rounded to bf16."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(stream_seed(seed, workload, what))
    return torch.randn(tuple(shape), generator=gen, device=dev,
                       dtype=torch.float32).to(torch.bfloat16)


def prompt_kv_rows(token_ids, seed: int, num_kv_heads: int, head_dim: int):
    """K and V rows (bf16 [n][num_kv_heads][head_dim]) for a request's
    tokens, each row a function of the token ids up to and including its
    own, as a model's K/V are: two requests whose token lists agree on a
    prefix get identical rows on that prefix and unrelated rows after it.
    Row i is N(0, 1) from a numpy stream keyed by (seed, a running 64-bit
    FNV-1a hash of token_ids[:i+1]), rounded to bf16."""
    h = 0xCBF29CE484222325
    k = np.empty((len(token_ids), num_kv_heads * head_dim), np.float32)
    v = np.empty_like(k)
    for i, t in enumerate(token_ids):
        for byte in int(t).to_bytes(4, "little", signed=True):
            h = ((h ^ byte) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
        g = np.random.default_rng([seed, h & 0xFFFFFFFF, h >> 32])
        k[i] = g.standard_normal(num_kv_heads * head_dim, dtype=np.float32)
        v[i] = g.standard_normal(num_kv_heads * head_dim, dtype=np.float32)
    shape = (len(token_ids), num_kv_heads, head_dim)
    return (torch.from_numpy(k).reshape(shape).to(torch.bfloat16),
            torch.from_numpy(v).reshape(shape).to(torch.bfloat16))
