"""GPU parity of automatic prefix caching.

"第 7 章推理框架" §7.1 (前缀共享, --enable-prefix-caching) and "GPU 学习日报
Day 28" §4.2 / §七: a request whose prompt starts with an earlier request's
tokens reuses that request's full KV blocks instead of writing them again.
The pool (pa_pool_append_tokens) hands such tokens slot -1, the cache write
(pa_reshape_and_cache) skips them, and the decode reads the earlier
request's physical blocks through the new request's table.

The scenario, on a pool small enough to force evictions:
  A  1000-token prompt, then one decode token (all blocks new);
  B  A's first 992 tokens + 300 of its own: 62 blocks found in the cache;
  A and B decode together, then both leave (their full blocks stay findable);
  D  470 tokens of its own: needs more fresh blocks than are free, so it
     evicts the least recently freed keyed blocks (B's suffix);
  E  A's whole prompt + 50 of its own: A's 62 full blocks are found again
     (freed, not evicted), the rest is new; D and E decode together.
Each token's K/V row is a function of the token ids up to it
(synth.prompt_kv_rows), as a model's are, so a skipped write loses nothing
only if the cached block really holds the same prefix.

Checks, per decode step: the GPU cache bytes of every block a live request
uses equal the oracle's cache rebuilt from the same writes (cached slots
skipped); the GPU output is within the oracle tolerance of the fp64 oracle
on that cache, and of the oracle on private, unshared copies of each
request's own rows (the two oracle results agree exactly); the shared blocks
are the physical ids A wrote.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from paged_kv_cache_429_b200 import (BlockPool, pa_decode, pa_get_device_error,
                                     pa_reshape_and_cache)
from parity_harness import BF16_TOL, FP8_TOL, cache_np, to_u16

pytestmark = pytest.mark.gpu

B = 16
HKV, HQ, D = 8, 32, 128
NB = 100
SM_SCALE = D ** -0.5


class Caches:
    """The GPU caches and the oracle's host caches, fed the same writes."""

    def __init__(self, fp8: bool, k_scale: float, v_scale: float):
        shape = (NB, HKV, B, D)
        self.fp8, self.k_scale, self.v_scale = fp8, k_scale, v_scale
        if fp8:
            self.gk = torch.full(shape, synth.SENTINEL_FP8, dtype=torch.uint8, device="cuda")
            self.hk = np.full(shape, synth.SENTINEL_FP8, dtype=np.uint8)
        else:
            self.gk = torch.full(shape, synth.SENTINEL_BF16, dtype=torch.int16,
                                 device="cuda").view(torch.bfloat16)
            self.hk = np.full(shape, synth.SENTINEL_BF16, dtype=np.uint16)
        self.gv, self.hv = self.gk.clone(), self.hk.copy()
        self.dtype = oracle.KV_FP8_E4M3 if fp8 else oracle.KV_BF16

    def write(self, krows, vrows, slots):
        slots = np.asarray(slots, np.int64)
        pa_reshape_and_cache(krows.cuda(), vrows.cuda(), self.gk, self.gv,
                             torch.from_numpy(slots).cuda(), k_scale=self.k_scale,
                             v_scale=self.v_scale)
        oracle.reshape_and_cache(to_u16(krows), to_u16(vrows), self.hk, self.hv, slots,
                                 self.dtype, self.k_scale, self.v_scale)


class Request:
    def __init__(self, seq_id, prompt, decode_tok, seed):
        self.id = seq_id
        self.tokens = np.concatenate([prompt, [decode_tok]]).astype(np.int32)
        self.k, self.v = synth.prompt_kv_rows(self.tokens, seed, HKV, D)
        self.n_prompt = len(prompt)


def admit(pool, caches, r):
    pool.add_seq(r.id)
    slots, cow, n_cached = pool.append_tokens(r.id, r.tokens[:r.n_prompt])
    assert cow is None
    assert np.all(slots[:n_cached] == -1) and np.all(slots[n_cached:] >= 0)
    # cached slots are -1 in the write as well: the kernel must skip them
    caches.write(r.k[:r.n_prompt], r.v[:r.n_prompt], slots)
    return n_cached


def decode_step(pool, caches, reqs, seed, partition_sizes=(0, 512)):
    """Append every request's decode token, write it, decode all of them."""
    for r in reqs:
        slots, cow, n_cached = pool.append_tokens(r.id, r.tokens[-1:])
        assert cow is None and n_cached == 0 and slots[0] >= 0
        caches.write(r.k[-1:], r.v[-1:], slots)
    ids = [r.id for r in reqs]
    maxb = max(pool.seq_num_blocks(i) for i in ids)
    tables, lens = pool.block_tables(ids, maxb)
    assert list(lens) == [len(r.tokens) for r in reqs]
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((len(reqs), HQ, D), generator=g).to(torch.bfloat16)

    # oracle on the shared cache, and on private copies of each request's rows
    kw = dict(kv_dtype=caches.dtype, k_scale=caches.k_scale, v_scale=caches.v_scale)
    ref = oracle.paged_decode(to_u16(q), caches.hk, caches.hv, tables, lens, SM_SCALE, **kw)
    for s, r in enumerate(reqs):
        n = len(r.tokens)
        nb = -(-n // B)
        sentinel = synth.SENTINEL_FP8 if caches.fp8 else synth.SENTINEL_BF16
        pk = np.full((nb, HKV, B, D), sentinel, dtype=caches.hk.dtype)
        pv = pk.copy()
        oracle.reshape_and_cache(to_u16(r.k), to_u16(r.v), pk, pv, np.arange(n), caches.dtype,
                                 caches.k_scale, caches.v_scale)
        priv = oracle.paged_decode(to_u16(q[s:s + 1]), pk, pv, np.arange(nb, dtype=np.int32)[None],
                                   np.array([n], np.int32), SM_SCALE, **kw)
        np.testing.assert_array_equal(priv[0], ref[s])

    # the GPU cache holds the oracle's bytes on every block in use
    used = sorted({int(b) for s, r in enumerate(reqs)
                   for b in tables[s, :-(-len(r.tokens) // B)]})
    idx = torch.tensor(used, device="cuda")
    np.testing.assert_array_equal(cache_np(caches.gk.index_select(0, idx)), caches.hk[used])
    np.testing.assert_array_equal(cache_np(caches.gv.index_select(0, idx)), caches.hv[used])

    tol = FP8_TOL if caches.fp8 else BF16_TOL
    qd, bt, cl = q.cuda(), torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    for ps in partition_sizes:
        out = torch.full((len(reqs), HQ, D), float("nan"), device="cuda")
        pa_decode(out, qd, caches.gk, caches.gv, bt, cl, int(lens.max()), SM_SCALE,
                  k_scale=caches.k_scale, v_scale=caches.v_scale, partition_size=ps)
        torch.cuda.synchronize()
        got = out.cpu().double().numpy()
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - ref)) <= tol, ps
    return tables


@pytest.mark.parametrize("fp8", [False, True])
def test_prefix_cache_hits_skipped_writes_and_evictions(fp8):
    pa_get_device_error()
    rng = np.random.default_rng(11)
    prompt_a = rng.integers(0, 32000, 1000)
    own_b = rng.integers(0, 32000, 300)
    own_b[0] = prompt_a[992] + 1                  # B's block 62 differs from A's
    reqs = {
        "A": Request(0, prompt_a, 7, 1),
        "B": Request(1, np.concatenate([prompt_a[:992], own_b]), 8, 1),
        "D": Request(3, rng.integers(0, 32000, 470), 9, 1),
        "E": Request(4, np.concatenate([prompt_a, rng.integers(0, 32000, 50)]), 10, 1),
    }
    # one per-tensor scale each for K and V over every row written (amax/448)
    k_scale = v_scale = 1.0
    if fp8:
        k_scale = float(np.float32(max(r.k.float().abs().max().item() for r in reqs.values()))
                        / np.float32(448.0))
        v_scale = float(np.float32(max(r.v.float().abs().max().item() for r in reqs.values()))
                        / np.float32(448.0))
    caches = Caches(fp8, k_scale, v_scale)
    pool = BlockPool(NB, shuffle_seed=5)
    pool.enable_prefix_caching()

    A, Bq, Dq, E = reqs["A"], reqs["B"], reqs["D"], reqs["E"]
    assert admit(pool, caches, A) == 0
    assert admit(pool, caches, Bq) == 992
    tables = decode_step(pool, caches, [A, Bq], seed=1)
    a_ids = list(tables[0, :63])
    b_ids = list(tables[1, :81])
    assert b_ids[:62] == a_ids[:62]               # B reads the blocks A wrote
    assert b_ids[62] != a_ids[62]
    assert all(pool.refcount(b) == 2 for b in a_ids[:62])

    pool.free_seq(A.id)
    pool.free_seq(Bq.id)
    assert pool.num_free == NB and pool.num_cached == 62 + 18

    # D needs 30 blocks while only 20 are unkeyed: 10 of B's suffix blocks
    # (the least recently freed keyed ones) are evicted and rewritten
    assert admit(pool, caches, Dq) == 0
    d_ids = set(int(b) for b in pool.block_tables([Dq.id], 30)[0][0])
    assert len(d_ids & set(b_ids[62:])) >= 10
    assert not d_ids & set(a_ids[:62])

    # E finds A's 62 full blocks again, after both of their users have left
    assert admit(pool, caches, E) == 992
    tables = decode_step(pool, caches, [Dq, E], seed=2)
    assert list(tables[1, :62]) == a_ids[:62]
    assert pa_get_device_error() == 0
