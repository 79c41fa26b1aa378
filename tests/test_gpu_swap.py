"""GPU tests of swapping blocks to pinned host memory and back.

Preemption by swapping ([Day28] "GPU 学习日报 Day 28" §六 question 4, §七,
FAQ Q3): a sequence's blocks move to a CPU pool, the GPU blocks are reused
by others, and the sequence later returns into different GPU blocks. The
host copy must hold exactly the oracle's bytes, and after the round trip the
decode output must be bit-identical (only physical ids changed).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from paged_kv_cache_429_b200 import (BlockPool, PagedAttentionError, pa_decode,
                                     pa_get_device_error, pa_swap_blocks)
from paged_kv_cache_429_b200.batch import DecodeBatch
from parity_harness import cache_np, oracle_caches

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean():
    pa_get_device_error()
    yield
    torch.cuda.empty_cache()


def pinned_cache(nb, like):
    t = torch.zeros((nb,) + tuple(like.shape[1:]), dtype=like.dtype)
    return t.pin_memory()


@pytest.mark.parametrize("name", ["tiny", "gqa_fp8"])
def test_swap_out_then_in_round_trip(name):
    w = synth.WORKLOADS[name]
    if name == "gqa_fp8":
        import dataclasses
        w = dataclasses.replace(w, num_seqs=6, len_lo=300, len_hi=700, pool_factor=2.0,
                                name="gqa_fp8_small")
    b = DecodeBatch.build(w, 0)
    b.step(partition_size=0)
    ref = b.out.clone()
    victim = 1
    cpu_pool = BlockPool(64)
    host_k, host_v = pinned_cache(64, b.k_cache), pinned_cache(64, b.v_cache)

    out_pairs = b.pool.swap_out(cpu_pool, victim)
    pa_swap_blocks(host_k, host_v, b.k_cache, b.v_cache, torch.from_numpy(out_pairs).cuda())
    torch.cuda.synchronize()
    assert pa_get_device_error() == 0

    # the host copy holds exactly the oracle's bytes of those blocks
    kc, vc = oracle_caches(b, subset=[victim])
    hk_ref = np.zeros_like(cache_np(host_k))
    hv_ref = np.zeros_like(hk_ref)
    oracle.swap_blocks(hk_ref, hv_ref, kc, vc, out_pairs)
    np.testing.assert_array_equal(cache_np(host_k), hk_ref)
    np.testing.assert_array_equal(cache_np(host_v), hv_ref)

    # the freed GPU blocks are taken by another sequence and overwritten, so
    # the victim comes back into other physical blocks
    b.pool.add_seq(999)
    b.pool.append(999, 16 * len(out_pairs))
    for g in out_pairs[:, 0]:
        b.k_cache[int(g)].view(torch.uint8).fill_(0x7F)
        b.v_cache[int(g)].view(torch.uint8).fill_(0x7F)

    in_pairs = b.pool.swap_in(cpu_pool, victim)
    assert not set(in_pairs[:, 1].tolist()) & set(out_pairs[:, 0].tolist())
    pairs_host = torch.from_numpy(in_pairs).pin_memory()  # pairs may live in pinned host memory
    pa_swap_blocks(b.k_cache, b.v_cache, host_k, host_v, pairs_host)
    tables, ctx = b.pool.block_tables(np.arange(w.num_seqs), b.max_blocks)
    assert np.array_equal(ctx, b.lens)
    bt = torch.from_numpy(tables).cuda()
    out = torch.empty_like(b.out)
    pa_decode(out, b.q, b.k_cache, b.v_cache, bt, b.context_lens, b.max_context_len,
              w.sm_scale, k_scale=b.k_scale, v_scale=b.v_scale, partition_size=0)
    torch.cuda.synchronize()
    assert pa_get_device_error() == 0
    assert torch.equal(out, ref)


def test_pageable_host_memory_is_refused():
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 1)
    pageable_k = torch.zeros((8,) + tuple(b.k_cache.shape[1:]), dtype=b.k_cache.dtype)
    pageable_v = torch.zeros_like(pageable_k)
    pairs = torch.tensor([[int(b.tables[0, 0]), 0]], dtype=torch.int64).cuda()
    with pytest.raises((PagedAttentionError, ValueError)):
        pa_swap_blocks(pageable_k, pageable_v, b.k_cache, b.v_cache, pairs)
    # straight through the C ABI as well: refused before any launch
    from paged_kv_cache_429_b200 import _lib
    rc = _lib.lib().pa_swap_blocks(
        pageable_k.data_ptr(), pageable_v.data_ptr(), b.k_cache.data_ptr(),
        b.v_cache.data_ptr(), pairs.data_ptr(), 1, b.k_cache[0].numel() * 2, b.num_blocks, 8,
        torch.cuda.current_stream().cuda_stream)
    assert rc == 1
    torch.cuda.synchronize()
    assert torch.all(pageable_k == 0)


def test_swap_pair_outside_either_pool_is_skipped_and_flagged():
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 2)
    host_k, host_v = pinned_cache(4, b.k_cache), pinned_cache(4, b.v_cache)
    pairs = torch.tensor([[0, 1], [1, 4], [b.num_blocks, 2]], dtype=torch.int64).cuda()
    pa_swap_blocks(host_k, host_v, b.k_cache, b.v_cache, pairs)
    torch.cuda.synchronize()
    assert pa_get_device_error() & 0x2
    assert torch.equal(host_k[1].view(torch.int16), b.k_cache[0].cpu().view(torch.int16))
    assert torch.all(host_k[[0, 2, 3]].view(torch.uint8) == 0)
