"""GPU parity of paged decode attention against the fp64 oracle.

Every workload is built through the block pool and the cache kernels, with
every slot first set to NaN, so any read of a slot outside a sequence shows
up as a non-finite output. The oracle rebuilds the cache from the same
source rows and the pool's host-side write log.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from paged_kv_cache_429_b200 import (PagedAttentionError, pa_decode,
                                     pa_get_device_error)
from paged_kv_cache_429_b200.batch import DecodeBatch
from parity_harness import (assert_cache_equal, max_abs_err, oracle_caches,
                            oracle_decode, tolerance)

pytestmark = pytest.mark.gpu
PA_DEVERR_CONTEXT_CLAMP = 0x4
PA_DEVERR_BLOCK_RANGE = 0x10


@pytest.fixture(autouse=True)
def _clean():
    pa_get_device_error()  # start each test with a clear error word
    yield
    torch.cuda.empty_cache()


def check_batch(batch, subset=None, paths=(None,)):
    """Run the decode step (new-token writes, then decode) on the GPU; check
    the cache bytes and then every decode path against the oracle."""
    kc, vc = oracle_caches(batch, subset)
    ref = oracle_decode(batch, kc, vc, subset)
    errs = {}
    for i, ps in enumerate(paths):
        if i == 0:
            batch.step(partition_size=ps)
            torch.cuda.synchronize()
            assert_cache_equal(batch, kc, vc, subset)
        else:
            batch.decode(partition_size=ps)
        torch.cuda.synchronize()
        errs[ps] = max_abs_err(batch.out, ref, subset)
    assert pa_get_device_error() == 0
    for ps, e in errs.items():
        assert e <= tolerance(batch), (ps, e)
    return errs


# --------------------------------------------------------------- workloads

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_workload(seed):
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], seed)
    check_batch(b, paths=(0, 16, 64, 512, -1))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_llama7b_workload(seed):
    b = DecodeBatch.build(synth.WORKLOADS["llama7b"], seed)
    check_batch(b, paths=(-1, 0, 512))


def sampled_subset(n, seed, must, count=32):
    """`count` sequences of an n-sequence batch: the listed ones plus a
    seeded draw of the rest."""
    rest = [s for s in range(n) if s not in must]
    pick = np.random.default_rng(100 + seed).choice(rest, count - len(must), replace=False)
    return sorted(set(must) | set(int(x) for x in pick))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_prefix_workload_sampled(seed):
    """32 of the 256 sequences (the first, the last writer to copy its
    shared partial block, the last one, which writes in place, and a seeded
    draw), all heads and dims."""
    b = DecodeBatch.build(synth.WORKLOADS["prefix"], seed)
    assert len([op for op in b.setup_ops + b.step_ops if op.kind == "copy"]) >= 1
    copies = [op for op in b.setup_ops + b.step_ops if op.kind == "copy"]
    n_pairs = sum(len(op.pairs) for op in copies)
    assert n_pairs == 255
    owners = set(int(o) for op in copies for o in op.owner)
    assert owners == set(range(255))              # every writer but the last copies
    subset = sampled_subset(256, seed, [0, 1, 254, 255])
    check_batch(b, subset, paths=(-1, 0, 512))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_gqa_fp8_workload_sampled(seed):
    b = DecodeBatch.build(synth.WORKLOADS["gqa_fp8"], seed)
    subset = sampled_subset(128, seed, [0, 63, 64, 127])
    check_batch(b, subset, paths=(-1, 0, 512))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_long_context_workload(seed):
    """All 8 sequences of 64K-128K tokens against the oracle: the
    workload's own 512-token split, the automatic choice, and the step with
    the new tokens' write fused into the decode (pa_decode_append)."""
    b = DecodeBatch.build(synth.WORKLOADS["long"], seed)
    kc, vc = oracle_caches(b)
    ref = oracle_decode(b, kc, vc)
    ws = b.workspace(512)
    for i, ps in enumerate((512, -1)):
        if i == 0:
            b.step(partition_size=ps, workspace=ws)
        else:
            b.decode(partition_size=ps, workspace=ws)
        torch.cuda.synchronize()
        assert max_abs_err(b.out, ref) <= tolerance(b), ps
    assert_cache_equal(b, kc, vc)
    # the fused step writes the same new-token bytes again and decodes
    b.out.fill_(float("nan"))
    b.step_fused(partition_size=512, workspace=ws)
    torch.cuda.synchronize()
    assert max_abs_err(b.out, ref) <= tolerance(b), "fused"
    assert_cache_equal(b, kc, vc)
    assert pa_get_device_error() == 0


# --------------------------------------------------------------- edge cases

EDGE_LENS = [1, 2, 15, 16, 17, 31, 32, 33, 100, 511, 512, 513, 1040]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (8, 2), (16, 2), (32, 2), (12, 1)])
def test_edge_lengths_heads_dtypes(D, fp8, hq, hkv):
    w = synth.Workload(f"edge{D}{int(fp8)}{hq}{hkv}", len(EDGE_LENS), hq, hkv, D, fp8,
                       pool_factor=1.5)
    b = DecodeBatch.build(w, 3, lens=np.array(EDGE_LENS))
    check_batch(b, paths=(0, 16, 512, -1))


def test_fp8_tensor_core_order_ties_and_large_batches():
    """The fp8 tensor-core decode ranks sequences by length (longest first)
    in batches of up to 256 and keeps the grid order beyond: equal lengths
    (ties broken by index), a batch of exactly 256, and one of 300 short
    sequences, every output against the oracle."""
    for S, lens in ((12, [640] * 6 + [129] * 6),
                    (256, np.random.default_rng(21).integers(1, 400, size=256)),
                    (300, np.random.default_rng(22).integers(1, 300, size=300))):
        w = synth.Workload(f"order{S}", S, 8, 2, 128, True, pool_factor=1.3)
        b = DecodeBatch.build(w, 4, lens=np.asarray(lens))
        check_batch(b, paths=(0,))


def test_fp8_tensor_core_chunk_boundaries():
    """Lengths on and around the 128-token chunks of the fp8 tensor-core
    decode, with GQA groups of 1, 4 and 8 (two instances of the kernel)."""
    lens = np.array([127, 128, 129, 255, 256, 257, 383, 384, 385, 1, 17, 8192])
    for hq, hkv in ((4, 4), (16, 4), (16, 2)):
        w = synth.Workload(f"chunks{hq}{hkv}", len(lens), hq, hkv, 128, True, pool_factor=1.2)
        b = DecodeBatch.build(w, 9, lens=lens)
        check_batch(b, paths=(0, -1))


SPLIT_EDGE_LENS = [1, 2, 15, 16, 17, 511, 512, 513, 1024, 1025, 2047, 2048, 2049, 2560, 3000,
                   3072]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("hq,hkv", [(16, 4), (64, 4)])
def test_split_chunks_of_several_partitions(D, fp8, hq, hkv):
    """160 sequences x 4 KV heads: enough CTAs that the split path streams
    chunks of several 512-token partitions per CTA (merged after each). The
    lengths cover one-token and partial last partitions and chunk
    boundaries (2048 / 2049 tokens for 4-partition chunks)."""
    rest = np.random.default_rng(11).integers(1, 3073, size=160 - len(SPLIT_EDGE_LENS))
    lens = np.concatenate([SPLIT_EDGE_LENS, rest])
    w = synth.Workload(f"owned{D}{int(fp8)}{hq}", len(lens), hq, hkv, D, fp8)
    b = DecodeBatch.build(w, 7, lens=lens)
    check_batch(b, subset=list(range(len(SPLIT_EDGE_LENS))) + [100, 159], paths=(512, 0))


def test_single_and_split_agree_closely():
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 4)
    b.step(partition_size=0)
    a = b.out.clone()
    b.decode(partition_size=32)
    assert torch.max(torch.abs(a - b.out)).item() <= 1e-5


def test_zero_length_context_gives_zeros():
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 5)
    b.step(partition_size=0)
    lens = b.context_lens.clone()
    lens[1] = 0
    for ps in (0, 64):
        out = torch.full_like(b.out, 7.0)
        pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, lens,
                  b.max_context_len, b.w.sm_scale, partition_size=ps)
        assert torch.all(out[1] == 0)
        assert torch.equal(out[0], b.out[0]) or torch.max(torch.abs(out[0] - b.out[0])) < 1e-5
    assert pa_get_device_error() == 0


def test_output_guards_untouched():
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 6)
    b.step(partition_size=0)
    n = b.out.numel()
    buf = torch.full((n + 2 * 64,), 123.0, device="cuda")
    out = buf[64:64 + n].view_as(b.out)
    for ps in (0, 32):
        pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
                  b.max_context_len, b.w.sm_scale, partition_size=ps)
        assert torch.all(buf[:64] == 123.0) and torch.all(buf[-64:] == 123.0)
        assert torch.max(torch.abs(out - b.out)).item() <= 1e-5


# ------------------------------------------------------------- invariances

def test_physical_block_relabelling_is_bit_identical():
    """Moving blocks to other physical ids (and the table with them) leaves
    every output bit unchanged ([Day28] §3.2: only the table translates)."""
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 7)
    for ps in (0, 32):
        b.step(partition_size=ps)
        ref = b.out.clone()
        pi = torch.randperm(b.num_blocks, generator=torch.Generator().manual_seed(1)).cuda()
        kc2 = torch.empty_like(b.k_cache)
        vc2 = torch.empty_like(b.v_cache)
        kc2[pi] = b.k_cache
        vc2[pi] = b.v_cache
        bt = b.block_tables.long()
        bt2 = torch.where(bt >= 0, pi[bt.clamp(min=0)], bt).to(torch.int32)
        out2 = torch.empty_like(b.out)
        pa_decode(out2, b.q, kc2, vc2, bt2, b.context_lens, b.max_context_len,
                  b.w.sm_scale, partition_size=ps)
        assert torch.equal(out2, ref)


def test_shared_prefix_equals_private_copies_bit_identical():
    """Sequences reading one shared set of prefix blocks give the same bits
    as with private copies ([Ch7] §7.1 前缀共享)."""
    w = dataclasses.replace(synth.WORKLOADS["prefix"], num_seqs=6, name="prefix6")
    b = DecodeBatch.build(w, 0)
    b.step(partition_size=0)
    ref = b.out.clone()
    nbpre = 62  # full prefix blocks, shared by all
    extra = w.num_seqs * nbpre
    kc2 = torch.cat([b.k_cache, b.k_cache[:1].repeat(extra, 1, 1, 1)])
    vc2 = torch.cat([b.v_cache, b.v_cache[:1].repeat(extra, 1, 1, 1)])
    bt2 = b.block_tables.clone()
    nxt = b.num_blocks
    for s in range(w.num_seqs):
        for j in range(nbpre):
            src = int(b.tables[s, j])
            kc2[nxt] = b.k_cache[src]
            vc2[nxt] = b.v_cache[src]
            bt2[s, j] = nxt
            nxt += 1
    out2 = torch.empty_like(b.out)
    pa_decode(out2, b.q, kc2, vc2, bt2, b.context_lens, b.max_context_len,
              w.sm_scale, partition_size=0)
    assert torch.equal(out2, ref)


# ------------------------------------------------------ device-side checks

def test_block_id_outside_pool_reads_zeros_and_is_flagged():
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 8)
    b.step(partition_size=0)
    bt = b.block_tables.clone()
    bt[0, 0] = b.num_blocks + 5
    bt[1, 0] = -3
    out = torch.empty_like(b.out)
    pa_decode(out, b.q, b.k_cache, b.v_cache, bt, b.context_lens,
              b.max_context_len, b.w.sm_scale, partition_size=0)
    assert pa_get_device_error() & PA_DEVERR_BLOCK_RANGE
    assert torch.all(torch.isfinite(out))
    assert torch.equal(out[2:], b.out[2:])


def test_context_longer_than_bound_is_clamped_and_flagged():
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 9)
    b.step(partition_size=0)
    lens = b.context_lens.clone()
    lens[0] = b.max_context_len + 1000
    out = torch.empty_like(b.out)
    pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, lens,
              b.max_context_len, b.w.sm_scale, partition_size=0)
    assert pa_get_device_error() & PA_DEVERR_CONTEXT_CLAMP
    assert torch.all(torch.isfinite(out[1:]))


def test_forced_split_without_workspace_is_rejected():
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 10)
    with pytest.raises(PagedAttentionError) as e:
        pa_decode(b.out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
                  b.max_context_len, b.w.sm_scale, partition_size=512,
                  workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 3
