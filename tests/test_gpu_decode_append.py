"""pa_decode_append: the decode step with the new tokens' cache write fused
into the decode launch.

The fused step must leave the caches and the output bit for bit as the
separate pa_reshape_and_cache + pa_decode step does (same bytes written,
same arithmetic read), on every path (single-pass, split, bf16, fp8, head
dims, GQA groups, shared prefixes whose last block is copied first), and
match the fp64 oracle; table entries outside the pool are not written and
are flagged.
"""
import numpy as np
import pytest
import torch

import synth
from paged_kv_cache_429_b200 import pa_decode_append, pa_get_device_error
from paged_kv_cache_429_b200.batch import DecodeBatch
from parity_harness import (assert_cache_equal, max_abs_err, oracle_caches,
                            oracle_decode, tolerance)

pytestmark = pytest.mark.gpu
PA_DEVERR_BLOCK_RANGE = 0x10


@pytest.fixture(autouse=True)
def _clean():
    pa_get_device_error()
    yield
    torch.cuda.empty_cache()


def as_bytes(t):
    return t.contiguous().view(torch.uint8)


def fused_vs_separate(b, ps):
    """Run the step both ways from the same cache state; return the fused
    step's output after checking caches and outputs are bit-identical."""
    k0, v0 = b.k_cache.clone(), b.v_cache.clone()
    ws = b.workspace(ps)
    b.step(partition_size=ps, workspace=ws)
    torch.cuda.synchronize()
    out_sep = b.out.clone()
    k_sep, v_sep = b.k_cache.clone(), b.v_cache.clone()
    b.k_cache.copy_(k0)
    b.v_cache.copy_(v0)
    b.out.fill_(float("nan"))
    b.step_fused(partition_size=ps, workspace=ws)
    torch.cuda.synchronize()
    assert pa_get_device_error() == 0
    assert torch.equal(as_bytes(b.k_cache), as_bytes(k_sep))
    assert torch.equal(as_bytes(b.v_cache), as_bytes(v_sep))
    assert torch.equal(b.out.view(torch.int32), out_sep.view(torch.int32))
    return b.out


@pytest.mark.parametrize("name,ps", [("tiny", 0), ("tiny", 32), ("llama7b", -1),
                                     ("llama7b", 512), ("gqa_fp8", -1), ("gqa_fp8", 512),
                                     ("prefix", -1)])
def test_fused_step_is_bit_identical_to_write_then_decode(name, ps):
    b = DecodeBatch.build(synth.WORKLOADS[name], 0)
    fused_vs_separate(b, ps)


EDGE_LENS = [1, 2, 15, 16, 17, 31, 32, 33, 100, 511, 512, 513, 1040]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("hq,hkv", [(8, 8), (32, 2), (12, 1)])
def test_fused_step_edge_lengths(D, fp8, hq, hkv):
    w = synth.Workload(f"app{D}{int(fp8)}{hq}{hkv}", len(EDGE_LENS), hq, hkv, D, fp8,
                       pool_factor=1.5)
    b = DecodeBatch.build(w, 5, lens=np.array(EDGE_LENS))
    for ps in (0, 16, 512):
        fused_vs_separate(b, ps)


def test_fused_step_matches_the_oracle():
    b = DecodeBatch.build(synth.WORKLOADS["gqa_fp8"], 1)
    subset = [0, 9, 127]
    kc, vc = oracle_caches(b, subset)
    ref = oracle_decode(b, kc, vc, subset)
    b.step_fused()
    torch.cuda.synchronize()
    assert pa_get_device_error() == 0
    assert_cache_equal(b, kc, vc, subset)
    assert max_abs_err(b.out, ref, subset) <= tolerance(b)


def test_out_of_pool_last_block_is_not_written_and_is_flagged():
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 6)
    bt = b.block_tables.clone()
    L0 = int(b.lens[0])
    bt[0, (L0 - 1) // 16] = b.num_blocks + 9   # sequence 0's last block
    k0, v0 = b.k_cache.clone(), b.v_cache.clone()
    out = torch.full_like(b.out, float("nan"))
    pa_decode_append(out, b.q, b.k_new, b.v_new, b.k_cache, b.v_cache, bt, b.context_lens,
                     b.max_context_len, b.w.sm_scale, partition_size=0)
    torch.cuda.synchronize()
    assert pa_get_device_error() & PA_DEVERR_BLOCK_RANGE
    assert torch.all(torch.isfinite(out))
    # sequence 0's new token went nowhere; the others' were written
    b2 = DecodeBatch.build(synth.WORKLOADS["tiny"], 6)
    b2.step(partition_size=0)
    torch.cuda.synchronize()
    real = b.tables[0, (L0 - 1) // 16]
    assert torch.equal(as_bytes(b.k_cache[real]), as_bytes(k0[real]))
    for s in range(1, b.w.num_seqs):
        L = int(b.lens[s])
        blk = b.tables[s, (L - 1) // 16]
        assert torch.equal(as_bytes(b.k_cache[blk]), as_bytes(b2.k_cache[blk]))
        assert torch.equal(out[s].view(torch.int32), b2.out[s].view(torch.int32))
