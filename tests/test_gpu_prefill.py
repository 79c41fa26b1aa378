"""GPU parity of chunked prefill attention against the fp64 oracle.

Each case fills a paged cache through the pool and reshape_and_cache (every
slot first set to NaN), then prefills the last n_s tokens of each sequence:
whole prompts (n = L), chunks after a cached prefix (n < L), and one-token
chunks (= decode).
"""

import numpy as np
import pytest
import torch

import oracle
import synth
from paged_kv_cache_429_b200 import pa_decode, pa_get_device_error, pa_prefill
from paged_kv_cache_429_b200.batch import DecodeBatch
from parity_harness import BF16_TOL, oracle_caches, to_u16

pytestmark = pytest.mark.gpu
PA_DEVERR_BLOCK_RANGE = 0x10


@pytest.fixture(autouse=True)
def _clean():
    pa_get_device_error()
    yield
    torch.cuda.empty_cache()


def build(hq, hkv, d, lens, chunks, seed=0):
    w = synth.Workload(f"prefill{hq}_{hkv}_{d}", len(lens), hq, hkv, d, False, pool_factor=1.3)
    b = DecodeBatch.build(w, seed, lens=np.array(lens))
    b.run_ops(b.step_ops)  # the whole context, chunk included, is in the cache
    T = int(sum(chunks))
    q = synth.randn_bf16((T, hq, d), seed, w.name, "q_prefill", "cuda")
    qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    return b, q, qs


def run_prefill(b, q, qs, chunks):
    out = torch.full((q.shape[0], q.shape[1], q.shape[2]), float("nan"), device="cuda")
    pa_prefill(out, q, b.k_cache, b.v_cache, b.block_tables,
               torch.from_numpy(qs).cuda(), b.context_lens, int(max(chunks)),
               b.max_context_len, b.w.sm_scale)
    torch.cuda.synchronize()
    return out


def check(b, q, qs, chunks):
    out = run_prefill(b, q, qs, chunks)
    assert pa_get_device_error() == 0
    kc, vc = oracle_caches(b)
    ref = oracle.paged_prefill(to_u16(q), kc, vc, b.tables, qs, b.lens.astype(np.int32),
                               b.w.sm_scale)
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got))
    err = float(np.max(np.abs(got - ref)))
    assert err <= BF16_TOL, err
    return out


LENS = [1, 15, 16, 17, 100, 513, 1040]
CHUNKS = [1, 15, 16, 5, 100, 64, 300]   # whole prompts, chunks, one token


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 2), (32, 8), (12, 1), (16, 1)])
def test_prefill_mixed_chunks(d, hq, hkv):
    b, q, qs = build(hq, hkv, d, LENS, CHUNKS)
    check(b, q, qs, CHUNKS)


def test_prefill_long_prompt():
    b, q, qs = build(32, 8, 128, [4096, 3000], [4096, 1000], seed=1)
    check(b, q, qs, [4096, 1000])


def test_one_token_chunks_match_decode():
    """A one-token chunk is a decode step ([Day28] FAQ Q4): the prefill and
    the decode compute the same function. They round P differently (the
    prefill to fp16, the decode to a high and a low bf16 half), so each is
    held to the oracle tolerance, and so is their difference."""
    lens = [33, 200, 1, 64]
    b, q, qs = build(16, 4, 128, lens, [1, 1, 1, 1], seed=2)
    pre = check(b, q, qs, [1, 1, 1, 1])
    dec = torch.empty_like(pre)
    pa_decode(dec, q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
              b.max_context_len, b.w.sm_scale, partition_size=0)
    torch.cuda.synchronize()
    kc, vc = oracle_caches(b)
    ref = oracle.paged_decode(to_u16(q), kc, vc, b.tables, b.lens.astype(np.int32),
                              b.w.sm_scale)
    assert float(np.max(np.abs(dec.double().cpu().numpy() - ref))) <= BF16_TOL
    assert torch.max(torch.abs(pre - dec)).item() <= BF16_TOL


def test_prefill_leaves_rows_outside_the_chunks_alone():
    b, q, qs = build(8, 8, 64, [40, 20], [10, 20], seed=3)
    big = torch.full((q.shape[0] + 8, 8, 64), 5.0, device="cuda")
    out = big[4:4 + q.shape[0]]
    pa_prefill(out, q, b.k_cache, b.v_cache, b.block_tables, torch.from_numpy(qs).cuda(),
               b.context_lens, 20, b.max_context_len, b.w.sm_scale)
    torch.cuda.synchronize()
    assert torch.all(big[:4] == 5.0) and torch.all(big[-4:] == 5.0)
    assert torch.all(torch.isfinite(out))


def test_block_id_outside_pool_reads_zeros_and_is_flagged():
    """Table entries outside [0, num_blocks) read as zero K/V and set
    PA_DEVERR_BLOCK_RANGE; other sequences are unaffected."""
    lens, chunks = [40, 200, 90], [40, 64, 30]
    b, q, qs = build(8, 2, 128, lens, chunks, seed=4)
    good = run_prefill(b, q, qs, chunks)
    assert pa_get_device_error() == 0
    bt = b.block_tables.clone()
    bt[0, 1] = b.num_blocks + 3
    bt[1, 0] = -7
    out = torch.full_like(good, float("nan"))
    pa_prefill(out, q, b.k_cache, b.v_cache, bt, torch.from_numpy(qs).cuda(), b.context_lens,
               int(max(chunks)), b.max_context_len, b.w.sm_scale)
    torch.cuda.synchronize()
    assert pa_get_device_error() & PA_DEVERR_BLOCK_RANGE
    assert torch.all(torch.isfinite(out))
    s2 = slice(int(qs[2]), int(qs[3]))
    assert torch.equal(out[s2], good[s2])
    # the oracle with those blocks' K/V zeroed gives the same answer
    kc, vc = oracle_caches(b)
    tables = b.tables.copy()
    zero_id = b.num_blocks  # an extra all-zero block appended to the caches
    kc = np.concatenate([kc, np.zeros_like(kc[:1])])
    vc = np.concatenate([vc, np.zeros_like(vc[:1])])
    tables[0, 1] = zero_id
    tables[1, 0] = zero_id
    ref = oracle.paged_prefill(to_u16(q), kc, vc, tables, qs, b.lens.astype(np.int32),
                               b.w.sm_scale)
    assert float(np.max(np.abs(out.double().cpu().numpy() - ref))) <= BF16_TOL


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_mha_long_chunks_span_many_query_tiles(d):
    """Group 1 (128 tokens per query tile, 256 per CTA): chunks that end
    inside the first or the second tile of a CTA and span several CTAs."""
    lens = [1500, 700, 257, 129]
    chunks = [1500, 300, 257, 128]
    b, q, qs = build(4, 4, d, lens, chunks, seed=5)
    check(b, q, qs, chunks)


@pytest.mark.parametrize("scale", [6.0, 24.0])
def test_prefill_large_scores_raise_the_running_max(scale):
    """Queries scaled up so that scores spread over tens of units in the
    exp2 domain: key tiles after a row's first one overflow the speculative
    pass (their P sum passes 2^15) and are redone max first, raising the
    running maximum and rescaling O in tensor memory, and some rows' weight
    concentrates on a late key. The result still matches the oracle."""
    lens = [2048, 1100, 300]
    chunks = [2048, 600, 300]
    b, q, qs = build(32, 8, 128, lens, chunks, seed=7)
    q = (q.float() * scale).to(torch.bfloat16)
    check(b, q, qs, chunks)
