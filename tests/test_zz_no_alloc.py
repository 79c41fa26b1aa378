"""pa_decode_no_alloc: split-context decode without a caller workspace.

Some callers cannot allocate device memory: a C program or plugin that is
handed only its input and output buffers, or a serving loop that forbids
cudaMalloc after start-up because it can synchronise the device. For them
the library keeps its split-context scratch in a fixed array of its own.
This file checks, through the C ABI, that two calls in a row give the same
output as pa_decode with a caller-allocated workspace, and that a launch
needing more scratch than the array holds is refused without launching.
It is collected last so that a run stopping at the first failure has
already run every other test; it also passes when run on its own.
"""
import numpy as np
import pytest
import torch

import synth
from paged_kv_cache_429_b200 import _lib, kv_dtype_of, pa_decode
from paged_kv_cache_429_b200.batch import DecodeBatch

pytestmark = pytest.mark.gpu

PATH_TOL = 1e-5          # agreement required between decode paths in these tests
PA_ERR_WORKSPACE = 3
SCRATCH_BYTES = 16 << 20  # PA_NO_ALLOC_SCRATCH_BYTES in include/pa.h


def call_no_alloc(b, out, partition_size, block_tables=None, max_context_len=None):
    bt = b.block_tables if block_tables is None else block_tables
    w = b.w
    return _lib.lib().pa_decode_no_alloc(
        out.data_ptr(), b.q.data_ptr(), b.k_cache.data_ptr(), b.v_cache.data_ptr(),
        kv_dtype_of(b.k_cache), b.k_scale, b.v_scale, bt.data_ptr(), bt.shape[1],
        b.context_lens.data_ptr(),
        b.max_context_len if max_context_len is None else max_context_len,
        w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, 16, b.num_blocks,
        w.sm_scale, partition_size, torch.cuda.current_stream().cuda_stream)


def reference_decode(b, ps):
    """pa_decode with a caller workspace whose every float is NaN, so a read
    of anything the call did not write would show in its output."""
    ws = b.workspace(ps)
    assert ws.numel() <= SCRATCH_BYTES
    ws.fill_(0xFF)   # 0xFFFFFFFF is a NaN in binary32
    ref = torch.full_like(b.out, float("nan"))
    pa_decode(ref, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
              b.max_context_len, b.w.sm_scale, k_scale=b.k_scale,
              v_scale=b.v_scale, partition_size=ps, workspace=ws)
    return ref


def test_two_calls_in_a_row_match_pa_decode():
    """The shared array keeps whatever the previous call left in it, so each
    call must read only what it wrote itself. The llama7b-shaped batch with
    512-token partitions fills several MB of the array; the tiny batch with
    32-token partitions (another partition count and row stride) then runs
    twice in a row on top of it, and llama7b runs again over the tiny
    batch's leftovers. Every result must match pa_decode run with a
    NaN-filled caller workspace."""
    big = DecodeBatch.build(synth.WORKLOADS["llama7b"], 1)
    big.step(partition_size=0)  # write the step's new tokens
    small = DecodeBatch.build(synth.WORKLOADS["tiny"], 0)
    small.step(partition_size=0)
    refs = {id(big): reference_decode(big, 512), id(small): reference_decode(small, 32)}
    for b, ps in ((big, 512), (small, 32), (small, 32), (big, 512)):
        out = torch.full_like(b.out, float("nan"))
        assert call_no_alloc(b, out, ps) == 0
        torch.cuda.synchronize()
        assert torch.all(torch.isfinite(out)), b.w.name
        assert torch.max(torch.abs(out - refs[id(b)])).item() <= PATH_TOL, b.w.name


def test_scratch_larger_than_the_array_is_refused():
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 2)
    # a table wide enough that 512-token partitions over its full width would
    # need more than the array: 4 seqs * 8 heads * P * (64 + 2) * 4 bytes
    P = SCRATCH_BYTES // (4 * 8 * 66 * 4) + 2
    width = P * 512 // 16
    bt = torch.full((4, width), -1, dtype=torch.int32, device="cuda")
    bt[:, :b.block_tables.shape[1]] = b.block_tables
    out = torch.full_like(b.out, 7.0)
    rc = call_no_alloc(b, out, 512, block_tables=bt, max_context_len=width * 16)
    torch.cuda.synchronize()
    assert rc == PA_ERR_WORKSPACE
    assert torch.all(out == 7.0)
    # a bad partition size is an argument error
    assert call_no_alloc(b, out, 0) == 1 and call_no_alloc(b, out, 100) == 1
    assert np.all(out.cpu().numpy() == 7.0)


def test_python_binding_matches_the_c_call():
    from paged_kv_cache_429_b200 import pa_decode_no_alloc
    b = DecodeBatch.build(synth.WORKLOADS["tiny"], 3)
    b.step(partition_size=0)
    a = torch.full_like(b.out, float("nan"))
    assert call_no_alloc(b, a, 64) == 0
    c = torch.full_like(b.out, float("nan"))
    pa_decode_no_alloc(c, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
                       b.max_context_len, b.w.sm_scale, partition_size=64)
    torch.cuda.synchronize()
    assert torch.equal(a, c)
