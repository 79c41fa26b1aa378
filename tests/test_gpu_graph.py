"""The library's calls can be captured in a CUDA graph.

They launch only on the given stream, never synchronise and allocate
nothing (the split path's workspace is the caller's), so a decode step —
the new tokens' write (after any copy-on-write copy) and the decode, or the
fused pa_decode_append — can be captured once and replayed. Capturing must
run nothing, and a replay must leave the caches and the output bit for bit
as the same step run eagerly from the same state.
"""
import pytest
import torch

import synth
from paged_kv_cache_429_b200 import pa_get_device_error
from paged_kv_cache_429_b200.batch import DecodeBatch

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean():
    pa_get_device_error()
    yield
    torch.cuda.empty_cache()


def as_bytes(t):
    return t.contiguous().view(torch.uint8)


def restore(b, k0, v0):
    b.k_cache.copy_(k0)
    b.v_cache.copy_(v0)
    b.out.zero_()
    torch.cuda.synchronize()


@pytest.mark.parametrize("name,ps", [("tiny", 0), ("tiny", 64), ("gqa_fp8", 0),
                                     ("gqa_fp8", 512)])
@pytest.mark.parametrize("fused", [False, True])
def test_captured_step_replays_the_eager_step(name, ps, fused):
    b = DecodeBatch.build(synth.WORKLOADS[name], 0, "cuda:0")
    ws = b.workspace(ps) if ps else None

    def step():
        if fused:
            b.step_fused(partition_size=ps, workspace=ws)
        else:
            b.step(partition_size=ps, workspace=ws)

    k0, v0 = b.k_cache.clone(), b.v_cache.clone()
    step()
    torch.cuda.synchronize()
    out_e, k_e, v_e = b.out.clone(), b.k_cache.clone(), b.v_cache.clone()

    # warm the launch path on a side stream, as graph capture expects
    restore(b, k0, v0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    restore(b, k0, v0)

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    torch.cuda.synchronize()
    # capturing ran nothing
    assert torch.count_nonzero(b.out) == 0
    assert torch.equal(as_bytes(b.k_cache), as_bytes(k0))

    for _ in range(2):  # the step is idempotent from this state
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(as_bytes(b.out), as_bytes(out_e))
        assert torch.equal(as_bytes(b.k_cache), as_bytes(k_e))
        assert torch.equal(as_bytes(b.v_cache), as_bytes(v_e))
    del g
    assert pa_get_device_error() == 0
