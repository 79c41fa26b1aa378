"""The Python binding's own checks, on CPU: tensors on the host are refused
(there is no CPU path to fall back to), as are wrong dtypes, ranks and
layouts — all before anything reaches the library."""
import pytest
import torch

import paged_kv_cache_429_b200 as pa

S, HQ, HKV, D, NB = 2, 4, 2, 64, 8


def decode_args(**over):
    a = dict(out=torch.empty(S, HQ, D), q=torch.empty(S, HQ, D, dtype=torch.bfloat16),
             k_cache=torch.empty(NB, HKV, 16, D, dtype=torch.bfloat16),
             v_cache=torch.empty(NB, HKV, 16, D, dtype=torch.bfloat16),
             block_tables=torch.zeros(S, 2, dtype=torch.int32),
             context_lens=torch.ones(S, dtype=torch.int32))
    a.update(over)
    return a


def call_decode(a):
    return pa.pa_decode(a["out"], a["q"], a["k_cache"], a["v_cache"], a["block_tables"],
                        a["context_lens"], 32, 0.125, partition_size=0)


def test_host_tensors_are_refused_by_every_launching_call():
    a = decode_args()
    with pytest.raises(ValueError, match="CUDA device"):
        call_decode(a)
    with pytest.raises(ValueError, match="CUDA device"):
        pa.pa_decode_no_alloc(a["out"], a["q"], a["k_cache"], a["v_cache"],
                              a["block_tables"], a["context_lens"], 32, 0.125)
    new = torch.empty(S, HKV, D, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA device"):
        pa.pa_decode_append(a["out"], a["q"], new, new.clone(), a["k_cache"], a["v_cache"],
                            a["block_tables"], a["context_lens"], 32, 0.125)
    with pytest.raises(ValueError, match="CUDA device"):
        pa.pa_reshape_and_cache(new, new.clone(), a["k_cache"], a["v_cache"],
                                torch.zeros(S, dtype=torch.int64))
    with pytest.raises(ValueError, match="CUDA device"):
        pa.pa_copy_blocks(a["k_cache"], a["v_cache"], torch.zeros(1, 2, dtype=torch.int64))
    with pytest.raises(ValueError, match="CUDA device"):
        pa.pa_prefill(torch.empty(3, HQ, D), torch.empty(3, HQ, D, dtype=torch.bfloat16),
                      a["k_cache"], a["v_cache"], a["block_tables"],
                      torch.tensor([0, 1, 3], dtype=torch.int32), a["context_lens"],
                      2, 32, 0.125)


@pytest.mark.parametrize("bad,exc,match", [
    (torch.empty(S, HQ, D, dtype=torch.float16), TypeError, "dtype"),   # output is fp32
    (torch.empty(S * HQ, D), ValueError, "dims"),
    (torch.empty(S, D, HQ).transpose(1, 2), ValueError, "contiguous"),
])
def test_output_checks_come_before_anything_else(bad, exc, match):
    # out is checked first, dtype -> rank -> layout -> device
    with pytest.raises(exc, match=match):
        call_decode(decode_args(out=bad))


@pytest.mark.parametrize("t,dtypes,ndim,exc,match", [
    (torch.empty(S, HQ, D), (torch.bfloat16,), 3, TypeError, "dtype"),
    (torch.zeros(S, 2, dtype=torch.int64), (torch.int32,), 2, TypeError, "dtype"),
    (torch.empty(S * HQ * D, dtype=torch.bfloat16), (torch.bfloat16,), 3, ValueError, "dims"),
    (torch.zeros(2, S, dtype=torch.int32).t(), (torch.int32,), 2, ValueError, "contiguous"),
    (torch.zeros(S, 2, dtype=torch.int32), (torch.int32,), 2, ValueError, "CUDA device"),
    ([1, 2], (torch.int32,), 1, TypeError, "torch.Tensor"),
])
def test_argument_checker(t, dtypes, ndim, exc, match):
    with pytest.raises(exc, match=match):
        pa._need(t, "arg", dtypes, ndim)
