"""The seeded synthetic inputs: the five workload shapes, the length
distributions, determinism and independence of the streams, and the NaN
sentinels that fill every cache slot no sequence owns."""
import dataclasses
import math

import numpy as np
import torch

import synth


def test_workload_shapes():
    W = synth.WORKLOADS
    shape = lambda w: (w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.kv_fp8)
    assert shape(W["tiny"]) == (4, 8, 8, 64, False) and W["tiny"].pool_blocks == 80
    assert shape(W["llama7b"]) == (64, 32, 32, 128, False)
    assert shape(W["prefix"]) == (256, 40, 40, 128, False) and W["prefix"].prefix_len == 1000
    assert shape(W["gqa_fp8"]) == (128, 32, 8, 128, True) and W["gqa_fp8"].group == 4
    assert shape(W["long"]) == (8, 64, 8, 128, False) and W["long"].partition_size == 512
    assert W["llama7b"].sm_scale == 1 / math.sqrt(128) and W["tiny"].sm_scale == 0.125


def test_uniform_lengths_cover_their_range_and_repeat_per_seed():
    for name in ("tiny", "llama7b", "gqa_fp8", "long"):
        w = synth.WORKLOADS[name]
        a = synth.draw_lengths(w, 0)
        assert a.dtype == np.int64 and a.shape == (w.num_seqs,)
        assert a.min() >= w.len_lo and a.max() <= w.len_hi
        np.testing.assert_array_equal(a, synth.draw_lengths(w, 0))
        assert not np.array_equal(a, synth.draw_lengths(w, 1))


def test_prefix_lengths_are_the_prefix_plus_a_clipped_lognormal_suffix():
    w = synth.WORKLOADS["prefix"]
    L = synth.draw_lengths(w, 0)
    suf = L - 1000
    assert suf.min() >= 1 and suf.max() <= 3072
    # median 300 (exp of ln 300), sigma 1: half the suffixes lie below 300
    assert 0.35 < np.mean(suf < 300) < 0.65
    big = synth.draw_lengths(dataclasses.replace(w, num_seqs=20000), 0) - 1000
    assert abs(np.median(big) - 300) < 15
    assert abs(np.std(np.log(big[(big > 1) & (big < 3072)])) - 1.0) < 0.05


def test_streams_are_independent_per_purpose():
    a = synth.rng(0, "llama7b", "q").standard_normal(4)
    b = synth.rng(0, "llama7b", "k_old").standard_normal(4)
    c = synth.rng(0, "prefix", "q").standard_normal(4)
    assert not np.allclose(a, b) and not np.allclose(a, c)
    assert synth.stream_seed(0, "llama7b", "q") == synth.stream_seed(0, "llama7b", "q")


def test_randn_bf16_draws():
    x = synth.randn_bf16((64, 1024), 0, "llama7b", "q")
    assert x.dtype == torch.bfloat16
    assert torch.equal(x, synth.randn_bf16((64, 1024), 0, "llama7b", "q"))
    assert not torch.equal(x, synth.randn_bf16((64, 1024), 0, "llama7b", "k_new"))
    f = x.float()
    assert abs(f.mean().item()) < 0.02 and abs(f.std().item() - 1.0) < 0.02


def test_sentinels_are_nan():
    b = torch.tensor([synth.SENTINEL_BF16], dtype=torch.int32).to(torch.int16)
    assert torch.isnan(b.view(torch.bfloat16).float()).all()
    f8 = torch.tensor([synth.SENTINEL_FP8], dtype=torch.uint8).view(torch.float8_e4m3fn)
    assert torch.isnan(f8.float()).all()


def test_prompt_rows_depend_on_the_whole_prefix():
    """Rows agree exactly where two token lists share a prefix and differ
    from the first differing token on, even if later tokens agree again."""
    a = [5, 6, 7, 8, 9]
    b = [5, 6, 1, 8, 9]
    ka, va = synth.prompt_kv_rows(a, 3, 2, 16)
    kb, vb = synth.prompt_kv_rows(b, 3, 2, 16)
    assert ka.dtype == torch.bfloat16 and ka.shape == (5, 2, 16)
    assert torch.equal(ka[:2], kb[:2]) and torch.equal(va[:2], vb[:2])
    for i in range(2, 5):
        assert not torch.equal(ka[i], kb[i]) and not torch.equal(va[i], vb[i])
    assert not torch.equal(ka, va)
    k2, _ = synth.prompt_kv_rows(a, 4, 2, 16)     # another seed, other rows
    assert not torch.equal(ka[0], k2[0])
    kx, _ = synth.prompt_kv_rows(a[:3], 3, 2, 16)  # a prefix alone: same rows
    assert torch.equal(kx, ka[:3])
