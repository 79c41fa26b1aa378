"""GPU parity of the cache writes against the oracle: bit-exact bytes."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_429_b200 import (pa_copy_blocks, pa_get_device_error,
                                     pa_reshape_and_cache)
from parity_harness import to_u16, to_u8

pytestmark = pytest.mark.gpu
PA_DEVERR_SLOT_RANGE = 0x1
PA_DEVERR_PAIR_RANGE = 0x2


@pytest.fixture(autouse=True)
def _clean():
    pa_get_device_error()
    yield
    torch.cuda.synchronize()


def bf16_dev(shape, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)


def cache_with_guards(nb, h, d, fp8, guard=3):
    """Cache tensor with `guard` canary blocks on each side; returns
    (full tensor, view of the nb usable blocks)."""
    if fp8:
        full = torch.full((nb + 2 * guard, h, 16, d), 0x5A, dtype=torch.uint8, device="cuda")
    else:
        full = torch.full((nb + 2 * guard, h, 16, d), 0x5A5A, dtype=torch.int16,
                          device="cuda").view(torch.bfloat16)
    return full, full[guard:guard + nb]


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("D", [64, 128])
def test_reshape_matches_oracle_bit_exact(fp8, D):
    T, H, NB = 300, 4, 40
    rng = np.random.default_rng(D + fp8)
    slots = rng.permutation(NB * 16)[:T].astype(np.int64)
    slots[::17] = -1  # padding tokens are skipped
    key, val = bf16_dev((T, H, D), 1), bf16_dev((T, H, D), 2)
    ks, vs = (3.9 / 448, 4.4 / 448) if fp8 else (1.0, 1.0)
    kfull, kc = cache_with_guards(NB, H, D, fp8)
    vfull, vc = cache_with_guards(NB, H, D, fp8)
    k0, v0 = kfull.clone(), vfull.clone()
    pa_reshape_and_cache(key, val, kc, vc, torch.from_numpy(slots).cuda(),
                         k_scale=ks, v_scale=vs)
    conv = to_u8 if fp8 else to_u16
    hk, hv = conv(k0[3:3 + NB]).copy(), conv(v0[3:3 + NB]).copy()
    oracle.reshape_and_cache(to_u16(key), to_u16(val), hk, hv, slots,
                             oracle.KV_FP8_E4M3 if fp8 else oracle.KV_BF16, ks, vs)
    np.testing.assert_array_equal(conv(kc), hk)
    np.testing.assert_array_equal(conv(vc), hv)
    # canary blocks on both sides untouched
    assert torch.equal(kfull[:3], k0[:3]) and torch.equal(kfull[-3:], k0[-3:])
    assert torch.equal(vfull[:3], v0[:3]) and torch.equal(vfull[-3:], v0[-3:])
    assert pa_get_device_error() == 0


@pytest.mark.parametrize("scale", [1.0, 0.5, 3.7 / 448, 5.3 / 448, 1e-3 / 448, 300.0 / 448])
def test_fp8_quantisation_exhaustive_bf16(scale):
    """Every bf16 bit pattern through the device quantiser (x / scale, E4M3
    RNE with saturation) equals the oracle's encoder bit for bit; NaN
    inputs must give a NaN code."""
    scale = float(np.float32(scale))
    bits = np.arange(65536, dtype=np.int64).astype(np.uint16)
    H, D = 4, 128
    T = 65536 // (H * D)
    src = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16).reshape(T, H, D)
    kc = torch.zeros((T, H, 16, D), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    slots = torch.arange(T, dtype=torch.int64, device="cuda") * 16  # offset 0 of block t
    pa_reshape_and_cache(src, src, kc, vc, slots, k_scale=scale, v_scale=scale)
    got = to_u8(kc[:, :, 0, :]).reshape(-1)
    ref = oracle.quantize_bf16_array(bits, scale)
    x = (bits.astype(np.uint32) << 16).view(np.float32)
    nan = np.isnan(x)
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert np.all((got[nan] & 0x7F) == 0x7F)
    np.testing.assert_array_equal(to_u8(vc[:, :, 0, :]).reshape(-1), got)


def test_reshape_out_of_range_slot_is_skipped_and_flagged():
    T, H, D, NB = 8, 2, 64, 4
    key, val = bf16_dev((T, H, D), 3), bf16_dev((T, H, D), 4)
    kfull, kc = cache_with_guards(NB, H, D, False)
    vfull, vc = cache_with_guards(NB, H, D, False)
    k0 = kfull.clone()
    slots = np.array([0, 1, NB * 16, 5, NB * 16 + 100, 2**40, 7, -5], dtype=np.int64)
    pa_reshape_and_cache(key, val, kc, vc, torch.from_numpy(slots).cuda())
    assert pa_get_device_error() & PA_DEVERR_SLOT_RANGE
    hk = to_u16(k0[3:3 + NB]).copy()
    hv = hk.copy()
    good = slots.copy()
    good[(good >= NB * 16)] = -1
    oracle.reshape_and_cache(to_u16(key), to_u16(val), hk, hv, good, oracle.KV_BF16)
    np.testing.assert_array_equal(to_u16(kc), hk)
    assert torch.equal(kfull[:3], k0[:3]) and torch.equal(kfull[-3:], k0[-3:])


@pytest.mark.parametrize("fp8", [False, True])
def test_copy_blocks_matches_oracle_bit_exact(fp8):
    NB, H, D = 64, 8, 128
    rng = np.random.default_rng(7)
    if fp8:
        k = torch.randint(0, 256, (NB, H, 16, D), dtype=torch.uint8, device="cuda")
    else:
        k = torch.randint(-32768, 32767, (NB, H, 16, D), dtype=torch.int16,
                          device="cuda").view(torch.bfloat16)
    v = k.flip(0).contiguous()
    perm = rng.permutation(NB)
    pairs = np.stack([perm[:20], perm[20:40]], axis=1).astype(np.int64)
    conv = to_u8 if fp8 else to_u16
    hk, hv = conv(k).copy(), conv(v).copy()
    pa_copy_blocks(k, v, torch.from_numpy(pairs).cuda())
    oracle.copy_blocks(hk, hv, pairs)
    np.testing.assert_array_equal(conv(k), hk)
    np.testing.assert_array_equal(conv(v), hv)
    assert pa_get_device_error() == 0


def test_copy_blocks_out_of_range_pair_is_skipped_and_flagged():
    NB, H, D = 8, 2, 64
    kfull, k = cache_with_guards(NB, H, D, False)
    vfull, v = cache_with_guards(NB, H, D, False)
    k.copy_(bf16_dev(k.shape, 9))
    v.copy_(bf16_dev(v.shape, 10))
    k0, v0 = kfull.clone(), vfull.clone()
    pairs = np.array([[1, 2], [3, NB], [-1, 4], [5, 6]], dtype=np.int64)
    pa_copy_blocks(k, v, torch.from_numpy(pairs).cuda())
    assert pa_get_device_error() & PA_DEVERR_PAIR_RANGE
    hk, hv = to_u16(k0[3:3 + NB]).copy(), to_u16(v0[3:3 + NB]).copy()
    oracle.copy_blocks(hk, hv, pairs[[0, 3]])
    np.testing.assert_array_equal(to_u16(k), hk)
    np.testing.assert_array_equal(to_u16(v), hv)
    assert torch.equal(kfull[:3], k0[:3]) and torch.equal(kfull[-3:], k0[-3:])
