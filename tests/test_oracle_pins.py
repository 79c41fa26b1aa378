"""Pins of the CPU oracle against things other than itself.

Each test fixes part of the oracle with something independent of its code:
numbers the pages print (tests/golden/, each with its citation), closed
forms, invariants, library routines (torch float64 SDPA, torch's float8
conversion) and a second, test-local brute-force formulation in numpy.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ----------------------------------------------------------------- helpers

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float values to bf16 (RNE, via torch) and return the bits."""
    t = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def make_case(rng, S, Hq, Hkv, D, lens, NB, B=16):
    """Random bf16 case: q, caches, block tables from a random permutation."""
    q = bf16_bits(rng.standard_normal((S, Hq, D)))
    kc = bf16_bits(rng.standard_normal((NB, Hkv, B, D)))
    vc = bf16_bits(rng.standard_normal((NB, Hkv, B, D)))
    maxb = max(1, max(-(-L // B) for L in lens))
    perm = rng.permutation(NB)
    bt = np.zeros((S, maxb), dtype=np.int32)
    k = 0
    for s, L in enumerate(lens):
        n = -(-L // B)
        bt[s, :n] = perm[k:k + n]
        k += n
    assert k <= NB
    return q, kc, vc, bt, np.asarray(lens, dtype=np.int32)


def numpy_attention(q, kc, vc, bt, lens, scale, B=16):
    """Second formulation: explicit K/V matrices by fancy indexing, then a
    softmax of the score vector — written independently of the oracle."""
    S, Hq, D = q.shape
    Hkv = kc.shape[1]
    g = Hq // Hkv
    out = np.zeros((S, Hq, D))
    qf = bits_to_f64(q)
    kf = bits_to_f64(kc)
    vf = bits_to_f64(vc)
    for s in range(S):
        L = int(lens[s])
        if L == 0:
            continue
        pos = np.arange(L)
        blocks = bt[s][pos // B]
        for hq in range(Hq):
            Km = kf[blocks, hq // g, pos % B, :]
            Vm = vf[blocks, hq // g, pos % B, :]
            z = scale * (Km @ qf[s, hq])
            w = np.exp(z - z.max())
            out[s, hq] = (w / w.sum()) @ Vm
    return out


# --------------------------------------------------- sizes and slots (pages)

def read_golden_rows(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


def test_kv_size_worked_examples(golden_dir):
    rows = read_golden_rows(os.path.join(golden_dir, "kv_size.txt"))
    assert len(rows) == 6
    for layers, heads, dim, nbytes, tokens, reqs, expected in rows:
        got = oracle.kv_cache_bytes(int(layers), int(heads), int(dim),
                                    int(nbytes), int(tokens), int(reqs))
        assert got == int(expected)
    # per-token form on its own (example 7-1: 0.625 MiB)
    assert oracle.kv_bytes_per_token(32, 40, 128, 2) == 655360
    assert oracle.kv_bytes_per_token(32, 40, 128, 2) / 2**20 == 0.625
    # fp8 halves it ([Ch7] §"KV cache 显存估算": bf16=2, fp8=1)
    assert 2 * oracle.kv_bytes_per_token(32, 40, 128, 1) == 655360


def test_block_table_example_slots(golden_dir):
    rows = read_golden_rows(os.path.join(golden_dir, "block_table_example.txt"))
    B = int(rows[0][1])
    table = [int(x) for x in rows[1][1:]]
    assert B == 16 and table == [7, 1, 3]
    for first, last, blk, s0, s1 in rows[2:]:
        for pos in range(int(first), int(last) + 1):
            got = oracle.slot(table, pos, B)
            assert got == int(s0) + (pos - int(first))
            assert got // B == int(blk)
        assert oracle.slot(table, int(last), B) == int(s1)


# ------------------------------------------------ attention: closed forms

def test_single_token_returns_its_value():
    rng = np.random.default_rng(1)
    q, kc, vc, bt, lens = make_case(rng, 3, 4, 4, 64, [1, 1, 1], 10)
    out = oracle.paged_decode(q, kc, vc, bt, lens, 0.125)
    for s in range(3):
        for h in range(4):
            np.testing.assert_array_equal(out[s, h], bits_to_f64(vc[bt[s, 0], h, 0]))


def test_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(2)
    lens = [37, 16, 5]
    q, kc, vc, bt, lens = make_case(rng, 3, 2, 2, 64, lens, 12)
    q[:] = 0
    out = oracle.paged_decode(q, kc, vc, bt, lens, 0.125)
    vf = bits_to_f64(vc)
    for s, L in enumerate(lens):
        pos = np.arange(L)
        for h in range(2):
            mean = vf[bt[s][pos // 16], h, pos % 16].mean(axis=0)
            np.testing.assert_allclose(out[s, h], mean, rtol=0, atol=1e-12)


def test_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(3)
    q, kc, vc, bt, lens = make_case(rng, 1, 1, 1, 128, [50], 6)
    kc[:] = kc[0, 0, 0]  # every key identical
    out = oracle.paged_decode(q, kc, vc, bt, lens, 1 / math.sqrt(128))
    vf = bits_to_f64(vc)
    pos = np.arange(50)
    mean = vf[bt[0][pos // 16], 0, pos % 16].mean(axis=0)
    np.testing.assert_allclose(out[0, 0], mean, rtol=0, atol=1e-12)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(4)
    q, kc, vc, bt, lens = make_case(rng, 1, 1, 1, 64, [40], 5)
    qf = bits_to_f64(q[0, 0])
    kc[:] = 0
    star = 23
    # key at position 23 is q itself scaled: z* = |q|^2 * 8 * scale >> others (0)
    kc[bt[0, star // 16], 0, star % 16] = bf16_bits(qf * 8.0)
    out = oracle.paged_decode(q, kc, vc, bt, lens, 1.0)
    z_star = float(bits_to_f64(kc[bt[0, star // 16], 0, star % 16]) @ qf)
    assert z_star > 50
    np.testing.assert_allclose(out[0, 0], bits_to_f64(vc[bt[0, star // 16], 0, star % 16]),
                               rtol=0, atol=1e-12)


def test_gqa_heads_read_kv_head_hq_over_group():
    """With V constant per KV head, query head hq must return the constant of
    KV head hq // g (contiguous groups), whatever q and K are."""
    rng = np.random.default_rng(5)
    S, Hq, Hkv, D = 2, 8, 2, 64
    q, kc, vc, bt, lens = make_case(rng, S, Hq, Hkv, D, [20, 33], 8)
    consts = [0.5, -2.0]
    for h in range(Hkv):
        vc[:, h] = bf16_bits(np.full(D, consts[h]))
    out = oracle.paged_decode(q, kc, vc, bt, lens, 0.125)
    for hq in range(Hq):
        np.testing.assert_allclose(out[:, hq], consts[hq // (Hq // Hkv)], atol=1e-12)


def test_empty_context_gives_zeros():
    rng = np.random.default_rng(6)
    q, kc, vc, bt, lens = make_case(rng, 2, 2, 2, 64, [0, 3], 4)
    out = oracle.paged_decode(q, kc, vc, bt, lens, 0.125)
    assert np.all(out[0] == 0.0)
    assert np.all(np.isfinite(out[1]))


def test_tail_slots_never_read():
    """NaN in unused slots of the last block and in unused blocks must not
    reach the output ([Day28] §4.2: waste is the unfilled part of the last
    block; its contents are not part of the sequence)."""
    rng = np.random.default_rng(7)
    lens = [17, 31, 1]
    q, kc, vc, bt, lens = make_case(rng, 3, 2, 2, 64, lens, 9)
    used = set()
    for s, L in enumerate(lens):
        for pos in range(int(L)):
            used.add((int(bt[s][pos // 16]), pos % 16))
    nan = bf16_bits(np.array([np.nan]))[0]
    for b in range(kc.shape[0]):
        for o in range(16):
            if (b, o) not in used:
                kc[b, :, o] = nan
                vc[b, :, o] = nan
    out = oracle.paged_decode(q, kc, vc, bt, lens, 0.125)
    assert np.all(np.isfinite(out))


# ------------------------------------------ attention: brute force, library

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_tiny_against_numpy_formulation(seed):
    rng = np.random.default_rng(100 + seed)
    lens = list(rng.integers(1, 21, size=4))
    q, kc, vc, bt, lens = make_case(rng, 4, 4, 2, 4, lens, 12)
    out = oracle.paged_decode(q, kc, vc, bt, lens, 0.5)
    ref = numpy_attention(q, kc, vc, bt, lens, 0.5)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_against_torch_sdpa_float64():
    """Tiny-config-shaped case (4 seqs, 8/8 heads, d64, L in [1, 256]) checked
    against torch's scaled_dot_product_attention in float64 on CPU over the
    gathered contiguous K/V."""
    rng = np.random.default_rng(11)
    lens = list(rng.integers(1, 257, size=4))
    q, kc, vc, bt, lens = make_case(rng, 4, 8, 8, 64, lens, 80)
    out = oracle.paged_decode(q, kc, vc, bt, lens, 1 / 8)
    qf, kf, vf = bits_to_f64(q), bits_to_f64(kc), bits_to_f64(vc)
    for s, L in enumerate(lens):
        pos = np.arange(int(L))
        K = torch.from_numpy(kf[bt[s][pos // 16], :, pos % 16]).permute(1, 0, 2)
        V = torch.from_numpy(vf[bt[s][pos // 16], :, pos % 16]).permute(1, 0, 2)
        Q = torch.from_numpy(qf[s]).unsqueeze(1)  # [H, 1, D]
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q, K, V, scale=1 / 8).squeeze(1).numpy()
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


def test_physical_block_permutation_invariance():
    """Renumbering physical blocks (moving their contents with them) changes
    nothing: the table translates positions ([OSPage] §PagedAttention 类比)."""
    rng = np.random.default_rng(12)
    lens = [45, 3, 64, 17]
    q, kc, vc, bt, lens = make_case(rng, 4, 4, 4, 64, lens, 16)
    out = oracle.paged_decode(q, kc, vc, bt, lens, 0.125)
    pi = rng.permutation(16)
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[pi] = kc
    vc2[pi] = vc
    bt2 = pi[bt].astype(np.int32)
    out2 = oracle.paged_decode(q, kc2, vc2, bt2, lens, 0.125)
    np.testing.assert_array_equal(out, out2)


def test_shared_prefix_equals_private_copies():
    """Two sequences pointing at the same prefix blocks give the same result
    as with private copies of those blocks ([Ch7] §7.1 前缀共享)."""
    rng = np.random.default_rng(13)
    q, kc, vc, bt, lens = make_case(rng, 2, 2, 2, 64, [40, 40], 10)
    bt_shared = bt.copy()
    bt_shared[1, :2] = bt[0, :2]  # seq 1 shares seq 0's first two blocks
    kc_priv, vc_priv = kc.copy(), vc.copy()
    kc_priv[bt[1, :2]] = kc[bt[0, :2]]
    vc_priv[bt[1, :2]] = vc[bt[0, :2]]
    a = oracle.paged_decode(q, kc, vc, bt_shared, lens, 0.125)
    b = oracle.paged_decode(q, kc_priv, vc_priv, bt, lens, 0.125)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("psize", [16, 32, 512])
def test_split_form_equals_single_pass(psize):
    rng = np.random.default_rng(14)
    lens = [1, 15, 16, 17, 513, 1100, 0]
    q, kc, vc, bt, lens = make_case(rng, 7, 4, 2, 64, lens, 200)
    a = oracle.paged_decode(q, kc, vc, bt, lens, 0.125)
    b = oracle.paged_decode_split(q, kc, vc, bt, lens, 0.125, psize)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


@pytest.mark.parametrize("psize", [16, 48, 512])
def test_split_form_equals_single_pass_fp8_gqa(psize):
    """The same identity on E4M3 caches (per-tensor scales) with GQA groups
    of 4: the partition + reduce form reaches the single-pass result."""
    rng = np.random.default_rng(17)
    lens = [1, 16, 31, 97, 700, 0]
    q, kc, vc, bt, lens = make_case(rng, 6, 8, 2, 128, lens, 120)
    k8 = oracle.quantize_bf16_array(kc, 0.01)
    v8 = oracle.quantize_bf16_array(vc, 0.02)
    kw = dict(kv_dtype=oracle.KV_FP8_E4M3, k_scale=0.01, v_scale=0.02)
    a = oracle.paged_decode(q, k8, v8, bt, lens, 128 ** -0.5, **kw)
    b = oracle.paged_decode_split(q, k8, v8, bt, lens, 128 ** -0.5, psize, **kw)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    assert np.all(a[5] == 0)  # empty context


def test_seq_subset_matches_full():
    rng = np.random.default_rng(15)
    q, kc, vc, bt, lens = make_case(rng, 5, 2, 2, 64, [5, 40, 18, 2, 33], 20)
    full = oracle.paged_decode(q, kc, vc, bt, lens, 0.125)
    sub = oracle.paged_decode(q, kc, vc, bt, lens, 0.125, seq_subset=[3, 1])
    np.testing.assert_array_equal(sub[[1, 3]], full[[1, 3]])
    assert np.all(np.isnan(sub[[0, 2, 4]]))


def test_bad_block_id_rejected():
    rng = np.random.default_rng(16)
    q, kc, vc, bt, lens = make_case(rng, 1, 1, 1, 64, [20], 4)
    bt[0, 1] = 4  # == num_blocks
    with pytest.raises(ValueError):
        oracle.paged_decode(q, kc, vc, bt, lens, 0.125)


# --------------------------------------------------------------------- fp8

def test_e4m3_decode_all_codes_against_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_decode(int(c)) for c in codes])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    # sign of zero too
    assert math.copysign(1.0, oracle.e4m3_decode(0x80)) == -1.0


def test_e4m3_decode_definition_points():
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x38) == 1.0
    assert math.isnan(oracle.e4m3_decode(0x7F))
    assert math.isnan(oracle.e4m3_decode(0xFF))
    assert oracle.e4m3_decode(0xFE) == -448.0


def test_e4m3_encode_boundaries():
    enc = oracle.e4m3_encode
    assert enc(464.0) == 0x7E          # tie between 448 and the NaN slot -> 448
    assert enc(1e30) == 0x7E and enc(-1e30) == 0xFE
    assert enc(float("inf")) == 0x7E and enc(float("-inf")) == 0xFE
    assert enc(float("nan")) == 0x7F
    assert enc(2.0 ** -10) == 0x00     # half of 2^-9: tie to even (0)
    assert enc(1.5 * 2.0 ** -10) == 0x01
    assert enc(2.5 * 2.0 ** -9) == 0x02  # tie between 2 and 3 -> 2
    assert enc(17.0) == 0x58           # 16 * 1.0625: tie -> mantissa 0
    assert enc(-0.0) == 0x80 and enc(0.0) == 0x00
    assert enc(448.0) == 0x7E and enc(449.0) == 0x7E
    # the subnormal/normal border: 15.5/16 of 2^-6 rounds up to 2^-6
    assert enc(2.0 ** -6 * (1 - 1 / 32)) == 0x08


@pytest.mark.parametrize("scale", [1.0, 0.5, 3.7 / 448, 5.3 / 448, 1e-3 / 448, 300.0 / 448])
def test_e4m3_quantize_exhaustive_bf16_against_torch(scale):
    """All 65,536 bf16 bit patterns: y = x / scale in binary32, then E4M3 RNE.
    torch's float8_e4m3fn conversion is RNE but turns |y| >= 464 into NaN
    instead of saturating, so it is the reference where |y| < 464; beyond,
    the saturation rule of the definition is checked directly."""
    scale = float(np.float32(scale))
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.quantize_bf16_array(bits, scale)
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float32)
    y = x / torch.tensor(scale, dtype=torch.float32)
    ref = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    yn = y.numpy()
    small = np.abs(yn) < 464
    np.testing.assert_array_equal(got[small], ref[small])
    big = (np.abs(yn) >= 464) & ~np.isnan(yn)
    expect_big = np.where(np.signbit(yn[big]), 0xFE, 0x7E).astype(np.uint8)
    np.testing.assert_array_equal(got[big], expect_big)
    assert np.all(got[np.isnan(yn)] == 0x7F)


def test_fp8_reshape_and_decode_use_dequantised_values():
    """fp8 decode equals bf16-free fp64 attention over decoded codes x scale."""
    rng = np.random.default_rng(17)
    S, H, D, NB = 2, 2, 64, 6
    lens = [20, 9]
    key = bf16_bits(rng.standard_normal((sum(lens), H, D)))
    val = bf16_bits(rng.standard_normal((sum(lens), H, D)))
    q = bf16_bits(rng.standard_normal((S, H, D)))
    kc = np.full((NB, H, 16, D), 0x7F, dtype=np.uint8)
    vc = np.full((NB, H, 16, D), 0x7F, dtype=np.uint8)
    bt = np.array([[4, 1], [0, 5]], dtype=np.int32)
    slots = np.array([bt[s][p // 16] * 16 + p % 16 for s, L in enumerate(lens)
                      for p in range(L)], dtype=np.int64)
    ks, vs = 4.0 / 448, 3.0 / 448
    oracle.reshape_and_cache(key, val, kc, vc, slots, oracle.KV_FP8_E4M3, ks, vs)
    # the cache bytes are exactly the element-wise quantisation
    np.testing.assert_array_equal(
        kc[slots // 16, :, slots % 16], oracle.quantize_bf16_array(key, np.float32(ks)))
    out = oracle.paged_decode(q, kc, vc, bt, np.array(lens), 0.125,
                              kv_dtype=oracle.KV_FP8_E4M3, k_scale=ks, v_scale=vs)
    lut = np.array([oracle.e4m3_decode(c) for c in range(256)])
    qf = bits_to_f64(q)
    for s, L in enumerate(lens):
        pos = np.arange(L)
        for h in range(H):
            K = lut[kc[bt[s][pos // 16], h, pos % 16]] * np.float64(np.float32(ks))
            V = lut[vc[bt[s][pos // 16], h, pos % 16]] * np.float64(np.float32(vs))
            z = 0.125 * (K @ qf[s, h])
            w = np.exp(z - z.max())
            np.testing.assert_allclose(out[s, h], (w / w.sum()) @ V, atol=1e-12)


# ------------------------------------------------------- copy and reshape

def test_copy_blocks_copies_whole_blocks():
    rng = np.random.default_rng(18)
    kc = rng.integers(0, 65535, size=(6, 2, 16, 64)).astype(np.uint16)
    vc = rng.integers(0, 65535, size=(6, 2, 16, 64)).astype(np.uint16)
    k0, v0 = kc.copy(), vc.copy()
    oracle.copy_blocks(kc, vc, np.array([[1, 4], [2, 0]]))
    np.testing.assert_array_equal(kc[4], k0[1])
    np.testing.assert_array_equal(vc[0], v0[2])
    for b in (1, 2, 3, 5):
        np.testing.assert_array_equal(kc[b], k0[b])
    with pytest.raises(ValueError):
        oracle.copy_blocks(kc, vc, np.array([[1, 6]]))


def test_swap_blocks_moves_blocks_between_pools():
    """(src, dst) pairs move whole K and V blocks between a 5-block device
    pool and an 8-block host pool and back; nothing else is touched."""
    rng = np.random.default_rng(20)
    gk = rng.integers(0, 65535, size=(5, 2, 16, 64)).astype(np.uint16)
    gv = rng.integers(0, 65535, size=(5, 2, 16, 64)).astype(np.uint16)
    hk = np.zeros((8, 2, 16, 64), dtype=np.uint16)
    hv = hk.copy()
    oracle.swap_blocks(hk, hv, gk, gv, np.array([[4, 7], [0, 2]]))
    np.testing.assert_array_equal(hk[7], gk[4])
    np.testing.assert_array_equal(hv[2], gv[0])
    for b in (0, 1, 3, 4, 5, 6):
        assert not hk[b].any() and not hv[b].any()
    bk, bv = np.zeros_like(gk), np.zeros_like(gv)
    oracle.swap_blocks(bk, bv, hk, hv, np.array([[7, 1], [2, 3]]))
    np.testing.assert_array_equal(bk[1], gk[4])
    np.testing.assert_array_equal(bv[3], gv[0])
    assert not bk[[0, 2, 4]].any() and not bv[[0, 2, 4]].any()
    with pytest.raises(ValueError):
        oracle.swap_blocks(hk, hv, gk, gv, np.array([[5, 0]]))  # src past the pool
    with pytest.raises(ValueError):
        oracle.swap_blocks(hk, hv, gk, gv, np.array([[0, 8]]))  # dst past the pool


def test_reshape_bf16_copies_bits_and_skips_negative_slots():
    rng = np.random.default_rng(19)
    key = rng.integers(0, 65535, size=(3, 2, 64)).astype(np.uint16)
    val = rng.integers(0, 65535, size=(3, 2, 64)).astype(np.uint16)
    kc = np.zeros((4, 2, 16, 64), dtype=np.uint16)
    vc = np.zeros((4, 2, 16, 64), dtype=np.uint16)
    oracle.reshape_and_cache(key, val, kc, vc, np.array([37, -1, 0]), oracle.KV_BF16)
    np.testing.assert_array_equal(kc[2, :, 5], key[0])
    np.testing.assert_array_equal(vc[0, :, 0], val[2])
    assert np.count_nonzero(kc) == np.count_nonzero(key[[0, 2]])
    with pytest.raises(ValueError):
        oracle.reshape_and_cache(key, val, kc, vc, np.array([64, 0, 0]), oracle.KV_BF16)


# ------------------------------------------------------------ utilisation

def read_golden_kv(path):
    out = {}
    for row in read_golden_rows(path):
        out[row[0]] = float(row[1])
    return out


def test_capacity_and_waste_worked_examples(golden_dir):
    g = read_golden_kv(os.path.join(golden_dir, "utilisation_examples.txt"))
    old = oracle.effective_capacity(g["capacity_kv_gb"], g["capacity_u_old"])
    new = oracle.effective_capacity(g["capacity_kv_gb"], g["capacity_u_new"])
    assert old == pytest.approx(g["capacity_eff_old_gb"])
    assert new == pytest.approx(g["capacity_eff_new_gb"])
    assert new / old == pytest.approx(g["capacity_gain"])
    waste = oracle.reserved_waste_bytes(int(g["reserve_tokens"]), int(g["used_tokens"]),
                                        int(g["llama7b_bytes_per_token"]))
    assert waste == int(g["unused_bytes"])
    assert int(g["reserve_tokens"]) - int(g["used_tokens"]) == int(g["unused_tokens"])
    # the per-token figure itself is the KV-size formula for Llama-7B fp16
    assert oracle.kv_bytes_per_token(32, 32, 128, 2) == int(g["llama7b_bytes_per_token"])


def test_paged_utilisation_closed_forms():
    assert oracle.paged_utilisation([16, 32, 160]) == 1.0
    assert oracle.paged_utilisation([1]) == 1 / 16
    assert oracle.paged_utilisation([17, 15]) == 32 / 48
    # the waste bound: at most 15 unused slots per sequence
    rng = np.random.default_rng(5)
    for _ in range(50):
        lens = rng.integers(1, 5000, size=rng.integers(1, 40))
        u = oracle.paged_utilisation(lens)
        held = sum(-(-int(L) // 16) * 16 for L in lens)
        assert held - sum(lens) <= 15 * len(lens)
        assert u >= 1 - 15 * len(lens) / held
    assert oracle.reserved_utilisation([400], 2048) == 400 / 2048
    assert oracle.reserved_utilisation([1024, 2048], 2048) == 0.75


# ---------------------------------------------------------------- prefill

def numpy_prefill(q, kc, vc, bt, qs, lens, scale, B=16):
    """Test-local second formulation: per sequence a [n x L] score matrix
    with an explicit causal mask, row softmax, times V."""
    T, Hq, D = q.shape
    Hkv = kc.shape[1]
    g = Hq // Hkv
    out = np.zeros((T, Hq, D))
    qf, kf, vf = bits_to_f64(q), bits_to_f64(kc), bits_to_f64(vc)
    for s in range(len(lens)):
        L, q0, n = int(lens[s]), int(qs[s]), int(qs[s + 1] - qs[s])
        pos = np.arange(L)
        qpos = L - n + np.arange(n)
        mask = pos[None, :] <= qpos[:, None]
        for hq in range(Hq):
            K = kf[bt[s][pos // B], hq // g, pos % B]
            V = vf[bt[s][pos // B], hq // g, pos % B]
            Z = scale * (qf[q0:q0 + n, hq] @ K.T)
            Z = np.where(mask, Z, -np.inf)
            W = np.exp(Z - Z.max(axis=1, keepdims=True))
            out[q0:q0 + n, hq] = (W / W.sum(axis=1, keepdims=True)) @ V
    return out


def prefill_case(rng, lens, chunks, Hq, Hkv, D, NB):
    q_total = sum(chunks)
    q = bf16_bits(rng.standard_normal((q_total, Hq, D)))
    _, kc, vc, bt, lens = make_case(rng, len(lens), Hq, Hkv, D, lens, NB)
    qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    return q, kc, vc, bt, qs, lens


@pytest.mark.parametrize("seed", [0, 1])
def test_prefill_against_numpy_formulation(seed):
    rng = np.random.default_rng(40 + seed)
    lens, chunks = [37, 5, 64, 100], [37, 5, 20, 1]   # full, full, chunked, decode-like
    q, kc, vc, bt, qs, lens = prefill_case(rng, lens, chunks, 4, 2, 16, 40)
    out = oracle.paged_prefill(q, kc, vc, bt, qs, lens, 0.25)
    ref = numpy_prefill(q, kc, vc, bt, qs, lens, 0.25)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_prefill_against_torch_sdpa_causal():
    """A whole prompt (no cached prefix) is causal attention."""
    rng = np.random.default_rng(42)
    q, kc, vc, bt, qs, lens = prefill_case(rng, [70], [70], 4, 4, 64, 8)
    out = oracle.paged_prefill(q, kc, vc, bt, qs, lens, 0.125)
    pos = np.arange(70)
    K = torch.from_numpy(bits_to_f64(kc)[bt[0][pos // 16], :, pos % 16]).permute(1, 0, 2)
    V = torch.from_numpy(bits_to_f64(vc)[bt[0][pos // 16], :, pos % 16]).permute(1, 0, 2)
    Q = torch.from_numpy(bits_to_f64(q)).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=0.125)
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def test_prefill_chunk_of_one_token_is_decode():
    rng = np.random.default_rng(43)
    lens = [33, 80, 1]
    q, kc, vc, bt, qs, lens = prefill_case(rng, lens, [1, 1, 1], 8, 2, 64, 20)
    pre = oracle.paged_prefill(q, kc, vc, bt, qs, lens, 0.125)
    dec = oracle.paged_decode(q, kc, vc, bt, lens, 0.125)
    np.testing.assert_array_equal(pre, dec)


def test_prefill_chunks_compose():
    """Prefilling a prompt in two chunks gives the rows of one whole pass."""
    rng = np.random.default_rng(44)
    q, kc, vc, bt, qs, lens = prefill_case(rng, [90], [90], 2, 2, 64, 8)
    whole = oracle.paged_prefill(q, kc, vc, bt, qs, lens, 0.125)
    first = oracle.paged_prefill(q[:50], kc, vc, bt, np.array([0, 50]), [50], 0.125)
    second = oracle.paged_prefill(q[50:], kc, vc, bt, np.array([0, 40]), [90], 0.125)
    np.testing.assert_array_equal(np.concatenate([first, second]), whole)


# ------------------------------------------------ block-table invariants
#
# The checker decides whether the host pool is correct, so each invariant it
# enforces is pinned here by a hand-built table that breaks exactly that
# invariant. The passing control is [Day28] §六's scenario written out by
# hand: request A holds 20 tokens in blocks [7, 1], request B forked from it
# shares both (refcount 2), then B's write into the partly filled block 1
# copies it to block 3 (A keeps [7, 1], B gets [7, 3]; block 1's refcount
# drops to 1).

DAY28_ROWS = [[7, 1], [7, 3]]
DAY28_LENS = [20, 21]
DAY28_NB = 10
DAY28_REFC = [0] * DAY28_NB
DAY28_REFC[7], DAY28_REFC[1], DAY28_REFC[3] = 2, 1, 1


def day28_check(rows=None, lens=None, refc=None, num_free=None, nb=DAY28_NB):
    return oracle.check_block_tables(
        DAY28_ROWS if rows is None else rows, DAY28_LENS if lens is None else lens,
        nb, 16, refcounts=DAY28_REFC if refc is None else refc,
        num_free=DAY28_NB - 3 if num_free is None else num_free)


def test_block_table_checker_accepts_the_day28_scenario():
    assert day28_check() == []
    # the [7, 1, 3] table of [Day28] §3.1 alone, 48 tokens (no waste) and 33
    # tokens (15 unused slots, the largest waste the bound allows)
    for L in (33, 48):
        assert oracle.check_block_tables([[7, 1, 3]], [L], 10, 16) == []


def test_block_table_checker_reports_one_block_too_many():
    """ceil(L/16) + 1 blocks: a whole unused block, 16 unused slots."""
    errs = oracle.check_block_tables([[7, 1, 3]], [32], 10, 16)
    assert any("3 blocks for 32 tokens, expected 2" in e for e in errs)
    assert any("16 unused slots" in e for e in errs)
    assert len(errs) == 2


def test_block_table_checker_reports_one_block_too_few():
    errs = oracle.check_block_tables([[7, 1]], [33], 10, 16)
    assert any("2 blocks for 33 tokens, expected 3" in e for e in errs)
    assert any("-1 unused slots" in e for e in errs)
    assert len(errs) == 2


def test_block_table_checker_waste_bound_is_fifteen_slots():
    """The bound itself, one slot on either side of it: 15 unused slots pass
    ([Day28] §4.2, FAQ Q2); the checker flags a waste of 16 even when only
    the waste test could catch it (the block count is checked separately)."""
    assert oracle.check_block_tables([[5]], [1], 10, 16) == []
    errs = oracle.check_block_tables([[5, 6]], [16], 10, 16)
    assert [e for e in errs if "unused slots" in e] == ["seq 0: 16 unused slots in its last block"]


@pytest.mark.parametrize("bad", [-1, DAY28_NB, DAY28_NB + 7])
def test_block_table_checker_reports_out_of_range_ids(bad):
    rows = [[7, 1], [7, bad]]
    refc = list(DAY28_REFC)
    refc[3] = 0
    errs = day28_check(rows=rows, refc=refc, num_free=DAY28_NB - 2)
    assert errs[0] == f"seq 1: block id {bad} out of range"
    # the id is counted as a use: conservation is off by that phantom block
    assert errs[1:] == [f"{DAY28_NB - 2} free + 3 used != {DAY28_NB}"]


@pytest.mark.parametrize("block,delta", [(7, +1), (7, -1), (1, +1), (3, -1), (0, +1)])
def test_block_table_checker_reports_refcount_off_by_one(block, delta):
    refc = list(DAY28_REFC)
    refc[block] += delta
    uses = DAY28_REFC[block]
    assert day28_check(refc=refc) == [
        f"block {block}: refcount {uses + delta} but {uses} table entries"]


@pytest.mark.parametrize("num_free", [DAY28_NB - 4, DAY28_NB - 2, 0, DAY28_NB])
def test_block_table_checker_reports_broken_conservation(num_free):
    """free + distinct used blocks must be N: a leaked block (one free too
    few) and a double-freed one (one too many) are both reported."""
    assert day28_check(num_free=num_free) == [f"{num_free} free + 3 used != {DAY28_NB}"]


def test_block_table_checker_counts_shared_blocks_once_for_conservation():
    """Block 7 appears in two tables but is one physical block: the sum is
    over distinct blocks, so 7 free + 3 used == 10 holds."""
    assert day28_check(num_free=7) == []
    assert day28_check(num_free=6) == ["6 free + 3 used != 10"]
