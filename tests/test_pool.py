"""Host block pool: the pages' scenarios and invariants, checked on CPU.

Invariants come from the oracle's checker (oracle.check_block_tables); slot
values from the oracle's slot function (pinned by the [7, 1, 3] example).
"""
import numpy as np
import pytest

import oracle
from paged_kv_cache_429_b200 import BlockPool, PagedAttentionError

B = 16


def tables_of(pool, ids):
    maxb = max([pool.seq_num_blocks(i) for i in ids] + [1])
    tables, ctx = pool.block_tables(ids, maxb)
    rows = [list(tables[k, :pool.seq_num_blocks(i)]) for k, i in enumerate(ids)]
    return tables, ctx, rows


def assert_invariants(pool, ids):
    tables, ctx, rows = tables_of(pool, ids)
    refc = [pool.refcount(b) for b in range(pool.num_blocks)]
    errs = oracle.check_block_tables(rows, ctx, pool.num_blocks, B,
                                     refcounts=refc, num_free=pool.num_free)
    assert errs == []


def test_day28_shared_prefix_cow_scenario():
    """Day 28 §六: A and B share their first blocks (refcount 2); when B
    writes into the shared block, B allocates a new one, copies, and the
    refcount drops by one."""
    pool = BlockPool(10)
    pool.add_seq(1)  # request A
    slots_a, cow = pool.append(1, 20)  # block 0 full, block 1 holds 4 tokens
    assert cow is None
    pool.fork(1, 2)  # request B
    _, _, rows = tables_of(pool, [1, 2])
    assert rows[0] == rows[1] and len(rows[0]) == 2
    assert [pool.refcount(b) for b in rows[0]] == [2, 2]
    slots_b, cow = pool.append(2, 1)
    assert cow is not None
    src, dst = cow
    assert src == rows[0][1] and dst not in rows[0]
    assert pool.refcount(src) == 1 and pool.refcount(dst) == 1
    assert pool.refcount(rows[0][0]) == 2
    _, _, rows2 = tables_of(pool, [1, 2])
    assert rows2[0] == rows[0]
    assert rows2[1] == [rows[0][0], dst]
    assert slots_b[0] == dst * B + 4
    assert slots_b[0] == oracle.slot(rows2[1], 20, B)
    assert_invariants(pool, [1, 2])


def test_thousand_token_prefix_shared_by_two_requests():
    """Day 28 §六 question: two requests sharing a 1000-token prefix. Paged,
    the prefix takes ceil(1000/16) = 63 blocks once (62 full + 8 tokens);
    contiguous allocation would hold 2 x 1000 token slots."""
    pool = BlockPool(200)
    pool.add_seq(0)
    pool.append(0, 1000)
    pool.fork(0, 1)
    assert pool.num_free == 200 - 63
    _, _, rows = tables_of(pool, [0, 1])
    assert len(rows[0]) == 63 and rows[0] == rows[1]
    assert all(pool.refcount(b) == 2 for b in rows[0])
    # 63 * 16 slots hold both prefixes; the contiguous layout needs 2000
    assert 63 * B < 2 * 1000
    assert_invariants(pool, [0, 1])


def test_on_demand_allocation_every_16_tokens():
    """[Ch7] §7.1: a new block only when the previous 16 slots are full."""
    pool = BlockPool(8)
    pool.add_seq(7)
    free0 = pool.num_free
    for n in range(1, 50):
        pool.append(7, 1)
        assert pool.num_free == free0 - (-(-n // B))
        assert_invariants(pool, [7])


def test_slots_follow_the_block_table():
    pool = BlockPool(64, shuffle_seed=3)
    pool.add_seq(0)
    slots, _ = pool.append(0, 100)
    _, _, rows = tables_of(pool, [0])
    for pos in range(100):
        assert slots[pos] == oracle.slot(rows[0], pos, B)


def test_shuffled_pool_hands_out_a_permutation():
    a, b = BlockPool(50, shuffle_seed=5), BlockPool(50, shuffle_seed=5)
    c = BlockPool(50, shuffle_seed=6)
    for p in (a, b, c):
        p.add_seq(0)
        p.append(0, 50 * B)
    ta = tables_of(a, [0])[2][0]
    assert sorted(ta) == list(range(50))
    assert ta == tables_of(b, [0])[2][0]
    assert ta != tables_of(c, [0])[2][0]
    assert ta != list(range(50))


def test_out_of_blocks_leaves_pool_unchanged():
    pool = BlockPool(4)
    pool.add_seq(0)
    with pytest.raises(PagedAttentionError) as e:
        pool.append(0, 4 * B + 1)
    assert e.value.status == 5
    assert pool.num_free == 4 and pool.seq_len(0) == 0
    pool.append(0, 4 * B)
    assert pool.num_free == 0


def test_cow_needs_a_free_block():
    pool = BlockPool(2)
    pool.add_seq(0)
    pool.append(0, 5)
    pool.fork(0, 1)
    pool.add_seq(2)
    pool.append(2, 16)  # takes the last free block
    with pytest.raises(PagedAttentionError) as e:
        pool.append(1, 1)
    assert e.value.status == 5
    assert_invariants(pool, [0, 1, 2])


def test_errors():
    pool = BlockPool(4)
    pool.add_seq(0)
    with pytest.raises(PagedAttentionError):
        pool.add_seq(0)
    with pytest.raises(PagedAttentionError) as e:
        pool.append(9, 1)
    assert e.value.status == 6
    with pytest.raises(PagedAttentionError):
        pool.fork(9, 1)
    pool.add_seq(1)
    with pytest.raises(PagedAttentionError):
        pool.fork(0, 1)
    with pytest.raises(PagedAttentionError):
        pool.free_seq(9)
    pool.append(0, 40)
    with pytest.raises(PagedAttentionError):
        pool.block_tables([0], 2)  # needs 3 columns
    assert pool.refcount(4) == -1 and pool.refcount(-1) == -1
    with pytest.raises(PagedAttentionError):
        BlockPool(4, block_size=8)


def test_free_returns_blocks_when_last_sharer_leaves():
    """Day 28 §五: a finished request returns its blocks to the pool."""
    pool = BlockPool(20)
    pool.add_seq(0)
    pool.append(0, 40)
    pool.fork(0, 1)
    pool.append(1, 10)
    pool.free_seq(0)
    assert_invariants(pool, [1])
    pool.free_seq(1)
    assert pool.num_free == 20


def test_prefix_workload_cow_count():
    """256 sequences share a 1000-token prefix (refcount 256 on its 63
    blocks); in id order every writer but the last copies the partial
    block, so 255 copy pairs; the last finds refcount 1 and writes in place."""
    pool = BlockPool(2000)
    pool.add_seq(0)
    pool.append(0, 1000)
    for s in range(1, 256):
        pool.fork(0, s)
    _, _, rows = tables_of(pool, [0])
    assert all(pool.refcount(b) == 256 for b in rows[0])
    pairs = []
    for s in range(256):
        _, cow = pool.append(s, 3)
        if cow:
            pairs.append(cow)
    assert len(pairs) == 255
    assert all(src == rows[0][62] for src, _ in pairs)
    assert len({d for _, d in pairs}) == 255
    assert pool.refcount(rows[0][62]) == 1
    assert all(pool.refcount(b) == 256 for b in rows[0][:62])
    assert_invariants(pool, list(range(256)))


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_keep_invariants(seed):
    """Waste bound ([Day28] §4.2: at most B-1 unused slots, all in the last
    block), refcounts and conservation hold after every operation."""
    rng = np.random.default_rng(seed)
    pool = BlockPool(96, shuffle_seed=seed)
    live, next_id = [], 0
    for _ in range(300):
        op = rng.integers(0, 10)
        if op < 2 or not live:
            pool.add_seq(next_id)
            live.append(next_id)
            next_id += 1
        elif op < 4:
            parent = live[rng.integers(len(live))]
            pool.fork(parent, next_id)
            live.append(next_id)
            next_id += 1
        elif op < 5:
            victim = live.pop(rng.integers(len(live)))
            pool.free_seq(victim)
        else:
            sid = live[rng.integers(len(live))]
            before = tables_of(pool, [sid])[2][0]
            L0 = pool.seq_len(sid)
            try:
                slots, cow = pool.append(sid, int(rng.integers(1, 40)))
            except PagedAttentionError as e:
                assert e.status == 5
                assert tables_of(pool, [sid])[2][0] == before
                continue
            after = tables_of(pool, [sid])[2][0]
            for i, sl in enumerate(slots):
                assert sl == oracle.slot(after, L0 + i, B)
            if cow:
                assert before[L0 // B] == cow[0] and after[L0 // B] == cow[1]
        assert_invariants(pool, live)


def test_swap_out_and_in_keeps_both_pools_consistent():
    """Preemption by swapping ([Day28] §六 question 4, FAQ Q3): the swapped
    sequence takes private CPU copies; blocks still shared stay on the GPU."""
    gpu, cpu = BlockPool(12, shuffle_seed=1), BlockPool(8)
    gpu.add_seq(1)
    gpu.append(1, 40)              # 3 blocks
    gpu.fork(1, 2)                 # seq 2 shares all three
    gpu.append(2, 1)               # CoW of the partial last block
    before = tables_of(gpu, [1])[2][0]
    free_gpu = gpu.num_free
    pairs = gpu.swap_out(cpu, 1)
    assert [int(a) for a in pairs[:, 0]] == before
    assert cpu.seq_len(1) == 40 and gpu.seq_len(1) == -1
    assert cpu.num_free == 8 - 3
    # blocks 0,1 still shared with seq 2 stay; the old last block is freed
    assert gpu.num_free == free_gpu + 1
    assert_invariants(gpu, [2])
    assert_invariants(cpu, [1])
    assert tables_of(cpu, [1])[2][0] == [int(b) for b in pairs[:, 1]]
    back = gpu.swap_in(cpu, 1)
    assert [int(a) for a in back[:, 0]] == [int(b) for b in pairs[:, 1]]
    assert cpu.num_free == 8 and gpu.seq_len(1) == 40
    assert_invariants(gpu, [1, 2])
    assert tables_of(gpu, [1])[2][0] == [int(b) for b in back[:, 1]]


def test_swap_errors_change_nothing():
    gpu, cpu = BlockPool(10), BlockPool(2)
    gpu.add_seq(0)
    gpu.append(0, 48)              # 3 blocks, more than the CPU pool holds
    with pytest.raises(PagedAttentionError) as e:
        gpu.swap_out(cpu, 0)
    assert e.value.status == 5
    assert gpu.seq_len(0) == 48 and cpu.num_free == 2 and gpu.num_free == 7
    with pytest.raises(PagedAttentionError) as e:
        gpu.swap_out(cpu, 9)
    assert e.value.status == 6
    cpu.add_seq(0)
    with pytest.raises(PagedAttentionError) as e:
        gpu.swap_out(cpu, 0)       # id already present in the destination
    assert e.value.status == 1


# ------------------------------------------------ automatic prefix caching

def test_prefix_caching_shares_whole_blocks_of_a_common_prompt():
    """Two requests with the same 1000-token system prompt ([Ch7] §7.1
    前缀共享; [Day28] §六 question 2): the second finds the first 62 full
    blocks (992 tokens) cached and gets slot -1 for them; the block holding
    prompt tokens 992-999 differs (other suffix) and is its own."""
    rng = np.random.default_rng(0)
    prompt = rng.integers(0, 32000, 1000)
    pool = BlockPool(200, shuffle_seed=3)
    pool.enable_prefix_caching()
    pool.add_seq(0)
    s0, _, c0 = pool.append_tokens(0, np.concatenate([prompt, rng.integers(0, 32000, 50)]))
    pool.add_seq(1)
    s1, _, c1 = pool.append_tokens(1, np.concatenate([prompt, rng.integers(0, 32000, 70)]))
    assert c0 == 0 and c1 == 992
    assert np.all(s1[:992] == -1) and np.all(s1[992:] >= 0)
    rows = tables_of(pool, [0, 1])[2]
    assert rows[0][:62] == rows[1][:62] and rows[0][62] != rows[1][62]
    assert all(pool.refcount(b) == 2 for b in rows[0][:62])
    # slots of the non-cached tokens follow the table
    for i in range(992, 1070):
        assert s1[i] == oracle.slot(rows[1], i, B)
    assert_invariants(pool, [0, 1])


def test_prefix_cache_survives_its_owner_and_is_evicted_last():
    rng = np.random.default_rng(1)
    prompt = rng.integers(0, 32000, 160)          # 10 full blocks
    pool = BlockPool(16)
    pool.enable_prefix_caching()
    pool.add_seq(0)
    pool.append_tokens(0, prompt)
    pool.free_seq(0)
    assert pool.num_free == 16 and pool.num_cached == 10
    pool.add_seq(1)
    _, _, c = pool.append_tokens(1, prompt)       # all found again
    assert c == 160 and pool.num_free == 6
    pool.free_seq(1)
    # a request that needs 13 fresh blocks evicts the 7 least recently freed;
    # blocks are freed last-first, so the prompt's tail goes, its head stays
    pool.add_seq(2)
    _, _, c = pool.append_tokens(2, rng.integers(0, 32000, 13 * 16))
    assert c == 0 and pool.num_cached == 10 - 7 + 13
    pool.add_seq(3)
    with pytest.raises(PagedAttentionError) as e:   # 3 cached + 7 fresh > 3 left
        pool.append_tokens(3, prompt)
    assert e.value.status == 5 and pool.seq_len(3) == 0
    pool.free_seq(2)
    _, _, c = pool.append_tokens(3, prompt)
    assert c == 3 * 16                              # the surviving head
    assert_invariants(pool, [3])


def test_prefix_cache_matches_only_an_identical_prefix():
    rng = np.random.default_rng(2)
    a = rng.integers(0, 32000, 64)
    b = a.copy()
    b[20] += 1                                    # differs inside block 1
    pool = BlockPool(20)
    pool.enable_prefix_caching()
    pool.add_seq(0)
    pool.append_tokens(0, a)
    pool.add_seq(1)
    _, _, c = pool.append_tokens(1, b)
    assert c == 16                                # block 0 only; then a miss
    pool.add_seq(2)
    _, _, c = pool.append_tokens(2, np.concatenate([a[16:32], a[:16], a[32:]]))
    assert c == 0                                 # same tokens, other order


def test_prefix_caching_with_incremental_decode_and_fork():
    rng = np.random.default_rng(3)
    toks = rng.integers(0, 32000, 40)
    pool = BlockPool(30)
    pool.enable_prefix_caching()
    pool.add_seq(0)
    pool.append_tokens(0, toks[:10])
    for t in toks[10:]:                           # one token per decode step
        pool.append_tokens(0, [t])
    pool.fork(0, 1)                               # shares the partial block too
    _, cow, _ = pool.append_tokens(1, [5])
    assert cow is not None                        # writer copies the shared block
    pool.add_seq(2)
    _, _, c = pool.append_tokens(2, toks)
    assert c == 32                                # the two blocks filled step by step
    assert_invariants(pool, [0, 1, 2])


def test_disabling_prefix_caching_forgets_keys():
    pool = BlockPool(8)
    pool.enable_prefix_caching()
    pool.add_seq(0)
    pool.append_tokens(0, list(range(32)))
    pool.free_seq(0)
    assert pool.num_cached == 2
    pool.enable_prefix_caching(False)
    assert pool.num_cached == 0 and pool.num_free == 8
    pool.enable_prefix_caching()
    pool.add_seq(1)
    _, _, c = pool.append_tokens(1, list(range(32)))
    assert c == 0


def test_append_decode_one_token_each():
    pool = BlockPool(12, shuffle_seed=4)
    for sid, n in ((1, 16), (2, 5), (3, 31)):
        pool.add_seq(sid)
        pool.append(sid, n)
    pool.fork(2, 4)                                  # 4 shares 2's partial block
    free0 = pool.num_free
    slots, cow = pool.append_decode([1, 2, 3, 4])
    # 2 writes first and copies; 4 is then the only owner and writes in place
    assert len(cow) == 1
    assert pool.num_free == free0 - 2                # seq 1's new block + 2's copy
    rows = tables_of(pool, [1, 2, 3, 4])[2]
    for sl, sid, row in zip(slots, (1, 2, 3, 4), rows):
        assert sl == oracle.slot(row, pool.seq_len(sid) - 1, B)
    assert_invariants(pool, [1, 2, 3, 4])
    with pytest.raises(PagedAttentionError):
        pool.append_decode([1, 1])                   # listed twice
    small = BlockPool(1)
    small.add_seq(0)
    small.append(0, 16)
    with pytest.raises(PagedAttentionError) as e:
        small.append_decode([0])
    assert e.value.status == 5 and small.seq_len(0) == 16


def test_seq_lens_matches_the_per_sequence_query():
    pool = BlockPool(64)
    for sid, n in ((5, 1), (9, 16), (2, 33)):
        pool.add_seq(sid)
        pool.append(sid, n)
    pool.fork(9, 11)
    ids = np.array([2, 11, 9, 5, 404], dtype=np.int64)
    lens = pool.seq_lens(ids)
    assert lens.tolist() == [33, 16, 16, 1, -1]
    assert lens.tolist() == [pool.seq_len(int(i)) for i in ids]
    assert pool.seq_lens(np.array([], dtype=np.int64)).tolist() == []
