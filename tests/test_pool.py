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
