"""Model-based randomized checks of the host block pool, on CPU.

A host "memory" (one 16-slot row per physical block, in the GPU pool and in
the host swap pool) is driven only by what the pool returns: the slots of
appended tokens, the copy-on-write pairs ([OSPage] §PagedAttention 写时复制;
[Day28] §4.2, §六 item 4) and the swap pairs ([Day28] §七, FAQ Q3). After
every operation each live sequence's tokens, read back through its block
table, must equal what was appended to it — so a write into a block another
sequence still shares, a copy that comes too late, a swap pair that misses a
block, or a cached prefix block ([Ch7] §7.1 前缀共享) holding different
tokens all fail. The structural invariants (refcounts, conservation, the
at-most-15-unused-slots waste bound of [Day28] §4.2) are checked by the
oracle's checker alongside.
"""
import numpy as np
import pytest

import oracle
from paged_kv_cache_429_b200 import BlockPool, PagedAttentionError

B = 16
OUT_OF_BLOCKS = 5


class Memory:
    def __init__(self, num_blocks):
        self.rows = np.full((num_blocks, B), -1, dtype=np.int64)

    def copy(self, src, dst):
        self.rows[dst] = self.rows[src]

    def write(self, slots, values):
        for s, v in zip(slots, values):
            if s >= 0:
                self.rows[s // B, s % B] = v


def table_row(pool, sid):
    n = pool.seq_num_blocks(sid)
    tables, ctx = pool.block_tables([sid], max(n, 1))
    return list(tables[0, :n]), int(ctx[0])


def read_back(pool, mem, sid):
    row, L = table_row(pool, sid)
    return [int(mem.rows[row[t // B], t % B]) for t in range(L)]


def check_pool(pool, ids):
    if not ids:
        return
    maxb = max(pool.seq_num_blocks(i) for i in ids) or 1
    tables, ctx = pool.block_tables(ids, maxb)
    rows = [list(tables[k, :pool.seq_num_blocks(i)]) for k, i in enumerate(ids)]
    refc = [pool.refcount(b) for b in range(pool.num_blocks)]
    assert oracle.check_block_tables(rows, ctx, pool.num_blocks, B, refcounts=refc,
                                     num_free=pool.num_free) == []


@pytest.mark.parametrize("seed", range(8))
def test_contents_follow_appends_forks_decodes_swaps_and_frees(seed):
    rng = np.random.default_rng(1000 + seed)
    gpu, cpu = BlockPool(72, shuffle_seed=seed), BlockPool(48, shuffle_seed=seed + 7)
    gmem, cmem = Memory(72), Memory(48)
    expect, where = {}, {}          # seq -> token values; seq -> "gpu" | "cpu"
    next_id, next_val = 0, 1

    def new_values(n):
        nonlocal next_val
        v = list(range(next_val, next_val + n))
        next_val += n
        return v

    for step in range(400):
        on_gpu = [s for s in expect if where[s] == "gpu"]
        on_cpu = [s for s in expect if where[s] == "cpu"]
        op = rng.integers(0, 12)
        try:
            if op == 0 or not expect:
                gpu.add_seq(next_id)
                expect[next_id], where[next_id] = [], "gpu"
                next_id += 1
            elif op == 1 and on_gpu:
                parent = on_gpu[rng.integers(len(on_gpu))]
                gpu.fork(parent, next_id)
                expect[next_id], where[next_id] = list(expect[parent]), "gpu"
                next_id += 1
            elif op in (2, 3, 4) and on_gpu:
                sid = on_gpu[rng.integers(len(on_gpu))]
                n = int(rng.integers(1, 40))
                slots, cow = gpu.append(sid, n)
                if cow:
                    gmem.copy(*cow)        # the copy comes before the writes
                vals = new_values(n)
                gmem.write(slots, vals)
                expect[sid] += vals
            elif op in (5, 6) and on_gpu:
                k = int(rng.integers(1, len(on_gpu) + 1))
                batch = [on_gpu[i] for i in rng.choice(len(on_gpu), size=k, replace=False)]
                slots, pairs = gpu.append_decode(batch)
                for src, dst in pairs:
                    gmem.copy(src, dst)
                vals = new_values(len(batch))
                gmem.write(slots, vals)
                for sid, v in zip(batch, vals):
                    expect[sid].append(v)
            elif op == 7 and expect:
                sid = list(expect)[rng.integers(len(expect))]
                (gpu if where[sid] == "gpu" else cpu).free_seq(sid)
                del expect[sid], where[sid]
            elif op in (8, 9) and on_gpu:
                sid = on_gpu[rng.integers(len(on_gpu))]
                for g, c in gpu.swap_out(cpu, sid):
                    cmem.rows[c] = gmem.rows[g]
                where[sid] = "cpu"
            elif op in (10, 11) and on_cpu:
                sid = on_cpu[rng.integers(len(on_cpu))]
                for c, g in gpu.swap_in(cpu, sid):
                    gmem.rows[g] = cmem.rows[c]
                where[sid] = "gpu"
        except PagedAttentionError as e:
            assert e.status == OUT_OF_BLOCKS, (step, op, e)
        for sid, vals in expect.items():
            pool, mem = (gpu, gmem) if where[sid] == "gpu" else (cpu, cmem)
            assert read_back(pool, mem, sid) == vals, (step, op, sid)
        check_pool(gpu, [s for s in expect if where[s] == "gpu"])
        check_pool(cpu, [s for s in expect if where[s] == "cpu"])


@pytest.mark.parametrize("seed", range(6))
def test_prefix_cached_blocks_hold_the_tokens_they_are_keyed_by(seed):
    """Prompts drawn from a few shared prefixes, incremental decode tokens,
    forks and frees with prefix caching on: every token read back through a
    table equals its token id, including those served from cached blocks
    (their slots are -1 and nothing is written)."""
    rng = np.random.default_rng(2000 + seed)
    pool = BlockPool(64, shuffle_seed=seed)
    pool.enable_prefix_caching(True)
    mem = Memory(64)
    prefixes = [list(rng.integers(1, 50, size=int(rng.integers(20, 70)))) for _ in range(3)]
    expect, next_id, hits = {}, 0, 0
    for step in range(300):
        op = rng.integers(0, 8)
        try:
            if op < 2 or not expect:
                sid = next_id
                next_id += 1
                pool.add_seq(sid)
                expect[sid] = []
                base = prefixes[rng.integers(len(prefixes))]
                toks = list(base[:int(rng.integers(1, len(base) + 1))])
                toks += list(rng.integers(1, 50, size=int(rng.integers(0, 20))))
                slots, cow, ncached = pool.append_tokens(sid, toks)
                hits += ncached
                if cow:
                    mem.copy(*cow)
                mem.write(slots, toks)
                expect[sid] += [int(t) for t in toks]
            elif op < 5:
                sid = list(expect)[rng.integers(len(expect))]
                toks = list(rng.integers(1, 50, size=int(rng.integers(1, 6))))
                slots, cow, ncached = pool.append_tokens(sid, toks)
                if cow:
                    mem.copy(*cow)
                mem.write(slots, toks)
                expect[sid] += [int(t) for t in toks]
            elif op == 5:
                parent = list(expect)[rng.integers(len(expect))]
                pool.fork(parent, next_id)
                expect[next_id] = list(expect[parent])
                next_id += 1
            else:
                sid = list(expect)[rng.integers(len(expect))]
                pool.free_seq(sid)
                del expect[sid]
        except PagedAttentionError as e:
            assert e.status == OUT_OF_BLOCKS, (step, op, e)
            # a failed append leaves the sequence as it was
        for sid, vals in expect.items():
            assert read_back(pool, mem, sid) == vals, (step, op, sid)
        assert pool.num_cached >= 0
    assert hits > 0  # the draws do hit the cache
