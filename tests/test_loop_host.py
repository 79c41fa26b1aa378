"""The continuous-batching loop's host scheduling, on CPU.

The three GPU calls the loop makes (cache writes, swaps, the decode) are
replaced by stand-ins that only check their arguments, so admission,
on-demand growth, preemption by swapping, resumption and retirement run
exactly as they do around the GPU. Checked after every step: both pools
conserve their blocks, every running request holds prompt + generated
tokens, the last-block waste bound of "GPU 学习日报 Day 28" §4.1 holds, and
the utilisation figures are consistent; over the run, requests are
preempted and resumed and finish, and the run is deterministic.
"""
import pytest
import torch

import paged_kv_cache_429_b200.serve_loop as sl

BS = 16


@pytest.fixture
def calls(monkeypatch):
    seen = {"write": 0, "swap_out": 0, "swap_in": 0, "decode": 0}

    def write(k, v, k_cache, v_cache, slots, **kw):
        seen["write"] += 1
        assert k.shape == v.shape and k.shape[0] == slots.numel()
        assert int(slots.min()) >= 0 and int(slots.max()) < k_cache.shape[0] * BS

    def swap(dst_k, dst_v, src_k, src_v, pairs, **kw):
        # the host cache has cpu_blocks rows, the device cache num_blocks
        seen["swap_out" if dst_k.shape[0] == CFG["cpu_blocks"] else "swap_in"] += 1
        assert pairs.ndim == 2 and pairs.shape[1] == 2 and pairs.shape[0] > 0

    def decode(out, q, k_cache, v_cache, tables, lens, max_len, scale, **kw):
        seen["decode"] += 1
        assert out.shape == q.shape and tables.shape[0] == q.shape[0] == lens.shape[0]
        assert int(lens.max()) == max_len and int(lens.min()) >= 1

    monkeypatch.setattr(sl, "pa_reshape_and_cache", write)
    monkeypatch.setattr(sl, "pa_swap_blocks", swap)
    monkeypatch.setattr(sl, "pa_decode", decode)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self, *a, **k: self)
    return seen


CFG = dict(num_q_heads=4, num_kv_heads=2, head_dim=64, num_blocks=384, cpu_blocks=1024,
           max_num_seqs=48, max_model_len=512, prompt_median=120.0, prompt_sigma=0.6,
           output_median=80.0, output_sigma=0.6, arrivals_per_step=2.0,
           watermark_blocks=4)


def check_state(loop):
    c = loop.cfg
    pool, cpu = loop.pool, loop.cpu_pool
    run_ids = [r.rid for r in loop.running]
    held = sum(pool.seq_num_blocks(i) for i in run_ids)
    assert held + pool.num_free == c.num_blocks  # nothing is shared: no forks
    swapped = sum(cpu.seq_num_blocks(r.rid) for r in loop.swapped)
    assert swapped + cpu.num_free == c.cpu_blocks
    for r in loop.running:
        L = pool.seq_len(r.rid)
        assert L == r.prompt_len + r.generated
        assert 0 <= pool.seq_num_blocks(r.rid) * BS - L <= BS - 1
    assert len(loop.running) <= c.max_num_seqs


def run(seed, steps=240):
    loop = sl.DecodeLoop(sl.LoopConfig(seed=seed, **CFG), device="cpu")
    trace = []
    for _ in range(steps):
        st = loop.step()
        check_state(loop)
        if st["running"]:
            assert 0 < st["reserved_util"] <= st["paged_util"] <= 1.0
            assert st["blocks_held"] * BS - st["tokens"] <= (BS - 1) * st["running"]
        trace.append((st["running"], st["waiting"], st["swapped"], st.get("tokens", 0)))
    return loop, trace


def test_scheduling_keeps_the_pools_consistent(calls):
    loop, trace = run(0)
    assert loop.preemptions > 0 and loop.finished > 0
    assert any(t[2] > 0 for t in trace)             # some requests sat swapped out
    assert calls["swap_out"] > 0 and calls["swap_in"] > 0
    assert calls["decode"] > 0 and calls["write"] > 0


def test_the_run_is_deterministic(calls):
    assert run(3, 120)[1] == run(3, 120)[1]
