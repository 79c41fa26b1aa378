"""GPU test of the continuous-batching decode loop.

Requests join and leave at every step, the pool is small enough that some
requests are preempted by swapping to host memory and resumed. The loop
records every cache operation it issued (writes with their source rows,
swaps with their pairs); the oracle replays them on its own copies of the
GPU and host caches. Then: the last step's decode output matches the oracle
within 2e-3, every live block's bytes match exactly, and the per-step
utilisation figures equal the oracle's plain definitions.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from paged_kv_cache_429_b200 import pa_get_device_error
from paged_kv_cache_429_b200.serve_loop import DecodeLoop, LoopConfig
from parity_harness import to_u16

pytestmark = pytest.mark.gpu


def replay(loop):
    c = loop.cfg
    gk = np.full((c.num_blocks, c.num_kv_heads, 16, c.head_dim), synth.SENTINEL_BF16, np.uint16)
    gv = gk.copy()
    hk = np.zeros((c.cpu_blocks, c.num_kv_heads, 16, c.head_dim), np.uint16)
    hv = hk.copy()
    for op in loop.log:
        if op[0] == "write":
            _, k, v, slots = op
            oracle.reshape_and_cache(to_u16(k), to_u16(v), gk, gv, slots, oracle.KV_BF16)
        elif op[0] == "swap_out":
            oracle.swap_blocks(hk, hv, gk, gv, op[1])
        else:
            oracle.swap_blocks(gk, gv, hk, hv, op[1])
    return gk, gv


def test_continuous_batching_loop_matches_oracle():
    cfg = LoopConfig(num_q_heads=8, num_kv_heads=4, head_dim=64, num_blocks=160,
                     cpu_blocks=600, max_num_seqs=16, max_model_len=512,
                     prompt_median=120, prompt_sigma=0.5, output_median=140,
                     output_sigma=0.5, arrivals_per_step=1.5, watermark_blocks=2, seed=7)
    loop = DecodeLoop(cfg, record=True)
    stats = loop.run(160)
    torch.cuda.synchronize()
    assert pa_get_device_error() == 0
    assert loop.finished > 0 and loop.preemptions > 0
    assert any(s["running"] >= 8 for s in stats)

    gk, gv = replay(loop)
    last = loop.last
    ref = oracle.paged_decode(to_u16(last["q"]), gk, gv, last["tables"], last["lens"],
                              loop.sm_scale)
    err = np.max(np.abs(last["out"].double().cpu().numpy() - ref))
    assert np.all(np.isfinite(ref)) and err <= 2e-3

    # every block a running request holds has the oracle's bytes
    live = sorted({int(b) for row, L in zip(last["tables"], last["lens"])
                   for b in row[:-(-int(L) // 16)]})
    idx = torch.tensor(live, device=loop.k_cache.device)
    np.testing.assert_array_equal(to_u16(loop.k_cache.index_select(0, idx)), gk[live])
    np.testing.assert_array_equal(to_u16(loop.v_cache.index_select(0, idx)), gv[live])

    # utilisation figures: the oracle's definitions on the recorded lengths
    for s in stats:
        if s["running"]:
            assert s["paged_util"] == pytest.approx(oracle.paged_utilisation(s["lens"]), abs=1e-12)
            assert s["reserved_util"] == pytest.approx(
                oracle.reserved_utilisation(s["lens"], cfg.max_model_len), abs=1e-12)
            assert s["paged_util"] >= s["reserved_util"]
