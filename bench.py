#!/usr/bin/env python3
"""Benchmark of the paged decode-attention step on B200.

One step = the whole hot path over one decode batch: write each sequence's
new token into its cache slot (pa_reshape_and_cache; pa_copy_blocks when a
step needs a copy-on-write), then decode attention through the block tables
(pa_decode). Default workload: 64 sequences, 32/32 heads, head_dim 128,
bf16 KV, context lengths U[512, 2048] (the Llama-7B-shaped layer).

Prints ONE JSON line (rank 0). `value` is the achieved HBM GB/s of the step
(algorithmic bytes: K/V of every context token, q, out, table entries and
the new-token write, over the device time), summed over ranks; `e2e` is the
same metric with the step's inputs copied from pinned host memory and the
output copied back, every step; `roofline` is the decode kernel alone.

  python bench.py [--gpus N --steps K --warmup W --workload NAME --impl ours|reference]
                  [--fuse] [--graph] [--partition-size P] [--op step|loop|swap|prefill]
                  [--also W[:P],... | --also none]

--fuse writes the new tokens inside the decode launch (pa_decode_append);
--graph captures one step as a CUDA graph and times its replays; --op
selects the continuous-batching loop, block swapping or chunked prefill,
each with its own line. --impl reference times the CPU oracle instead.
--also measures more decode workloads in the same run (same steps and
warm-up) and summarises each under `also`; with the default workload the
long-context one on the automatic partitions and the fp8 one ride along.

With torchrun (N > 1) every rank decodes its own batch (its own sequences,
its own pool; no collective on the data path): weak scaling.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "paged decode attention: achieved HBM GB/s (% of B200 peak), decode tokens/s"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2**20
DECODE_SOURCES = ["paged_kv_cache_429_b200/csrc/decode.cuh",
                  "paged_kv_cache_429_b200/csrc/decode_tc.cuh",
                  "paged_kv_cache_429_b200/csrc/kv_quant.cuh",
                  "paged_kv_cache_429_b200/csrc/ptx.cuh"]


# ----------------------------------------------------------------- helpers

def describe(w: synth.Workload) -> str:
    if w.prefix_len:
        lens = f"shared {w.prefix_len}-token prefix + lognormal(median {w.suffix_median:g}) suffix"
    else:
        lens = f"L~U[{w.len_lo},{w.len_hi}]"
    kv = "fp8_e4m3" if w.kv_fp8 else "bf16"
    return (f"{w.name}: {w.num_seqs} seqs, {w.num_q_heads}/{w.num_kv_heads} heads, "
            f"d{w.head_dim}, {kv} KV, block 16, {lens}")


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            peaks = json.load(f)
        return float(peaks["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s pool measurement)"


def _code_only(text: str) -> str:
    """Source text without comments and blank space, so that the hash
    changes with the compiled code only."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.strip() for line in text.splitlines() if line.strip())


def decode_source_hash() -> str:
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


PREFILL_SOURCES = ["paged_kv_cache_429_b200/csrc/prefill.cuh",
                   "paged_kv_cache_429_b200/csrc/ptx.cuh"]


def prefill_source_hash() -> str:
    h = hashlib.sha256()
    for rel in PREFILL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_prefill_traffic():
    """DRAM bytes per prefill launch from the committed ncu summary, if it
    was taken on the current prefill kernel source."""
    try:
        text = open(os.path.join(ROOT, "profiles", "paged_prefill_16x2048.md")).read()
    except OSError:
        return None
    m_hash = re.search(r"prefill_source_sha256_16:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not (m_hash and m_tr) or m_hash.group(1) != prefill_source_hash():
        return None
    return int(m_tr.group(1))


def profiled_traffic(workload: str, partition_size: int = None):
    """DRAM bytes per decode launch from the committed ncu summary of this
    workload (the entry for this partition size when the summary has one),
    if it was taken on the current decode kernel source."""
    path = os.path.join(ROOT, "profiles", f"paged_decode_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"decode_source_sha256_16:\s*([0-9a-f]+)", text)
    m_tr = None
    if partition_size is not None:
        m_tr = re.search(r"dram_bytes_per_launch_ps%d:\s*([0-9]+)" % partition_size, text)
    if m_tr is None:
        m_tr = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not (m_hash and m_tr) or m_hash.group(1) != decode_source_hash():
        return None
    return int(m_tr.group(1))


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting",
               0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x10: "sync_boost",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.error = None
        try:
            import pynvml
            self.nv = pynvml
            pynvml.nvmlInit()
            self.h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report no clocks
            self.nv, self.error = None, repr(e)

    def _handle(self, idx):
        nv = self.nv
        try:
            props = torch.cuda.get_device_properties(idx)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId_v2(bus.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(idx)

    def _sample(self):
        nv = self.nv
        mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append(mhz)
        for b, name in self.REASONS.items():
            if bits & b:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception as e:
                self.error = repr(e)
                return
            time.sleep(self.period)

    def start(self):
        if self.nv:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread:
            self._stop.set()
            self._thread.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "note": self.error}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


def l2_note(step_bytes: int) -> str:
    """How the timed steps stand to the L2 cache (no flush is done)."""
    if step_bytes > L2_BYTES:
        return (f"inputs larger than L2: {step_bytes / 1e9:.2f} GB per step vs "
                f"{L2_BYTES / 2**20:.0f} MiB L2; no flush")
    return (f"inputs fit in L2 ({step_bytes / 2**20:.2f} MiB per step vs "
            f"{L2_BYTES / 2**20:.0f} MiB L2) and stay resident: a launch-bound "
            f"case, not an HBM bandwidth figure")


def quantiles_ms(xs, fracs=(0.1, 0.5, 0.9)):
    """Nearest-rank quantiles of a list of durations, rounded to ns."""
    s = sorted(xs)
    return [round(s[min(len(s) - 1, int(f * (len(s) - 1) + 0.5))], 6) for f in fracs]


def init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world, device):
    if world > 1:
        import torch.distributed as dist
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def reduce_timing(elapsed_ms: float, nbytes: float, world: int, device):
    """(max elapsed ms over ranks, total bytes over ranks)."""
    if world == 1:
        return elapsed_ms, nbytes
    import torch.distributed as dist
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    b = torch.tensor([nbytes], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return float(t.item()), float(b.item())


# ------------------------------------------------------------- our GPU arm

def run_ours(args, world, rank, local):
    from paged_kv_cache_429_b200.batch import DecodeBatch

    device = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload]
    if args.partition_size is not None:
        import dataclasses
        w = dataclasses.replace(w, partition_size=args.partition_size)
    batch = DecodeBatch.build(w, args.seed + rank, device)
    # the earlier tokens' source rows were only needed to fill the cache
    batch.k_old = batch.v_old = None
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream(device)
    ps = w.partition_size
    ws = batch.workspace(ps if ps != 0 else 0)

    step_writes = sum((op.row1 - op.row0) for op in batch.step_ops if op.kind == "write")
    eb = 1 if w.kv_fp8 else 2
    reshape_bytes = step_writes * w.num_kv_heads * w.head_dim * (2 * 2 + 2 * eb) + 8 * step_writes
    decode_bytes = batch.algorithmic_bytes()
    unique_kv = batch.unique_kv_bytes() if w.prefix_len else 0
    step_bytes = decode_bytes + reshape_bytes
    n_copy_launches = sum(1 for op in batch.step_ops if op.kind == "copy")
    n_write_launches = sum(1 for op in batch.step_ops if op.kind == "write")

    fuse = args.fuse

    def one_step(ev=None):
        if fuse:
            # copy-on-write copies, then one decode launch that also writes
            # the new tokens (events bracket both: the decode launch and any
            # copies in front of it)
            if ev is not None:
                ev[0].record(stream)
            batch.step_fused(partition_size=ps, workspace=ws)
        else:
            batch.run_ops(batch.step_ops)
            if ev is not None:
                ev[0].record(stream)
            batch.decode(partition_size=ps, workspace=ws)
        if ev is not None:
            ev[1].record(stream)

    # which decode path runs (split launches a second, reduce kernel)
    split = ps > 0 or (ps < 0 and ws is not None and _auto_split(batch, ws))
    launches_per_step = (0 if fuse else n_write_launches) + n_copy_launches + (2 if split else 1)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize(device)
    run_step = one_step
    if args.graph:
        # the whole step captured once (on torch's capture stream) and
        # replayed on this stream: no host work per step
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            one_step()
        torch.cuda.synchronize(device)
        run_step = graph.replay
        for _ in range(args.warmup):
            run_step()
        torch.cuda.synchronize(device)

    # ---- device-resident timing: K whole steps, nothing else on the stream
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier(world, device)
    torch.cuda.synchronize(device)
    clocks.start()
    t0.record(stream)
    for i in range(K):
        run_step()
    t1.record(stream)
    torch.cuda.synchronize(device)
    clocks.stop()
    barrier(world, device)
    elapsed = t0.elapsed_time(t1)
    max_ms, total_bytes = reduce_timing(elapsed, step_bytes * K, world, device)

    # ---- the decode launch alone (roofline): events around each decode of
    # a second run of steps
    KD = min(K, 500)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(KD)]
    clocks_dec = ClockSampler(local)
    clocks_dec.start()
    for i in range(KD):
        one_step(evs[i])
    torch.cuda.synchronize(device)
    clocks_dec.stop()
    dec_ms = [a.elapsed_time(b) for a, b in evs]
    value = total_bytes / (max_ms * 1e-3) / 1e9
    ms_per_step = max_ms / K
    dec_avg_ms = sum(dec_ms) / len(dec_ms)

    # ---- end to end: pinned host inputs in, output back, every step
    e2e = run_e2e(batch, args, ps, ws, stream, device, world, step_bytes)

    if rank != 0:
        return None
    peak, peak_src = measured_peak()
    # the fused launch also reads and writes the step's new tokens
    kernel_bytes = decode_bytes + (reshape_bytes if fuse else 0)
    achieved = kernel_bytes / (dec_avg_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3" if w.kv_fp8 else "bf16", "data": "synthetic",
        "config": {
            "workload": describe(w), "global_batch": w.num_seqs * world,
            "seq_len": f"U[{w.len_lo},{w.len_hi}]" if not w.prefix_len else "prefix+suffix",
            "parallelism": f"dp{world} (independent sequence shards, no collective)",
            "decode_path": "split-context" if split else "single-pass",
            "new_token_write": "fused into the decode launch (pa_decode_append)" if fuse
                               else "separate pa_reshape_and_cache launch",
            "partition_size": ps,
            "step_launch": "one CUDA graph replay" if args.graph else "eager calls",
            "l2": l2_note(decode_bytes),
            "seed": args.seed,
        },
        "tokens_per_s": round(w.num_seqs * world / (ms_per_step * 1e-3), 1),
        **({"unique_kv_bytes_per_step": unique_kv,
            "unique_kv_gbs": round(unique_kv * world / (ms_per_step * 1e-3) / 1e9, 2)}
           if w.prefix_len else {}),
        "pct_of_peak": round(100 * value / world / peak, 2),
        "pct_of_8tbs_datasheet": round(100 * value / world / 8000.0, 2),
        "e2e": e2e,
        "gpu_launches": launches_per_step * K,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": profiled_traffic(w.name, ps),
                     "kernel": "paged_decode_kernel" + (" (new-token write fused)" if fuse else "")
                               + (" + reduce" if split else ""),
                     "algorithmic_bytes_per_launch": kernel_bytes,
                     "avg_launch_ms": round(dec_avg_ms, 6),
                     "launch_ms_p10_p50_p90": quantiles_ms(dec_ms),
                     "launches_timed": len(dec_ms), "peak_source": peak_src,
                     "clocks": clocks_dec.summary()},
        "clocks": clocks.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(batch, args.cpu_seconds)
    return line


def also_specs(args):
    """The extra decode workloads of a step run: (name, partition size or
    None for the workload's own). By default the long-context workload on
    the automatic partitions and the fp8 one ride along with the default
    workload, so one run measures every decode configuration's kernel."""
    spec = args.also
    if spec is None:
        spec = ("long:-1,gqa_fp8" if args.workload == "llama7b" and not args.fuse
                and not args.graph and args.partition_size is None else "none")
    if spec.strip().lower() == "none":
        return []
    out = []
    for item in spec.split(","):
        item = item.strip()
        if not item:
            continue
        name, _, ps = item.partition(":")
        if name not in synth.WORKLOADS:
            raise SystemExit(f"--also: unknown workload {name!r}")
        out.append((name, int(ps) if ps else None))
    return out


def also_summary(line):
    """The part of an extra workload's line kept under 'also'."""
    r = line["roofline"]
    return {
        "workload": line["config"]["workload"], "dtype": line["dtype"],
        "decode_path": line["config"]["decode_path"],
        "partition_size": line["config"]["partition_size"],
        "value": line["value"], "unit": line["unit"], "ms_per_step": line["ms_per_step"],
        "tokens_per_s": line["tokens_per_s"], "e2e": line["e2e"]["value"],
        "roofline": {k: r[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic",
                                       "kernel", "algorithmic_bytes_per_launch",
                                       "avg_launch_ms", "peak_source")},
        "clocks": line["clocks"],
    }


def _auto_split(batch, ws) -> bool:
    """Mirror of the library's automatic choice, for reporting only."""
    w = batch.w
    sms = torch.cuda.get_device_properties(batch.device).multi_processor_count
    units = w.num_seqs * w.num_kv_heads
    cap = min(batch.max_context_len, batch.max_blocks * 16)
    return (units < 2 * 3 * sms or cap > 16384) and cap > 512


def run_e2e(batch, args, ps, ws, stream, device, world, step_bytes):
    """The step through the public calls (pa_reshape_and_cache,
    pa_copy_blocks, pa_decode) with host buffers: every step copies its
    inputs (q, the new K/V, slots, copy pairs, block tables, context
    lengths; packed in one pinned buffer) host -> device and its output
    device -> host. Two slots of device buffers let step i+1's upload and
    step i-1's download run on their own streams while step i computes."""
    from paged_kv_cache_429_b200 import (pa_copy_blocks, pa_decode, pa_decode_append,
                                         pa_reshape_and_cache)
    b = batch
    fuse = args.fuse
    items = [("q", b.q), ("k_new", b.k_new), ("v_new", b.v_new),
             ("tables", b.block_tables), ("lens", b.context_lens)]
    for i, op in enumerate(b.step_ops):
        if op.kind == "write":
            items.append((f"slots{i}", b._dev_slots[id(op)]))
        else:
            items.append((f"pairs{i}", b._dev_pairs[id(op)]))
    offs, total = {}, 0
    for name, t in items:
        offs[name] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    host_in = torch.empty(total, dtype=torch.uint8).pin_memory()
    for name, t in items:
        nb = t.numel() * t.element_size()
        host_in[offs[name]:offs[name] + nb] = t.contiguous().view(-1).view(torch.uint8).cpu()
    NSLOT = 2
    slots = []
    for _ in range(NSLOT):
        buf = torch.empty(total, dtype=torch.uint8, device=device)
        views = {}
        for name, t in items:
            nb = t.numel() * t.element_size()
            views[name] = buf[offs[name]:offs[name] + nb].view(t.dtype).view(t.shape)
        slots.append({"buf": buf, "v": views,
                      "out": torch.empty(b.out.shape, dtype=b.out.dtype, device=device),
                      "host_out": torch.empty(b.out.shape, dtype=b.out.dtype).pin_memory(),
                      "up": torch.cuda.Event(), "done": torch.cuda.Event(),
                      "down": torch.cuda.Event()})
    up_stream = torch.cuda.Stream(device)
    down_stream = torch.cuda.Stream(device)
    h2d = total
    d2h = b.out.numel() * b.out.element_size()

    def e2e_step(i):
        sl = slots[i % NSLOT]
        v = sl["v"]
        up_stream.wait_event(sl["done"])        # the slot's last step has read its inputs
        with torch.cuda.stream(up_stream):
            sl["buf"].copy_(host_in, non_blocking=True)
        sl["up"].record(up_stream)
        stream.wait_event(sl["up"])
        stream.wait_event(sl["down"])           # the slot's last output has been read back
        for j, op in enumerate(b.step_ops):
            if op.kind == "copy":
                pa_copy_blocks(b.k_cache, b.v_cache, v[f"pairs{j}"], stream=stream)
            elif not fuse:
                pa_reshape_and_cache(v["k_new"][op.row0:op.row1], v["v_new"][op.row0:op.row1],
                                     b.k_cache, b.v_cache, v[f"slots{j}"], k_scale=b.k_scale,
                                     v_scale=b.v_scale, stream=stream)
        if fuse:
            pa_decode_append(sl["out"], v["q"], v["k_new"], v["v_new"], b.k_cache, b.v_cache,
                             v["tables"], v["lens"], b.max_context_len, b.w.sm_scale,
                             k_scale=b.k_scale, v_scale=b.v_scale, partition_size=ps,
                             workspace=ws, stream=stream)
        else:
            pa_decode(sl["out"], v["q"], b.k_cache, b.v_cache, v["tables"], v["lens"],
                      b.max_context_len, b.w.sm_scale, k_scale=b.k_scale, v_scale=b.v_scale,
                      partition_size=ps, workspace=ws, stream=stream)
        sl["done"].record(stream)
        down_stream.wait_event(sl["done"])
        with torch.cuda.stream(down_stream):
            sl["host_out"].copy_(sl["out"], non_blocking=True)
        sl["down"].record(down_stream)

    for i in range(max(NSLOT, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize(device)
    K = max(50, args.steps)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize(device)
    t0.record(stream)
    for i in range(K):
        e2e_step(i)
    for sl in slots:
        stream.wait_event(sl["down"])
    t1.record(stream)
    torch.cuda.synchronize(device)
    barrier(world, device)
    # the last step's output, read back, equals the device-resident step's
    last = slots[(K - 1) % NSLOT]
    same = bool(torch.equal(last["host_out"], b.out.cpu()))
    max_ms, total_bytes = reduce_timing(t0.elapsed_time(t1), step_bytes * K, world, device)
    return {"value": round(total_bytes / (max_ms * 1e-3) / 1e9, 2), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K,
            "ms_per_step": round(max_ms / K, 6),
            "pipeline": f"{NSLOT} slots; upload and download on their own streams",
            "output_matches_device_step": same}


# ------------------------------------------------------- CPU oracle timing

def oracle_host_inputs(w: synth.Workload, seed: int):
    """Host-only inputs of the workload's shape for the oracle: lengths from
    synth, each sequence's blocks taken in order from a seeded permutation
    of the pool, every pool slot filled with N(0,1) bf16 values."""
    lens = synth.draw_lengths(w, seed)
    nblk = -(-lens // 16)
    nb = w.pool_blocks or int(np.ceil(w.pool_factor * nblk.sum()))
    perm = synth.rng(seed, w.name, "pool").permutation(nb).astype(np.int32)
    tables = np.full((w.num_seqs, int(nblk.max())), -1, np.int32)
    k = 0
    for s in range(w.num_seqs):
        tables[s, :nblk[s]] = perm[k:k + nblk[s]]
        k += nblk[s]
    shape = (nb, w.num_kv_heads, 16, w.head_dim)
    kc = synth.randn_bf16(shape, seed, w.name, "k_old").view(torch.int16).numpy().view(np.uint16)
    vc = synth.randn_bf16(shape, seed, w.name, "v_old").view(torch.int16).numpy().view(np.uint16)
    q = synth.randn_bf16((w.num_seqs, w.num_q_heads, w.head_dim), seed, w.name,
                         "q").view(torch.int16).numpy().view(np.uint16)
    return lens, tables, kc, vc, q


def seq_bytes(w, L):
    eb = 1 if w.kv_fp8 else 2
    return (L * w.num_kv_heads * w.head_dim * eb * 2 + w.num_q_heads * w.head_dim * 6
            + (-(-L // 16)) * 4 + 4)


def time_oracle(w, inputs, budget_s: float, steps=None):
    """Oracle decode, one sequence per step (round robin), on this host's
    cores (the oracle is single-threaded). Returns (GB/s, steps, seconds)."""
    import oracle
    lens, tables, kc, vc, q = inputs
    n, nbytes, t_total = 0, 0, 0.0
    while True:
        s = n % w.num_seqs
        t = time.perf_counter()
        oracle.paged_decode(q, kc, vc, tables, lens.astype(np.int32), w.sm_scale,
                            seq_subset=[s])
        t_total += time.perf_counter() - t
        nbytes += seq_bytes(w, int(lens[s]))
        n += 1
        if (steps is not None and n >= steps) or (steps is None and t_total >= budget_s):
            break
    return nbytes / t_total / 1e9, n, t_total


def cpu_baseline(batch, budget_s):
    w = batch.w
    inputs = oracle_host_inputs(w, batch.seed)
    gbs, n, secs = time_oracle(w, inputs, budget_s)
    return {"value": round(gbs, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": (f"{n} single-sequence decode steps of the {w.name} workload "
                       f"(round robin over its {w.num_seqs} sequences), {secs:.1f} s "
                       f"of single-threaded fp64 oracle time; host has "
                       f"{os.cpu_count()} cores")}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    w = synth.WORKLOADS[args.workload]
    inputs = oracle_host_inputs(w, args.seed)
    time_oracle(w, inputs, 0, steps=max(1, args.warmup))
    gbs, n, secs = time_oracle(w, inputs, 0, steps=max(1, args.steps))
    ms_per_step = secs / n * 1e3
    sample = (f"one sequence per step (round robin over the {w.num_seqs} sequences of "
              f"the {w.name} workload), single-threaded fp64 oracle; host has "
              f"{os.cpu_count()} cores")
    return {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 6), "unit": UNIT,
        "n_gpus": world, "steps": n, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(w), "global_batch": w.num_seqs,
                   "parallelism": "single host thread"},
        "cpu_baseline": {"value": round(gbs, 6), "unit": UNIT, "cores": 1,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ------------------------------------------------------- other operations

def run_loop(args):
    """Continuous-batching decode loop (requests join and leave each step;
    preemption by swapping): decode tokens/s over the whole loop, host work
    included, and KV utilisation of the paged pool vs max-length reservation."""
    from paged_kv_cache_429_b200.serve_loop import DecodeLoop, LoopConfig
    cfg = LoopConfig(num_q_heads=32, num_kv_heads=32, head_dim=128, num_blocks=16384,
                     cpu_blocks=8192, max_num_seqs=256, max_model_len=4096,
                     prompt_median=600, prompt_sigma=0.7, output_median=300,
                     output_sigma=0.7, arrivals_per_step=4.0, watermark_blocks=64,
                     seed=args.seed)
    loop = DecodeLoop(cfg)
    loop.run(args.warmup)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    stats = loop.run(args.steps)
    torch.cuda.synchronize()
    secs = time.perf_counter() - t0
    live = [st for st in stats if st["running"]]
    tokens = sum(st["running"] for st in live)
    mean = lambda k: sum(st[k] for st in live) / max(len(live), 1)
    # the decode's algorithmic bytes per step (K and V of every context
    # token, q, out, table entries, lengths) and its time at the copy peak
    eb = 2
    dec_bytes = [st["tokens"] * cfg.num_kv_heads * cfg.head_dim * eb * 2
                 + st["running"] * cfg.num_q_heads * cfg.head_dim * 6
                 + st["blocks_held"] * 4 + 4 * st["running"] for st in live]
    peak, peak_src = measured_peak()
    bound_ms = 1e3 * (sum(dec_bytes) / max(len(stats), 1)) / (peak * 1e9)
    return {
        "op": "loop", "metric": "continuous-batching decode loop: decode tokens/s "
        "(one attention layer, host scheduling included)",
        "value": round(tokens / secs, 1), "unit": "tokens/s", "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 4),
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "32/32 heads, d128, bf16, pool 16384 blocks, "
                   "max_num_seqs 256, max_model_len 4096, prompts lognormal(600), "
                   "outputs lognormal(300), Poisson arrivals 4/step", "seed": args.seed},
        "mean_running": round(mean("running"), 1),
        "kv_utilisation_paged": round(mean("paged_util"), 4),
        "kv_utilisation_reserved_max_len": round(mean("reserved_util"), 4),
        "min_kv_utilisation_paged": round(min(st["paged_util"] for st in live), 4),
        "preemptions": loop.preemptions, "finished": loop.finished,
        "decode_gb_per_step": round(sum(dec_bytes) / max(len(stats), 1) / 1e9, 4),
        "decode_at_peak_ms_per_step": round(bound_ms, 4),
        "step_over_decode_at_peak": round((1e3 * secs / args.steps) / bound_ms, 3) if bound_ms else None,
        "peak_gbs": peak, "peak_source": peak_src,
    }


def run_swap(args):
    """Swap-out of whole sequences to pinned host memory and back in."""
    from paged_kv_cache_429_b200 import BlockPool, pa_swap_blocks
    from paged_kv_cache_429_b200.batch import DecodeBatch
    w = synth.WORKLOADS["llama7b"]
    b = DecodeBatch.build(w, args.seed)
    b.k_old = b.v_old = None
    seqs = list(range(16))
    nblk = sum(b.pool.seq_num_blocks(s) for s in seqs)
    cpu = BlockPool(nblk)
    hk = torch.empty((nblk,) + tuple(b.k_cache.shape[1:]), dtype=b.k_cache.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_pairs = np.concatenate([b.pool.swap_out(cpu, s) for s in seqs])
    in_pairs = np.concatenate([b.pool.swap_in(cpu, s) for s in seqs])
    po, pi = torch.from_numpy(out_pairs).cuda(), torch.from_numpy(in_pairs).cuda()
    block_bytes = b.k_cache[0].numel() * b.k_cache.element_size()
    moved = 2 * block_bytes * len(out_pairs)
    times = {"out": [], "in": []}
    for it in range(args.warmup + args.steps):
        for d, (dk, dv, sk, sv, pr) in (("out", (hk, hv, b.k_cache, b.v_cache, po)),
                                         ("in", (b.k_cache, b.v_cache, hk, hv, pi))):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            pa_swap_blocks(dk, dv, sk, sv, pr)
            e1.record()
            torch.cuda.synchronize()
            if it >= args.warmup:
                times[d].append(e0.elapsed_time(e1))
    gbs = {d: moved / (statistics.median(t) * 1e-3) / 1e9 for d, t in times.items()}
    return {
        "op": "swap", "metric": "pa_swap_blocks GB/s (device <-> pinned host), one launch",
        "value": round(min(gbs.values()), 2), "unit": "GB/s",
        "swap_out_gbs": round(gbs["out"], 2), "swap_in_gbs": round(gbs["in"], 2),
        "bytes_per_direction": moved, "blocks": len(out_pairs), "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "data": "synthetic",
        "config": {"workload": "16 sequences of the llama7b workload (32 KV heads, d128, bf16)"},
    }


def run_prefill(args):
    """Chunked prefill attention: 16 whole 2048-token prompts, 32 query /
    8 KV heads, d128, bf16 KV (the prompts' K/V already in the cache)."""
    from paged_kv_cache_429_b200 import pa_prefill
    from paged_kv_cache_429_b200.batch import DecodeBatch
    S, Hq, Hkv, D, L = 16, 32, 8, 128, 2048
    w = synth.Workload("prefill", S, Hq, Hkv, D, False, pool_factor=1.2)
    b = DecodeBatch.build(w, args.seed, lens=np.full(S, L))
    b.run_ops(b.step_ops)
    b.k_old = b.v_old = None
    q = synth.randn_bf16((S * L, Hq, D), args.seed, w.name, "q_prefill", "cuda")
    qs = torch.arange(0, S * L + 1, L, dtype=torch.int32, device="cuda")
    out = torch.empty((S * L, Hq, D), dtype=torch.float32, device="cuda")
    flops = S * Hq * 4 * D * (L * (L + 1) // 2)
    def once():
        pa_prefill(out, q, b.k_cache, b.v_cache, b.block_tables, qs, b.context_lens, L, L,
                   w.sm_scale)
    for _ in range(args.warmup):
        once()
    # K launches back to back, events only around the loop; the inputs
    # (2.3 GB of Q, K/V and output) exceed L2, so no flush is done
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device())
    torch.cuda.synchronize()
    clocks.start()
    t0.record()
    for _ in range(K):
        once()
    t1.record()
    torch.cuda.synchronize()
    clocks.stop()
    ms = t0.elapsed_time(t1) / K
    tflops = flops / (ms * 1e-3) / 1e12
    # a kernel timed alone: the burst figure is the peak; the sustained one
    # (a seconds-long loop under the power cap, as this loop is) is reported
    # beside it
    peak, peak_source = 1590.0, "fallback (1.59 PFLOP/s pool measurement)"
    peak_sus, peak_sus_source = 1400.0, "fallback (about 1.4 PFLOP/s sustained)"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
        peak = float(peaks["bf16_tflops"])
        peak_source = "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
        peak_sus = float(peaks["bf16_tflops_sustained"])
        peak_sus_source = "measured (MEASURED_PEAKS.json bf16_tflops_sustained)"
    except (OSError, KeyError, ValueError):
        pass
    return {
        "op": "prefill", "metric": "chunked prefill attention TFLOP/s (causal, QK and PV)",
        "value": round(tflops, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{S} whole {L}-token prompts, {Hq}/{Hkv} heads, d{D}, bf16 KV",
                   "l2": "inputs larger than L2 (Q 268 MB, K/V 134 MB, output 537 MB); no flush"},
        "gpu_launches": K,
        "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                     "peak_source": peak_source,
                     "peak_sustained": peak_sus, "frac_of_sustained": round(tflops / peak_sus, 4),
                     "peak_sustained_source": peak_sus_source,
                     "traffic": profiled_prefill_traffic(),
                     "kernel": "paged_prefill_kernel (tcgen05, tensor-memory accumulators)"},
        "clocks": clocks.summary(),
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--op", choices=["step", "loop", "swap", "prefill"], default="step",
                    help="step: the decode step (default); loop: continuous batching; "
                         "swap: block swapping to host memory")
    ap.add_argument("--workload", default="llama7b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--partition-size", type=int, default=None)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="capture one step in a CUDA graph and time its replays")
    ap.add_argument("--also", default=None,
                    help="more decode workloads measured in the same run, each WORKLOAD or "
                         "WORKLOAD:PARTITION_SIZE, comma-separated, summarised under 'also' "
                         "(default with the default workload: long:-1,gqa_fp8; 'none' for none)")
    ap.add_argument("--fuse", action="store_true",
                    help="write the new tokens inside the decode launch (pa_decode_append) "
                         "instead of a separate pa_reshape_and_cache launch")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        # the CPU oracle arm: rank 0 alone runs it, other ranks exit at once
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if args.op != "step":
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        line = {"loop": run_loop, "swap": run_swap, "prefill": run_prefill}[args.op](args)
        print(json.dumps(line), flush=True)
        return
    world, rank, local = init_dist()
    if args.gpus != world and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    try:
        line = run_ours(args, world, rank, local)
        also = []
        for wname, ps in also_specs(args):
            import copy
            import gc
            gc.collect()
            torch.cuda.empty_cache()
            sub_args = copy.copy(args)
            sub_args.workload, sub_args.partition_size = wname, ps
            sub_args.no_cpu_baseline, sub_args.fuse, sub_args.graph = True, False, False
            sub = run_ours(sub_args, world, rank, local)
            if sub is not None:
                also.append(also_summary(sub))
        if line is not None:
            if also:
                line["also"] = also
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
