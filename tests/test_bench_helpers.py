"""Host-side helpers of bench.py: launch-time quantiles and the gating of the
ncu traffic figure on the decode source it was captured from; the CPU
oracle arm (--impl reference) and its JSON line."""
import json

import pytest

import bench


def test_quantiles_are_nearest_rank():
    xs = [float(v) for v in range(11, 0, -1)]  # order must not matter
    assert bench.quantiles_ms(xs) == [2.0, 6.0, 10.0]
    assert bench.quantiles_ms([0.25]) == [0.25, 0.25, 0.25]
    assert bench.quantiles_ms([1.0, 3.0]) == [1.0, 3.0, 3.0]


def test_l2_note_says_which_side_of_l2_the_step_is():
    assert bench.l2_note(1_354_125_840).startswith("inputs larger than L2: 1.35 GB")
    small = bench.l2_note(1_050_000)
    assert small.startswith("inputs fit in L2") and "not an HBM bandwidth figure" in small


def test_code_only_ignores_comments_and_blank_lines():
    a = "int x = 1;  // one\n\n/* block\n comment */ int y = 2;\n"
    b = "int x = 1;\n   int y = 2;   \n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only("int x = 1;") != bench._code_only("int x = 2;")


def _profile(tmp_path, name, text):
    d = tmp_path / "profiles"
    d.mkdir(exist_ok=True)
    (d / f"paged_decode_{name}.md").write_text(text)


def test_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "decode_source_hash", lambda: "0123456789abcdef")
    _profile(tmp_path, "same", "decode_source_sha256_16: 0123456789abcdef\n"
                               "dram_bytes_per_launch: 1365135360\n")
    _profile(tmp_path, "stale", "decode_source_sha256_16: fedcba9876543210\n"
                                "dram_bytes_per_launch: 1365135360\n")
    _profile(tmp_path, "nohash", "dram_bytes_per_launch: 1365135360\n")
    assert bench.profiled_traffic("same") == 1365135360
    assert bench.profiled_traffic("stale") is None
    assert bench.profiled_traffic("nohash") is None
    assert bench.profiled_traffic("missing") is None


def test_prefill_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d = tmp_path / "profiles"
    d.mkdir()
    f = d / "paged_prefill_16x2048.md"
    assert bench.profiled_prefill_traffic() is None          # no profile
    monkeypatch.setattr(bench, "prefill_source_hash", lambda: "00112233aabbccdd")
    f.write_text("prefill_source_sha256_16: 00112233aabbccdd\ndram_bytes_per_launch: 893372416\n")
    assert bench.profiled_prefill_traffic() == 893372416
    monkeypatch.setattr(bench, "prefill_source_hash", lambda: "ffffffffffffffff")
    assert bench.profiled_prefill_traffic() is None          # kernel changed since


def test_committed_profiles_match_the_current_sources():
    """The DRAM bytes the bench reports come from profiles taken on the
    current kernel sources: every decode workload's and the prefill's."""
    for w in ("llama7b", "gqa_fp8", "prefix"):
        assert bench.profiled_traffic(w) is not None, w
    assert bench.profiled_traffic("long", 512) is not None
    assert bench.profiled_traffic("long", -1) is not None
    assert bench.profiled_prefill_traffic() is not None


def test_traffic_per_partition_size(tmp_path, monkeypatch):
    """A summary with entries per partition size gives each path its own
    bytes, and the plain entry when the size has none."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "decode_source_hash", lambda: "0123456789abcdef")
    _profile(tmp_path, "split", "decode_source_sha256_16: 0123456789abcdef\n"
                                "dram_bytes_per_launch_ps512: 3669506560\n"
                                "dram_bytes_per_launch_ps-1: 3598697472\n")
    _profile(tmp_path, "both", "decode_source_sha256_16: 0123456789abcdef\n"
                               "dram_bytes_per_launch: 100\n"
                               "dram_bytes_per_launch_ps512: 200\n")
    assert bench.profiled_traffic("split", 512) == 3669506560
    assert bench.profiled_traffic("split", -1) == 3598697472
    assert bench.profiled_traffic("split", 0) is None
    assert bench.profiled_traffic("both", 512) == 200
    assert bench.profiled_traffic("both", 0) == 100
    assert bench.profiled_traffic("both") == 100


def _run_main(argv, capsys, monkeypatch, env=None):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    for k, v in (env or {}).items():
        monkeypatch.setenv(k, v)
    bench.main(argv)
    return [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]


def test_reference_arm_line(capsys, monkeypatch):
    """--impl reference times the CPU oracle and prints the contract's line."""
    lines = _run_main(["--impl", "reference", "--steps", "3", "--warmup", "3"], capsys,
                      monkeypatch)
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "GB/s"
    assert d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["higher_is_better"] is True and d["gpu_launches"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("llama7b")


def test_reference_arm_other_ranks_print_nothing(capsys, monkeypatch):
    lines = _run_main(["--impl", "reference", "--steps", "3", "--warmup", "3"], capsys,
                      monkeypatch, env={"WORLD_SIZE": "2", "RANK": "1", "LOCAL_RANK": "1"})
    assert lines == []


def test_warmup_below_three_is_refused():
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--steps", "3", "--warmup", "2"])


def test_also_specs():
    import argparse
    ns = argparse.Namespace(also=None, workload="llama7b", fuse=False, graph=False,
                            partition_size=None)
    assert bench.also_specs(ns) == [("long", -1), ("gqa_fp8", None)]
    ns.fuse = True                      # a non-default run adds nothing by itself
    assert bench.also_specs(ns) == []
    ns.also = "prefix, long:512"
    assert bench.also_specs(ns) == [("prefix", None), ("long", 512)]
    ns.also = "none"
    assert bench.also_specs(ns) == []
    ns.also = "nosuch"
    with pytest.raises(SystemExit):
        bench.also_specs(ns)
