"""Host-side helpers of bench.py: launch-time quantiles and the gating of the
ncu traffic figure on the decode source it was captured from."""
import bench


def test_quantiles_are_nearest_rank():
    xs = [float(v) for v in range(11, 0, -1)]  # order must not matter
    assert bench.quantiles_ms(xs) == [2.0, 6.0, 10.0]
    assert bench.quantiles_ms([0.25]) == [0.25, 0.25, 0.25]
    assert bench.quantiles_ms([1.0, 3.0]) == [1.0, 3.0, 3.0]


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
