"""Host-side logic of bench.py on CPU: the a / D + b fit of the activation memory, the clock
record parsing, and the per-launch DRAM traffic that the line reports only while the kernel
sources and the launch shapes it was captured with are unchanged."""
import hashlib
import json
import os

import bench


def test_fit_inverse_d_recovers_a_and_b():
    sweep = [{"D": D, "workspace_gb": 12.0 / D + 0.5} for D in (1, 2, 4, 8, 16)]
    f = bench.fit_inverse_d(sweep)
    assert abs(f["a_gb"] - 12.0) < 1e-9 and abs(f["b_gb"] - 0.5) < 1e-9
    assert f["max_abs_residual_gb"] < 1e-9
    assert bench.fit_inverse_d(sweep[:1]) is None and bench.fit_inverse_d([]) is None


def _tree(tmp_path, src_text, api_line, entry):
    root = tmp_path / "r"
    csrc = root / "memory_efficient_exact_chunk_b200" / "csrc"
    csrc.mkdir(parents=True)
    (root / "profiles").mkdir()
    (csrc / "gemm_tc.cu").write_text(src_text)
    (csrc / "sbp_api.cu").write_text(api_line)
    (root / "profiles" / "traffic.json").write_text(json.dumps({"k@w": entry}))
    return str(root)


def test_traffic_only_for_the_captured_sources_and_shapes(tmp_path, monkeypatch):
    src = "// kernel\n"
    rel = "memory_efficient_exact_chunk_b200/csrc/gemm_tc.cu"
    api = "memory_efficient_exact_chunk_b200/csrc/sbp_api.cu"
    good = hashlib.sha256(src.encode()).hexdigest()[:16]
    entry = {"sources": [rel], "sources_sha256_16": good, "dram_bytes_per_launch": 4.9e8,
             "requires": [[api, "kVocabBlock = 16384;"]]}
    line = "constexpr int64_t kVocabBlock = 16384;\n"
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path / "a", src, line, entry))
    assert bench.traffic_from_profiles("k@w") == 4.9e8
    assert bench.traffic_from_profiles("other@w") is None
    # another vocabulary block, or an edited kernel file: the stored figure no longer applies
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path / "b", src, line.replace("16384", "8192"),
                                             entry))
    assert bench.traffic_from_profiles("k@w") is None
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path / "c", src + " ", line, entry))
    assert bench.traffic_from_profiles("k@w") is None


def test_committed_traffic_entries_are_well_formed():
    """Every entry of profiles/traffic.json names existing sources, a summary under profiles/
    that exists, and a positive per-launch figure.  (Whether the sources still match is what
    the bench checks at run time: a stale entry reports traffic null.)"""
    path = os.path.join(bench.ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return
    with open(path) as fh:
        entries = json.load(fh)
    for key, e in entries.items():
        assert "@" in key
        assert e["dram_bytes_per_launch"] > 0
        assert os.path.exists(os.path.join(bench.ROOT, e["summary"])), key
        for rel in e["sources"]:
            assert os.path.exists(os.path.join(bench.ROOT, rel)), (key, rel)


def test_parse_clocks_reasons_and_median():
    rec = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1500, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "0, [N/A], 1965, 10, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    c = bench.parse_clocks(rec)
    assert c == {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}
    hot = rec[:1] + ["0, 900, 1965, 500, 0x8, Not Active, Active, Not Active, Not Active"]
    assert bench.parse_clocks(hot)["reasons"] == ["hw_thermal_slowdown"]
    assert bench.parse_clocks(["x"]) is None and bench.parse_clocks([]) is None


def test_clock_sampler_stop_reads_and_removes_its_file(tmp_path):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as fh:
        fh.write("0, 1800, 1965, 900, 0x4, Not Active, Not Active, Not Active, Active\n")

    class Done:                       # a sampler process that has already exited
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    s.proc = Done()
    s.fh = open(str(tmp_path / "unused"), "w")
    assert s.stop() == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                        "samples": 1}
    assert not (tmp_path / "clocks.csv").exists()
