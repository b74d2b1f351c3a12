"""Host-side logic of bench.py on CPU: the a / D + b fit of the activation memory, and the
per-launch DRAM traffic that the line reports only while the kernel file and the vocabulary
block it was captured with are unchanged."""
import hashlib

import bench


def test_fit_inverse_d_recovers_a_and_b():
    sweep = [{"D": D, "workspace_gb": 12.0 / D + 0.5} for D in (1, 2, 4, 8, 16)]
    f = bench.fit_inverse_d(sweep)
    assert abs(f["a_gb"] - 12.0) < 1e-9 and abs(f["b_gb"] - 0.5) < 1e-9
    assert f["max_abs_residual_gb"] < 1e-9
    assert bench.fit_inverse_d(sweep[:1]) is None and bench.fit_inverse_d([]) is None


def _tree(tmp_path, src_text, api_block, stored_hash, bytes_per_launch="4.9e8"):
    root = tmp_path / "r"
    csrc = root / "memory_efficient_exact_chunk_b200" / "csrc"
    csrc.mkdir(parents=True)
    (root / "profiles").mkdir()
    (csrc / "gemm_tc.cu").write_text(src_text)
    (csrc / "sbp_api.cu").write_text(f"constexpr int64_t kVocabBlock = {api_block};\n")
    (root / "profiles" / "lmhead_ce_32k_gemm_tc.md").write_text(
        f"dram_bytes_per_launch = {bytes_per_launch}\nkernel_source_sha256_16 = {stored_hash}\n")
    return str(root)


def test_traffic_only_for_the_captured_kernel_and_block(tmp_path, monkeypatch):
    src = "// kernel\n"
    good = hashlib.sha256(src.encode() + b"kVocabBlock=16384").hexdigest()[:16]
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path / "a", src, 16384, good))
    assert bench.traffic_from_profiles("gemm_tc.cu", "lmhead_ce_32k") == 4.9e8
    # another vocabulary block, or an edited kernel file: the stored figure no longer applies
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path / "b", src, 8192, good))
    assert bench.traffic_from_profiles("gemm_tc.cu", "lmhead_ce_32k") is None
    monkeypatch.setattr(bench, "ROOT", _tree(tmp_path / "c", src + " ", 16384, good))
    assert bench.traffic_from_profiles("gemm_tc.cu", "lmhead_ce_32k") is None


def test_committed_traffic_matches_the_kernel_file():
    """The committed profile was captured on the committed kernel file: after an edit of
    gemm_tc.cu the DRAM-traffic capture in profiles/ has to be taken again (until then the
    bench line reports traffic null)."""
    assert bench.traffic_from_profiles("gemm_tc.cu", "lmhead_ce_32k") is not None


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
