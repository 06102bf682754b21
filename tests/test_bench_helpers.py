"""CPU checks of bench.py's bookkeeping helpers (no GPU)."""
import bench


def test_code_only_ignores_comments_and_spacing():
    a = "int f(int x) {  // add one\n    return x + 1; /* done */\n}\n"
    b = "int f(int x) {\n  return x + 1;\n}"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(b.replace("+ 1", "+ 2"))


def test_kernel_source_hash_is_stable_and_scoped():
    files = bench.KERNEL_SOURCES["gemm_nvfp4_f32"]
    assert bench.csrc_hash(files) == bench.csrc_hash(files)
    assert bench.csrc_hash(files) != bench.csrc_hash()          # a subset hashes differently from the whole tree
    assert bench.ncu_traffic("no-such-kernel") is None



def test_issue_roofline_arithmetic(monkeypatch):
    w = 19169808.0
    monkeypatch.setattr(bench, "ncu_warp_insts", lambda key: w if key == "k" else None)
    n = 4096 * 4096
    r = bench.issue_roofline("k", 0.0327, n, 148, 1965.0)
    assert r["bound"] == "alu" and r["unit"] == "G warp-inst/s"
    assert abs(r["peak"] - 148 * 4 * 1.965) < 1e-9                 # G warp instructions per second
    assert abs(r["achieved"] - w / 32.7e-6 / 1e9) < 1e-6
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    assert abs(r["thread_inst_per_element"] - 32.0 * w / n) < 1e-9
    assert abs(r["issue_bound_ms"] - w / (r["peak"] * 1e9) * 1e3) < 1e-12
    assert bench.issue_roofline("other", 0.03, n, 148, 1965.0) is None


def test_clock_summary_reads_median_clock_and_active_reasons():
    s = bench.ClockSampler(0)
    s.out = ("0, 1965, 1965, 600.5, 0x0, Not Active, Not Active, Not Active, Not Active\n"
             "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n"
             "0, 1900, 1965, [N/A], 0x0, Not Active, Not Active, Not Active, Not Active\n"
             "garbage line\n")
    r = s.summary()
    assert r["samples"] == 3 and r["sm_mhz"] == 1900.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"] and r["power_w_max"] == 990.0
    s.out = "0, 1200, 1965, 700, 0x8, Active, Not Active, Active, Not Active\n"
    assert s.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    s.out = ""
    assert s.summary()["reasons"] == ["no samples"]


def test_measured_peaks_fall_back_to_the_recipe_figures(monkeypatch, tmp_path):
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks() == (6650.0, 1590.0, 1400.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6534.8, "bf16_tflops": 1633.5,
                                                              "bf16_tflops_sustained": 1390.6}))
    assert bench.measured_peaks() == (6534.8, 1633.5, 1390.6, "measured")


def test_ncu_figures_are_read_only_for_the_current_sources(monkeypatch, tmp_path):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.txt").write_text(
        "# kernel-key bytes hash source\n"
        "gemm_nvfp4_f32 111 oldhash ncu\n"
        "gemm_nvfp4_f32 222 newhash ncu\n"
        "quant1d_mxfp4_rot_sr 333 oldhash ncu\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "csrc_hash", lambda files=None: "newhash")
    assert bench.ncu_traffic("gemm_nvfp4_f32") == 222.0
    assert bench.ncu_traffic("quant1d_mxfp4_rot_sr") is None          # taken on other sources: stale
    assert bench.ncu_warp_insts("gemm_nvfp4_f32") is None               # no issue file


def test_row_partitioned_oracle_step_equals_the_single_threaded_one():
    import numpy as np
    import oracle
    import synth
    x = synth.cfg2_X()[:40].copy()
    par = bench._oracle_step_parallel(oracle, x, 4)
    single = [oracle.quantize(x, oracle.MXFP4, oracle.RNE, rotate=True),
              oracle.quantize(x, oracle.MXFP4, oracle.SR, rotate=True, seed=7)]
    for a, b in zip(single, par):
        for k in ("codes", "scales"):
            assert np.array_equal(a[k], b[k])


def test_default_arguments_keep_the_default_run_short(monkeypatch):
    monkeypatch.setattr("sys.argv", ["bench.py"])
    a = bench.parse()
    assert (a.gpus, a.steps, a.warmup, a.impl) == (1, 200, 20, "libqfp4")
    assert a.warmup >= 3
