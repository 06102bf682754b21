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
