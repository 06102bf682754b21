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
