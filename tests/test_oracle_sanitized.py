"""The oracle under AddressSanitizer and UndefinedBehaviorSanitizer (CPU):
every entry point over small and ragged shapes and every option combination,
with output buffers of exactly the sizes the header states."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_oracle_is_clean_under_address_and_undefined_behaviour_sanitizers(tmp_path):
    exe = tmp_path / "drive"
    cc = subprocess.run(["gcc", "-O1", "-g", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                         "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
                         "-I", os.path.join(ROOT, "oracle"), os.path.join(ROOT, "oracle", "qfp4_oracle.c"),
                         os.path.join(ROOT, "tests", "oracle_sanitize_drive.c"), "-lm", "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300,
                         env=dict(os.environ, ASAN_OPTIONS="detect_leaks=1", UBSAN_OPTIONS="print_stacktrace=1"))
    assert run.returncode == 0, run.stderr[-4000:]
    assert int(run.stdout.strip()) > 200          # the valid combinations ran to completion
