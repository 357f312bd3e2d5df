"""The CPU oracle under AddressSanitizer and UndefinedBehaviorSanitizer.

tests/sanitize_oracle.c calls every oracle entry point (decode step, chunk,
bypass, import/dequant, the fp32 recurrence, the BDR reading study, hash and
precision map) on small seeded inputs with ragged tile counts; it is compiled
together with oracle/lrs_oracle.c with -fsanitize=address,undefined and run.
Any out-of-bounds access, use after free, leak or undefined integer operation
aborts the run with the sanitizer's report. No GPU."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ORACLE = os.path.join(os.path.dirname(HERE), "oracle")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is needed")
def test_oracle_is_clean_under_asan_and_ubsan(tmp_path):
    exe = str(tmp_path / "sanitize_oracle")
    cmd = ["gcc", "-std=c11", "-O1", "-g", "-ffp-contract=off", "-fno-omit-frame-pointer",
           "-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-I", ORACLE,
           os.path.join(HERE, "sanitize_oracle.c"), os.path.join(ORACLE, "lrs_oracle.c"),
           "-o", exe, "-lm", "-lpthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0",
               UBSAN_OPTIONS="print_stacktrace=1")
    r = subprocess.run([exe], capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, (r.stdout + r.stderr)[-4000:]
    assert "0 failures" in r.stdout
