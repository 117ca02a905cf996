"""The C oracle under AddressSanitizer and UndefinedBehaviorSanitizer.

tests/oracle_asan_driver.c calls every oracle entry point on small inputs in
heap arrays of exactly their size, edge cases included; built here with the
sanitizers, any out-of-bounds access, use after free, leak or undefined
arithmetic in the oracle fails the test (an off-by-one in the gather loop,
planted in a copy, is reported as a heap-buffer-overflow)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not on PATH")
def test_oracle_is_clean_under_sanitizers(tmp_path):
    exe = str(tmp_path / "oracle_asan")
    cmd = ["gcc", "-O1", "-g", "-std=c11", "-Wall", "-Werror", "-Wno-unknown-pragmas",
           "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
           "-fno-omit-frame-pointer", os.path.join(HERE, "oracle_asan_driver.c"),
           os.path.join(ROOT, "oracle", "pa_oracle.c"), "-lm", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0",
               UBSAN_OPTIONS="print_stacktrace=1")
    r = subprocess.run([exe], capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "ok" in r.stdout
