"""The C ABI from plain C: include/pa.h compiles as strict C99 (-pedantic
-Werror) and a C program linked against libpa.so makes the host-side calls
(tests/abi_c_client.c); no GPU is involved."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
PKG = os.path.join(ROOT, "paged_kv_cache_334_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not on PATH")
def test_plain_c_client_builds_links_and_runs(tmp_path):
    from paged_kv_cache_334_b200 import build
    build.build()
    exe = str(tmp_path / "abi_c_client")
    cmd = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
           "-I" + os.path.join(ROOT, "include"), os.path.join(HERE, "abi_c_client.c"),
           "-L" + PKG, "-lpa", "-Wl,-rpath," + PKG, "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "ok" in r.stdout


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not on PATH")
def test_header_compiles_as_cpp(tmp_path):
    src = tmp_path / "inc.cpp"
    src.write_text('#include "pa.h"\nint main() { return pa_version() > 0 ? 0 : 1; }\n')
    r = subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only",
                        "-I" + os.path.join(ROOT, "include"), str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
