"""The boundary from C: tests/c_abi/host_checks.c, a C99 program that
includes include/attn.h and links libattn.so, is compiled with -std=c99
-pedantic -Werror and run.  Its cases return before any launch, so this
runs without a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_client_compiles_links_and_runs(tmp_path):
    from exact_tiled_attention_39_b200 import build
    lib = build.build()
    libdir = os.path.dirname(lib)
    exe = tmp_path / "host_checks"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi", "host_checks.c"),
           "-o", str(exe), "-L", libdir, "-lattn", f"-Wl,-rpath,{libdir}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr
    assert "ok" in res.stdout
