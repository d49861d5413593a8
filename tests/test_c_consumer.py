"""The C ABI from a plain C99 translation unit: tests/c/sekv_c_consumer.c includes
include/sekv.h, links the in-tree libsekv.so and checks descriptor sizes, the
block-size formula, status strings and pre-launch argument errors (host-only
calls, no GPU)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "hierarchical_kv_cache_span_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_compiles_as_c99_and_host_entry_points_work(tmp_path):
    if not os.path.exists(os.path.join(PKG, "libsekv.so")):
        pytest.fail("libsekv.so is not built")
    exe = str(tmp_path / "sekv_c_consumer")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "sekv_c_consumer.c"), "-L", PKG, "-lsekv", f"-Wl,-rpath,{PKG}",
           "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
