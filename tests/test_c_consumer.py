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


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_binding_field_offsets_equal_the_header(tmp_path):
    """every field of the Python binding's descriptors sits at the offset the C header
    gives it (sizes alone would not catch two fields swapped, or a field added into
    the struct's tail padding)"""
    import ctypes

    from hierarchical_kv_cache_span_b200 import sekv as S

    structs = [("sekv_build_desc", S.sekv_build_desc), ("sekv_decode_desc", S.sekv_decode_desc),
               ("sekv_fetch_desc", S.sekv_fetch_desc)]
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "sekv.h"', "int main(void) {"]
    expect = []
    for cname, cls in structs:
        lines.append(f'    printf("{cname} %zu\\n", sizeof({cname}));')
        expect.append(f"{cname} {ctypes.sizeof(cls)}")
        for f in cls._fields_:
            name = f[0]
            lines.append(f'    printf("{cname}.{name} %zu\\n", offsetof({cname}, {name}));')
            expect.append(f"{cname}.{name} {getattr(cls, name).offset}")
    lines += ["    return 0;", "}"]
    src = tmp_path / "offsets.c"
    src.write_text("\n".join(lines) + "\n")
    exe = str(tmp_path / "offsets")
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split("\n")[:-1] == expect
