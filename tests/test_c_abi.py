"""include/abattn.h is a C header: a strict C99 program compiles against it without
warnings, links libabattn.so and queries it (no GPU call)."""

import os
import shutil
import subprocess

import pytest

import block_sparse_attention_ibcs_b200 as ab

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_header_compiles_as_c99_and_links(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    ab.lib()  # the library is built
    libdir = os.path.dirname(ab.LIB_PATH)
    exe = str(tmp_path / "abi_from_c")
    cmd = [cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(HERE, "c", "abi_from_c.c"), "-L", libdir, "-labattn", f"-Wl,-rpath,{libdir}",
           "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    tok = out.stdout.split()
    r, n, rb, version = tok[0], tok[1], tok[2], tok[-1]
    assert int(r) == 0 and int(rb) == -2
    assert out.stdout.split(" ", 3)[3].rsplit(" ", 1)[0] == (
        f"{ab.ab_status_string(0)}|{ab.ab_status_string(-2)}")
    p = ab.params(1, 2, 1024, 64)
    assert int(n) == ab.ab_workspace_bytes(p)
    assert int(version) == ab.ab_version()
