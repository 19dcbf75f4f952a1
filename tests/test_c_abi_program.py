"""include/vi.h from plain C: a C99 program compiles against the header with
every warning enabled, links libvi.so, and gets the documented answers from
the host-only calls (version, status strings, an argument rejection, an empty
call), with no GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "abi_check.c")
LIBDIR = os.path.join(ROOT, "clip_temporal_modules_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_compiles_as_c99_and_library_links(tmp_path):
    from clip_temporal_modules_b200 import build
    build.build()
    exe = tmp_path / "abi_check"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), "-o", str(exe), SRC,
                           "-L", LIBDIR, "-lvi", f"-Wl,-rpath,{LIBDIR}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "status -3 = VI_ERR_UNSUPPORTED" in out.stdout
    assert "bad F % N -> VI_ERR_INVALID_ARG" in out.stdout
    assert "empty conv -> VI_OK" in out.stdout
