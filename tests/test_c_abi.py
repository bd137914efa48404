"""The boundary is a C ABI: include/bca.h compiles as strict C99, and a plain C program
(tests/c_abi/plan_host.c) built with gcc against it and libbca.so creates a host-only
plan, reads its statistics and mask rows, and gets the documented error codes.  The
expected numbers are closed forms of the block-causal mask, not library output."""
import os
import shutil
import subprocess

import pytest

from block_causal_attention_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GCC = shutil.which("gcc")


@pytest.mark.skipif(GCC is None, reason="gcc not available")
def test_header_is_strict_c99():
    r = subprocess.run([GCC, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only", "-x", "c",
                        os.path.join(ROOT, "include", "bca.h")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


@pytest.mark.skipif(GCC is None, reason="gcc not available")
def test_plain_c_caller(tmp_path):
    libdir = os.path.dirname(_abi.LIB_PATH)
    exe = str(tmp_path / "plan_host")
    r = subprocess.run([GCC, "-std=c99", "-Wall", "-Wextra", "-Werror", "-O1", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c_abi", "plan_host.c"), "-L", libdir, "-lbca",
                        f"-Wl,-rpath,{libdir}", "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    nq, nk, pairs, row0, row255 = map(int, r.stdout.split())
    # 2 chunks of 2 x 8 x 8 = 128 tokens, block-causal: chunk 0 sees itself, chunk 1 both
    assert (nq, nk) == (256, 256)
    assert pairs == 128 * 128 + 128 * 256
    assert (row0, row255) == (128, 256)
