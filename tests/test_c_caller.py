"""The boundary is a plain C ABI: a C program (tests/c/moe_c_caller.c) compiled with gcc against
include/moe.h and linked to libmoe.so, without Python or torch, runs the host-side entry
points (sizing, the capacity rule, argument validation).  Needs no GPU."""

import os
import shutil
import subprocess

import pytest

import sparse_mixture_experts_warp_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c_program_links_and_runs(tmp_path):
    lib = M.library_path()
    assert os.path.exists(lib)
    exe = tmp_path / "moe_c_caller"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-O1",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "moe_c_caller.c"),
                    "-L", libdir, "-l:libmoe.so", "-Wl,-rpath," + libdir,
                    "-o", str(exe)], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAILED" not in r.stdout
    assert "ok: Switch capacity 80" in r.stdout
