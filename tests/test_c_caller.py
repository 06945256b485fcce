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


CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile_gpu_caller(tmp_path):
    lib = M.library_path()
    libdir = os.path.dirname(lib)
    exe = tmp_path / "moe_c_gpu"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-O1",
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                    os.path.join(ROOT, "tests", "c", "moe_c_gpu.c"),
                    "-L", libdir, "-l:libmoe.so", "-Wl,-rpath," + libdir,
                    "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                    "-Wl,-rpath," + os.path.join(CUDA, "lib64"),
                    "-o", str(exe)], check=True, capture_output=True, text=True)
    return exe


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_gpu_c_program_compiles(tmp_path):
    """The GPU caller builds from plain C99 against include/moe.h and the CUDA runtime."""
    assert os.path.exists(_compile_gpu_caller(tmp_path))


@pytest.mark.gpu
@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_gpu_c_program_runs_the_layer(tmp_path):
    """A plain C program allocates device memory with cudaMalloc, runs moe_layer_forward on a
    seeded Mixtral-shaped layer (T = 300 tokens, D = 512, 8 experts of width 1024, top-2) and
    writes the output; every element is compared with the oracle here (bf16 tolerance 2e-2,
    max relative error over the tensor), and the balance statistics too."""
    import numpy as np
    import torch

    import moe_check as C
    from oracle import moe_oracle as O
    from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, scaled

    exe = _compile_gpu_caller(tmp_path)
    w = scaled(WORKLOADS["mixtral"], T=300, D=512, F=1024)
    inp = C.inputs_for(w, device="cpu")
    for name, t in [("x", inp.x), ("wg", inp.Wg), ("wgate", inp.W_gate), ("wup", inp.W_up),
                    ("wdown", inp.W_down)]:
        t.contiguous().view(torch.int16).numpy().tofile(str(tmp_path / f"{name}.bin"))
    r = subprocess.run([str(exe), str(tmp_path), str(w.T), str(w.D), str(w.E), str(w.F),
                        str(w.k)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    raw = np.fromfile(str(tmp_path / "out.bin"), dtype=np.int16).reshape(w.T, w.D)
    got = torch.from_numpy(raw).view(torch.bfloat16).double().numpy()
    ref = O.layer_forward(C.wdict(w), C.np64(inp.x), C.np64(inp.Wg), None, C.np64(inp.W_gate),
                          C.np64(inp.W_up), C.np64(inp.W_down))
    err = C.max_rel(got, ref["out"])
    assert err <= C.TOL_OUT["bf16"], f"C caller output max rel err {err:.3e}"
    st = M.MoeStats.from_buffer_copy((tmp_path / "stats.bin").read_bytes())
    np.testing.assert_allclose(st.aux, ref["stats"]["aux"], rtol=1e-4)
    assert st.n_routes == w.T * w.k and st.n_dropped == 0


NVCC = os.path.join(CUDA, "bin", "nvcc")


@pytest.mark.skipif(not os.path.exists(NVCC), reason="nvcc not installed")
def test_streamk_schedule_closed_forms(tmp_path):
    """The stream-K schedule of the decode k-split products (common.cuh), compiled for the
    host: the owner of every k-block and the partial-slot bound per tile agree with a
    brute-force table over several thousand (tiles, nkb, slots, grid)."""
    exe = tmp_path / "streamk_schedule"
    subprocess.run([NVCC, "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "sparse_mixture_experts_warp_b200", "csrc"),
                    os.path.join(ROOT, "tests", "c", "streamk_schedule.cu"), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok:"), r.stdout
