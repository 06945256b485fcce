"""The tcgen05 grouped GEMM (moe_expert_up / moe_expert_down) on ragged groups, against the
oracle's expert formulas evaluated in fp64 on the same bf16 rows.

Groups include an empty one, a single row, sizes just below and above the 128-row tile, and
a multi-tile group; F = 192 leaves half of the last 128-column SwiGLU tile outside the matrix.
Rows outside the groups must stay untouched.
"""

import numpy as np
import pytest
import torch

import sparse_mixture_experts_warp_b200 as M
from sparse_mixture_experts_warp_b200.workloads import Workload
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def _case(act, D, F, counts, extra_rows=5, seed=3):
    G = len(counts)
    w = Workload("gemm", T=1, D=D, E=G, F=F, k=1, act=act)
    d = M.desc_of(w)
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    n = int(sum(counts))
    rows = n + extra_rows
    a = torch.randn(rows, D, generator=g, device="cuda").to(torch.bfloat16)
    Wg = (torch.randn(G, F, D, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    Wu = (torch.randn(G, F, D, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    Wd = (torch.randn(G, D, F, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32,
                           device="cuda")
    sentinel = torch.tensor(-12345.0, dtype=torch.bfloat16)
    h = torch.full((rows, F), sentinel.item(), dtype=torch.bfloat16, device="cuda")
    y = torch.full((rows, D), sentinel.item(), dtype=torch.bfloat16, device="cuda")
    return d, G, a, Wg if act == "swiglu" else None, Wu, Wd, offsets, h, y, n, sentinel


@pytest.mark.parametrize("act", ["swiglu", "relu"])
@pytest.mark.parametrize("D,F,counts", [
    (256, 192, [0, 1, 127, 129, 300]),
    (128, 512, [5, 0, 0, 256, 3]),
    (512, 256, [1000]),
    # token tiles of the weights-as-M schedule: N = 16 and 32 (17 rows), three token tiles
    # (513 rows: 256 + 256 + 1), 64 live features in the last feature tile (F = 320)
    (256, 320, [17, 16, 513, 0, 33]),
])
def test_grouped_gemm_ragged(act, D, F, counts):
    d, G, a, Wg, Wu, Wd, offsets, h, y, n, sentinel = _case(act, D, F, counts)
    M.moe_expert_up(d, G, F, a, offsets, Wg, Wu, h)
    M.moe_expert_down(d, G, F, h, offsets, Wd, y)
    torch.cuda.synchronize()
    assert M.get_device_error() == 0
    off = offsets.cpu().numpy()
    a64 = a.double().cpu().numpy()
    h_gpu = h.double().cpu().numpy()
    y_gpu = y.double().cpu().numpy()
    for e in range(G):
        lo, hi = off[e], off[e + 1]
        if hi == lo:
            continue
        xr = a64[lo:hi]
        wu = Wu[e].double().cpu().numpy()
        if act == "swiglu":
            wg = Wg[e].double().cpu().numpy()
            gpre, upre = xr @ wg.T, xr @ wu.T
            h_ref = O.silu(gpre) * upre
        else:
            h_ref = np.maximum(xr @ wu.T, 0.0)
        # h is rounded once to bf16: 2^-8 relative to the row scale, plus accumulation order
        scale = np.abs(h_ref).max()
        assert np.abs(h_gpu[lo:hi] - h_ref).max() <= 1e-2 * scale + 1e-6
        # down projection of the GPU's own bf16 h
        y_ref = h_gpu[lo:hi] @ Wd[e].double().cpu().numpy().T
        assert np.abs(y_gpu[lo:hi] - y_ref).max() <= 1e-2 * np.abs(y_ref).max() + 1e-6
    # rows outside every group are untouched
    assert torch.all(h[n:] == sentinel.to("cuda"))
    assert torch.all(y[n:] == sentinel.to("cuda"))


def test_grouped_gemm_repeatable():
    d, G, a, Wg, Wu, Wd, offsets, h, y, n, _ = _case("swiglu", 256, 192, [3, 200, 77])
    M.moe_expert_ffn(d, G, 192, a, offsets, Wg, Wu, Wd, h, y)
    y1 = y.clone()
    M.moe_expert_ffn(d, G, 192, a, offsets, Wg, Wu, Wd, h, y)
    torch.cuda.synchronize()
    assert torch.equal(y1[:n], y[:n])


@pytest.mark.parametrize("var,val", [("MOE_GEMM_TILE", "128"), ("MOE_GEMM_TILE", "256k32"),
                                     ("MOE_GEMM_TILE", "pair"), ("MOE_GEMM_SWAP", "0"),
                                     ("MOE_GEMM_SWAP", "1")])
def test_grouped_gemm_other_tiles_in_subprocess(var, val):
    """The other tile shapes (128-row tiles with a double TMEM buffer; 256-row tiles with
    32-element k-blocks; 256 x 256 tiles on a CTA pair) are selected per process by
    MOE_GEMM_TILE, and the weights-as-M schedule by MOE_GEMM_SWAP=1 (every grouped call, the
    one-group case included; MOE_GEMM_SWAP=0 is the default, the row tiles); run this file's
    ragged cases under each in a child process."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, **{var: val})
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__,
                        "-k", "ragged or repeatable"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
