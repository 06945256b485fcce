"""moe_permute_noalloc, the dispatch permutation for callers that cannot allocate device memory.

Such callers (a plugin handed only its input and output buffers by an engine whose allocator
owns the device memory) cannot provide the scratch buffer moe_permute takes; the no-alloc
entry point keeps that scratch in a fixed device array inside the library instead.  This test
calls it through the C ABI twice in a row, on two different routings, and checks each result
against moe_permute's: the permutation is integer work, so they must agree bit for bit (the
tolerance of the other permute checks).  The second call reuses the shared array the first one
left behind.  It also checks the size limit is refused before anything runs.

The file name sorts last so that a run stopping at its first failure has run every other test.
"""

import ctypes

import pytest
import torch

import sparse_mixture_experts_warp_b200 as M
from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, make_inputs, scaled

pytestmark = pytest.mark.gpu


def _route(w, seed):
    inp = make_inputs(w, seed=seed, device="cuda", experts=False)
    d = M.desc_of(w)
    K = w.E if w.select == "expert" else w.k
    ids = torch.empty((w.E, w.c) if w.select == "expert" else (w.T, K), dtype=torch.int32,
                      device="cuda")
    gates = torch.empty((w.T, K), dtype=torch.float32, device="cuda")
    M.moe_route(d, inp.x, inp.Wg, inp.bias, ids, gates)
    return d, inp.x, ids


def _outputs(w, d):
    A = M.rows_max(d)
    K = w.E if w.select == "expert" else w.k
    return dict(
        x_perm=torch.zeros((A, w.D), dtype=torch.bfloat16, device="cuda"),
        counts=torch.zeros(w.E, dtype=torch.int32, device="cuda"),
        offsets=torch.zeros(w.E + 1, dtype=torch.int32, device="cuda"),
        row_src=torch.full((A,), -7, dtype=torch.int32, device="cuda"),
        inv=torch.full((w.T * K,), -7, dtype=torch.int32, device="cuda"),
    )


def _compare(w, d, x, ids):
    ref = _outputs(w, d)
    M.moe_permute(d, ids, x, ref["x_perm"], ref["counts"], ref["offsets"], ref["row_src"],
                  ref["inv"])
    got = _outputs(w, d)
    M.moe_permute_noalloc(d, ids, x, got["x_perm"], got["counts"], got["offsets"],
                          got["row_src"], got["inv"])
    torch.cuda.synchronize()
    n = int(ref["offsets"][-1].item())
    assert torch.equal(got["counts"], ref["counts"])
    assert torch.equal(got["offsets"], ref["offsets"])
    assert torch.equal(got["row_src"][:n], ref["row_src"][:n])
    assert torch.equal(got["inv"], ref["inv"])
    assert torch.equal(got["x_perm"][:n], ref["x_perm"][:n])


@pytest.mark.parametrize("name,shape", [
    ("mixtral", dict(T=700, D=512, F=1024)),
    ("switch", dict(T=3000, D=256, E=16, F=512)),     # capacity drop
    ("v3", dict(T=300, D=512, E=64, F=256, F_shared=256)),
    # more than 65536 assignments: the histogram path that uses the fixed scratch array
    ("mixtral", dict(T=40000, D=128, F=128)),
    ("v3", dict(T=9000, D=128, E=64, F=128, F_shared=128)),
])
def test_noalloc_permute_matches_permute_on_two_calls(name, shape):
    w = scaled(WORKLOADS[name], **shape)
    for seed in (11, 12):                  # two calls in a row, different routings
        d, x, ids = _route(w, seed)
        _compare(w, d, x, ids)


def test_noalloc_permute_rejects_oversized_problems_before_launch():
    w = scaled(WORKLOADS["v3"], T=300_000, D=512, F=256, F_shared=256)
    d = M.desc_of(w)
    # ceil(300000*8/1024) * 256 histogram entries exceed the fixed array
    assert -(-w.T * w.k // 1024) * w.E > 65536
    st = M.lib().moe_permute_noalloc(ctypes.byref(d), 16, 16, 16, 16, 16, 16, 16, None)
    assert st == 2      # MOE_ERR_UNSUPPORTED
