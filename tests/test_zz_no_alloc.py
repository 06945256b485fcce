"""moe_permute_noalloc, the dispatch permutation for callers that cannot allocate device memory.

Such callers (a plugin handed only its input and output buffers by an engine whose allocator
owns the device memory) cannot provide the scratch buffer moe_permute takes; the no-alloc
entry point keeps that scratch in a fixed device array inside the library instead.  This test
calls it through the C ABI twice in a row, on two different routings, and checks each result
against moe_permute's: the permutation is integer work, so they must agree bit for bit (the
tolerance of the other permute checks).  The second call reuses the shared array the first one
left behind.  A host-only test (no GPU needed) checks that a problem beyond the array's size is
refused before any pointer is looked at or anything is launched.

The file name sorts last so that a run stopping at its first failure has run every other test.
"""

import ctypes

import pytest
import torch

import sparse_mixture_experts_warp_b200 as M
from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, make_inputs, scaled


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


# The permute takes its one-pass path (E <= 8 and at most 16384 assignments), its one-CTA
# index path (at most 2048 assignments otherwise) or its cluster index path (at most 65536)
# without touching the scratch array; above those sizes it builds per-block histograms in it.
@pytest.mark.gpu
@pytest.mark.parametrize("name,shape", [
    ("mixtral", dict(T=700, D=512, F=1024)),            # one-pass path
    ("switch", dict(T=3000, D=256, E=16, F=512)),      # cluster index path, capacity drop
    ("v3", dict(T=300, D=512, E=64, F=256, F_shared=256)),
    # histogram paths, in the fixed scratch array
    ("mixtral", dict(T=40000, D=128, F=128)),           # 80000 assignments, E = 8
    ("v3", dict(T=9000, D=128, E=64, F=128, F_shared=128)),   # 72000 assignments
    ("switch", dict(T=70000, D=128, E=16, F=128)),     # 70000 assignments, capacity clamp
])
def test_noalloc_permute_matches_permute_on_two_calls(name, shape):
    w = scaled(WORKLOADS[name], **shape)
    for seed in (11, 12):                  # two calls in a row, different routings
        d, x, ids = _route(w, seed)
        _compare(w, d, x, ids)


def test_noalloc_permute_rejects_oversized_problems_before_launch():
    """Host-only: the size check comes before the pointer checks, so with every pointer NULL an
    oversized problem still answers MOE_ERR_UNSUPPORTED, and a size that fits answers
    MOE_ERR_INVALID_ARG; neither launches anything (no GPU is needed)."""
    w = scaled(WORKLOADS["v3"], T=300_000, D=512, F=256, F_shared=256)
    d = M.desc_of(w)
    # ceil(300000*8/1024) * 256 histogram entries exceed the fixed array
    assert -(-w.T * w.k // 1024) * w.E > 65536
    nulls = [None] * 7
    assert M.lib().moe_permute_noalloc(ctypes.byref(d), *nulls, None) == 2  # UNSUPPORTED
    small = M.desc_of(scaled(WORKLOADS["v3"], T=300, D=512, F=256, F_shared=256))
    assert M.lib().moe_permute_noalloc(ctypes.byref(small), *nulls, None) == 1  # INVALID_ARG
