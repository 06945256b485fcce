"""Failure detection without a GPU fault: every wait of the grouped GEMM is bounded.

The test hook moe_debug_inject(1) makes CTA 0's TMA producer arm a ring stage without loading
it -- a barrier that nothing will complete.  The MMA issuer's bounded wait must run out, the
kernel must record MOE_ERR_TIMEOUT in the device error word and finish (the other CTAs run
normally), and the context must stay usable: the next call, without the hook, is correct.
"""

import numpy as np
import pytest
import torch

import sparse_mixture_experts_warp_b200 as M
from sparse_mixture_experts_warp_b200.workloads import Workload
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def _small():
    G, D, F = 3, 256, 256
    w = Workload("wait", T=1, D=D, E=G, F=F, k=1)
    d = M.desc_of(w)
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    counts = [100, 300, 60]
    a = torch.randn(sum(counts), D, generator=g, device="cuda").to(torch.bfloat16)
    Wg = (torch.randn(G, F, D, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    Wu = (torch.randn(G, F, D, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32,
                           device="cuda")
    h = torch.zeros(sum(counts), F, dtype=torch.bfloat16, device="cuda")
    return d, G, F, a, Wg, Wu, offsets, h


def test_withheld_stage_times_out_and_context_stays_usable():
    d, G, F, a, Wg, Wu, offsets, h = _small()
    assert M.get_device_error() == 0
    M.debug_inject(1)
    try:
        M.moe_expert_up(d, G, F, a, offsets, Wg, Wu, h)
        status, code = M.device_error_status()        # synchronises: ~2 s bounded wait
    finally:
        M.debug_inject(0)
    assert status == 5, (status, hex(code))           # MOE_ERR_TIMEOUT
    assert 0x100 <= code < 0x200
    assert M.get_device_error() == 0                   # the word was cleared
    # the context is still usable and the next call is correct
    h.zero_()
    M.moe_expert_up(d, G, F, a, offsets, Wg, Wu, h)
    torch.cuda.synchronize()
    assert M.get_device_error() == 0
    off = offsets.cpu().numpy()
    for e in range(G):
        xr = a[off[e]:off[e + 1]].double().cpu().numpy()
        ref = O.silu(xr @ Wg[e].double().cpu().numpy().T) * (xr @ Wu[e].double().cpu().numpy().T)
        got = h[off[e]:off[e + 1]].double().cpu().numpy()
        assert np.abs(got - ref).max() <= 1e-2 * np.abs(ref).max() + 1e-6


def test_inject_rejects_unknown_fault_kinds():
    with pytest.raises(M.MoeError):
        M.debug_inject(7)
