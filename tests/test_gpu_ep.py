"""The expert-parallel layer on one GPU: G logical ranks held by one process exchange their rows
through LocalAllToAll (device copies standing in for the All-to-All), so route, permute, the
exchange plan, the block reorder kernel, the local grouped GEMMs on Eg = E / G experts, the
reverse exchange and the combine all run on the device.

Each rank's output is compared with the single-device layer on the same tokens and full expert
set (moe_layer_forward): in a dropless layer every row meets the same kernels in the same k
order, so they must agree bit for bit.  Under a capacity limit the single-device layer may
split its down projection along K on the device (when the kept rows leave SMs idle) while the
ranks, each with fewer experts, decide for themselves, so y's fp32 summation order can differ:
there the outputs must agree within bf16 rounding.  Every rank is also compared with the oracle
(routing from the GPU's fp32 logits, every token, the bf16 tolerance)."""

import numpy as np
import pytest
import torch

import moe_check as C
import sparse_mixture_experts_warp_b200 as M
from sparse_mixture_experts_warp_b200 import ep
from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, scaled

pytestmark = pytest.mark.gpu

CASES = {
    "mixtral_G2": (scaled(WORKLOADS["mixtral"], T=300, D=512, F=1024), 2),
    "mixtral_G4": (scaled(WORKLOADS["mixtral"], T=200, D=256, F=512), 4),
    "mixtral_G8_one_expert_each": (scaled(WORKLOADS["mixtral"], T=150, D=256, F=256), 8),
    # per-rank capacity limit: each rank drops by its own batch, as one device would
    "switch_drop_G2": (scaled(WORKLOADS["switch"], T=400, D=256, E=16, F=512), 2),
}


@pytest.mark.parametrize("name", list(CASES))
def test_expert_parallel_layer_matches_single_device(name):
    w, G = CASES[name]
    Eg = w.E // G
    per_rank = [C.inputs_for(w, seed=20 + r) for r in range(G)]
    full = per_rank[0]           # router and expert weights: rank 0's draw, shared by all
    ranks = []
    for r in range(G):
        sl = slice(r * Eg, (r + 1) * Eg)
        ranks.append(ep.EpRank(
            rank=r, x=per_rank[r].x, Wg=full.Wg, bias=full.bias,
            W_gate=full.W_gate[sl].contiguous() if full.W_gate is not None else None,
            W_up=full.W_up[sl].contiguous(), W_down=full.W_down[sl].contiguous(),
            out=torch.empty_like(per_rank[r].x)))
    plans, keep = ep.ep_layer_forward(w, ranks, ep.LocalAllToAll(G))
    torch.cuda.synchronize()
    assert M.get_device_error() == 0
    del keep
    sent = sum(p.send_total for p in plans)
    assert sent == sum(p.recv_total for p in plans) > 0
    for r in range(G):
        inp = per_rank[r]
        ref = C.run_layer(w, type(inp)(inp.x, full.Wg, full.bias, full.W_gate, full.W_up,
                                       full.W_down))[0]
        if w.overflow == "drop":
            diff = (ranks[r].out.float() - ref.float()).abs().max().item()
            assert diff <= 1e-2 * ref.float().abs().max().item(), \
                f"rank {r}: differs from the single-device layer by {diff}"
        else:
            assert torch.equal(ranks[r].out, ref), \
                f"rank {r}: differs from the single-device layer"
        v = ranks[r].views
        C.check_routing(w, type(inp)(inp.x, full.Wg, full.bias, full.W_gate, full.W_up,
                                     full.W_down), v)
        C.check_sampled_output(w, type(inp)(inp.x, full.Wg, full.bias, full.W_gate, full.W_up,
                                            full.W_down), ranks[r].out, v, list(range(w.T)))
