"""The library's calls capture into a CUDA graph as they are (no allocation, no host
synchronisation, every launch on the caller's stream): a captured moe_layer_forward replays to
the same bits as the eager call, and replays keep matching after the inputs change in place."""

import pytest
import torch

import sparse_mixture_experts_warp_b200 as M
from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, scaled
import moe_check as C

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,w", [
    ("mixtral_small", scaled(WORKLOADS["mixtral"], T=700, D=512, F=1024)),
    ("v3_small", scaled(WORKLOADS["v3"], T=300, D=512, E=64, F=256, F_shared=256)),
])
def test_graph_replay_matches_eager(name, w):
    inp = C.inputs_for(w)
    d = M.desc_of(w)
    ws = M.empty_workspace(d, "cuda")
    out = torch.empty_like(inp.x)

    def fwd(stream=None):
        M.moe_layer_forward(d, inp.x, inp.Wg, inp.bias, inp.W_gate, inp.W_up, inp.W_down,
                            inp.Ws_gate, inp.Ws_up, inp.Ws_down, out, ws, stream)

    fwd()
    torch.cuda.synchronize()
    eager = out.clone()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    out.zero_()
    with torch.cuda.graph(g, stream=cap):
        fwd(cap)
    g.replay()
    torch.cuda.synchronize()
    assert M.get_device_error() == 0
    assert torch.equal(out, eager)
    # new token values in the same buffer: the replay routes and computes them afresh
    inp2 = C.inputs_for(w, seed=1)
    inp.x.copy_(inp2.x)
    g.replay()
    torch.cuda.synchronize()
    replayed = out.clone()
    fwd()
    torch.cuda.synchronize()
    assert torch.equal(replayed, out)
    assert not torch.equal(replayed, eager)
