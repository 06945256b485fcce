"""moe_expert_up_ws / moe_expert_down_ws: the small-batch (decode) schedule of the expert
products.  With a few executed rows the products are split along K into fp32 partials in the
scratch and summed in a fixed order before the activation; the result equals the fused grouped
GEMM up to fp32 summation order (both round the same fp32 value to bf16 once), the split path
really runs (kernel launch count), and without scratch the fused product runs (bit-identical).
Layer-level parity of the schedule against the oracle is in test_gpu_parity.py (decode cases).
"""

import pytest
import torch

import sparse_mixture_experts_warp_b200 as M
from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, scaled
import moe_check as C

pytestmark = pytest.mark.gpu

# bf16 ulp is 2^-8 relative; two roundings of values that differ only in fp32 summation order
TOL = 2.0 ** -7

CASES = {
    # one token of a SwiGLU layer: up split 4 (gate and up), down split 8
    "swiglu_T1": scaled(WORKLOADS["mixtral"], T=1, D=1024, F=2048),
    # ReLU, two tokens over 16 experts: up split, down split
    "relu_T2": scaled(WORKLOADS["switch"], T=2, D=1024, E=16, F=1024, zipf_s=0.0),
    # F not a multiple of 256: the up product's partial block starts at column 1536
    "swiglu_T1_F1408": scaled(WORKLOADS["mixtral"], T=1, D=1024, F=1408),
    # GELU
    "gelu_T3": scaled(WORKLOADS["switch"], act="gelu", T=3, D=1024, E=16, F=512,
                      overflow="dropless", gate="renorm", k=2, zipf_s=0.0),
    # stream-K (the split tiles would take more than one wave of SMs): the Mixtral width at one
    # and two tokens (gate + up: 224 and 448 tiles, two k-ranges each), and a single ReLU
    # product of 112 tiles split five ways
    "swiglu_T1_full": scaled(WORKLOADS["mixtral"], T=1),
    "swiglu_T2_full": scaled(WORKLOADS["mixtral"], T=2),
    "relu_T1_wide": scaled(WORKLOADS["switch"], act="relu", T=1, D=4096, E=8, F=14336,
                           overflow="dropless", gate="renorm", k=2, zipf_s=0.0),
}


def _x_perm(w, inp, v):
    """The grouped token rows, by moe_permute (a layer forward that gathers its rows inside the
    up projection leaves the workspace's x_perm unwritten)."""
    d = M.desc_of(w)
    xp = torch.empty_like(v["x_perm"])
    M.moe_permute(d, v["expert_ids"], inp.x, xp, v["counts"], v["offsets"], v["row_src"],
                  v["inv"], v["scratch"])
    return xp


def _rel(a, b):
    den = b.abs().max().item()
    return (a - b).abs().max().item() / den if den > 0 else (a - b).abs().max().item()


@pytest.mark.parametrize("name", list(CASES))
def test_ws_products_match_fused_products(name):
    w = CASES[name]
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    d = M.desc_of(w)
    n = int(v["offsets"][w.E].item())              # executed rows
    assert n > 0
    scratch = v["scratch"]
    h0 = torch.zeros_like(v["h"])
    h1 = torch.zeros_like(v["h"])
    xp = _x_perm(w, inp, v)
    M.moe_expert_up(d, w.E, w.F, xp, v["offsets"], inp.W_gate, inp.W_up, h0)
    k0 = M.kernel_launches()
    M.moe_expert_up_ws(d, w.E, w.F, xp, v["offsets"], inp.W_gate, inp.W_up, h1, scratch)
    up_launches = M.kernel_launches() - k0
    y0 = torch.zeros_like(v["y"])
    y1 = torch.zeros_like(v["y"])
    M.moe_expert_down(d, w.E, w.F, h0, v["offsets"], inp.W_down, y0)
    k0 = M.kernel_launches()
    M.moe_expert_down_ws(d, w.E, w.F, h0, v["offsets"], inp.W_down, y1, scratch)
    down_launches = M.kernel_launches() - k0
    torch.cuda.synchronize()
    assert M.get_device_error() == 0
    # one split launch (SwiGLU: the gate and up products together, W_up's n-tiles after
    # W_gate's) plus the summing pass
    assert up_launches == 2
    assert down_launches == 2
    assert _rel(h1[:n].float(), h0[:n].float()) <= TOL
    assert _rel(y1[:n].float(), y0[:n].float()) <= TOL


def test_ws_without_scratch_runs_the_fused_products():
    w = CASES["swiglu_T1"]
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    d = M.desc_of(w)
    h0, h1 = torch.zeros_like(v["h"]), torch.zeros_like(v["h"])
    xp = _x_perm(w, inp, v)
    M.moe_expert_up(d, w.E, w.F, xp, v["offsets"], inp.W_gate, inp.W_up, h0)
    k0 = M.kernel_launches()
    M.moe_expert_up_ws(d, w.E, w.F, xp, v["offsets"], inp.W_gate, inp.W_up, h1, None)
    assert M.kernel_launches() - k0 == 1
    y0, y1 = torch.zeros_like(v["y"]), torch.zeros_like(v["y"])
    M.moe_expert_down(d, w.E, w.F, h0, v["offsets"], inp.W_down, y0)
    M.moe_expert_down_ws(d, w.E, w.F, h0, v["offsets"], inp.W_down, y1, None)
    torch.cuda.synchronize()
    assert torch.equal(h0, h1) and torch.equal(y0, y1)


def test_ws_with_many_rows_runs_the_fused_products():
    # 700 tokens x top-2: far more rows than the schedule's limits
    w = scaled(WORKLOADS["mixtral"], T=700, D=512, F=1024)
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    d = M.desc_of(w)
    h0, h1 = torch.zeros_like(v["h"]), torch.zeros_like(v["h"])
    xp = _x_perm(w, inp, v)
    M.moe_expert_up(d, w.E, w.F, xp, v["offsets"], inp.W_gate, inp.W_up, h0)
    M.moe_expert_up_ws(d, w.E, w.F, xp, v["offsets"], inp.W_gate, inp.W_up, h1,
                       v["scratch"])
    torch.cuda.synchronize()
    assert torch.equal(h0, h1)


@pytest.mark.parametrize("name", ["switch_full", "switch_small_k2", "swiglu_T1", "relu_T2"])
def test_layer_combine_sums_the_down_split(name):
    """Under a capacity limit the down projection may split K on the device (fp32 partials);
    moe_layer_forward then lets the combine sum each kept row's partials (split order, one bf16
    rounding), write it to y and weight it, instead of a separate summing launch (the decode
    cases keep the summing kernel of their host-side split).  Either way y and the layer output
    equal, bit for bit, those of the step entry points (moe_expert_down_ws sums with its own
    kernel, moe_combine reads y)."""
    w = {"switch_full": WORKLOADS["switch"],
         "switch_small_k2": scaled(WORKLOADS["switch"], T=3000, D=256, E=16, F=512, k=2),
         **CASES}[name]
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    d = M.desc_of(w)
    n = int(v["offsets"][w.E].item())
    assert n > 0
    y1 = torch.zeros_like(v["y"])
    M.moe_expert_down_ws(d, w.E, w.F, v["h"], v["offsets"], inp.W_down, y1, v["scratch"])
    out1 = torch.empty_like(out)
    M.moe_combine(d, y1, v["inv"], v["gates"], None, out1)
    torch.cuda.synchronize()
    assert M.get_device_error() == 0
    assert torch.equal(y1[:n], v["y"][:n])
    assert torch.equal(out1, out)
