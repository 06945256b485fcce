"""Parity of moe_layer_backward (selection fixed) with the oracle's layer_backward.

The oracle is called with the GPU forward's fp32 router logits, so both sides hold the same
selection; it evaluates every product in fp64 from the same bf16 inputs.  The CUDA path rounds
dY, the recomputed pre-activations, dH, [da | db] and the per-row dX to bf16 once each (2^-9
relative), so gradients are compared by max |gpu - oracle| / max |oracle| over each tensor
<= 3e-2.  Cases: SwiGLU with softmax + renormalised gates; Switch-style top-1 with raw gates,
ReLU experts and a capacity limit (dropped assignments carry no gradient); sigmoid +
selection bias + GELU with k = 3; an expert that receives no rows (its weight gradients are
exactly zero); the full Mixtral layer width at T = 64; expert choice; and layers with one or two
shared experts (moe_layer_backward_ex, whose shared weights get gradients too).
"""

import numpy as np
import pytest
import torch

import sparse_mixture_experts_warp_b200 as M
from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, scaled
from oracle import moe_oracle as O
import moe_check as C

pytestmark = pytest.mark.gpu

W = WORKLOADS
TOL = 3e-2
# fp32 layers: every product accumulates in fp32 from fp32 operands (no bf16 rounding); the
# gradients meet the forward's fp32 bound
TOL_F32 = 1e-5

CASES = {
    "swiglu_softmax_renorm": scaled(W["mixtral"], T=300, D=256, E=8, k=2, F=256),
    "relu_raw_capacity": scaled(W["switch"], T=400, D=256, E=16, F=256, capacity_factor=1.0,
                                zipf_s=0.0),
    "gelu_sigmoid_bias_k3": scaled(W["v3"], T=200, D=256, E=8, k=3, F=192, n_shared=0,
                                   F_shared=0, act="gelu"),
    "empty_expert": scaled(W["mixtral"], T=5, D=128, E=16, k=2, F=128),
    "mixtral_width_T64": scaled(W["mixtral"], T=64),
    # DeepSeek-V3 routing (256 experts, top-8, sigmoid + selection bias) without the shared
    # expert, at D = 256, F = 128 so the fp64 oracle stays small: 256 groups along K in the
    # weight gradients, E = 256 in the router backward and dW_g
    "v3_routing_E256": scaled(W["v3"], T=128, D=256, F=128, n_shared=0, F_shared=0),
    # expert choice: every expert keeps its top-c tokens; a picked pair's merge weight is its
    # softmax probability (tokens picked by several experts and by none)
    "expert_choice": scaled(W["ec"], T=500, D=256, E=16, F=256, c=62),
    # shared experts (weight 1 on every token): DeepSeek-style sigmoid + bias top-4 with one
    # shared expert, and softmax top-2 with two of them
    "v3_shared": scaled(W["v3"], T=200, D=256, E=16, k=4, F=128, F_shared=256),
    "two_shared": scaled(W["mixtral"], T=150, D=128, E=8, F=128, n_shared=2, F_shared=192),
    # fp32 layers (CUDA-core path): the tiny MoE the pages train (D=32, E=4, F=48, top-2), and
    # fp32 variants of expert choice, ReLU with a capacity limit, GELU, and shared experts
    "tiny_f32": W["tiny"],
    "f32_expert_choice": scaled(W["ec"], dtype="f32", T=120, D=32, E=6, F=24, c=30, clusters=4,
                                w_std=0.2, wg_std=0.2),
    "f32_relu_drop": scaled(W["switch"], dtype="f32", T=300, D=32, E=8, F=48, zipf_s=1.1,
                            w_std=0.15, wg_std=0.15),
    "f32_gelu": scaled(W["tiny"], act="gelu", T=40),
    "f32_sigmoid_shared": scaled(W["v3"], dtype="f32", T=90, D=64, E=16, F=32, k=3, n_shared=2,
                                 F_shared=40, w_std=0.1, wg_std=0.1),
}


def _rel(got, ref):
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / den) if den > 0 else float(np.abs(got).max())


def run_backward(w, inp, dout, aux_grad, train=False, with_out=False):
    """Forward (moe_layer_forward, or moe_layer_forward_train that saves the expert
    pre-activations) then moe_layer_backward."""
    d = M.desc_of(w)
    ws = M.empty_workspace(d, "cuda")
    out = torch.empty_like(inp.x)
    bws = M.empty_backward_workspace(d, "cuda")
    if train:
        M.moe_layer_forward_train(d, inp.x, inp.Wg, inp.bias, inp.W_gate, inp.W_up, inp.W_down,
                                  out, ws, bws)
    else:
        M.moe_layer_forward(d, inp.x, inp.Wg, inp.bias, inp.W_gate, inp.W_up, inp.W_down,
                            inp.Ws_gate, inp.Ws_up, inp.Ws_down, out, ws)
    E, D, F = w.E, w.D, w.F
    f32 = dict(dtype=torch.float32, device="cuda")
    assert not (train and w.dtype == "f32")
    dx = torch.empty_like(inp.x)
    dWg = torch.empty(E, D, **f32)
    dWgate = torch.empty(E, F, D, **f32) if w.act == "swiglu" else None
    dWup = torch.empty(E, F, D, **f32)
    dWdown = torch.empty(E, D, F, **f32)
    grads = dict(dx=dx, dWg=dWg, dW_gate=dWgate, dW_up=dWup, dW_down=dWdown)
    if w.n_shared:
        S, Fs = w.n_shared, w.F_shared
        sh = (inp.Ws_gate, inp.Ws_up, inp.Ws_down, torch.empty(S, Fs, D, **f32),
              torch.empty(S, Fs, D, **f32), torch.empty(S, D, Fs, **f32))
        grads.update(dWs_gate=sh[3], dWs_up=sh[4], dWs_down=sh[5])
        M.moe_layer_backward_ex(d, inp.x, inp.Wg, inp.W_gate, inp.W_up, inp.W_down, sh, dout,
                                aux_grad, ws, dx, dWg, dWgate, dWup, dWdown, bws)
    else:
        M.moe_layer_backward(d, inp.x, inp.Wg, inp.W_gate, inp.W_up, inp.W_down, dout, aux_grad,
                             ws, dx, dWg, dWgate, dWup, dWdown, bws,
                             flags=M.BWD_PREACT_SAVED if train else 0)
    torch.cuda.synchronize()
    assert M.get_device_error() == 0
    if with_out:
        grads["out"] = out
    return M.layer_views(d, ws), grads


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(name):
    w = CASES[name]
    inp = C.inputs_for(w)
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    dout = torch.randn(w.T, w.D, generator=g, device="cuda").to(inp.x.dtype)
    aux_grad = 0.5
    v, got = run_backward(w, inp, dout, aux_grad)
    ref = O.layer_backward(C.wdict(w), C.np64(inp.x), C.np64(inp.Wg), C.np64(inp.bias),
                           C.np64(inp.W_gate), C.np64(inp.W_up), C.np64(inp.W_down),
                           C.np64(dout), aux_grad, logits=v["logits"].double().cpu().numpy(),
                           Ws_gate=C.np64(inp.Ws_gate), Ws_up=C.np64(inp.Ws_up),
                           Ws_down=C.np64(inp.Ws_down))
    for key in ("dx", "dWg", "dW_gate", "dW_up", "dW_down", "dWs_gate", "dWs_up", "dWs_down"):
        if ref.get(key) is None:
            continue
        err = _rel(C.np64(got[key]), ref[key])
        tol = TOL_F32 if w.dtype == "f32" else TOL
        assert err <= tol, f"{name}: {key} max rel err {err:.3e}"
    # experts without rows get exactly zero weight gradients
    counts = v["counts"].cpu().numpy()
    for e in np.nonzero(counts == 0)[0]:
        assert torch.all(got["dW_down"][e] == 0) and torch.all(got["dW_up"][e] == 0)
    if name == "empty_expert":
        assert (counts == 0).any()


def test_backward_is_deterministic():
    w = CASES["swiglu_softmax_renorm"]
    inp = C.inputs_for(w)
    dout = torch.ones(w.T, w.D, device="cuda", dtype=torch.bfloat16)
    _, a = run_backward(w, inp, dout, 1.0)
    a = {k: v.clone() for k, v in a.items() if v is not None}
    _, b = run_backward(w, inp, dout, 1.0)
    for k in a:
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("name", ["swiglu_softmax_renorm", "gelu_sigmoid_bias_k3"])
def test_saved_preactivations_give_identical_results(name):
    # moe_layer_forward_train stores the up projection's accumulators; the backward then skips
    # its recompute -- the same GEMM on the same operands, so every result is bit-identical
    w = CASES[name]
    inp = C.inputs_for(w)
    g = torch.Generator(device="cuda")
    g.manual_seed(12)
    dout = torch.randn(w.T, w.D, generator=g, device="cuda").to(torch.bfloat16)
    _, a = run_backward(w, inp, dout, 0.3, train=False, with_out=True)
    a = {k: v.clone() for k, v in a.items() if v is not None}
    _, b = run_backward(w, inp, dout, 0.3, train=True, with_out=True)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_backward_with_transposed_weight_copies_in_subprocess():
    """MOE_BWD_WEIGHT_TRANSPOSE=1 makes the dgrad products use K-major transposed copies of the
    weights instead of reading them MN-major; run this file's parity cases under it."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, MOE_BWD_WEIGHT_TRANSPOSE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__,
                        "-k", "matches_oracle and not mixtral_width"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


def test_backward_with_128_row_weight_gradient_tiles_in_subprocess():
    """MOE_WGRAD_TILE=128 runs the weight-gradient products on 128-row tiles with two TMEM
    accumulators instead of the default 256-row tiles; run this file's parity cases under it
    (the E = 256 case takes 64-element k-blocks there, 32-element ones by default)."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, MOE_WGRAD_TILE="128")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__,
                        "-k", "matches_oracle and not mixtral_width"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
