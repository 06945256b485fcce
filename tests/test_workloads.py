"""The seeded input generators (sparse_mixture_experts_warp_b200/workloads.py) follow the
recipe the tests and the bench rely on (CPU only, reduced sizes): determinism per seed, the
stated distributions, the Zipf-scaled router offset carried through a constant feature, the
token clusters of the expert-choice workload, and the separation of router keys that keeps the
selection stable under fp32 rounding."""

import math

import numpy as np
import torch

from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, make_inputs, scaled
import moe_check as C


def test_same_seed_same_inputs_and_other_seed_other_inputs():
    w = scaled(WORKLOADS["mixtral"], T=64, D=128, F=64)
    a, b = make_inputs(w, seed=0), make_inputs(w, seed=0)
    for name in ("x", "Wg", "W_gate", "W_up", "W_down"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    c = make_inputs(w, seed=1)
    assert not torch.equal(a.x, c.x) and not torch.equal(a.W_up, c.W_up)


def test_stated_distributions():
    # x ~ N(0, 1); router and expert weights ~ N(0, 0.02^2); bf16 operands
    w = scaled(WORKLOADS["mixtral"], T=512, D=512, F=256)
    inp = make_inputs(w, seed=0)
    assert inp.x.dtype == torch.bfloat16 and inp.W_up.dtype == torch.bfloat16
    assert abs(inp.x.float().std().item() - 1.0) < 0.01
    for t in (inp.Wg, inp.W_gate, inp.W_up, inp.W_down):
        assert abs(t.float().std().item() / 0.02 - 1.0) < 0.02
        assert abs(t.float().mean().item()) < 0.002
    # the selection-only bias of the sigmoid workload ~ N(0, 0.1^2), fp32
    v = scaled(WORKLOADS["v3"], T=16, D=64, E=256, F=64, F_shared=64)
    b = make_inputs(v, seed=0, experts=False).bias
    assert b.dtype == torch.float32 and abs(b.std().item() / 0.1 - 1.0) < 0.15


def test_zipf_offset_is_carried_by_a_constant_feature():
    # o_e = -1.1 ln r_e with r a seeded permutation of 1..E, stored in W_g[:, 0] (bf16) and
    # multiplied by x[:, 0] = 1 for every token
    w = scaled(WORKLOADS["switch"], T=300, D=64, F=64)
    inp = make_inputs(w, seed=0, experts=False)
    assert torch.all(inp.x[:, 0] == 1.0)
    got = np.sort(inp.Wg[:, 0].float().numpy())
    want = np.sort(torch.tensor([-1.1 * math.log(r) for r in range(1, w.E + 1)])
                   .to(torch.bfloat16).float().numpy())
    np.testing.assert_array_equal(got, want)
    # the prior it induces is p_e proportional to r_e^-1.1: the most favoured expert's offset
    assert got.max() == 0.0


def test_expert_choice_tokens_come_from_clusters_with_unit_variance():
    # mu_j ~ N(0, I/2), x_t = mu_{c(t)} + N(0, I/2): marginal variance 1, and tokens of the same
    # cluster are closer to each other than to other clusters' tokens
    w = scaled(WORKLOADS["ec"], T=2000, D=256, F=64, c=100)
    x = make_inputs(w, seed=0, experts=False).x.float()
    assert abs(x.var().item() - 1.0) < 0.05
    # cluster ids are not returned: two tokens of one cluster have cosine ~ 1/2 (the shared
    # mean carries half the variance), of different clusters ~ 0, so each token's most similar
    # other token (one of ~250 in its cluster) sits well above 1/4
    xn = x / x.norm(dim=1, keepdim=True)
    sim = xn[:400] @ xn.T
    sim[torch.arange(400), torch.arange(400)] = -2.0
    assert (sim.max(dim=1).values > 0.25).float().mean().item() > 0.95


def test_router_keys_are_separated_for_the_parity_checks():
    # every token's k+1 largest router keys (fp64 keys of the rounded inputs) are pairwise
    # at least 1e-3 apart, so fp32 logits select the same experts as the fp64 oracle
    for w in (scaled(WORKLOADS["mixtral"], T=256, D=256, F=64),
              scaled(WORKLOADS["switch"], T=256, D=64, F=64),
              scaled(WORKLOADS["v3"], T=128, D=64, E=64, F=64, F_shared=64, n_shared=0)):
        inp = C.inputs_for(w, device="cpu")
        keys = C.key_fn_for(w)(C.np64(inp.x), C.np64(inp.Wg), C.np64(inp.bias))
        top = -np.sort(-keys, axis=1)[:, :w.k + 1]
        assert (top[:, :-1] - top[:, 1:]).min() >= 1e-3, w.name
