"""Exact ties in the selection, on the GPU, against the oracle's lowest-index rule.

The pages rank with torch.topk and leave ties open; the reading taken here is that an equal key
goes to the lower expert index (token choice) or the lower token index (expert choice).  The
generators keep keys apart so that selection is stable under rounding; these cases put exact
ties back on purpose:

* token choice: two router rows W_g[a] = W_g[b] (and, under sigmoid, equal selection biases)
  give bit-identical fp32 logits for every token, so wherever a and b sit among a token's k+1
  largest keys the rule decides their order or which of them is kept.  Every router path is
  covered: the mma.sync router (bf16, E <= 8, by default) and the tensor-core router fused
  with the selection (bf16, the other cases by default, E <= 8 in a subprocess), the
  grouped-GEMM router product (bf16, E % 32 == 0, in a subprocess) and the CUDA-core router
  (fp32 always, bf16 in a subprocess).
* sigmoid with a selection bias: two experts whose router rows are zero have sigma(0) = 1/2
  exactly, and equal biases then make their keys equal although the merge weights leave the
  bias out.
* expert choice: a token row copied over another puts two tokens with identical probabilities
  across an expert's c-th place; the lower token id must be the one taken.

All other keys keep the generators' separation (the duplicated columns are left out of the key
function), so the oracle, routing from the GPU's own fp32 logits, takes every other decision the
same way.  Routing and permutation are compared bit for bit, outputs within the usual tolerance
for every token.
"""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_warp_b200.workloads import (WORKLOADS, make_inputs, scaled,
                                                          separate_keys)
import moe_check as C

pytestmark = pytest.mark.gpu

W = WORKLOADS

# name: (workload, duplicated router rows (src, dst), zero router rows with one shared bias)
TOKEN_CASES = {
    # E <= 8 (the mma.sync router under MOE_ROUTER=fast): softmax top-2 renormalised; two
    # tied pairs
    "e8_softmax_top2": (scaled(W["mixtral"], T=300, D=1024, F=256), [(2, 5), (6, 7)], ()),
    # E = 8, top-1 with the raw softmax gate: a tie at the top must go to the lower id
    "e8_top1_raw": (scaled(W["switch"], T=400, D=1024, E=8, F=256, zipf_s=0.0,
                             overflow="dropless"), [(1, 4)], ()),
    # E = 8, sigmoid + bias: zero router rows 1 and 6 with equal biases
    "e8_sigmoid_bias": (scaled(W["v3"], T=200, D=1024, E=8, k=3, F=256, F_shared=256),
                          [], (1, 6)),
    # E = 64 (the grouped-GEMM router product under MOE_ROUTER=gemm), sigmoid + bias, top-6:
    # pairs inside one 32-expert register slot and across two
    "e64_sigmoid_top6": (scaled(W["v3"], T=97, D=1024, E=64, k=6, F=256, F_shared=256),
                          [(3, 4), (10, 41)], ()),
    # E = 32, softmax top-1, raw gate, capacity drop
    # (Zipf offsets: the most popular expert is copied onto the last one, "popular")
    "e32_softmax_top1_drop": (scaled(W["switch"], T=300, D=256, E=32, F=256),
                               "popular", ()),
    # CUDA-core router (fp32): tiny layer, softmax top-2
    "f32_softmax_top2": (scaled(W["tiny"], T=64), [(0, 3)], ()),
    # CUDA-core router (fp32): sigmoid + bias, zero rows with equal biases
    "f32_sigmoid_bias": (scaled(W["v3"], dtype="f32", T=90, D=64, E=16, F=32, k=3, n_shared=1,
                                F_shared=40, w_std=0.1, wg_std=0.1), [(2, 9)], (4, 12)),
}


def _tie_token_inputs(w, dup, zero, seed=0):
    inp = make_inputs(w, seed, "cuda")
    if dup == "popular":
        s = O.router_logits(C.np64(inp.x), C.np64(inp.Wg))
        a = int(np.bincount(s.argmax(axis=1), minlength=w.E).argmax())
        dup = [(a, w.E - 1 if a != w.E - 1 else w.E - 2)]
    for a, b in dup:
        inp.Wg[b] = inp.Wg[a]
        if inp.bias is not None:
            inp.bias[b] = inp.bias[a]
    if zero:
        inp.Wg[list(zero)] = 0
        # bias 0.45 puts the tied keys (sigma(0) + 0.45 = 0.95) among the best few
        inp.bias[list(zero)] = 0.45
    drop = {b for _, b in dup} | set(list(zero)[1:])
    keep = [e for e in range(w.E) if e not in drop]

    def key_fn(x, Wg, b):
        return O.routing_keys(x, Wg, b, w.score)[:, keep]

    separate_keys(w, inp, seed, key_fn, key_gap=1e-3)
    return inp, dup


@pytest.mark.parametrize("name", list(TOKEN_CASES))
def test_token_choice_ties_go_to_the_lower_expert(name):
    w, dup, zero = TOKEN_CASES[name]
    inp, dup = _tie_token_inputs(w, dup, zero)
    out, v = C.run_layer(w, inp)
    logits = v["logits"]
    # the ties are really there: bit-identical fp32 logits
    for a, b in dup:
        assert torch.equal(logits[:, a], logits[:, b]), f"logits of experts {a}, {b} differ"
    for e in zero:
        assert torch.all(logits[:, e] == 0)
    C.check_logits(w, inp, v)
    ref = C.check_routing(w, inp, v)
    # ... and they decided something: tokens for which both tied experts are among the k+1
    # largest keys (which of them is kept, or their slot order)
    s = logits.double().cpu().numpy()
    if w.score == "softmax":
        key = s
    else:
        key = O.sigmoid(s) + inp.bias.double().cpu().numpy()[None, :]
    top = np.argsort(-key, axis=1, kind="stable")[:, :w.k + 1]
    pairs = list(dup) + ([tuple(zero)] if zero else [])
    decided = 0
    ids = ref["ids"]
    for a, b in pairs:
        a, b = min(a, b), max(a, b)
        both = np.isin(top, [a, b]).sum(axis=1) == 2
        decided += int(both.sum())
        for t in np.nonzero(both)[0]:
            row = ids[t].tolist()
            # the lower id is kept whenever the higher one is, and comes first
            if b in row:
                assert a in row and row.index(a) < row.index(b)
    assert decided > 0, "no token has both tied experts among its k+1 best keys"
    C.check_sampled_output(w, inp, out, v, list(range(w.T)))


EC_CASES = {
    "ec_small": scaled(W["ec"], T=1000, D=256, E=16, F=256, c=125),
    # router product on the tcgen05 engine (E = 64)
    "ec_e64": scaled(W["ec"], T=777, D=512, E=64, F=256, c=50),
    "ec_f32": scaled(W["ec"], dtype="f32", T=120, D=32, E=6, F=24, c=30, clusters=4, w_std=0.2,
                     wg_std=0.2),
}


def _boundary_gaps(p, c):
    srt = -np.sort(-p, axis=0)
    return srt[c - 1] - srt[c]


def _top_c(p, e, c):
    return set(np.argsort(-p[:, e], kind="stable")[:c].tolist())


def _plant_ec_tie(w, inp, p, e_star, lower, avoid, keep=()):
    """Copies the token at expert e_star's c-th place over a token ranked below that place,
    chosen with a lower token id (lower=True) or a higher one.  p (the oracle's probabilities,
    kept in step with the copies row by row) must then show every expert's c-th/(c+1)-th gap
    either >= 1e-6 or exactly 0 (a copied pair), and the relations of earlier plants (`keep`:
    (expert, token taken, token left out)) must still hold.  Returns (t_c, t_copy, new p)."""
    c = w.c
    order = np.argsort(-p[:, e_star], kind="stable")
    t_c = int(order[c - 1])
    for t in order[c + 1:].tolist():
        if t in avoid or (t < t_c) != lower:
            continue
        p2 = p.copy()
        p2[t] = p[t_c]
        gaps = _boundary_gaps(p2, c)
        if gaps[e_star] != 0.0 or not np.all((gaps == 0.0) | (gaps >= 1e-6)):
            continue
        if not all(i in _top_c(p2, e, c) and o not in _top_c(p2, e, c) for e, i, o in keep):
            continue
        inp.x[t] = inp.x[t_c]
        return t_c, int(t), p2
    raise AssertionError("no token to copy keeps the other boundaries separated")


@pytest.mark.parametrize("name", list(EC_CASES))
def test_expert_choice_ties_go_to_the_lower_token(name):
    w = EC_CASES[name]
    inp = C.inputs_for(w)
    p = O.softmax_probs_of(C.np64(inp.x), C.np64(inp.Wg))
    # expert 0: the copy has the lower id and must displace the token that held the c-th place;
    # expert 1: the copy has the higher id and must stay out
    t0, u0, p = _plant_ec_tie(w, inp, p, 0, lower=True, avoid=set())
    t1, u1, p = _plant_ec_tie(w, inp, p, 1, lower=False, avoid={t0, u0},
                              keep=[(0, u0, t0)])
    assert u0 in _top_c(p, 0, w.c) and t0 not in _top_c(p, 0, w.c)
    assert t1 in _top_c(p, 1, w.c) and u1 not in _top_c(p, 1, w.c)
    out, v = C.run_layer(w, inp)
    logits = v["logits"]
    assert torch.equal(logits[t0], logits[u0]) and torch.equal(logits[t1], logits[u1])
    C.check_logits(w, inp, v)
    ref = C.check_routing(w, inp, v)
    picked = v["expert_ids"].cpu().numpy()
    assert u0 in picked[0] and t0 not in picked[0]
    assert t1 in picked[1] and u1 not in picked[1]
    np.testing.assert_array_equal(picked, ref["ids"])
    C.check_sampled_output(w, inp, out, v, list(range(w.T)))


# The same ties through the router paths other than the default (MOE_ROUTER is read once per
# process): the tensor-core router takes the E = 8 cases (the mma.sync router has them by
# default; MOE_ROUTER=fast only confirms that), the grouped-GEMM product the E = 32 and E = 64
# ones, the CUDA-core router every bf16 case.
ROUTER_MODES = {
    "tc": "e8_",
    "fast": "e8_",
    "gemm": "e32_ or e64_ or ec_e64",
    "simt": "e8_ or e32_ or e64_ or ec_small or ec_e64",
}


@pytest.mark.parametrize("mode", list(ROUTER_MODES))
def test_ties_through_other_router_paths_in_subprocess(mode):
    import os
    import subprocess
    import sys
    env = dict(os.environ, MOE_ROUTER=mode)
    sel = f"not subprocess and ({ROUTER_MODES[mode]})"
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__, "-k", sel],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout, r.stdout[-3000:]
