"""Pins of the CPU oracle to facts the pages and mathematics fix (no GPU).

Each test ties one oracle function to something other than itself: a worked
example printed on a page (fixtures in tests/golden/, each citing its page and
section), a closed form, brute force over a tiny input, or a reduction of the
layer to a textbook computation (a dense FFN, soft routing).
"""

import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def cfg(**kw):
    base = dict(T=8, D=6, E=4, F=5, k=2, c=0, score="softmax", select="token",
                gate="renorm", overflow="dropless", capacity_factor=0.0,
                act="swiglu", n_shared=0, F_shared=0, aux_alpha=1e-2)
    base.update(kw)
    return base


def rand_layer(rng, c, with_bias=False):
    x = rng.standard_normal((c["T"], c["D"]))
    Wg = rng.standard_normal((c["E"], c["D"]))
    Wgate = rng.standard_normal((c["E"], c["F"], c["D"])) / math.sqrt(c["D"])
    Wup = rng.standard_normal((c["E"], c["F"], c["D"])) / math.sqrt(c["D"])
    Wdown = rng.standard_normal((c["E"], c["D"], c["F"])) / math.sqrt(c["F"])
    b = rng.standard_normal(c["E"]) * 0.3 if with_bias else None
    return x, Wg, b, Wgate, Wup, Wdown


# ---------------------------------------------------------------- router ----

def test_router_logits_basis_vector_gives_weight_column():
    # s = W_g . x with x the d-th basis vector is column d of W_g (shape [E, D]).
    rng = np.random.default_rng(1)
    Wg = rng.standard_normal((5, 7))
    for d in range(7):
        x = np.zeros((1, 7))
        x[0, d] = 1.0
        np.testing.assert_array_equal(O.router_logits(x, Wg)[0], Wg[:, d])


def test_router_logits_is_linear_in_x():
    rng = np.random.default_rng(2)
    Wg = rng.standard_normal((3, 4))
    a, b = rng.standard_normal((1, 4)), rng.standard_normal((1, 4))
    np.testing.assert_allclose(O.router_logits(2 * a - b, Wg),
                               2 * O.router_logits(a, Wg) - O.router_logits(b, Wg), atol=1e-12)


def test_softmax_rows_are_distributions_and_shift_invariant():
    rng = np.random.default_rng(3)
    s = rng.standard_normal((6, 5)) * 4
    p = O.softmax_rows(s)
    np.testing.assert_allclose(p.sum(1), 1.0, atol=1e-15)
    np.testing.assert_allclose(O.softmax_rows(s + 100.0), p, atol=1e-14)
    # ratio of two probabilities is e^{s_i - s_j}
    np.testing.assert_allclose(p[:, 0] / p[:, 1], np.exp(s[:, 0] - s[:, 1]), rtol=1e-12)


def test_sigmoid_closed_forms():
    assert O.sigmoid(np.array([0.0]))[0] == 0.5
    np.testing.assert_allclose(O.sigmoid(np.array([math.log(3.0)])), [0.75], rtol=1e-15)
    np.testing.assert_allclose(O.sigmoid(np.array([-math.log(3.0)])), [0.25], rtol=1e-15)


# ------------------------------------------------------------ selection ----

def test_page_router_example_top2_renormalised():
    g = gold("tiny_moe_router_example.json")
    logits = np.log(np.array([g["router_probs"]]))
    ids, gates, probs = O.route_token_choice(logits, g["k"], "softmax", "renorm")
    assert ids[0].tolist() == g["topk_indices"]
    np.testing.assert_allclose(np.take_along_axis(probs, ids, 1)[0], g["topk_weights"], rtol=1e-12)
    np.testing.assert_allclose(gates[0], g["renormalized"], rtol=1e-12)
    ids_raw, gates_raw, _ = O.route_token_choice(logits, g["k"], "softmax", "raw")
    np.testing.assert_allclose(gates_raw[0], g["topk_weights"], rtol=1e-12)


@pytest.mark.parametrize("E,k", [(4, 2), (6, 3), (8, 1), (5, 5)])
def test_topk_matches_bruteforce_enumeration(E, k):
    # The chosen set maximises the key sum over all C(E, k) subsets, and its
    # members come in descending key order.
    rng = np.random.default_rng(10 + E * 7 + k)
    keys = rng.standard_normal((40, E))
    ids = O.topk_desc(keys, k)
    for t in range(keys.shape[0]):
        best = max(itertools.combinations(range(E), k), key=lambda S: sum(keys[t, list(S)]))
        assert sorted(ids[t].tolist()) == sorted(best)
        vals = keys[t, ids[t]]
        assert np.all(vals[:-1] > vals[1:])


def test_topk_ties_go_to_lower_index():
    keys = np.array([[1.0, 3.0, 3.0, 0.0, 3.0]])
    assert O.topk_desc(keys, 2)[0].tolist() == [1, 2]
    assert O.topk_desc(keys, 3)[0].tolist() == [1, 2, 4]


def test_renormalised_gates_equal_softmax_over_selected_logits():
    # [TKR] gate Step 2: g_i = e^{s_i} / sum_{j in TopK} e^{s_j} (variant b)
    # equals softmax over all experts followed by renormalisation (variant a).
    rng = np.random.default_rng(4)
    s = rng.standard_normal((20, 6)) * 2
    ids, gates, _ = O.route_token_choice(s, 3, "softmax", "renorm")
    for t in range(20):
        sel = s[t, ids[t]]
        direct = [math.exp(v) / sum(math.exp(u) for u in sel) for v in sel]
        np.testing.assert_allclose(gates[t], direct, rtol=1e-12)
    np.testing.assert_allclose(gates.sum(1), 1.0, atol=1e-15)


def test_switch_raw_gate_is_top1_softmax_value():
    rng = np.random.default_rng(5)
    s = rng.standard_normal((30, 8))
    ids, gates, probs = O.route_token_choice(s, 1, "softmax", "raw")
    np.testing.assert_allclose(gates[:, 0], probs.max(1), rtol=1e-15)
    assert np.all(gates <= 1.0)
    assert np.all(ids[:, 0] == s.argmax(1))


def test_sigmoid_bias_changes_selection_but_not_merge_weights():
    # logits chosen so that sigma(s) ranks expert 0 > 1 > 2, while the bias
    # lifts expert 2 above expert 1 for selection only.
    s = np.array([[2.0, 1.0, 0.5]])
    b = np.array([0.0, 0.0, 0.15])
    ids, gates, _ = O.route_token_choice(s, 2, "sigmoid", "renorm", bias=b)
    assert ids[0].tolist() == [0, 2]
    a0, a2 = 1 / (1 + math.exp(-2.0)), 1 / (1 + math.exp(-0.5))
    np.testing.assert_allclose(gates[0], [a0 / (a0 + a2), a2 / (a0 + a2)], rtol=1e-14)
    ids_nb, _, _ = O.route_token_choice(s, 2, "sigmoid", "renorm", bias=None)
    assert ids_nb[0].tolist() == [0, 1]


def test_expert_choice_bruteforce_and_exact_counts():
    rng = np.random.default_rng(6)
    T, E, c = 7, 3, 2
    s = rng.standard_normal((T, E)) * 2
    picked, p = O.route_expert_choice(s, c)
    assert picked.shape == (E, c)
    for e in range(E):
        best = max(itertools.combinations(range(T), c), key=lambda S: sum(p[list(S), e]))
        assert picked[e].tolist() == sorted(best)
    counts, kept, offsets, row_src, inv = O.dispatch_expert_choice(picked, T)
    assert counts.tolist() == [c] * E and offsets.tolist() == [0, 2, 4, 6]


# -------------------------------------------------------------- dispatch ----

def test_page_dispatch_example():
    g = gold("tiny_moe_dispatch_example.json")
    ids = np.array(g["topk_indices"])
    counts, kept, offsets, row_src, inv = O.dispatch_token_choice(ids, g["num_experts"])
    e = g["expert_id"]
    rows = row_src[offsets[e]:offsets[e + 1]]
    k = ids.shape[1]
    assert (rows // k).tolist() == g["token_indices"]
    assert (rows % k).tolist() == g["route_slots"]
    assert ((ids == e).tolist() == g["mask"])
    # inverse permutation
    for r, a in enumerate(row_src):
        assert inv[a] == r


def test_counts_sum_to_routes_and_permutation_is_bijection():
    gt = gold("tiny_moe_route_totals.json")
    for cnt in gt["printed_counts"]:
        assert sum(cnt) == gt["routes"] == gt["N"] * gt["K"]
    rng = np.random.default_rng(7)
    s = rng.standard_normal((gt["N"], 4))
    ids, _, _ = O.route_token_choice(s, gt["K"])
    counts, kept, offsets, row_src, inv = O.dispatch_token_choice(ids, 4)
    assert counts.sum() == gt["routes"]
    assert sorted(row_src.tolist()) == list(range(gt["routes"]))
    assert sorted(inv.tolist()) == list(range(gt["routes"]))


def test_capacity_formula_and_switch_value():
    # [TKR] capacity factor: buffer = CF * tokens/N * k; Switch workload: 80 slots.
    assert O.capacity(1.25, 8192, 1, 128) == 80
    assert O.capacity(1.0, 10, 2, 4) == 5
    assert O.capacity(1.1, 10, 1, 4) == 3          # 2.75 rounds up


def test_capacity_drops_later_assignments_first():
    ids = np.array([[0], [0], [1], [0], [0]])
    counts, kept, offsets, row_src, inv = O.dispatch_token_choice(ids, 2, cap=2)
    assert counts.tolist() == [4, 1] and kept.tolist() == [2, 1]
    assert inv.tolist() == [0, 1, 2, -1, -1]
    assert row_src.tolist() == [0, 1, 2]


# ----------------------------------------------------------- expert FFN ----

def test_swiglu_closed_form_scalar():
    # D = F = 1: out = w_down * SiLU(w_gate * x) * (w_up * x); SiLU(ln 3) = (3/4) ln 3.
    x = np.array([[1.0]])
    out = O.swiglu_expert(x, [[math.log(3.0)]], [[2.0]], [[0.5]])
    np.testing.assert_allclose(out, [[0.5 * 0.75 * math.log(3.0) * 2.0]], rtol=1e-15)
    # gate and up are not interchangeable: swapping them changes the result
    out_sw = O.swiglu_expert(x, [[2.0]], [[math.log(3.0)]], [[0.5]])
    assert abs(out_sw[0, 0] - out[0, 0]) > 0.1
    # a zero gate pre-activation closes the gate
    assert O.swiglu_expert(x, [[0.0]], [[5.0]], [[1.0]])[0, 0] == 0.0


def _swiglu_by_loops(xv, Wgate, Wup, Wdown):
    D, F = len(xv), len(Wgate)
    h = []
    for f in range(F):
        a = sum(Wgate[f][d] * xv[d] for d in range(D))
        u = sum(Wup[f][d] * xv[d] for d in range(D))
        h.append(a / (1 + math.exp(-a)) * u)
    return [sum(Wdown[d][f] * h[f] for f in range(F)) for d in range(D)]


def test_single_expert_layer_is_the_dense_ffn():
    c = cfg(E=1, k=1, T=3)
    rng = np.random.default_rng(8)
    x, Wg, _, Wgate, Wup, Wdown = rand_layer(rng, c)
    r = O.layer_forward(c, x, Wg, None, Wgate, Wup, Wdown)
    for t in range(c["T"]):
        ref = _swiglu_by_loops(x[t].tolist(), Wgate[0].tolist(), Wup[0].tolist(), Wdown[0].tolist())
        np.testing.assert_allclose(r["out"][t], ref, rtol=1e-12, atol=1e-14)


def test_relu_expert_closed_form():
    x = np.array([[1.0, -2.0]])
    Wup = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])      # pre-act [1, -2, -1]
    Wdown = np.array([[1.0, 1.0, 1.0], [2.0, 0.0, 5.0]])
    np.testing.assert_allclose(O.relu_expert(x, Wup, Wdown), [[1.0, 2.0]])


# -------------------------------------------------------------- combine ----

def test_page_combine_example_accumulates_both_experts():
    g = gold("tiny_moe_combine_example.json")
    # ReLU experts with W_up = I, W_down = (e+1) I: E_e(x) = (e+1) x for x > 0.
    D, E = 3, 4
    c = cfg(T=1, D=D, E=E, F=D, k=2, act="relu")
    Wup = np.stack([np.eye(D)] * E)
    Wdown = np.stack([(e + 1) * np.eye(D) for e in range(E)])
    x = np.array([[0.5, 1.0, 2.0]])
    # router probs [0.2, 0.1, 0.6, 0.1]: top-2 = experts 2, 0 -> 0.75, 0.25
    logits = np.log(np.array([[0.2, 0.1, 0.6, 0.1]]))
    r = O.layer_forward(c, x, np.zeros((E, D)), None, None, Wup, Wdown, logits=logits)
    assert r["ids"][0].tolist() == g["experts"]
    np.testing.assert_allclose(r["gates"][0], g["weights"], rtol=1e-12)
    expect = sum(w * (e + 1) * x[0] for e, w in zip(g["experts"], g["weights"]))
    np.testing.assert_allclose(r["out"][0], expect, rtol=1e-12)


# ----------------------------------------------------- balance statistics ----

def test_page_imbalance_example():
    g = gold("moe_comparison_imbalance.json")
    st = O.balance_stats(np.full((1, 4), 0.25), g["counts"], g["total"], g["total"], 1e-2)
    assert sum(g["counts"]) == g["total"] and g["total"] / 4 == g["ideal_mean"]
    assert st["max_over_mean"] == g["max_over_mean"]
    assert st["n_dropped"] == 0


@pytest.mark.parametrize("case", ["case_A", "case_B"])
def test_page_importance_and_load_cases(case):
    g = gold("tiny_moe_balance_cases.json")
    cs = g[case]
    c = cfg(T=2, E=2, k=1, D=1, F=1, aux_alpha=0.01)
    r = O.route(c, np.log(np.array(cs["probs"])))
    assert r["ids"][:, 0].tolist() == cs["routes"]
    st = r["stats"]
    np.testing.assert_allclose(st["P"], cs["importance"], rtol=1e-12)
    np.testing.assert_allclose(st["f"], cs["load"], rtol=1e-12)
    expect = 0.01 * 2 * sum(p * f for p, f in zip(cs["importance"], cs["load"]))
    np.testing.assert_allclose(st["aux"], expect, rtol=1e-12)
    # case A puts both routes on the expert with the larger importance: 1.02 alpha;
    # case B balances the routes: exactly the reference value 1 * alpha.
    np.testing.assert_allclose(st["aux"] / 0.01, {"case_A": 1.02, "case_B": 1.0}[case], rtol=1e-12)


def test_balanced_reference_value_is_alpha():
    g = gold("tiny_moe_balance_cases.json")
    for E in (2, 4, 8):
        st = O.balance_stats(np.full((5, E), 1.0 / E), [3] * E, 3 * E, 3 * E, 0.01)
        np.testing.assert_allclose(st["aux"], 0.01 * g["balanced_reference_value"], rtol=1e-12)


def test_load_counts_routes_over_tokens_times_k():
    rng = np.random.default_rng(9)
    c = cfg(T=50, E=6, k=2)
    r = O.route(c, rng.standard_normal((50, 6)))
    np.testing.assert_allclose(r["stats"]["f"].sum(), 1.0, atol=1e-15)
    np.testing.assert_allclose(r["stats"]["P"].sum(), 1.0, atol=1e-14)


# ---------------------------------------------------------- whole layer ----

@pytest.mark.parametrize("score,act,bias", [("softmax", "swiglu", False),
                                            ("softmax", "relu", False),
                                            ("sigmoid", "swiglu", True)])
def test_dropless_equals_dense_masked(score, act, bias):
    c = cfg(T=12, D=8, E=5, F=7, k=2, score=score, act=act)
    rng = np.random.default_rng(11)
    x, Wg, b, Wgate, Wup, Wdown = rand_layer(rng, c, with_bias=bias)
    r = O.layer_forward(c, x, Wg, b, Wgate, Wup, Wdown)
    dense = O.dense_masked_forward(c, x, Wg, b, Wgate, Wup, Wdown)
    np.testing.assert_allclose(r["out"], dense, rtol=1e-12, atol=1e-13)


def test_topk_equal_E_with_renorm_is_soft_routing():
    c = cfg(T=9, D=5, E=4, F=6, k=4)
    rng = np.random.default_rng(12)
    x, Wg, _, Wgate, Wup, Wdown = rand_layer(rng, c)
    r = O.layer_forward(c, x, Wg, None, Wgate, Wup, Wdown)
    soft = O.soft_routing_forward(c, x, Wg, Wgate, Wup, Wdown)
    np.testing.assert_allclose(r["out"], soft, rtol=1e-12, atol=1e-13)


def test_large_capacity_equals_dropless_and_overflow_rows_are_zero():
    c = cfg(T=16, D=6, E=4, F=5, k=1, overflow="drop", capacity_factor=100.0, gate="raw")
    rng = np.random.default_rng(13)
    x, Wg, _, Wgate, Wup, Wdown = rand_layer(rng, c)
    Wg[0] += 3.0 * x.mean(0)          # make expert 0 popular
    big = O.layer_forward(c, x, Wg, None, Wgate, Wup, Wdown)
    free = O.layer_forward(dict(c, overflow="dropless"), x, Wg, None, Wgate, Wup, Wdown)
    np.testing.assert_allclose(big["out"], free["out"], rtol=1e-13, atol=1e-14)
    small = O.layer_forward(dict(c, capacity_factor=1.0), x, Wg, None, Wgate, Wup, Wdown)
    cap = O.capacity(1.0, 16, 1, 4)
    assert small["cap"] == cap == 4
    dropped = np.nonzero(small["inv"] < 0)[0]
    assert len(dropped) == small["stats"]["n_dropped"] > 0
    for t in dropped:                          # k = 1: assignment id == token id
        assert np.all(small["out"][t] == 0.0)
    kept = np.nonzero(small["inv"] >= 0)[0]
    np.testing.assert_allclose(small["out"][kept], free["out"][kept], rtol=1e-13, atol=1e-14)
    # the tokens kept by each expert are its earliest ones
    for e in range(4):
        toks = [t for t in range(16) if free["ids"][t, 0] == e]
        assert [t for t in toks if small["inv"][t] >= 0] == toks[:cap]


def test_expert_choice_c_equal_T_is_soft_routing_and_unpicked_rows_are_zero():
    c = cfg(T=6, D=5, E=3, F=4, k=0, c=6, select="expert")
    rng = np.random.default_rng(14)
    x, Wg, _, Wgate, Wup, Wdown = rand_layer(rng, c)
    r = O.layer_forward(c, x, Wg, None, Wgate, Wup, Wdown)
    soft = O.soft_routing_forward(c, x, Wg, Wgate, Wup, Wdown)
    np.testing.assert_allclose(r["out"], soft, rtol=1e-12, atol=1e-13)
    c2 = dict(c, c=1)
    r2 = O.layer_forward(c2, x, Wg, None, Wgate, Wup, Wdown)
    picked = set(r2["ids"].reshape(-1).tolist())
    assert r2["counts"].tolist() == [1, 1, 1]
    for t in range(6):
        if t not in picked:
            assert np.all(r2["out"][t] == 0.0)
    np.testing.assert_allclose(r2["stats"]["f"], [1 / 3] * 3, rtol=1e-15)


def test_shared_expert_adds_with_weight_one():
    c = cfg(T=5, D=4, E=3, F=3, k=1, n_shared=1, F_shared=6)
    rng = np.random.default_rng(15)
    x, Wg, _, Wgate, Wup, Wdown = rand_layer(rng, c)
    Sg, Su, Sd = (rng.standard_normal((1, 6, 4)), rng.standard_normal((1, 6, 4)),
                  rng.standard_normal((1, 4, 6)))
    r = O.layer_forward(c, x, Wg, None, Wgate, Wup, Wdown, Sg, Su, Sd)
    base = O.layer_forward(dict(c, n_shared=0), x, Wg, None, Wgate, Wup, Wdown)
    for t in range(5):
        ref = _swiglu_by_loops(x[t].tolist(), Sg[0].tolist(), Su[0].tolist(), Sd[0].tolist())
        np.testing.assert_allclose(r["out"][t] - base["out"][t], ref, rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("kw", [dict(), dict(overflow="drop", capacity_factor=1.0, k=1, gate="raw"),
                                dict(select="expert", k=0, c=3),
                                dict(score="sigmoid", n_shared=1, F_shared=4)])
def test_sampled_rows_agree_with_full_layer(kw):
    c = cfg(T=10, D=6, E=4, F=5, **kw)
    rng = np.random.default_rng(16)
    x, Wg, b, Wgate, Wup, Wdown = rand_layer(rng, c, with_bias=c["score"] == "sigmoid")
    S = None
    if c["n_shared"]:
        S = (rng.standard_normal((1, 4, 6)), rng.standard_normal((1, 4, 6)),
             rng.standard_normal((1, 6, 4)))
    full = O.layer_forward(c, x, Wg, b, Wgate, Wup, Wdown, *(S or ()))
    rows = O.layer_forward_rows(c, [0, 3, 7, 9], x, Wg, b, Wgate, Wup, Wdown, *(S or ()))
    np.testing.assert_allclose(rows["out_rows"], full["out"][[0, 3, 7, 9]], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- GELU ----

def test_gelu_closed_forms():
    # GELU(z) = z * Phi(z); Phi(1) = 0.8413447460685429 (standard normal table value).
    phi1 = 0.8413447460685429
    np.testing.assert_allclose(O.gelu(np.array([0.0, 1.0, -1.0])),
                               [0.0, phi1, -(1.0 - phi1)], rtol=1e-14, atol=1e-16)
    big = np.array([8.0, -8.0])
    np.testing.assert_allclose(O.gelu(big), [8.0, 0.0], atol=1e-12)
    # classic FFN with GELU, D = F = 1: out = w_down * GELU(w_up * x)
    np.testing.assert_allclose(O.gelu_expert(np.array([[2.0]]), [[0.5]], [[3.0]]),
                               [[3.0 * phi1]], rtol=1e-14)


def test_gelu_layer_is_dense_masked():
    c = cfg(T=10, D=6, E=4, F=5, k=2, act="gelu")
    rng = np.random.default_rng(21)
    x, Wg, _, _, Wup, Wdown = rand_layer(rng, c)
    r = O.layer_forward(c, x, Wg, None, None, Wup, Wdown)
    dense = O.dense_masked_forward(c, x, Wg, None, None, Wup, Wdown)
    np.testing.assert_allclose(r["out"], dense, rtol=1e-12, atol=1e-13)


# ------------------------------------------------- monitoring statistics ----

def test_router_entropy_closed_forms():
    # uniform probabilities over E experts: entropy ln E; a one-hot row: 0
    for E in (2, 8, 64):
        st = O.balance_stats(np.full((3, E), 1.0 / E), [1] * E, E, E, 0.01)
        np.testing.assert_allclose(st["entropy"], math.log(E), rtol=1e-14)
    st = O.balance_stats(np.array([[1.0, 0.0, 0.0], [0.0, 0.0, 1.0]]), [1, 0, 1], 2, 2, 0.01)
    assert st["entropy"] == 0.0
    # two tokens, p = [1/2, 1/2] and [1/4, 3/4]: mean of ln 2 and H(1/4)
    h2 = -(0.25 * math.log(0.25) + 0.75 * math.log(0.75))
    st = O.balance_stats(np.array([[0.5, 0.5], [0.25, 0.75]]), [1, 1], 2, 2, 0.01)
    np.testing.assert_allclose(st["entropy"], (math.log(2) + h2) / 2, rtol=1e-14)


def test_count_percentiles_of_the_page_example():
    # [9,4,2,1] sorted = [1,2,4,9]; position q*(E-1): 0.95*3 = 2.85 -> 4 + 0.85*5 = 8.25,
    # 0.99*3 = 2.97 -> 4 + 0.97*5 = 8.85 (linear interpolation between order statistics)
    g = gold("moe_comparison_imbalance.json")
    st = O.balance_stats(np.full((1, 4), 0.25), g["counts"], g["total"], g["total"], 1e-2)
    np.testing.assert_allclose(st["count_p95"], 8.25, rtol=1e-12)
    np.testing.assert_allclose(st["count_p99"], 8.85, rtol=1e-12)


# ------------------------------------------------ group-limited selection ----
# [RAT] variant (c) (choose groups, then experts inside them); [CMP] "Group/node limited" row
# and the DeepSeek-V3 note (256 experts on 8 nodes, a token's top-8 on at most 4 nodes).

def test_group_limit_hand_example():
    # E = 4 in 2 groups {0,1} {2,3}; keys [0.9, 0.1 | 0.89, 0.88], k = 2.  Plain top-2 is
    # {0, 2} (two groups).  With one group allowed, group 0 (best key 0.9 > 0.89) is kept and
    # the top-2 inside it is [0, 1] -- the limit trades expert 2 (0.89) for expert 1 (0.1).
    s = np.array([[0.9, 0.1, 0.89, 0.88]])
    ids, _, _ = O.route_token_choice(s, 2, "softmax", "renorm")
    assert ids.tolist() == [[0, 2]]
    ids, gates, _ = O.route_token_choice(s, 2, "softmax", "renorm", n_group=2, topk_group=1)
    assert ids.tolist() == [[0, 1]]
    p = np.exp(s[0]) / np.exp(s[0]).sum()
    np.testing.assert_allclose(gates[0], [p[0] / (p[0] + p[1]), p[1] / (p[0] + p[1])], rtol=1e-14)
    assert O.group_limit_mask(s, 2, 1).tolist() == [[True, True, False, False]]
    # equal group scores go to the lower group index
    t = np.array([[0.5, 0.1, 0.5, 0.2]])
    assert O.group_limit_mask(t, 2, 1).tolist() == [[True, True, False, False]]


def test_group_limit_reduces_to_plain_topk():
    rng = np.random.default_rng(31)
    s = rng.normal(size=(50, 16))
    b = rng.normal(scale=0.1, size=16)
    for score, bias in (("softmax", None), ("sigmoid", b)):
        plain = O.route_token_choice(s, 3, score, "renorm", bias)
        for n_group, topk_group in ((1, 1), (4, 4), (16, 16)):
            lim = O.route_token_choice(s, 3, score, "renorm", bias, n_group, topk_group)
            assert np.array_equal(plain[0], lim[0])
            np.testing.assert_array_equal(plain[1], lim[1])


def test_group_limit_invariants_at_the_node_shape():
    # V3 node shape: E = 256 in 8 groups of 32, top-8 on at most 4 groups
    rng = np.random.default_rng(32)
    s = rng.normal(size=(300, 256))
    b = rng.normal(scale=0.1, size=256)
    a = O.sigmoid(s)
    key = a + b
    plain, _, _ = O.route_token_choice(s, 8, "sigmoid", "renorm", b)
    ids, gates, _ = O.route_token_choice(s, 8, "sigmoid", "renorm", b, n_group=8, topk_group=4)
    groups = ids // 32
    assert all(len(set(row)) <= 4 for row in groups.tolist())
    # the token's best expert is always kept (its group has the largest score)
    assert np.array_equal(ids[:, 0], np.argmax(key, axis=1))
    # with distinct keys, a plain top-k that already spans <= 4 groups is unchanged
    spans = np.array([len(set(row)) for row in (plain // 32).tolist()])
    same = spans <= 4
    assert same.any() and (~same).any()
    assert np.array_equal(ids[same], plain[same])
    # otherwise the limited set is the top-8 inside the 4 groups of largest best key
    for t in np.nonzero(~same)[0][:20]:
        gbest = key[t].reshape(8, 32).max(axis=1)
        keep = sorted(np.argsort(-gbest, kind="stable")[:4].tolist())
        cand = [e for e in range(256) if e // 32 in keep]
        want = sorted(cand, key=lambda e: (-key[t, e], e))[:8]
        assert ids[t].tolist() == want
    np.testing.assert_allclose(gates.sum(axis=1), 1.0, rtol=1e-14)


def test_group_limited_dropless_layer_is_dense_masked():
    c = cfg(T=12, D=6, E=8, F=5, k=2)
    c.update(n_group=4, topk_group=1)
    rng = np.random.default_rng(33)
    x, Wg, _, Wgate, Wup, Wdown = rand_layer(rng, c)
    r = O.layer_forward(c, x, Wg, None, Wgate, Wup, Wdown)
    dense = O.dense_masked_forward(c, x, Wg, None, Wgate, Wup, Wdown)
    np.testing.assert_allclose(r["out"], dense, rtol=1e-12, atol=1e-13)
    assert all(len(set(row)) == 1 for row in (r["ids"] // 2).tolist())


# ------------------------------------------------------------- backward ----
# [TKR] "門控網路的梯度流" (selection fixed; selected gate scores carry the gradient, unselected
# experts none) and [TINY] section 9 (task loss + weight x aux loss).  The backward is pinned
# against central finite differences of the (separately pinned) forward oracle.

def _loss(c, x, Wg, b, Wgate, Wup, Wdown, dout, aux_grad, Ws=(None, None, None)):
    r = O.layer_forward(c, x, Wg, b, Wgate, Wup, Wdown, *Ws)
    return float(np.sum(dout * r["out"])) + aux_grad * r["stats"]["aux"], r["ids"]


def _check_fd(c, params, grads, b, dout, aux_grad, rng, shared=()):
    """Directional derivatives of the loss along 3 random directions per parameter, by
    central differences, against the analytic gradients; the selection must not move."""
    eps = 1e-6
    names = ["x", "Wg", "Wgate", "Wup", "Wdown"]
    for name, val in params.items():
        if val is None:
            continue
        for _ in range(3):
            v = rng.standard_normal(val.shape)
            plus, minus = dict(params), dict(params)
            plus[name], minus[name] = val + eps * v, val - eps * v
            args_p = [plus[n] for n in names]
            args_m = [minus[n] for n in names]
            sp = tuple(plus.get(n) for n in shared) if shared else (None, None, None)
            sm = tuple(minus.get(n) for n in shared) if shared else (None, None, None)
            lp, ids_p = _loss(c, args_p[0], args_p[1], b, *args_p[2:], dout, aux_grad, sp)
            lm, ids_m = _loss(c, args_m[0], args_m[1], b, *args_m[2:], dout, aux_grad, sm)
            assert np.array_equal(ids_p, ids_m)                   # the selection did not move
            fd = (lp - lm) / (2 * eps)
            an = float(np.sum(grads[name] * v))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


@pytest.mark.parametrize("kw", [
    dict(score="softmax", gate="renorm", act="swiglu"),
    dict(score="softmax", gate="raw", act="relu", k=1, overflow="drop", capacity_factor=1.0),
    dict(score="sigmoid", gate="renorm", act="gelu", k=3),
    dict(score="sigmoid", gate="raw", act="swiglu", k=2),
])
def test_backward_matches_finite_differences(kw):
    c = cfg(T=9, D=6, E=5, F=4, aux_alpha=0.05)
    c.update(kw)
    rng = np.random.default_rng(41)
    x, Wg, b, Wgate, Wup, Wdown = rand_layer(rng, c, with_bias=(c["score"] == "sigmoid"))
    if c["act"] != "swiglu":
        Wgate = None
    dout = rng.standard_normal((c["T"], c["D"]))
    aux_grad = 0.7
    gr = O.layer_backward(c, x, Wg, b, Wgate, Wup, Wdown, dout, aux_grad)
    if c["overflow"] == "drop":
        assert (np.asarray(gr["forward"]["inv"]) < 0).any()      # some assignments dropped
    params = {"x": x, "Wg": Wg, "Wgate": Wgate, "Wup": Wup, "Wdown": Wdown}
    grads = {"x": gr["dx"], "Wg": gr["dWg"], "Wgate": gr["dW_gate"], "Wup": gr["dW_up"],
             "Wdown": gr["dW_down"]}
    eps = 1e-6
    for name, val in params.items():
        if val is None:
            continue
        for _ in range(3):
            v = rng.standard_normal(val.shape)
            plus, minus = dict(params), dict(params)
            plus[name], minus[name] = val + eps * v, val - eps * v
            lp, ids_p = _loss(c, plus["x"], plus["Wg"], b, plus["Wgate"], plus["Wup"],
                              plus["Wdown"], dout, aux_grad)
            lm, ids_m = _loss(c, minus["x"], minus["Wg"], b, minus["Wgate"], minus["Wup"],
                              minus["Wdown"], dout, aux_grad)
            assert np.array_equal(ids_p, ids_m)                   # the selection did not move
            fd = (lp - lm) / (2 * eps)
            an = float(np.sum(grads[name] * v))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_backward_gate_path_reaches_selected_logits_only():
    # softmax + renorm: the gate gradient is a softmax Jacobian over the selected logits --
    # zero on unselected experts ([TKR]) and summing to zero over the selected ones
    rng = np.random.default_rng(42)
    s = rng.standard_normal((20, 8))
    ids, _, _ = O.route_token_choice(s, 3)
    dg = rng.standard_normal((20, 3))
    ds = O.gate_logit_grad(s, ids, dg, "softmax", "renorm")
    mask = np.zeros_like(ds, dtype=bool)
    np.put_along_axis(mask, ids, True, axis=1)
    assert np.all(ds[~mask] == 0.0)
    np.testing.assert_allclose(ds.sum(axis=1), 0.0, atol=1e-14)


def test_backward_single_expert_is_the_dense_ffn_backward():
    # E = 1, k = 1: the gate is 1 and the layer is the dense FFN; with aux_grad = 0 the layer
    # gradients are the FFN's: dW_down = dout^T h, dx = (dh . u . SiLU'(a)) W_gate + ... .
    c = cfg(T=7, D=5, E=1, F=3, k=1)
    rng = np.random.default_rng(43)
    x, Wg, _, Wgate, Wup, Wdown = rand_layer(rng, c)
    dout = rng.standard_normal((7, 5))
    gr = O.layer_backward(c, x, Wg, None, Wgate, Wup, Wdown, dout, aux_grad=0.0)
    a, u = x @ Wgate[0].T, x @ Wup[0].T
    h = O.silu(a) * u
    dh = dout @ Wdown[0]
    sg = 1 / (1 + np.exp(-a))
    da = dh * u * (sg * (1 + a * (1 - sg)))
    np.testing.assert_allclose(gr["dW_down"][0], dout.T @ h, rtol=1e-12)
    np.testing.assert_allclose(gr["dW_gate"][0], da.T @ x, rtol=1e-12)
    np.testing.assert_allclose(gr["dx"], da @ Wgate[0] + (dh * O.silu(a)) @ Wup[0], rtol=1e-12,
                               atol=1e-13)
    assert np.all(gr["dWg"] == 0.0)


def test_backward_shared_experts_match_finite_differences():
    # DeepSeek-style layer: sigmoid top-3 with a selection bias plus two always-on shared
    # experts ([CMP] "shared direct path", weight 1); the shared weights get gradients too
    c = cfg(T=9, D=6, E=6, F=4, k=3, score="sigmoid", n_shared=2, F_shared=5, aux_alpha=0.05)
    rng = np.random.default_rng(44)
    x, Wg, b, Wgate, Wup, Wdown = rand_layer(rng, c, with_bias=True)
    Sg = rng.standard_normal((2, 5, 6)) / math.sqrt(6)
    Su = rng.standard_normal((2, 5, 6)) / math.sqrt(6)
    Sd = rng.standard_normal((2, 6, 5)) / math.sqrt(5)
    dout = rng.standard_normal((c["T"], c["D"]))
    gr = O.layer_backward(c, x, Wg, b, Wgate, Wup, Wdown, dout, 0.7, Ws_gate=Sg, Ws_up=Su,
                          Ws_down=Sd)
    params = {"x": x, "Wg": Wg, "Wgate": Wgate, "Wup": Wup, "Wdown": Wdown, "Sg": Sg,
              "Su": Su, "Sd": Sd}
    grads = {"x": gr["dx"], "Wg": gr["dWg"], "Wgate": gr["dW_gate"], "Wup": gr["dW_up"],
             "Wdown": gr["dW_down"], "Sg": gr["dWs_gate"], "Su": gr["dWs_up"],
             "Sd": gr["dWs_down"]}
    _check_fd(c, params, grads, b, dout, 0.7, rng, shared=("Sg", "Su", "Sd"))


def test_backward_shared_expert_alone_is_the_dense_ffn_backward():
    # the shared expert's weight gradients are those of the dense SwiGLU FFN on all tokens
    c = cfg(T=7, D=5, E=3, F=4, k=1, n_shared=1, F_shared=3)
    rng = np.random.default_rng(45)
    x, Wg, _, Wgate, Wup, Wdown = rand_layer(rng, c)
    Sg = rng.standard_normal((1, 3, 5))
    Su = rng.standard_normal((1, 3, 5))
    Sd = rng.standard_normal((1, 5, 3))
    dout = rng.standard_normal((7, 5))
    gr = O.layer_backward(c, x, Wg, None, Wgate, Wup, Wdown, dout, 0.0, Ws_gate=Sg, Ws_up=Su,
                          Ws_down=Sd)
    a, u = x @ Sg[0].T, x @ Su[0].T
    np.testing.assert_allclose(gr["dWs_down"][0], dout.T @ (O.silu(a) * u), rtol=1e-12)
    dh = dout @ Sd[0]
    np.testing.assert_allclose(gr["dWs_up"][0], (dh * O.silu(a)).T @ x, rtol=1e-12)


@pytest.mark.parametrize("act", ["swiglu", "relu"])
def test_backward_expert_choice_matches_finite_differences(act):
    # expert choice: each expert keeps its top-c tokens (held fixed); the merge weight of a
    # picked (token, expert) is its softmax probability
    c = cfg(T=10, D=6, E=4, F=4, k=0, c=4, select="expert", act=act, aux_alpha=0.05)
    rng = np.random.default_rng(46)
    x, Wg, _, Wgate, Wup, Wdown = rand_layer(rng, c)
    if act != "swiglu":
        Wgate = None
    dout = rng.standard_normal((c["T"], c["D"]))
    gr = O.layer_backward(c, x, Wg, None, Wgate, Wup, Wdown, dout, 0.7)
    inv = np.asarray(gr["forward"]["inv"]).reshape(10, 4)
    assert (inv < 0).any() and (inv >= 0).sum(axis=1).max() > 1   # unpicked and multi-picked
    params = {"x": x, "Wg": Wg, "Wgate": Wgate, "Wup": Wup, "Wdown": Wdown}
    grads = {"x": gr["dx"], "Wg": gr["dWg"], "Wgate": gr["dW_gate"], "Wup": gr["dW_up"],
             "Wdown": gr["dW_down"]}
    _check_fd(c, params, grads, None, dout, 0.7, rng)


def test_backward_expert_choice_unpicked_token_gets_router_gradient_only():
    # a token no expert picked contributes nothing to out: its dx is the router term ds W_g
    # alone, and with aux_grad = 0 its ds is zero (no merge weight of its own)
    c = cfg(T=12, D=5, E=3, F=4, k=0, c=3, select="expert")
    rng = np.random.default_rng(47)
    x, Wg, _, Wgate, Wup, Wdown = rand_layer(rng, c)
    dout = rng.standard_normal((12, 5))
    gr = O.layer_backward(c, x, Wg, None, Wgate, Wup, Wdown, dout, 0.0)
    inv = np.asarray(gr["forward"]["inv"]).reshape(12, 3)
    un = np.nonzero((inv < 0).all(axis=1))[0]
    assert len(un) > 0
    assert np.all(gr["dlogits"][un] == 0.0) and np.all(gr["dx"][un] == 0.0)
