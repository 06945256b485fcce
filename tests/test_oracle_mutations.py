"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake in the oracle -- a dropped term, a wrong sign, axis or
index, swapped or untransposed operands, a wrong normaliser or rounding, a step left out -- by
replacing one oracle function for the duration of the case (pytest's monkeypatch restores it),
then calls the pins of tests/test_oracle_pins.py directly and requires that at least one of
them fails.  A mistake in the forward pass must be caught by a forward pin (the backward pins,
which compare the analytic gradients with finite differences of the forward, are left out for
it), a mistake in the backward by a backward pin.  A pin "fails" when it raises: an assertion,
or an error such as a shape mismatch that the mistake provokes.  The unmodified oracle passes
every pin (test_oracle_pins.py itself, and the control case below).
"""

import math

import numpy as np
import pytest

from oracle import moe_oracle as O
import test_oracle_pins as P


def _pin_calls():
    """Every pin of test_oracle_pins.py with each of its parametrisations."""
    calls = []
    for name in sorted(dir(P)):
        if not name.startswith("test_"):
            continue
        fn = getattr(P, name)
        params = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not params:
            calls.append((name, fn, {}))
            continue
        argnames, values = params[0].args[0], params[0].args[1]
        if isinstance(argnames, str):
            argnames = [a.strip() for a in argnames.split(",")]
        for vals in values:
            if len(argnames) == 1:
                vals = (vals,)
            calls.append((f"{name}{list(vals)}", fn, dict(zip(argnames, vals))))
    return calls


PINS = _pin_calls()


BACKWARD = ("silu_grad", "gelu_grad", "expert_backward", "gate_logit_grad", "layer_backward")


def _first_failing_pin(stage=None):
    """Name of the first pin that fails (None: all pass).  stage "forward" / "backward" runs
    only the forward pins or only the backward (finite-difference) pins."""
    for name, fn, kwargs in PINS:
        if stage is not None and (("backward" in name) != (stage == "backward")):
            continue
        try:
            fn(**kwargs)
        except Exception:            # an assertion, or an error the planted mistake provokes
            return name
    return None


# ---- the planted mistakes: (oracle function, builder taking the original) ----

def _a(v):
    return np.asarray(v, dtype=np.float64)


def _reversed_dispatch(orig):
    # overflow keeps the LATEST assignments of an expert (rows in descending token order)
    def f(ids, E, cap=None):
        ids = np.asarray(ids, dtype=np.int64)
        T, k = ids.shape
        counts, kept, offsets, rs, iv = orig(ids[::-1], E, cap)
        row_src = (T - 1 - rs // k) * k + rs % k
        inv = np.full(T * k, -1, dtype=np.int64)
        for a, r in enumerate(iv):
            if r >= 0:
                inv[(T - 1 - a // k) * k + a % k] = r
        return counts, kept, offsets, row_src, inv
    return f


def _bias_in_merge(orig):
    # the selection-only bias also enters the sigmoid merge weights
    def f(logits, k, score="softmax", gate="renorm", bias=None, n_group=1, topk_group=1):
        ids, g, imp = orig(logits, k, score, gate, bias, n_group, topk_group)
        if score == "sigmoid" and bias is not None:
            w = O.sigmoid(logits) + _a(bias)[None, :]
            psel = np.take_along_axis(w, ids, axis=1)
            g = psel / psel.sum(axis=1, keepdims=True) if gate == "renorm" else psel
        return ids, g, imp
    return f


def _ec_least_probable(orig):
    def f(logits, c):
        picked, p = orig(logits, c)
        low = np.sort(np.argsort(p, axis=0, kind="stable")[:c].T, axis=1)
        return low, p
    return f


def _combine_assigns(orig):
    # the last contribution overwrites the token row instead of accumulating
    def f(T, D, y_rows, inv, gates, K, shared=None):
        out = np.zeros((T, D))
        inv = np.asarray(inv).reshape(T, K)
        gates = _a(gates).reshape(T, K)
        for t in range(T):
            for j in range(K):
                if inv[t, j] >= 0:
                    out[t] = gates[t, j] * y_rows[inv[t, j]]
        if shared is not None:
            for ys in shared:
                out += ys
        return out
    return f


def _stats_with(change):
    def build(orig):
        def f(importance_rows, counts, n_kept, n_routes, alpha):
            st = orig(importance_rows, counts, n_kept, n_routes, alpha)
            change(st, np.asarray(counts, dtype=np.float64), alpha)
            return st
        return f
    return build


def _f_over_experts(st, counts, alpha):
    st["f"] = counts / len(counts)
    st["aux"] = alpha * len(counts) * float(np.sum(st["f"] * st["P"]))


def _aux_without_E(st, counts, alpha):
    st["aux"] = st["aux"] / len(counts)


def _max_over_median(st, counts, alpha):
    st["max_over_mean"] = float(counts.max() / np.median(counts))


def _entropy_in_bits(st, counts, alpha):
    st["entropy"] = st["entropy"] / math.log(2.0)


def _group_by_sum(orig):
    def f(keys, n_group, topk_group):
        keys = _a(keys)
        T, E = keys.shape
        size = E // n_group
        scores = keys.reshape(T, n_group, size).sum(axis=2)
        best = O.topk_desc(scores, topk_group)
        allowed = np.zeros((T, n_group), dtype=bool)
        np.put_along_axis(allowed, best, True, axis=1)
        return np.repeat(allowed, size, axis=1)
    return f


def _swap_gate_up_grads(orig):
    def f(act, xr, dy, Wgate, Wup, Wdown):
        dx, dwg, dwu, dwd = orig(act, xr, dy, Wgate, Wup, Wdown)
        if dwg is not None:
            dwg, dwu = dwu, dwg
        return dx, dwg, dwu, dwd
    return f


MUTANTS = {
    # score
    "logits drop the first input feature":
        ("router_logits", lambda o: lambda x, Wg: o(_a(x)[:, 1:], _a(Wg)[:, 1:])),
    "logits with W_g not transposed":
        ("router_logits", lambda o: lambda x, Wg: _a(x) @ _a(Wg)),
    "softmax over tokens instead of experts":
        ("softmax_rows", lambda o: lambda s: o(_a(s).T).T),
    "softmax of the negated logits":
        ("softmax_rows", lambda o: lambda s: o(-_a(s))),
    "sigmoid with the wrong sign":
        ("sigmoid", lambda o: lambda s: o(-_a(s))),
    # select
    "top-k takes the smallest keys":
        ("topk_desc", lambda o: lambda keys, k: o(-_a(keys), k)),
    "top-k ties go to the higher index":
        ("topk_desc", lambda o: lambda keys, k: (_a(keys).shape[1] - 1) - o(_a(keys)[:, ::-1], k)),
    "top-k slots in ascending key order":
        ("topk_desc", lambda o: lambda keys, k: o(keys, k)[:, ::-1]),
    "gates not renormalised":
        ("route_token_choice",
         lambda o: lambda logits, k, score="softmax", gate="renorm", *a, **kw:
             o(logits, k, score, "raw", *a, **kw)),
    "selection ignores the selection bias":
        ("route_token_choice",
         lambda o: lambda logits, k, score="softmax", gate="renorm", bias=None, *a, **kw:
             o(logits, k, score, gate, None, *a, **kw)),
    "selection bias enters the merge weights": ("route_token_choice", _bias_in_merge),
    "expert choice takes the least probable tokens": ("route_expert_choice", _ec_least_probable),
    "group score is the sum of its keys": ("group_limit_mask", _group_by_sum),
    # dispatch
    "capacity rounded down":
        ("capacity", lambda o: lambda cf, T, k, E: int(math.floor(float(cf) * T * k / E))),
    "capacity without the factor k":
        ("capacity", lambda o: lambda cf, T, k, E: o(cf, T, 1, E)),
    "overflow keeps the latest assignments": ("dispatch_token_choice", _reversed_dispatch),
    # experts
    "SwiGLU with gate and up swapped":
        ("swiglu_expert", lambda o: lambda xr, Wg, Wu, Wd: o(xr, Wu, Wg, Wd)),
    "SwiGLU without the SiLU":
        ("swiglu_expert",
         lambda o: lambda xr, Wg, Wu, Wd: ((_a(xr) @ _a(Wg).T) * (_a(xr) @ _a(Wu).T)) @ _a(Wd).T),
    "SiLU replaced by the sigmoid":
        ("silu", lambda o: lambda z: 1.0 / (1.0 + np.exp(-z))),
    "ReLU expert without the ReLU":
        ("relu_expert", lambda o: lambda xr, Wu, Wd: (_a(xr) @ _a(Wu).T) @ _a(Wd).T),
    "GELU by the tanh approximation":
        ("gelu", lambda o: lambda z: 0.5 * _a(z) * (1.0 + np.tanh(
            math.sqrt(2.0 / math.pi) * (_a(z) + 0.044715 * _a(z) ** 3)))),
    # merge
    "combine ignores the gates":
        ("combine", lambda o: lambda T, D, y, inv, gates, K, shared=None:
            o(T, D, y, inv, np.ones_like(_a(gates)), K, shared)),
    "combine drops the shared experts":
        ("combine", lambda o: lambda T, D, y, inv, gates, K, shared=None:
            o(T, D, y, inv, gates, K, None)),
    "combine assigns instead of accumulating": ("combine", _combine_assigns),
    # statistics
    "load f normalised by the expert count": ("balance_stats", _stats_with(_f_over_experts)),
    "aux loss without the factor E": ("balance_stats", _stats_with(_aux_without_E)),
    "imbalance as max over median": ("balance_stats", _stats_with(_max_over_median)),
    "entropy in bits": ("balance_stats", _stats_with(_entropy_in_bits)),
    # backward
    "SiLU derivative without the z term":
        ("silu_grad", lambda o: lambda z: 1.0 / (1.0 + np.exp(-z))),
    "gate gradient with the wrong sign":
        ("gate_logit_grad", lambda o: lambda *a, **kw: -o(*a, **kw)),
    "expert weight gradients of gate and up swapped": ("expert_backward", _swap_gate_up_grads),
}


def test_the_unmodified_oracle_passes_every_pin():
    assert _first_failing_pin() is None


@pytest.mark.parametrize("mistake", list(MUTANTS))
def test_a_pin_catches_the_planted_mistake(mistake, monkeypatch):
    attr, build = MUTANTS[mistake]
    monkeypatch.setattr(O, attr, build(getattr(O, attr)))
    stage = "backward" if attr in BACKWARD else "forward"
    assert _first_failing_pin(stage) is not None, f"no {stage} pin catches: {mistake}"
