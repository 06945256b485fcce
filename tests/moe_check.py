"""Helpers of the GPU parity tests: run the CUDA layer through the C ABI and compare it with
the CPU oracle on the same seeded inputs.

Tolerances (from the layer's arithmetic):
  * routing (expert ids, counts, offsets, row order, inverse permutation, dropped sets) is
    compared bit-exactly, the oracle routing from the GPU's own fp32 logits;
  * router logits: for every token t and expert e, |gpu - oracle| / sum_d |x[t,d] Wg[e,d]|
    <= 1e-5.  The denominator is the condition number of the fp32 dot product: its rounding
    error is bounded relative to the sum of the magnitudes of its terms, so the bound holds per
    logit whatever the logit's own size (a logit near zero, or E = 1);
  * gates / probabilities: relative 1e-5 (fp32 exp and division);
  * layer output: max |gpu - oracle| / max |oracle| over the compared rows <= 2e-2 for bf16
    operands (bf16 rounding of h, y and out, each 2^-9 relative), <= 1e-5 for fp32; rows the
    method zeroes (dropped or unpicked tokens) must be exactly zero.
"""

from __future__ import annotations

import numpy as np
import torch

import sparse_mixture_experts_warp_b200 as M
from sparse_mixture_experts_warp_b200.workloads import make_inputs
from oracle import moe_oracle as O

TOL_OUT = {"bf16": 2e-2, "f32": 1e-5}
TOL_LOGITS = 1e-5
TOL_GATES = 1e-5


def key_fn_for(w):
    if w.select == "expert":
        return lambda x, Wg, b: O.softmax_probs_of(x, Wg)
    if w.n_group > 1 and w.topk_group < w.n_group:
        # group-limited: separate the k+1 best keys, the topk_group+1 best group scores and
        # the k+1 best keys inside the kept groups
        def fn(x, Wg, b):
            key = O.routing_keys(x, Wg, b, w.score)
            gs = key.reshape(key.shape[0], w.n_group, -1).max(axis=2)
            inside = np.where(O.group_limit_mask(key, w.n_group, w.topk_group), key, -1e30)
            return [(key, w.k + 1), (gs, w.topk_group + 1), (inside, w.k + 1)]
        return fn
    return lambda x, Wg, b: O.routing_keys(x, Wg, b, w.score)


def inputs_for(w, seed=0, device="cuda"):
    if w.select == "expert":
        return make_inputs(w, seed, device, key_fn=key_fn_for(w), ec_gap=1e-6)
    return make_inputs(w, seed, device, key_fn=key_fn_for(w), key_gap=1e-3)


def np64(t):
    if t is None:
        return None
    return t.detach().float().cpu().double().numpy()


def run_layer(w, inp):
    d = M.desc_of(w)
    ws = M.empty_workspace(d, inp.x.device)
    out = torch.empty_like(inp.x)
    M.moe_layer_forward(d, inp.x, inp.Wg, inp.bias, inp.W_gate, inp.W_up, inp.W_down,
                        inp.Ws_gate, inp.Ws_up, inp.Ws_down, out, ws)
    torch.cuda.synchronize()
    err = M.get_device_error()
    assert err == 0, f"device error word {err:#x}"
    return out, M.layer_views(d, ws)


def max_rel(a, b):
    den = np.max(np.abs(b))
    if den == 0:
        return float(np.max(np.abs(a)))
    return float(np.max(np.abs(a - b)) / den)


def logit_condition(x, Wg):
    """cond[t, e] = sum_d |x[t, d] * Wg[e, d]|, the scale of one fp32 dot product's rounding
    error (each of its D products and partial sums is rounded relative to this sum)."""
    return np.abs(x) @ np.abs(Wg).T


def check_logits(w, inp, v, rows=None):
    """GPU fp32 logits against the oracle's fp64 router product (optionally sampled rows),
    per token and expert: |gpu - oracle| <= 1e-5 * sum_d |x_d Wg[e, d]|.  A logit whose terms
    are all zero (cond = 0) must be exactly zero."""
    x = np64(inp.x) if rows is None else np64(inp.x[torch.as_tensor(rows, device=inp.x.device)])
    Wg = np64(inp.Wg)
    ref = O.router_logits(x, Wg)
    got = v["logits"].double().cpu().numpy()
    if rows is not None:
        got = got[rows]
    cond = logit_condition(x, Wg)
    diff = np.abs(got - ref)
    zero = cond == 0.0
    assert np.all(diff[zero] == 0.0), "a logit with no nonzero term is not exactly zero"
    rel = diff[~zero] / cond[~zero]
    err = float(rel.max()) if rel.size else 0.0
    assert err <= TOL_LOGITS, f"router logit error {err:.3e} of sum|x*Wg| (tolerance 1e-5)"
    return err


def wdict(w):
    return dict(T=w.T, D=w.D, E=w.E, F=w.F, k=w.k, c=w.c, score=w.score, select=w.select,
                gate=w.gate, overflow=w.overflow, capacity_factor=w.capacity_factor, act=w.act,
                n_shared=w.n_shared, F_shared=w.F_shared, aux_alpha=w.aux_alpha,
                n_group=w.n_group, topk_group=w.topk_group)


def check_routing(w, inp, v):
    """Routing, permutation and statistics bit-exact / within fp32 rounding, with the oracle
    routing from the GPU's fp32 logits."""
    logits = v["logits"].double().cpu().numpy()
    ref = O.route(wdict(w), logits, np64(inp.bias))
    ids = v["expert_ids"].cpu().numpy()
    np.testing.assert_array_equal(ids, ref["ids"])
    counts = v["counts"].cpu().numpy()
    offsets = v["offsets"].cpu().numpy()
    np.testing.assert_array_equal(counts, ref["counts"])
    np.testing.assert_array_equal(offsets, ref["offsets"])
    n = int(offsets[-1])
    np.testing.assert_array_equal(v["row_src"].cpu().numpy()[:n], ref["row_src"])
    np.testing.assert_array_equal(v["inv"].cpu().numpy().reshape(-1), ref["inv"])
    gates = v["gates"].double().cpu().numpy()
    np.testing.assert_allclose(gates, np.asarray(ref["gates"]).reshape(gates.shape),
                               rtol=TOL_GATES, atol=1e-7)
    # gathered rows are exact copies of their tokens (when the layer writes them: with the
    # gathering up projection it reads them straight from x and x_perm stays unwritten)
    K = ref["K"]
    if n and not M.gather_fusion(M.desc_of(w)):
        src_tok = torch.as_tensor(ref["row_src"] // K, device=inp.x.device, dtype=torch.long)
        assert torch.equal(v["x_perm"][:n], inp.x[src_tok])
    st = ref["stats"]
    np.testing.assert_allclose(v["importance"].double().cpu().numpy(), st["P"], rtol=1e-5,
                               atol=1e-7)
    np.testing.assert_allclose(v["f"].double().cpu().numpy(), st["f"], rtol=1e-6, atol=1e-9)
    s = M.stats_of(v["stats"])
    np.testing.assert_allclose(s["aux"], st["aux"], rtol=1e-5)
    np.testing.assert_allclose(s["max_over_mean"], st["max_over_mean"], rtol=1e-6)
    assert s["n_dropped"] == st["n_dropped"]
    assert s["n_kept"] == int(ref["kept"].sum())
    np.testing.assert_allclose(s["count_p95"], st["count_p95"], rtol=1e-6)
    np.testing.assert_allclose(s["count_p99"], st["count_p99"], rtol=1e-6)
    # entropy from fp32 logits: fp32 exp/log over E terms per token, averaged over T
    np.testing.assert_allclose(s["entropy"], st["entropy"], rtol=1e-4, atol=1e-6)
    return ref


def check_full_output(w, inp, out, ref_route):
    """Whole-layer output against the oracle's fp64 evaluation (all rows)."""
    r = O.layer_forward(wdict(w), np64(inp.x), np64(inp.Wg), np64(inp.bias), np64(inp.W_gate),
                        np64(inp.W_up), np64(inp.W_down), np64(inp.Ws_gate), np64(inp.Ws_up),
                        np64(inp.Ws_down), logits=None)
    # the oracle routed from its own logits: gaps in the inputs make that routing identical
    np.testing.assert_array_equal(r["ids"], ref_route["ids"])
    got = out.double().cpu().numpy()
    err = max_rel(got, r["out"])
    assert err <= TOL_OUT[w.dtype], f"layer output max rel err {err:.3e}"
    zero_rows = np.nonzero(np.all(r["out"] == 0.0, axis=1))[0]
    assert np.all(got[zero_rows] == 0.0)
    return err


def expert_weights_streamer(inp):
    """weights_of(e) for the oracle: one expert's weights copied to the host as fp64."""
    def weights_of(e):
        g = np64(inp.W_gate[e]) if inp.W_gate is not None else None
        return g, np64(inp.W_up[e]), np64(inp.W_down[e])
    return weights_of


def check_sampled_output(w, inp, out, v, tokens):
    """Sampled output rows at full size: oracle routes the whole batch from the GPU's logits
    and evaluates only the sampled tokens' experts."""
    logits = v["logits"].double().cpu().numpy()
    tk = torch.as_tensor(tokens, device=inp.x.device, dtype=torch.long)
    x_rows = np.zeros((w.T, w.D))
    x_rows[tokens] = np64(inp.x[tk])
    r = O.layer_forward_rows(wdict(w), tokens, x_rows, None, np64(inp.bias), None, None, None,
                             np64(inp.Ws_gate), np64(inp.Ws_up), np64(inp.Ws_down),
                             logits=logits, weights_of=expert_weights_streamer(inp))
    got = out[tk].double().cpu().numpy()
    ref = r["out_rows"]
    err = max_rel(got, ref)
    assert err <= TOL_OUT[w.dtype], f"sampled output max rel err {err:.3e}"
    for i in range(len(tokens)):
        if np.all(ref[i] == 0.0):
            assert np.all(got[i] == 0.0)
    return err


def stratified_rows(offsets, rng, every_slice=True):
    """Executed rows to check at full size.  The grouped GEMM tiles each expert's rows from the
    expert's first row in 256-row tiles made of two 128-row MMA halves, whose rows sit in the
    four 32-lane quarters of the TMEM accumulator; so the 32-row slices of each expert, counted
    from its first row, are exactly its (tile, half, lane quarter) cells.  One random row from
    every slice (or, with every_slice=False, from one random slice per expert), plus each
    expert's last row (the ragged tail of its last tile)."""
    rows = set()
    for e in range(len(offsets) - 1):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi <= lo:
            continue
        starts = list(range(lo, hi, 32))
        if not every_slice:
            starts = [starts[int(rng.integers(len(starts)))]]
        for s in starts:
            rows.add(int(rng.integers(s, min(s + 32, hi))))
        rows.add(hi - 1)
    return sorted(rows)


def check_stratified_output(w, inp, out, v, seed=123, every_slice=True, extra_tokens=()):
    """Full-size output parity on a tile-stratified sample (stratified_rows).

    Each sampled executed row's expert output y (before its gate) is compared with the
    oracle's evaluation of that assignment; every token owning a sampled row, every token of
    one row per 32-token slice of the shared experts' group (the tokens themselves) and
    `extra_tokens` are compared on the whole layer output, the oracle routing the batch from
    the GPU's fp32 logits.  Returns (rows checked, tokens checked, y error, output error)."""
    rng = np.random.default_rng(seed)
    offsets = v["offsets"].cpu().numpy()
    row_src = v["row_src"].cpu().numpy()
    K = w.E if w.select == "expert" else w.k
    rows = stratified_rows(offsets, rng, every_slice)
    tokens = {int(row_src[r]) // K for r in rows}
    if w.n_shared:
        tokens.update(stratified_rows(np.array([0, w.T]), rng, every_slice))
    tokens.update(int(t) for t in extra_tokens)
    tokens = sorted(tokens)
    logits = v["logits"].double().cpu().numpy()
    tk = torch.as_tensor(tokens, device=inp.x.device, dtype=torch.long)
    x_rows = np.zeros((w.T, w.D))
    x_rows[tokens] = np64(inp.x[tk])
    r = O.layer_forward_rows(wdict(w), tokens, x_rows, None, np64(inp.bias), None, None, None,
                             np64(inp.Ws_gate), np64(inp.Ws_up), np64(inp.Ws_down),
                             logits=logits, weights_of=expert_weights_streamer(inp))
    # expert outputs of the sampled rows
    ref_y = np.stack([r["y_assign"][(int(row_src[q]) // K, int(row_src[q]) % K)] for q in rows])
    got_y = np64(v["y"][torch.as_tensor(rows, device=inp.x.device, dtype=torch.long)])
    err_y = max_rel(got_y, ref_y)
    assert err_y <= TOL_OUT[w.dtype], f"sampled expert rows max rel err {err_y:.3e}"
    if w.n_shared:
        for i in range(w.n_shared):
            got_s = np64(v["y_shared"][i][tk])
            err_s = max_rel(got_s, r["shared_rows"][i])
            assert err_s <= TOL_OUT[w.dtype], f"shared expert {i} rows max rel err {err_s:.3e}"
    # whole-layer output of the tokens
    got = out[tk].double().cpu().numpy()
    ref = r["out_rows"]
    err = max_rel(got, ref)
    assert err <= TOL_OUT[w.dtype], f"sampled output max rel err {err:.3e}"
    for i in range(len(tokens)):
        if np.all(ref[i] == 0.0):
            assert np.all(got[i] == 0.0)
    return len(rows), len(tokens), err_y, err
