"""CPU oracle for the forward pass of one sparse MoE FFN layer (fp64, numpy).

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously correct
statement of what the layer computes, used to check the CUDA library.  Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import it.  It shares no code with the CUDA path and imports nothing from
the product package; the product path never calls it.

Every function follows the pages it cites.  The pages (web articles) are:

  [TKR]  "Top-k 路由（Top-k Routing）", compassingai.com concept page
  [RAT]  "Mixture of Experts (MoE): 解释 MoE 的路由算法（Top-k / expert choice /
         soft routing）与取舍", talentme M4-080
  [GLO]  "Top-K Routing (MoE)", ayinedjimi-consultants glossary
  [CMP]  "别只比较 Top-k：同一个数字，可能对应完全不同的专家工作量",
         ailearn moe-comparison
  [TINY] "从 Dense FFN 到 MoE：用一个 Tiny Transformer 理解 Router、Top-K 与负载均衡",
         f3dlife

Arithmetic is float64 throughout, from the (bf16- or fp32-valued) inputs.
Library primitives used as steps: numpy matmul, exp, and a stable argsort.

Readings where the pages are silent (each one is listed in the design notes):
  * ties in top-k / top-c go to the lower expert / token index;
  * within a token, slot j holds the j-th largest key;
  * rows of one expert are ordered by (token, slot) ascending, as torch.where
    orders them in [TINY] section 5;
  * under a capacity limit C = ceil(CF*T*k/E), the first C assignments of an
    expert in (token, slot) order keep their slot, the rest are dropped and
    contribute zero; gates are not renormalised after a drop;
  * load f_e counts nominal (pre-capacity) routes over T*k;
  * under sigmoid affinity the importance P_e is the mean of the affinities
    normalised to sum 1 over experts;
  * under expert choice the merge weight is the softmax probability, a token
    taken by several experts sums their contributions, an untaken token gets 0;
  * shared experts are added with weight 1;
  * group-limited selection scores a group by its largest selection key and
    keeps each token's topk_group best groups (ties -> lower group index)
    before the top-k.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(worked examples of the pages, closed forms, brute force and reductions to
dense/soft routing; the backward by central finite differences of the forward);
none is "parity unpinned".  ``tests/test_oracle_mutations.py`` plants plausible
mistakes in these functions, one at a time, and checks that a pin of the same
stage catches each.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "router_logits", "softmax_rows", "sigmoid", "routing_keys",
    "topk_desc", "group_limit_mask", "route_token_choice", "route_expert_choice",
    "capacity", "dispatch_token_choice", "dispatch_expert_choice",
    "swiglu_expert", "relu_expert", "gelu", "gelu_expert", "expert_rows",
    "combine", "balance_stats", "layer_forward", "layer_forward_rows",
    "silu_grad", "gelu_grad", "expert_backward", "gate_logit_grad", "layer_backward",
    "dense_masked_forward", "soft_routing_forward",
]


# --------------------------------------------------------------------------
# Score: router logits and affinity
# --------------------------------------------------------------------------

def router_logits(x, Wg):
    """s = W_g . x for every token: logits[t, e] = sum_d Wg[e, d] * x[t, d].

    [TKR] "門控函式的數學形式" Step 1 (W_g in R^{N x d}); [TINY] section 4
    (router = nn.Linear(D, E, bias=False), weight stored [E, D]).
    """
    x = np.asarray(x, dtype=np.float64)
    Wg = np.asarray(Wg, dtype=np.float64)
    return x @ Wg.T


def softmax_rows(s):
    """Softmax over the experts of each token (max-subtracted for range).

    [TKR] gate Step 2, variant (a); [TINY] section 4 (F.softmax over dim=-1).
    """
    s = np.asarray(s, dtype=np.float64)
    z = np.exp(s - s.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def sigmoid(s):
    """Sigmoid affinity sigma(s) = 1 / (1 + e^{-s}), per expert.

    [CMP] "评分、Top-k、合并权重和实际执行" Score step (DeepSeek-V3 uses a
    Sigmoid affinity).
    """
    s = np.asarray(s, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-s))


def routing_keys(x, Wg, bias=None, score="softmax"):
    """Per-token keys that top-k selection ranks.

    Softmax: the logits themselves (softmax is monotone within a row, so the
    top-k of probabilities and of logits coincide).  Sigmoid: sigma(s) + b,
    the selection-only bias of [CMP] "Select" / [RAT] variant (d).
    """
    s = router_logits(x, Wg)
    if score == "softmax":
        return s
    k = sigmoid(s)
    if bias is not None:
        k = k + np.asarray(bias, dtype=np.float64)[None, :]
    return k


def softmax_probs_of(x, Wg):
    """Soft probabilities of every token (expert-choice keys), [TINY] section 4."""
    return softmax_rows(router_logits(x, Wg))


# --------------------------------------------------------------------------
# Select: token choice top-k, expert choice top-c
# --------------------------------------------------------------------------

def topk_desc(keys, k):
    """Indices of the k largest keys per row, largest first; ties -> lower index.

    [TKR] gate "top_k_indices = argtopk"; [TINY] section 4 (torch.topk).  A
    stable sort of -key keeps equal keys in index order.
    """
    keys = np.asarray(keys, dtype=np.float64)
    order = np.argsort(-keys, axis=1, kind="stable")
    return order[:, :k]


def group_limit_mask(keys, n_group, topk_group):
    """Experts each token may select under group-limited routing.

    [RAT] routing variant (c): groups are chosen first, then experts inside
    the chosen groups; [CMP] "Group/node limited" row (the candidate set
    shrinks to the experts of the allowed devices or nodes) and its
    DeepSeek-V3 note (256 experts on 8 nodes, a token's top-8 on at most 4
    nodes).  The experts are split into n_group contiguous groups of
    E / n_group.  The pages do not say how a group is scored; the reading
    here: a group scores its largest selection key, and each token keeps its
    topk_group highest-scoring groups (ties -> lower group index).
    Returns a boolean [T, E] mask.
    """
    keys = np.asarray(keys, dtype=np.float64)
    T, E = keys.shape
    if E % n_group:
        raise ValueError("n_group must divide E")
    size = E // n_group
    scores = keys.reshape(T, n_group, size).max(axis=2)
    best = topk_desc(scores, topk_group)
    allowed = np.zeros((T, n_group), dtype=bool)
    np.put_along_axis(allowed, best, True, axis=1)
    return np.repeat(allowed, size, axis=1)


def route_token_choice(logits, k, score="softmax", gate="renorm", bias=None,
                       n_group=1, topk_group=1):
    """Token-choice routing from router logits.

    Returns (ids[T,k] int, gates[T,k], probs_for_importance[T,E]).

    * softmax + renorm (Mixtral, tiny): p = softmax(s); pick the k largest;
      g_j = p_j / sum_sel p   -- [GLO] TopKRouter, [TINY] section 4,
      [RAT] variant (a).  Equal to softmax over the selected logits
      ([TKR] gate Step 2, variant (b)).
    * softmax + raw (Switch): top-1 of softmax, gate = the softmax value,
      no renormalisation -- [TKR] gate Step 2 note on Switch Transformer.
    * sigmoid (+ optional selection-only bias): select on sigma(s) + b,
      merge weight sigma(s_j) / sum_sel sigma(s)  (bias excluded) --
      [CMP] "Select" / "Merge" steps, DeepSeek-V3 row of the family table.
    * n_group > 1 and topk_group < n_group: the top-k runs over the experts of
      the token's topk_group best groups only (group_limit_mask); merge
      weights and importance are unchanged in form.
    """
    s = np.asarray(logits, dtype=np.float64)
    T, E = s.shape
    if score == "softmax":
        p = softmax_rows(s)
        key = s
        weight = p
        imp = p
    elif score == "sigmoid":
        a = sigmoid(s)
        key = a + (np.asarray(bias, dtype=np.float64)[None, :] if bias is not None else 0.0)
        weight = a
        imp = a / a.sum(axis=1, keepdims=True)
    else:
        raise ValueError(score)
    if n_group > 1 and topk_group < n_group:
        key = np.where(group_limit_mask(key, n_group, topk_group), key, -np.inf)
    ids = topk_desc(key, k)
    psel = np.take_along_axis(weight, ids, axis=1)
    if gate == "renorm":
        g = psel / psel.sum(axis=1, keepdims=True)
    elif gate == "raw":
        g = psel
    else:
        raise ValueError(gate)
    return ids.astype(np.int64), g, imp


def route_expert_choice(logits, c):
    """Expert-choice routing: every expert takes its c most probable tokens.

    [TKR] "Token-Choice vs Expert-Choice" table (each expert picks top-C
    tokens); [RAT] routing class (2).  p = softmax over experts per token;
    per expert column, the c largest p (ties -> lower token id), reported in
    ascending token order.  Returns (picked[E,c], probs[T,E]); the merge weight
    of (t, e) is probs[t, e].
    """
    p = softmax_rows(logits)
    T, E = p.shape
    picked = np.empty((E, c), dtype=np.int64)
    for e in range(E):
        order = np.argsort(-p[:, e], kind="stable")[:c]
        picked[e] = np.sort(order)
    return picked, p


# --------------------------------------------------------------------------
# Execute: capacity and dispatch
# --------------------------------------------------------------------------

def capacity(capacity_factor, T, k, E):
    """Expert buffer = CF * (tokens per batch / N) * k, rounded up.

    [TKR] "容量因子" (capacity factor) formula.  The page gives no rounding;
    ceil, evaluated in double as CF*T*k/E.
    """
    return int(math.ceil(float(capacity_factor) * T * k / E))


def dispatch_token_choice(ids, E, cap=None):
    """Group assignments by expert (the torch.where step of [TINY] section 5).

    Assignment a = t*k + j is token t's j-th choice.  Rows of expert e are its
    assignments in ascending a (token, then slot).  With a capacity `cap`
    ([CMP] capacity + overflow table: Switch skips the expert for an
    overflowing token), only the first `cap` of each expert keep a row.

    Returns counts[E] (nominal), kept[E], offsets[E+1] (exclusive scan of kept),
    row_src[A_kept] (assignment id per row), inv[T*k] (row per assignment, -1
    if dropped).
    """
    ids = np.asarray(ids, dtype=np.int64)
    T, k = ids.shape
    flat = ids.reshape(-1)
    counts = np.zeros(E, dtype=np.int64)
    rank = np.empty_like(flat)
    for a, e in enumerate(flat):              # plain running count per expert
        rank[a] = counts[e]
        counts[e] += 1
    kept = counts.copy() if cap is None else np.minimum(counts, cap)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    inv = np.full(T * k, -1, dtype=np.int64)
    row_src = np.empty(int(offsets[-1]), dtype=np.int64)
    for a, e in enumerate(flat):
        if cap is None or rank[a] < cap:
            r = offsets[e] + rank[a]
            inv[a] = r
            row_src[r] = a
    return counts, kept, offsets, row_src, inv


def dispatch_expert_choice(picked, T):
    """Rows of expert e are its picked tokens in ascending token order.

    Assignment id of (t, e) is t*E + e; inv[T*E] is the row of (t, e) or -1
    (token t not picked by e).  Every expert has exactly c rows.
    """
    picked = np.asarray(picked, dtype=np.int64)
    E, c = picked.shape
    counts = np.full(E, c, dtype=np.int64)
    offsets = np.arange(E + 1, dtype=np.int64) * c
    row_src = np.empty(E * c, dtype=np.int64)
    inv = np.full(T * E, -1, dtype=np.int64)
    for e in range(E):
        for i, t in enumerate(picked[e]):
            r = e * c + i
            row_src[r] = t * E + e
            inv[t * E + e] = r
    return counts, counts.copy(), offsets, row_src, inv


# --------------------------------------------------------------------------
# Expert compute
# --------------------------------------------------------------------------

def silu(z):
    return z / (1.0 + np.exp(-z))


def swiglu_expert(xr, Wgate, Wup, Wdown):
    """One SwiGLU expert on a block of rows.

    [TINY] section 3: gate = SiLU(x W_gate), value = x W_up,
    hidden = gate (.) value, output = hidden W_down, with nn.Linear weights
    gate/up [F, D] and down [D, F].
    """
    xr = np.asarray(xr, dtype=np.float64)
    g = xr @ np.asarray(Wgate, dtype=np.float64).T
    u = xr @ np.asarray(Wup, dtype=np.float64).T
    return (silu(g) * u) @ np.asarray(Wdown, dtype=np.float64).T


def relu_expert(xr, Wup, Wdown):
    """Classic two-matrix FFN D -> F -> D with a ReLU in between.

    [TINY] section 2-3 (the classic D -> 4D -> D FFN; the Switch-style layer
    here uses ReLU as its activation).
    """
    xr = np.asarray(xr, dtype=np.float64)
    h = np.maximum(xr @ np.asarray(Wup, dtype=np.float64).T, 0.0)
    return h @ np.asarray(Wdown, dtype=np.float64).T


def gelu(z):
    """Exact GELU, z * Phi(z) = z * (1 + erf(z / sqrt 2)) / 2 ([TINY] section 3: the classic
    FFN's nn.GELU(), whose default is this erf form)."""
    from scipy.special import erf
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))


def gelu_expert(xr, Wup, Wdown):
    """Classic two-matrix FFN D -> F -> D with GELU in between ([TINY] section 3)."""
    xr = np.asarray(xr, dtype=np.float64)
    return gelu(xr @ np.asarray(Wup, dtype=np.float64).T) @ np.asarray(Wdown, dtype=np.float64).T


def expert_rows(act, xr, e, W_gate, W_up, W_down):
    if act == "swiglu":
        return swiglu_expert(xr, W_gate[e], W_up[e], W_down[e])
    if act == "relu":
        return relu_expert(xr, W_up[e], W_down[e])
    if act == "gelu":
        return gelu_expert(xr, W_up[e], W_down[e])
    raise ValueError(act)


# --------------------------------------------------------------------------
# Merge: weighted combine back to token rows
# --------------------------------------------------------------------------

def combine(T, D, y_rows, inv, gates, K, shared=None):
    """out[t] = sum_j gates[t, j] * y_rows[inv[t, j]]  (+ sum of shared outputs).

    [TKR] "Combine" (output = sum of gate_score_i * y_i); [TINY] section 6:
    accumulate (index_add), never assign.  A dropped or unpicked assignment
    (inv = -1) contributes 0.  Shared experts add with weight 1.
    """
    out = np.zeros((T, D), dtype=np.float64)
    inv = np.asarray(inv).reshape(T, K)
    gates = np.asarray(gates, dtype=np.float64).reshape(T, K)
    for t in range(T):
        for j in range(K):
            r = inv[t, j]
            if r >= 0:
                out[t] += gates[t, j] * y_rows[r]
    if shared is not None:
        for ys in shared:
            out += ys
    return out


# --------------------------------------------------------------------------
# Balance statistics
# --------------------------------------------------------------------------

def balance_stats(importance_rows, counts, n_kept, n_routes, alpha):
    """Load statistics and the auxiliary balance loss.

    P_e = mean_t importance_rows[t, e] (average routing probability, before
    selection); f_e = counts_e / n_routes (share of routes each expert gets,
    [TINY] section 8: one_hot(topk).mean over (tokens, k)); aux = alpha * E *
    sum_e f_e P_e ([TKR] "負載均衡" formula, [TINY] section 8).  Also
    max/mean of the counts ([CMP] "先数 assignments": [9,4,2,1] -> 2.25) and
    the number of dropped routes (n_routes - n_kept).  Monitoring figures of
    [CMP] "监控至少要覆盖分布、容量与网络": the mean router entropy -sum p log p of
    the importance rows, and the 95th/99th percentiles of the counts (linear
    interpolation between order statistics).
    """
    counts = np.asarray(counts, dtype=np.float64)
    E = counts.shape[0]
    P = np.asarray(importance_rows, dtype=np.float64).mean(axis=0)
    f = counts / float(n_routes)
    aux = alpha * E * float(np.sum(f * P))
    mean = counts.sum() / E
    rows = np.asarray(importance_rows, dtype=np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        plogp = np.where(rows > 0, rows * np.log(rows), 0.0)
    return {
        "P": P, "f": f, "aux": aux,
        "max_over_mean": float(counts.max() / mean) if mean > 0 else 0.0,
        "n_dropped": int(n_routes - n_kept),
        # [CMP] monitoring list: router entropy and P95/P99 of the per-expert counts
        "entropy": float(-plogp.sum(axis=1).mean()),
        "count_p95": float(np.percentile(counts, 95)),
        "count_p99": float(np.percentile(counts, 99)),
    }


# --------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------

def _np(a):
    if a is None:
        return None
    if hasattr(a, "detach"):          # a torch tensor handed in by a test
        a = a.detach().float().cpu().numpy()
    return np.asarray(a, dtype=np.float64)


def route(w, logits, bias=None):
    """Score + select + merge weights from given logits (fp32 GPU logits in
    the bit-exact checks, or the oracle's own fp64 logits).

    `w` is a mapping/object with fields k, c, E, T, score, select, gate,
    overflow, capacity_factor, aux_alpha.
    """
    g = _get(w)
    if g["select"] == "token":
        ids, gates, imp = route_token_choice(logits, g["k"], g["score"], g["gate"], bias,
                                             g["n_group"], g["topk_group"])
        cap = capacity(g["capacity_factor"], g["T"], g["k"], g["E"]) if g["overflow"] == "drop" else None
        counts, kept, offsets, row_src, inv = dispatch_token_choice(ids, g["E"], cap)
        K = g["k"]
        n_routes = g["T"] * g["k"]
    else:
        picked, p = route_expert_choice(logits, g["c"])
        ids, gates, imp = picked, p, p
        counts, kept, offsets, row_src, inv = dispatch_expert_choice(picked, g["T"])
        K = g["E"]
        n_routes = g["E"] * g["c"]
        cap = None
    stats = balance_stats(imp, counts, int(kept.sum()), n_routes, g["aux_alpha"])
    return dict(ids=ids, gates=gates, importance=imp, counts=counts, kept=kept,
                offsets=offsets, row_src=row_src, inv=inv, K=K, cap=cap, stats=stats)


def _get(w):
    keys = ["T", "D", "E", "F", "k", "c", "score", "select", "gate", "overflow",
            "capacity_factor", "act", "n_shared", "F_shared", "aux_alpha"]
    optional = {"n_group": 1, "topk_group": 1}      # no group limit unless given
    if isinstance(w, dict):
        out = {k: w[k] for k in keys}
        out.update({k: w.get(k, v) for k, v in optional.items()})
        return out
    out = {k: getattr(w, k) for k in keys}
    out.update({k: getattr(w, k, v) for k, v in optional.items()})
    return out


def layer_forward(w, x, Wg, bias, W_gate, W_up, W_down,
                  Ws_gate=None, Ws_up=None, Ws_down=None, logits=None):
    """The whole forward pass (Gate -> Dispatch -> Expert compute -> Combine,
    [TKR] lifecycle; [CMP] Score -> Select -> Merge -> Execute).

    `logits`, when given, replaces the router product (used to route from the
    GPU's fp32 logits).  Returns a dict with the routing, the stats, the
    per-row expert outputs and out[T, D].
    """
    g = _get(w)
    x = _np(x)
    s = router_logits(x, _np(Wg)) if logits is None else _np(logits)
    r = route(g, s, _np(bias))
    Wgt, Wu, Wd = _np(W_gate), _np(W_up), _np(W_down)
    D = g["D"]
    y = np.zeros((len(r["row_src"]), D), dtype=np.float64)
    off = r["offsets"]
    K = r["K"]
    for e in range(g["E"]):
        rows = slice(off[e], off[e + 1])
        if off[e + 1] == off[e]:
            continue
        src_tok = r["row_src"][rows] // K
        y[rows] = expert_rows(g["act"], x[src_tok], e, Wgt, Wu, Wd)
    shared = None
    if g["n_shared"]:
        Sg, Su, Sd = _np(Ws_gate), _np(Ws_up), _np(Ws_down)
        shared = [swiglu_expert(x, Sg[i], Su[i], Sd[i]) for i in range(g["n_shared"])]
    out = combine(g["T"], D, y, r["inv"], r["gates"], K, shared)
    r.update(logits=s, y_rows=y, shared=shared, out=out)
    return r


def layer_forward_rows(w, tokens, x, Wg, bias, W_gate, W_up, W_down,
                       Ws_gate=None, Ws_up=None, Ws_down=None, logits=None,
                       weights_of=None):
    """out[t] for a sample of tokens at full size.

    Routing and dispatch are computed for the whole batch (a drop depends on
    earlier tokens); only the sampled tokens' expert rows are evaluated.
    `weights_of(e)` (optional) returns (W_gate[e], W_up[e], W_down[e]) as fp64
    arrays, so that a caller can stream expert weights from device memory one
    expert at a time.  Besides out_rows, the result holds each evaluated
    assignment's expert output before its gate (y_assign[(t, j)]) and each
    shared expert's output on the sampled tokens (shared_rows[i]).
    """
    g = _get(w)
    x = _np(x)
    s = router_logits(x, _np(Wg)) if logits is None else _np(logits)
    r = route(g, s, _np(bias))
    K = r["K"]
    tokens = [int(t) for t in tokens]
    need = {}
    for t in tokens:
        for j in range(K):
            row = r["inv"][t * K + j]
            if row >= 0:
                e = j if g["select"] == "expert" else int(r["ids"][t, j])
                need.setdefault(e, []).append((t, j))
    if weights_of is None:
        Wgt, Wu, Wd = _np(W_gate), _np(W_up), _np(W_down)

        def weights_of(e):
            return (Wgt[e] if Wgt is not None else None), Wu[e], Wd[e]
    out = {t: np.zeros(g["D"], dtype=np.float64) for t in tokens}
    gates = np.asarray(r["gates"], dtype=np.float64).reshape(g["T"], K)
    y_assign = {}
    for e in sorted(need):
        wg_e, wu_e, wd_e = weights_of(e)
        ts = [t for t, _ in need[e]]
        if g["act"] == "swiglu":
            ye = swiglu_expert(x[ts], wg_e, wu_e, wd_e)
        elif g["act"] == "gelu":
            ye = gelu_expert(x[ts], wu_e, wd_e)
        else:
            ye = relu_expert(x[ts], wu_e, wd_e)
        for i, (t, j) in enumerate(need[e]):
            out[t] += gates[t, j] * ye[i]
            y_assign[(t, j)] = ye[i]
    shared_rows = []
    if g["n_shared"]:
        Sg, Su, Sd = _np(Ws_gate), _np(Ws_up), _np(Ws_down)
        for i in range(g["n_shared"]):
            ys = swiglu_expert(x[tokens], Sg[i], Su[i], Sd[i])
            shared_rows.append(ys)
            for n, t in enumerate(tokens):
                out[t] += ys[n]
    r.update(logits=s, out_rows=np.stack([out[t] for t in tokens]) if tokens else
             np.zeros((0, g["D"])), y_assign=y_assign, shared_rows=shared_rows)
    return r


# --------------------------------------------------------------------------
# Backward pass with the selection fixed
# --------------------------------------------------------------------------
# [TKR] "門控網路的梯度流": the discrete top-k is not differentiated; the gate
# scores of the selected experts carry the gradient, unselected experts get
# none from the gates.  [TINY] section 9: total loss = task loss + weight x
# router aux loss; selected experts' gate/up/down matrices, the selected route
# weights (task loss) and the soft importance (balance loss) get gradients;
# the expert indices are fixed integers.  The loss here is
#   L = <dout, out> + aux_grad * aux,
# i.e. dout = dL/dout and aux_grad = dL/daux are given.  The selection-only
# bias is not trained by gradients (the pages update it by a rule).

def silu_grad(z):
    """d/dz of z * sigma(z) = sigma(z) * (1 + z * (1 - sigma(z)))."""
    z = np.asarray(z, dtype=np.float64)
    sg = 1.0 / (1.0 + np.exp(-z))
    return sg * (1.0 + z * (1.0 - sg))


def gelu_grad(z):
    """d/dz of z * Phi(z) = Phi(z) + z * phi(z)."""
    from scipy.special import erf
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * (1.0 + erf(z / math.sqrt(2.0))) + z * np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)


def expert_backward(act, xr, dy, Wgate, Wup, Wdown):
    """Gradients of one expert FFN on its rows xr, given dy = dL/dy_rows.

    Returns (dx_rows, dW_gate or None, dW_up, dW_down).  Chain rule through
    [TINY] section 3's expert (SwiGLU: h = SiLU(x W_gate^T) * (x W_up^T),
    y = h W_down^T; the classic FFN with ReLU or GELU).
    """
    xr = np.asarray(xr, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    Wu = np.asarray(Wup, dtype=np.float64)
    Wd = np.asarray(Wdown, dtype=np.float64)
    if act == "swiglu":
        Wg = np.asarray(Wgate, dtype=np.float64)
        a = xr @ Wg.T
        b = xr @ Wu.T
        h = silu(a) * b
        dh = dy @ Wd
        da = dh * b * silu_grad(a)
        db = dh * silu(a)
        return da @ Wg + db @ Wu, da.T @ xr, db.T @ xr, dy.T @ h
    z = xr @ Wu.T
    if act == "relu":
        h, dz_dh = np.maximum(z, 0.0), (z > 0).astype(np.float64)
    elif act == "gelu":
        h, dz_dh = gelu(z), gelu_grad(z)
    else:
        raise ValueError(act)
    dz = (dy @ Wd) * dz_dh
    return dz @ Wu, None, dz.T @ xr, dy.T @ h


def gate_logit_grad(logits, ids, dgates, score="softmax", gate="renorm", bias=None):
    """dL/ds from dL/dg of the merge weights, the selection ids held fixed.

    softmax + renorm: g_j = softmax over the selected logits ([TKR] masked
    softmax), so ds_i = g_i (dg_i - sum_j g_j dg_j) for selected i, 0
    otherwise ([TKR]: unselected experts' gate derivative is 0).
    softmax + raw: g_j = p_{id_j}, p = softmax over all E:
    ds = p (.) (dp - <p, dp>), dp scattered from dg.
    sigmoid + renorm: g_j = a_j / sum_sel a (a = sigma(s)):
    da_i = (dg_i - sum_j g_j dg_j) / sum_sel a, ds = da a (1 - a).
    sigmoid + raw: da_i = dg_i, ds = da a (1 - a).
    """
    s = np.asarray(logits, dtype=np.float64)
    T, E = s.shape
    ids = np.asarray(ids)
    dg = np.asarray(dgates, dtype=np.float64)
    ds = np.zeros((T, E), dtype=np.float64)
    for t in range(T):
        sel = ids[t]
        if score == "softmax":
            if gate == "renorm":
                z = np.exp(s[t, sel] - s[t, sel].max())
                g = z / z.sum()
                ds[t, sel] = g * (dg[t] - np.dot(g, dg[t]))
            else:
                p = softmax_rows(s[t:t + 1])[0]
                dp = np.zeros(E)
                np.add.at(dp, sel, dg[t])
                ds[t] = p * (dp - np.dot(p, dp))
        else:
            a = sigmoid(s[t])
            da = np.zeros(E)
            if gate == "renorm":
                asel = a[sel]
                g = asel / asel.sum()
                np.add.at(da, sel, (dg[t] - np.dot(g, dg[t])) / asel.sum())
            else:
                np.add.at(da, sel, dg[t])
            ds[t] = da * a * (1.0 - a)
    return ds


def layer_backward(w, x, Wg, bias, W_gate, W_up, W_down, dout, aux_grad=1.0, logits=None,
                   Ws_gate=None, Ws_up=None, Ws_down=None):
    """Gradients of L = <dout, out> + aux_grad * aux for one MoE layer, the
    routing of layer_forward held fixed.

    Per kept assignment (t, j) -> row r of expert e: dy_r = g[t,j] dout[t] and
    dg[t,j] = <dout[t], y_r>; a dropped (or, under expert choice, unpicked)
    assignment has neither.  Experts: expert_backward on their rows.
    Router: token choice -- ds = gate_logit_grad(dg); expert choice -- the
    merge weight of (t, e) is the softmax probability p[t, e] itself, so
    ds = p (.) (dp - <p, dp>) with dp[t, e] = dg[t, e] on picked pairs, 0
    elsewhere (the picked sets are held fixed, as the top-k is).  Plus the
    balance-loss term: aux = alpha E sum_e f_e P_e with f fixed (counts) and
    P_e = mean_t of the importance rows, so dP_e = aux_grad alpha E f_e / T,
    pushed through softmax over all E (ds = p (dq - <p, dq>)) or through
    q = a / sum_e a under sigmoid (da = (dq - <q, dq>) / sum a, ds = da a (1-a)).
    Shared experts ([CMP] "shared direct path", weight 1) see dout on every
    token: dx gains their input gradient and dWs_* their weight gradients.
    dW_g = ds^T x, and dx = sum_j dx_rows[r(t, j)] + ds W_g (+ shared).
    """
    g = _get(w)
    x = _np(x)
    Wg = _np(Wg)
    r = layer_forward(w, x, Wg, bias, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down,
                      logits=logits)
    s, K, T, E = r["logits"], r["K"], g["T"], g["E"]
    dout = np.asarray(dout, dtype=np.float64)
    inv = np.asarray(r["inv"]).reshape(T, K)
    gates = np.asarray(r["gates"], dtype=np.float64).reshape(T, K)
    y = r["y_rows"]
    A = len(r["row_src"])
    dy = np.zeros((A, g["D"]), dtype=np.float64)
    dgates = np.zeros((T, K), dtype=np.float64)
    for t in range(T):
        for j in range(K):
            row = inv[t, j]
            if row >= 0:
                dy[row] = gates[t, j] * dout[t]
                dgates[t, j] = float(np.dot(dout[t], y[row]))
    Wgt, Wu, Wd = _np(W_gate), _np(W_up), _np(W_down)
    dWgate = np.zeros_like(Wgt) if Wgt is not None else None
    dWup, dWdown = np.zeros_like(Wu), np.zeros_like(Wd)
    dx_rows = np.zeros((A, g["D"]), dtype=np.float64)
    off = r["offsets"]
    for e in range(E):
        rows = slice(off[e], off[e + 1])
        if off[e + 1] == off[e]:
            continue
        xr = x[r["row_src"][rows] // K]
        dxr, dge, due, dde = expert_backward(g["act"], xr, dy[rows],
                                             Wgt[e] if Wgt is not None else None, Wu[e], Wd[e])
        dx_rows[rows] = dxr
        if dge is not None:
            dWgate[e] = dge
        dWup[e], dWdown[e] = due, dde
    if g["select"] == "token":
        ds = gate_logit_grad(s, r["ids"], dgates, g["score"], g["gate"], _np(bias))
    else:
        p = softmax_rows(s)
        dp = np.where(inv >= 0, dgates, 0.0)
        ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    f = r["stats"]["f"]
    dq = np.broadcast_to(aux_grad * g["aux_alpha"] * E * f / T, (T, E))
    if g["score"] == "softmax":
        p = softmax_rows(s)
        ds = ds + p * (dq - np.sum(p * dq, axis=1, keepdims=True))
    else:
        a = sigmoid(s)
        q = a / a.sum(axis=1, keepdims=True)
        da = (dq - np.sum(q * dq, axis=1, keepdims=True)) / a.sum(axis=1, keepdims=True)
        ds = ds + da * a * (1.0 - a)
    dx = ds @ Wg
    for t in range(T):
        for j in range(K):
            if inv[t, j] >= 0:
                dx[t] += dx_rows[inv[t, j]]
    dWs = None
    if g["n_shared"]:
        Sg, Su, Sd = _np(Ws_gate), _np(Ws_up), _np(Ws_down)
        dWs = (np.zeros_like(Sg), np.zeros_like(Su), np.zeros_like(Sd))
        for i in range(g["n_shared"]):
            dxs, dgs, dus, dds = expert_backward("swiglu", x, dout, Sg[i], Su[i], Sd[i])
            dx += dxs
            dWs[0][i], dWs[1][i], dWs[2][i] = dgs, dus, dds
    return dict(forward=r, dx=dx, dWg=ds.T @ x, dW_gate=dWgate, dW_up=dWup, dW_down=dWdown,
                dWs_gate=dWs[0] if dWs else None, dWs_up=dWs[1] if dWs else None,
                dWs_down=dWs[2] if dWs else None, dgates=dgates, dlogits=ds, dy_rows=dy)


# --------------------------------------------------------------------------
# Second paths (used only to pin the first)
# --------------------------------------------------------------------------

def dense_masked_forward(w, x, Wg, bias, W_gate, W_up, W_down):
    """Every expert on every token, then keep only each token's selected
    experts with their gates.  Equal to the dropless sparse layer."""
    g = _get(w)
    x = _np(x)
    s = router_logits(x, _np(Wg))
    ids, gates, _ = route_token_choice(s, g["k"], g["score"], g["gate"], _np(bias),
                                       g["n_group"], g["topk_group"])
    Wgt, Wu, Wd = _np(W_gate), _np(W_up), _np(W_down)
    T = x.shape[0]
    allout = np.stack([expert_rows(g["act"], x, e, Wgt, Wu, Wd) for e in range(g["E"])], 1)
    mask = np.zeros((T, g["E"]), dtype=np.float64)
    for t in range(T):
        for j in range(g["k"]):
            mask[t, ids[t, j]] = gates[t, j]
    return np.einsum("te,ted->td", mask, allout)


def soft_routing_forward(w, x, Wg, W_gate, W_up, W_down):
    """Soft routing y = sum_i g_i(x) E_i(x) over all experts with softmax g
    ([RAT] routing class (3))."""
    g = _get(w)
    x = _np(x)
    p = softmax_rows(router_logits(x, _np(Wg)))
    Wgt, Wu, Wd = _np(W_gate), _np(W_up), _np(W_down)
    allout = np.stack([expert_rows(g["act"], x, e, Wgt, Wu, Wd) for e in range(g["E"])], 1)
    return np.einsum("te,ted->td", p, allout)
