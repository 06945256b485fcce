"""Seeded synthetic workloads for the sparse MoE FFN layer.

This module only draws random numbers and names shapes.  It holds none of the
layer's arithmetic: where a workload needs its router keys to be well
separated (so that a top-k or top-c selection is stable under rounding), the
caller passes in the function that computes those keys.

The five workloads are the layer shapes the pages talk about:

* ``tiny``     -- the tiny fp32 MoE of "从 Dense FFN 到 MoE：用一个 Tiny Transformer
  理解 Router、Top-K 与负载均衡" (f3dlife), sections 3-4: D=32, E=4, F=48, top-2.
* ``mixtral``  -- Mixtral-8x7B layer shape (8 experts, top-2, SwiGLU F=14336).
* ``switch``   -- Switch-style top-1 with ReLU experts and a capacity limit.
* ``v3``       -- DeepSeek-V3 layer shape (256 routed + 1 shared, sigmoid, top-8,
  selection-only bias).
* ``ec``       -- expert-choice routing at the DeepSeekMoE-16B layer shape.

Recipe (seed 0 unless told otherwise): every tensor is drawn as fp32 from a
``torch.Generator`` on the target device, scaled by its standard deviation and,
for bf16 workloads, rounded once to bf16 (round-to-nearest-even, torch's
``.to(torch.bfloat16)``).  Tensors are drawn in a fixed order so that a given
(seed, device) always gives the same inputs.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int                 # tokens in the batch
    D: int                 # hidden size
    E: int                 # routed experts
    F: int                 # expert intermediate size
    k: int = 0             # token-choice top-k (0 under expert choice)
    c: int = 0             # expert-choice tokens per expert (0 under token choice)
    score: str = "softmax"     # "softmax" | "sigmoid"
    select: str = "token"      # "token" | "expert"
    gate: str = "renorm"       # "renorm" | "raw"
    overflow: str = "dropless"  # "dropless" | "drop"
    capacity_factor: float = 0.0
    act: str = "swiglu"        # "swiglu" | "relu" | "gelu"
    dtype: str = "bf16"        # "bf16" | "f32"
    n_shared: int = 0
    F_shared: int = 0
    aux_alpha: float = 1e-2
    n_group: int = 1           # group-limited selection: expert groups (1 = no limit)
    topk_group: int = 1        # groups each token may use
    x_std: float = 1.0
    w_std: float = 0.02
    wg_std: float = 0.02
    bias_std: float = 0.0      # selection-only bias b_e ~ N(0, bias_std)
    zipf_s: float = 0.0        # Zipf-scaled per-expert logit offset (0 = none)
    clusters: int = 0          # token clusters for the expert-choice router
    description: str = ""

    def as_dict(self) -> dict:
        return asdict(self)


WORKLOADS = {
    "tiny": Workload(
        "tiny", T=64, D=32, E=4, F=48, k=2, dtype="f32",
        x_std=1.0, w_std=1.0 / math.sqrt(32), wg_std=1.0 / math.sqrt(32),
        description="tiny MoE: D=32, E=4 SwiGLU F=48, softmax top-2 renormalised, "
                    "dropless, fp32, x[64,32]"),
    "mixtral": Workload(
        "mixtral", T=4096, D=4096, E=8, F=14336, k=2,
        description="Mixtral-8x7B layer: D=4096, E=8 SwiGLU F=14336, softmax top-2 "
                    "renormalised, dropless, bf16, x[4096,4096]"),
    "switch": Workload(
        "switch", T=8192, D=768, E=128, F=3072, k=1, gate="raw", overflow="drop",
        capacity_factor=1.25, act="relu", zipf_s=1.1,
        description="Switch top-1: D=768, E=128 ReLU F=3072, softmax value as gate, "
                    "capacity ceil(1.25*T/E)=80, overflow dropped, bf16, x[8192,768]"),
    "v3": Workload(
        "v3", T=4096, D=7168, E=256, F=2048, k=8, score="sigmoid", n_shared=1,
        F_shared=2048, bias_std=0.1,
        description="DeepSeek-V3 layer: D=7168, 256 routed + 1 shared SwiGLU F=2048, "
                    "sigmoid, selection-only bias, top-8 renormalised, dropless, bf16"),
    "ec": Workload(
        "ec", T=16384, D=2048, E=64, F=1408, c=512, select="expert", clusters=8,
        description="expert choice at DeepSeekMoE-16B shape: D=2048, E=64 SwiGLU "
                    "F=1408, softmax, each expert takes its top c=512 tokens, bf16"),
}


def capacity_of(w: Workload) -> int:
    """Slots per expert under the drop policy, C = ceil(CF * T * k / E), in double."""
    if w.overflow != "drop":
        return 0
    return int(math.ceil(float(w.capacity_factor) * w.T * w.k / w.E))


def rows_max(w: Workload) -> int:
    """Upper bound on the rows the experts execute (A): T*k, E*C or E*c."""
    if w.select == "expert":
        return w.E * w.c
    if w.overflow == "drop":
        return min(w.T * w.k, w.E * capacity_of(w))
    return w.T * w.k


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields changed (smaller parity cases)."""
    d = w.as_dict()
    d.update(changes)
    return Workload(**d)


def _dt(w: Workload):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def _randn(gen, shape, std, device):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


@dataclass
class Inputs:
    x: torch.Tensor                  # [T, D]
    Wg: torch.Tensor                 # [E, D] router weight (nn.Linear layout)
    bias: torch.Tensor | None        # [E] fp32 selection-only bias
    W_gate: torch.Tensor | None      # [E, F, D]
    W_up: torch.Tensor               # [E, F, D]
    W_down: torch.Tensor             # [E, D, F]
    Ws_gate: torch.Tensor | None = None   # [S, Fs, D]
    Ws_up: torch.Tensor | None = None     # [S, Fs, D]
    Ws_down: torch.Tensor | None = None   # [S, D, Fs]
    resampled: int = 0               # token rows redrawn to separate router keys
    extra: dict = field(default_factory=dict)


def make_inputs(w: Workload, seed: int = 0, device="cpu", experts: bool = True,
                key_fn=None, key_gap: float = 0.0, ec_gap: float = 0.0,
                max_rounds: int = 64) -> Inputs:
    """Draw the seeded inputs of one workload.

    key_fn(x_rows[fp64 numpy], Wg[fp64 numpy], bias[fp64 numpy|None]) -> keys[n,E]
    is the caller's routing-key function.  When it is given with key_gap > 0
    (token choice), every token whose k+1 largest keys are not pairwise
    separated by key_gap has its x row redrawn from a sub-seed until they are.
    key_fn may instead return a list of (scores[n,m], j) pairs: then the j
    largest scores of every row of every pair must be pairwise separated.
    With ec_gap > 0 (expert choice, key_fn returning probabilities), the
    tokens sitting at each expert's c-th / (c+1)-th boundary are redrawn
    until the boundary gap is at least ec_gap.
    """
    dt = _dt(w)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    T, D, E, F = w.T, w.D, w.E, w.F

    # x: token activations
    if w.clusters:
        # 8-cluster mixture: mu_j ~ N(0, I/2), x_t = mu_{c(t)} + N(0, I/2), c(t) uniform
        mu = _randn(gen, (w.clusters, D), math.sqrt(0.5), device)
        cid = torch.randint(0, w.clusters, (T,), generator=gen, device=device)
        x = mu[cid] + _randn(gen, (T, D), math.sqrt(0.5), device)
    else:
        x = _randn(gen, (T, D), w.x_std, device)
    Wg = _randn(gen, (E, D), w.wg_std, device)
    if w.zipf_s:
        # Zipf-scaled offset o_e = -s * ln r_e, r a seeded permutation of 1..E,
        # carried inside W_g.x through a constant feature x[:,0] = 1.
        r = torch.randperm(E, generator=gen, device=device).to(torch.float32) + 1.0
        Wg[:, 0] = -w.zipf_s * torch.log(r)
        x[:, 0] = 1.0
    bias = None
    if w.bias_std:
        bias = _randn(gen, (E,), w.bias_std, device)

    x = x.to(dt)
    Wg = Wg.to(dt)

    W_gate = W_up = W_down = None
    Ws_gate = Ws_up = Ws_down = None
    if experts:
        W_gate = _randn(gen, (E, F, D), w.w_std, device).to(dt) if w.act == "swiglu" else None
        W_up = _randn(gen, (E, F, D), w.w_std, device).to(dt)
        W_down = _randn(gen, (E, D, F), w.w_std, device).to(dt)
        if w.n_shared:
            S, Fs = w.n_shared, w.F_shared
            Ws_gate = _randn(gen, (S, Fs, D), w.w_std, device).to(dt)
            Ws_up = _randn(gen, (S, Fs, D), w.w_std, device).to(dt)
            Ws_down = _randn(gen, (S, D, Fs), w.w_std, device).to(dt)

    inp = Inputs(x, Wg, bias, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down)
    if key_fn is not None and (key_gap > 0 or ec_gap > 0):
        _separate_keys(w, inp, seed, key_fn, key_gap, ec_gap, max_rounds)
    return inp


def separate_keys(w: Workload, inp: Inputs, seed: int, key_fn, key_gap: float = 0.0,
                  ec_gap: float = 0.0, max_rounds: int = 64) -> Inputs:
    """The key-separation step of make_inputs on inputs a caller has already edited (for
    example router rows made equal on purpose, whose tied keys key_fn leaves out)."""
    if key_fn is not None and (key_gap > 0 or ec_gap > 0):
        _separate_keys(w, inp, seed, key_fn, key_gap, ec_gap, max_rounds)
    return inp


def _redraw(w, inp, rows, seed, rnd):
    """Redraw x rows `rows` (sorted) from sub-seed (seed, round)."""
    device = inp.x.device
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000003 + 7919 * (rnd + 1))
    n = len(rows)
    if w.clusters:
        mu_g = torch.Generator(device=device)
        mu_g.manual_seed(seed)
        mu = _randn(mu_g, (w.clusters, w.D), math.sqrt(0.5), device)
        cid = torch.randint(0, w.clusters, (n,), generator=g, device=device)
        new = mu[cid] + _randn(g, (n, w.D), math.sqrt(0.5), device)
    else:
        new = _randn(g, (n, w.D), w.x_std, device)
    if w.zipf_s:
        new[:, 0] = 1.0
    idx = torch.as_tensor(rows, device=device, dtype=torch.long)
    inp.x[idx] = new.to(inp.x.dtype)


def _separate_keys(w, inp, seed, key_fn, key_gap, ec_gap, max_rounds):
    import numpy as np
    Wg = inp.Wg.float().cpu().double().numpy()
    b = inp.bias.double().cpu().numpy() if inp.bias is not None else None
    keys = key_fn(inp.x.float().cpu().double().numpy(), Wg, b)
    redrawn = set()
    for rnd in range(max_rounds):
        bad = []
        if w.select == "token" and key_gap > 0:
            pairs = keys if isinstance(keys, list) else [(keys, w.k + 1)]
            worst = np.zeros(pairs[0][0].shape[0], dtype=bool)
            for sc, j in pairs:
                m = min(j, sc.shape[1])
                top = -np.sort(-sc, axis=1)[:, :m]
                gaps = top[:, :-1] - top[:, 1:]
                worst |= (gaps < key_gap).any(axis=1)
            bad = np.nonzero(worst)[0].tolist()
        elif w.select == "expert" and ec_gap > 0 and w.c < w.T:
            c = w.c
            order = np.argsort(-keys, axis=0, kind="stable")   # per expert column
            col = np.arange(w.E)
            gap = keys[order[c - 1], col] - keys[order[c], col]
            for e in np.nonzero(gap < ec_gap)[0]:
                bad.extend([int(order[c - 1, e]), int(order[c, e])])
            bad = sorted(set(bad))
        if not bad:
            inp.resampled = len(redrawn)
            return
        redrawn.update(bad)
        _redraw(w, inp, bad, seed, rnd)
        idx = torch.as_tensor(bad, dtype=torch.long, device=inp.x.device)
        new = key_fn(inp.x[idx].float().cpu().double().numpy(), Wg, b)
        if isinstance(keys, list):
            for (sc, _), (nsc, _) in zip(keys, new):
                sc[bad] = nsc
        else:
            keys[bad] = new
    raise RuntimeError(f"could not separate router keys of workload {w.name} "
                       f"in {max_rounds} rounds")
