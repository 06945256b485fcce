"""Parity of the CUDA layer with the CPU oracle (through the C ABI, on cuda:0).

Small cases run the whole oracle and compare every output element; they are sized to span
several 128-row GEMM tiles, more than one 1024-assignment permute block, and ragged tails.
The full-size workloads (Mixtral, Switch, DeepSeek-V3, expert choice) compare the routing and
permutation of the whole batch bit-exactly, the router logits of every token, and a sample of
output rows that the oracle evaluates one by one.
"""

import numpy as np
import pytest
import torch

from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, scaled
import moe_check as C
import sparse_mixture_experts_warp_b200 as M

pytestmark = pytest.mark.gpu

W = WORKLOADS
SMALL = {
    "tiny": W["tiny"],
    "tiny_T1": scaled(W["tiny"], T=1),
    "tiny_T37": scaled(W["tiny"], T=37),
    "tiny_k_eq_E": scaled(W["tiny"], T=50, k=4),
    "f32_relu_drop": scaled(W["switch"], dtype="f32", T=300, D=32, E=8, F=48, zipf_s=1.1,
                            w_std=0.15, wg_std=0.15),
    "f32_sigmoid_shared": scaled(W["v3"], dtype="f32", T=90, D=64, E=16, F=32, k=3,
                                 n_shared=2, F_shared=40, w_std=0.1, wg_std=0.1),
    "f32_expert_choice": scaled(W["ec"], dtype="f32", T=120, D=32, E=6, F=24, c=30, clusters=4,
                                w_std=0.2, wg_std=0.2),
    "mixtral_small": scaled(W["mixtral"], T=700, D=512, F=1024),
    "switch_small": scaled(W["switch"], T=3000, D=256, E=16, F=512),
    "v3_small": scaled(W["v3"], T=300, D=512, E=64, F=256, F_shared=256),
    "ec_small": scaled(W["ec"], T=1000, D=256, E=16, F=256, c=125),
    # router shapes.  By default bf16 with E <= 8 and D = 256 * NW (4 <= NW <= 16) runs the
    # mma.sync router and the rest the tensor-core router; in subprocesses below the router
    # cases also run through the tensor-core router (MOE_ROUTER=tc), the mma.sync router
    # (MOE_ROUTER=fast), the grouped-GEMM router product (E % 32 == 0: MOE_ROUTER=gemm) and
    # the CUDA-core router (MOE_ROUTER=simt).  E <= 8, ragged token counts
    "router_E8_T1": scaled(W["mixtral"], T=1, D=4096, F=256),
    "router_E8_T37": scaled(W["mixtral"], T=37, D=1024, F=256),
    "router_E6_T300": scaled(W["mixtral"], T=300, D=2048, E=6, F=256),
    "router_E8_switch_k1": scaled(W["switch"], T=500, D=1024, E=8, F=256),
    "router_E8_sigmoid_shared": scaled(W["v3"], T=200, D=1024, E=8, k=2, F=256, F_shared=256),
    # E >= 32: ragged T, one to four k-ranges per 128-token tile
    "router_E32_switch": scaled(W["switch"], T=300, D=256, E=32, F=256),
    "router_E64_v3": scaled(W["v3"], T=97, D=1024, E=64, k=6, F=256, F_shared=256),
    "router_E64_ec": scaled(W["ec"], T=777, D=512, E=64, F=256, c=50),
    # tensor-core router: E not a multiple of 16 (N = 48 of which 40 live, 64 TMEM columns;
    # 8 tiles, 4 k-ranges of 3 k-blocks), one k-range per tile over more tiles than SMs, and
    # expert choice over 256 experts (the largest E with the DeepSeek-V3 group limit is
    # groups_E256_v3_node below)
    "router_E40_T1000": scaled(W["switch"], T=1000, D=768, E=40, F=128, capacity_factor=2.0),
    "groups_E256_v3_node": scaled(W["v3"], T=130, D=1024, F=128, F_shared=128, n_group=8,
                                  topk_group=4),
    "router_E16_T20000": scaled(W["mixtral"], T=20000, D=128, E=16, k=2, F=64),
    "router_E256_ec": scaled(W["ec"], T=600, D=512, E=256, F=128, c=10),
    # three k-blocks: a cluster of three CTAs, one k-block each; E = 24 (N = 32, 24 live)
    "router_E24_ks3": scaled(W["mixtral"], T=130, D=192, E=24, k=3, F=128),
    # the classic D -> F -> D expert with GELU (bf16 tensor-core epilogue, fp32 CUDA cores)
    "gelu_bf16": scaled(W["switch"], act="gelu", T=500, D=256, E=16, F=512, overflow="dropless",
                        gate="renorm", k=2, zipf_s=0.0),
    "gelu_f32": scaled(W["tiny"], act="gelu", T=40),
    # degenerate and extreme shapes: one expert (the layer is the dense FFN, every gate 1), the
    # largest top-k (k = 32 of 64 experts: tensor-core router, 32 arg-max rounds, the general
    # combine), and the smallest bf16 widths (D = F = 64: one k-block, 64 live features in a
    # 128-feature SwiGLU tile)
    "single_expert_E1": scaled(W["mixtral"], T=100, D=256, E=1, k=1, F=256),
    "max_k32": scaled(W["mixtral"], T=64, D=256, E=64, k=32, F=128),
    "bf16_D64_F64": scaled(W["mixtral"], T=50, D=64, F=64),
    # more than 65536 assignments: the multi-block permute path
    "large_A": scaled(W["mixtral"], T=33000, D=128, F=128),
    # group-limited selection: fast router (groups of 2 experts, softmax; groups of 2, sigmoid
    # with selection bias), generic fp32 router (groups of 4), tensor-core router (groups of
    # 32 = one register slot, and of 64 = two slots)
    "groups_E8_softmax": scaled(W["mixtral"], T=300, D=1024, E=8, k=2, F=256, n_group=4,
                                  topk_group=1),
    "groups_E8_sigmoid": scaled(W["v3"], T=200, D=1024, E=8, k=3, F=256, F_shared=256,
                                  n_group=4, topk_group=2),
    "groups_f32_generic": scaled(W["v3"], dtype="f32", T=90, D=64, E=16, F=32, k=3,
                                 n_shared=1, F_shared=40, w_std=0.1, wg_std=0.1, n_group=4,
                                 topk_group=2),
    "groups_E64_size32": scaled(W["v3"], T=300, D=512, E=64, F=256, F_shared=256,
                                    n_group=2, topk_group=1),
    "groups_E128_size64": scaled(W["v3"], T=300, D=512, E=128, k=4, F=256, F_shared=256,
                                    n_group=2, topk_group=1),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_layer_matches_oracle(name):
    w = SMALL[name]
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    C.check_logits(w, inp, v)
    ref = C.check_routing(w, inp, v)
    C.check_full_output(w, inp, out, ref)


def test_layer_is_deterministic():
    w = SMALL["mixtral_small"]
    inp = C.inputs_for(w)
    out1, v1 = C.run_layer(w, inp)
    o1, rs1 = out1.clone(), v1["row_src"].clone()
    out2, v2 = C.run_layer(w, inp)
    assert torch.equal(o1, out2)
    assert torch.equal(rs1, v2["row_src"])


@pytest.mark.parametrize("name", ["mixtral_small", "switch_small", "v3_small", "ec_small",
                                  "router_E8_T1"])
def test_layer_statistics_equal_the_statistics_entry_point(name):
    """moe_layer_forward computes the balance statistics in the combine's first block; they equal,
    bit for bit, what moe_balance_stats computes from the same counts, offsets, importance and
    entropy."""
    w = SMALL[name]
    inp = C.inputs_for(w)
    _, v = C.run_layer(w, inp)
    d = M.desc_of(w)
    f = torch.full_like(v["f"], float("nan"))
    stats = torch.zeros_like(v["stats"])
    M.moe_balance_stats(d, v["counts"], v["offsets"], v["importance"], f, stats,
                        entropy=v["entropy"])
    torch.cuda.synchronize()
    assert torch.equal(f, v["f"])
    assert torch.equal(stats, v["stats"])


def test_capacity_drops_give_zero_rows():
    w = SMALL["switch_small"]
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    inv = v["inv"].cpu().numpy().reshape(-1)
    dropped = np.nonzero(inv < 0)[0]
    assert len(dropped) > 0
    assert torch.all(out[torch.as_tensor(dropped, device=out.device)] == 0)
    counts = v["counts"].cpu().numpy()
    assert counts.sum() == w.T * w.k


def test_expert_choice_every_expert_gets_c():
    w = SMALL["ec_small"]
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    assert np.all(v["counts"].cpu().numpy() == w.c)
    picked = v["expert_ids"].cpu().numpy()
    assert np.all(np.diff(picked, axis=1) > 0)         # ascending token order per expert
    unpicked = sorted(set(range(w.T)) - set(picked.reshape(-1).tolist()))
    if unpicked:
        assert torch.all(out[torch.as_tensor(unpicked, device=out.device)] == 0)


FULL = ["mixtral", "switch", "v3", "ec"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    """The whole batch's routing and permutation bit-exact, every logit within its bound, and
    a tile-stratified output sample: one executed row from every 32-row slice of every expert
    (every expert x 256-row tile x 128-row MMA half x TMEM lane quarter) plus each expert's
    last row, checked on its expert output and on its token's layer output."""
    w = W[name]
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    C.check_logits(w, inp, v)
    ref = C.check_routing(w, inp, v)
    # include rows the method zeroes, when there are any
    extra = []
    if w.select == "expert":
        picked = set(ref["ids"].reshape(-1).tolist())
        extra = [t for t in range(w.T) if t not in picked][:4]
    elif w.overflow == "drop":
        extra = np.nonzero(ref["inv"] < 0)[0][:4].tolist()   # k = 1: assignment == token
    nrows, ntok, _, _ = C.check_stratified_output(w, inp, out, v, extra_tokens=extra)
    assert nrows >= int(np.count_nonzero(ref["kept"])) and ntok > 0


# small-T (decode) regime at the full Mixtral layer shape: a few rows per expert, every weight
# tile streamed for them; all tokens are checked against the oracle
@pytest.mark.parametrize("T", [1, 8, 64, 200])
def test_decode_regime_mixtral_shape(T):
    w = scaled(W["mixtral"], T=T)
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    C.check_logits(w, inp, v)
    C.check_routing(w, inp, v)
    C.check_sampled_output(w, inp, out, v, list(range(T)))


# mid-size batches at the full Mixtral layer shape: ~256 and ~512 rows per expert, where the
# down projection takes the 128-row tiles (whole waves of CTAs) and the up projection the
# 256-row tiles at 2048 tokens; routing bit-exact, a tile-stratified output sample
@pytest.mark.parametrize("T", [1024, 2048])
def test_mid_size_mixtral_shape(T):
    w = scaled(W["mixtral"], T=T)
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    C.check_logits(w, inp, v)
    C.check_routing(w, inp, v)
    nrows, ntok, _, _ = C.check_stratified_output(w, inp, out, v, seed=125)
    assert nrows > 0 and ntok > 0


# A few executed rows (bf16) take the k-split expert schedule: fp32 partials of the up and down
# products summed by splitk.cu.  ReLU at the full Switch layer with its capacity limit (up split
# 3, down split 8) and GELU (splits 4 and 2); SwiGLU is covered by router_E8_T1 (up split 7)
# and T = 1 above (up 2, down 4).  Every token against the oracle, which evaluates only the
# experts in use.
DECODE = {
    "switch_relu_T2": scaled(W["switch"], T=2),
    "gelu_T3": scaled(W["switch"], act="gelu", T=3, D=1024, E=16, F=512, overflow="dropless",
                      gate="renorm", k=2, zipf_s=0.0),
}


@pytest.mark.parametrize("name", list(DECODE))
def test_decode_split_schedule(name):
    w = DECODE[name]
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    C.check_logits(w, inp, v)
    C.check_routing(w, inp, v)
    C.check_sampled_output(w, inp, out, v, list(range(w.T)))


def test_decode_without_streamk_in_subprocess():
    """MOE_STREAMK=0: split products whose equal k-ranges take more than one wave of SMs keep
    them (by default they run stream-K: equal shares of all tiles' k-blocks per SM); the decode
    cases pass both ways."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, MOE_STREAMK="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__, "-k",
                        "(decode or router_E8_T1) and not in_subprocess"], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout, r.stdout[-3000:]


def test_decode_split_schedule_matches_fused_path_in_subprocess():
    """MOE_DECODE_SPLITK=0 keeps the fused grouped GEMMs at every size; the decode cases pass
    there too."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, MOE_DECODE_SPLITK="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__, "-k",
                        "decode_split_schedule and not subprocess or decode_regime and 1]"],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


# The E = 8 router at larger token counts.  Tensor-core router: 40 to 94 tiles, 1 to 3
# k-ranges, a ragged last tile.  mma.sync router (MOE_ROUTER=fast): each CTA routes several
# 16-token batches, the last one ragged (T=5000, D=4096: 34 tokens per CTA; T=9000, D=1024:
# 61; T=12000, D=4096: 82).  Logits of every token, the whole routing, permutation and
# statistics are compared with the oracle.
@pytest.mark.parametrize("T,D", [(5000, 4096), (9000, 1024), (12000, 4096)])
def test_router_many_batches(T, D):
    w = scaled(W["mixtral"], T=T, D=D, F=256)
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    C.check_logits(w, inp, v)
    C.check_routing(w, inp, v)



# Group-limited routing: every token's experts lie in at most topk_group groups, and the full
# DeepSeek-V3 node shape (256 experts on 8 groups, top-8 on at most 4) matches the oracle.
@pytest.mark.parametrize("name", [n for n in SMALL if n.startswith("groups_")])
def test_group_limit_spans_at_most_topk_group_groups(name):
    w = SMALL[name]
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    ids = v["expert_ids"].cpu().numpy()
    size = w.E // w.n_group
    assert max(len(set(row)) for row in (ids // size).tolist()) <= w.topk_group


def test_v3_node_limited_full_size():
    w = scaled(W["v3"], n_group=8, topk_group=4)
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    C.check_logits(w, inp, v)
    ref = C.check_routing(w, inp, v)
    groups = ref["ids"] // 32
    assert max(len(set(row)) for row in groups.tolist()) <= 4
    # every expert that received rows: one row from one of its 32-row slices, and its last row
    C.check_stratified_output(w, inp, out, v, seed=124, every_slice=False)


def test_layer_with_gather_fusion_in_subprocess():
    """MOE_GATHER_FUSION=1 makes moe_layer_forward gather the token rows inside the up
    projection (the permutation writes indices only, x_perm stays unwritten); the small-case
    parity tests pass there too."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, MOE_GATHER_FUSION="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__, "-k",
                        "small_layer_matches_oracle"], env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


@pytest.mark.parametrize("name", ["mixtral_small", "switch_small", "v3_small", "ec_small"])
def test_gathering_up_projection_matches_the_permuted_one(name):
    """moe_permute without x_perm + moe_expert_up_gather gives the same h, bit for bit, as
    moe_permute with x_perm + moe_expert_up (the same products in the same k order; only the
    way the A rows reach shared memory differs), and moe_permute's x_perm rows are the tokens'."""
    w = SMALL[name]
    inp = C.inputs_for(w)
    out, v = C.run_layer(w, inp)
    d = M.desc_of(w)
    A = M.rows_max(d)
    x_perm = torch.empty(A, w.D, dtype=inp.x.dtype, device="cuda")
    M.moe_permute(d, v["expert_ids"], inp.x, x_perm, v["counts"], v["offsets"], v["row_src"],
                  v["inv"])
    n = int(v["offsets"][-1].item())
    K = w.E if w.select == "expert" else w.k
    tok = (v["row_src"][:n] // K).long()
    assert torch.equal(x_perm[:n], inp.x[tok])
    h1 = torch.zeros(A, w.F, dtype=inp.x.dtype, device="cuda")
    h2 = torch.zeros(A, w.F, dtype=inp.x.dtype, device="cuda")
    M.moe_expert_up(d, w.E, w.F, x_perm, v["offsets"], inp.W_gate, inp.W_up, h1)
    M.moe_expert_up_gather(d, w.E, w.F, inp.x, v["row_src"], A, v["offsets"], inp.W_gate,
                           inp.W_up, h2)
    torch.cuda.synchronize()
    assert M.get_device_error() == 0
    assert torch.equal(h1[:n], h2[:n])


# The router paths other than the default tensor-core router, each on the router cases it
# can take (MOE_ROUTER is read once per process).
ROUTER_MODES = {
    "tc": "router_E8 or router_E6_ or groups_E8 or router_many_batches or single_expert",
    "fast": "router_E8 or router_E6_ or groups_E8 or router_many_batches",
    "gemm": "router_E32 or router_E64 or router_E256 or groups_E64 or groups_E128 or groups_E256",
    "simt": "router_E8_T37 or router_E6_ or router_E64_v3 or router_E40 or groups_E64 or "
            "router_E256_ec or groups_E256",
}


@pytest.mark.parametrize("mode", list(ROUTER_MODES))
def test_other_router_paths_in_subprocess(mode):
    import os
    import subprocess
    import sys
    env = dict(os.environ, MOE_ROUTER=mode)
    sel = f"(small_layer_matches_oracle or router_many_batches) and ({ROUTER_MODES[mode]})"
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__, "-k", sel],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout, r.stdout[-3000:]


def test_switch_layer_without_adaptive_split_in_subprocess():
    """MOE_ADAPTIVE_SPLIT=0: the down projection of capacity-limited layers writes bf16 directly
    whatever its tile count (by default the grouped GEMM splits K on the device when the
    executed rows leave most SMs idle, as in the Switch layer); the Switch cases pass both
    ways."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, MOE_ADAPTIVE_SPLIT="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__, "-k",
                        "(small_layer_matches_oracle or full_size_workload or capacity_drops) "
                        "and (switch or f32_relu_drop or router_E40)"],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout, r.stdout[-3000:]


def test_layer_with_weights_as_m_tiles_in_subprocess():
    """MOE_GEMM_SWAP=1 runs every expert product of the layer (bf16, inference) on the
    weights-as-M tiles instead of the row tiles: token tiles of up to 256 rows with N rounded to
    16, gathered or tiled token loads; the layer cases pass there too."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, MOE_GEMM_SWAP="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__, "-k",
                        "small_layer_matches_oracle or full_size_workload or decode_regime or "
                        "gathering_up_projection or v3_node_limited"],
                       env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout, r.stdout[-3000:]


def test_permutation_without_cluster_kernel_in_subprocess():
    """MOE_PERMUTE_CLUSTER=0: between 2048 and 65536 assignments the permutation indexes with the
    one-CTA kernel (up to 8192) or the three-kernel histogram path instead of one cluster of up
    to 8 CTAs; the cases in that range pass both ways."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, MOE_PERMUTE_CLUSTER="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__, "-k",
                        "(small_layer_matches_oracle or full_size_workload or capacity_drops) "
                        "and (switch or v3 or router_E16_T20000 or router_E40 or groups_E64 or "
                        "groups_E128 or router_E256_ec)"],
                       env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout, r.stdout[-3000:]


def test_layer_without_programmatic_dependent_launch_in_subprocess():
    """MOE_PDL=0 launches every kernel without programmatic stream serialization (each waits
    for the previous one to finish before it is scheduled); the small-case parity tests pass
    there too."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, MOE_PDL="0")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", __file__, "-k",
                        "small_layer_matches_oracle or full_size_workload and mixtral"],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
