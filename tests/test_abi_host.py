"""Host-side checks of the C ABI (no GPU): the library loads, exports every function
include/moe.h declares, sizes the grouped buffers and workspace, and rejects bad arguments
before anything is launched."""

import ctypes
import math

import pytest

import sparse_mixture_experts_warp_b200 as M
from sparse_mixture_experts_warp_b200.build import build
from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, capacity_of, rows_max


@pytest.fixture(scope="module", autouse=True)
def built():
    build()


def test_library_exports_every_declared_function():
    L = M.lib()
    names = M.header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
    assert L.moe_version().decode().startswith("moe-b200")


def test_status_strings():
    assert M.status_string(0) == "ok"
    assert "invalid" in M.status_string(1)
    assert "unsupported" in M.status_string(2)
    assert "timed out" in M.status_string(5)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_rows_capacity_workspace(name):
    w = WORKLOADS[name]
    d = M.desc_of(w)
    assert M.rows_max(d) == rows_max(w)
    assert M.capacity(d) == capacity_of(w)
    ws = M.workspace_size(d)
    es = 2 if w.dtype == "bf16" else 4
    A = rows_max(w)
    # at least x_perm + h + y
    assert ws >= A * (2 * w.D + w.F) * es
    assert M.scratch_size(d) > 0


def test_switch_capacity_is_80():
    d = M.desc_of(WORKLOADS["switch"])
    assert M.capacity(d) == 80 == math.ceil(1.25 * 8192 / 128)
    assert M.rows_max(d) == min(8192, 128 * 80)


def _bad(**kw):
    d = M.desc_of(WORKLOADS["mixtral"])
    for k, v in kw.items():
        setattr(d, k, v)
    return d


@pytest.mark.parametrize("kw,status", [
    (dict(k=0), 1), (dict(k=9), 1), (dict(D=0), 1), (dict(E=0), 1), (dict(T=-1), 1),
    (dict(score=7), 1), (dict(dtype=3), 1), (dict(E=300, k=2), 2), (dict(D=4100), 2),
    (dict(F=100), 2), (dict(overflow=1, capacity_factor=0.0), 1),
    (dict(select=1, c=0), 1), (dict(select=1, c=5000), 1), (dict(select=1, c=8, score=1), 2),
    (dict(act=3), 1),
    # group-limited selection (Mixtral: E = 8, k = 2)
    (dict(n_group=3, topk_group=1), 1),              # 3 does not divide 8
    (dict(n_group=4, topk_group=0), 1), (dict(n_group=4, topk_group=5), 1),
    (dict(n_group=8, topk_group=1), 1),              # 1 group of 1 expert < k = 2
    (dict(n_group=-1), 1), (dict(select=1, c=8, n_group=2, topk_group=1), 2),
    (dict(E=96, n_group=32, topk_group=4), 2),       # groups of 3 experts
])
def test_invalid_descriptors_are_rejected(kw, status):
    v = ctypes.c_size_t()
    assert M.lib().moe_workspace_size(ctypes.byref(_bad(**kw)), ctypes.byref(v)) == status


def test_group_limited_descriptors_are_accepted():
    v = ctypes.c_size_t()
    for kw in (dict(n_group=4, topk_group=1), dict(n_group=2, topk_group=2),
               dict(n_group=0, topk_group=0), dict(E=256, k=8, n_group=8, topk_group=4),
               dict(E=64, k=6, n_group=2, topk_group=1)):
        assert M.lib().moe_workspace_size(ctypes.byref(_bad(**kw)), ctypes.byref(v)) == 0, kw


def test_null_pointers_rejected_before_launch():
    d = M.desc_of(WORKLOADS["mixtral"])
    L = M.lib()
    st = L.moe_route(ctypes.byref(d), None, None, None, None, None, None, None, None, None, 0,
                     None)
    assert st == 1
    st = L.moe_permute(ctypes.byref(d), None, None, None, None, None, None, None, None, 0, None)
    assert st == 1
    st = L.moe_combine(ctypes.byref(d), None, None, None, None, None, None)
    assert st == 1
    st = L.moe_expert_ffn(ctypes.byref(d), 8, 14336, None, 8192, None, None, None, None, None,
                          None, None)
    assert st == 1
    st = L.moe_expert_up_ws(ctypes.byref(d), 8, 14336, None, 8192, None, None, None, None,
                            None, 0, None)
    assert st == 1
    st = L.moe_expert_down_ws(ctypes.byref(d), 8, 14336, None, 8192, None, None, None, None, 0,
                              None)
    assert st == 1
    # misaligned pointers are refused too
    st = L.moe_combine(ctypes.byref(d), 0x1001, 0x2000, 0x3000, None, 0x4000, None)
    assert st == 1


def test_scratch_holds_the_small_batch_partials():
    # the routed experts' k-split partials (at most 8 splits, fp32) fit in moe_scratch_size
    # whenever the schedule may run: A <= 256 for the down product, A <= 16 for the up product
    # (gate and up partial sets for SwiGLU, each rounded to 256 bytes), plus the alignment slack
    from sparse_mixture_experts_warp_b200.workloads import scaled
    for T in (1, 2, 8, 64, 128):
        w = scaled(WORKLOADS["mixtral"], T=T)
        d = M.desc_of(w)
        A = rows_max(w)
        need = 0
        if A <= 256:
            need = 8 * A * w.D * 4
        if A <= 16:
            one = -(-8 * A * w.F * 4 // 256) * 256
            need = max(need, 2 * one)
        assert M.scratch_size(d) >= need + 256, T
    # large batches do not pay for it
    big = M.desc_of(WORKLOADS["mixtral"])
    assert M.scratch_size(big) < 8 * 2 * 4096 * 4


def test_workspace_too_small_or_misaligned():
    d = M.desc_of(WORKLOADS["tiny"])
    need = M.workspace_size(d)
    v = M.MoeLayerViews()
    L = M.lib()
    assert L.moe_layer_views(ctypes.byref(d), 0x10000, need - 1, ctypes.byref(v)) == 3
    assert L.moe_layer_views(ctypes.byref(d), 0x10010, need, ctypes.byref(v)) == 3
    assert L.moe_layer_views(ctypes.byref(d), 0x10000, need, ctypes.byref(v)) == 0
    # views are laid out inside the workspace, 256-byte aligned, in range
    ptrs = [v.logits, v.expert_ids, v.gates, v.importance, v.entropy, v.counts, v.offsets,
            v.row_src, v.inv, v.x_perm, v.h, v.y, v.f, v.stats, v.scratch]
    for p in ptrs:
        assert 0x10000 <= p < 0x10000 + need and p % 256 == 0
    assert len(set(ptrs)) == len(ptrs)
    assert v.rows == 128


def test_header_entry_points_cite_the_pages():
    text = open(M.HEADER).read()
    for title in ("Top-k 路由", "Tiny MoE", "moe-comparison"):
        assert title in text


def test_backward_validation_before_launch():
    v = ctypes.c_size_t()
    L = M.lib()
    # bf16 and fp32 layers: token choice or expert choice, with or without shared experts
    for kw, st in ((dict(dtype=0), 0), (dict(select=1, c=8), 0), (dict(n_shared=1, F_shared=64), 0),
                   (dict(k=0), 1), (dict(E=300, k=2), 2)):
        assert L.moe_backward_workspace_size(ctypes.byref(_bad(**kw)), ctypes.byref(v)) == st, kw
    # shared experts need moe_layer_backward_ex's weights (moe_layer_backward passes none) and
    # the plain forward (moe_layer_forward_train does not run them)
    sh = _bad(n_shared=1, F_shared=64)
    p = 0x10000
    assert L.moe_layer_backward(ctypes.byref(sh), p, p, p, p, p, p, 1.0, p, 1 << 30, p, p, p, p,
                                p, p, 1 << 30, 0, None) == 1
    assert L.moe_layer_forward_train(ctypes.byref(sh), p, p, None, p, p, p, p, p, 1 << 30, p,
                                     1 << 30, None) == 2
    d = M.desc_of(WORKLOADS["mixtral"])
    assert L.moe_backward_workspace_size(ctypes.byref(d), ctypes.byref(v)) == 0
    assert v.value > 0
    # null pointers and unknown flags are rejected before anything is launched
    st = L.moe_layer_backward(ctypes.byref(d), None, None, None, None, None, None, 1.0, None, 0,
                              None, None, None, None, None, None, 0, 0, None)
    assert st in (1, 3)
    st = L.moe_layer_forward_train(ctypes.byref(d), None, None, None, None, None, None, None,
                                   None, 0, None, 0, None)
    assert st == 3                     # MOE_ERR_WORKSPACE: no backward workspace


def test_empty_batch_returns_before_any_launch():
    # T = 0: argument checks only, no kernel is enqueued (the pointers are never dereferenced)
    from sparse_mixture_experts_warp_b200.workloads import scaled
    w = scaled(WORKLOADS["mixtral"], T=0)
    d = M.desc_of(w)
    assert M.rows_max(d) == 0
    need = M.workspace_size(d)
    L = M.lib()
    n0 = L.moe_kernel_launches()
    st = L.moe_layer_forward(ctypes.byref(d), 0x1000, 0x2000, None, 0x3000, 0x4000, 0x5000, None,
                             None, None, 0x6000, 0x10000, need, None)
    assert st == 0
    st = L.moe_route(ctypes.byref(d), 0x1000, 0x2000, None, 0x3000, 0x4000, None, None, None,
                     0x10000, M.scratch_size(d), None)
    assert st == 0
    st = L.moe_combine(ctypes.byref(d), 0x1000, 0x2000, 0x3000, None, 0x4000, None)
    assert st == 0
    assert L.moe_kernel_launches() == n0
    # the workspace check still applies
    assert L.moe_layer_forward(ctypes.byref(d), 0x1000, 0x2000, None, 0x3000, 0x4000, 0x5000,
                               None, None, None, 0x6000, 0x10000, need - 1, None) == 3
