"""Python binding of the sm_100a sparse MoE FFN layer (include/moe.h).

Argument marshalling only: every step of the layer runs in the CUDA library libmoe.so.
PyTorch supplies device memory and the stream.  There is no fallback: if the library is
missing, every call raises.

The functions keep the C names (moe_route, moe_permute, moe_expert_up, moe_expert_down,
moe_expert_ffn, moe_expert_up_ws, moe_expert_down_ws, moe_combine, moe_balance_stats,
moe_layer_forward) and take torch tensors.
"""

from __future__ import annotations

import ctypes
import os
import re

import torch

__all__ = [
    "MoeDesc", "MoeStats", "MoeLayerViews", "MoeError", "lib", "library_path", "desc_of",
    "header_functions", "status_string", "rows_max", "capacity", "scratch_size",
    "workspace_size", "layer_views", "moe_route", "moe_permute", "moe_expert_up",
    "moe_expert_down", "moe_expert_ffn", "moe_expert_up_ws", "moe_expert_down_ws",
    "moe_permute_noalloc", "moe_combine", "moe_balance_stats", "moe_layer_backward_ex",
    "moe_expert_up_gather", "gather_fusion",
    "MoeBwdShared",
    "moe_layer_forward", "get_device_error", "empty_scratch", "empty_workspace",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_PKG)
HEADER = os.path.join(_ROOT, "include", "moe.h")

SOFTMAX, SIGMOID = 0, 1
TOKEN_CHOICE, EXPERT_CHOICE = 0, 1
RENORM, RAW = 0, 1
DROPLESS, CAPACITY_DROP = 0, 1
SWIGLU, RELU, GELU = 0, 1, 2
F32, BF16 = 0, 1


class MoeDesc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("D", ctypes.c_int32), ("E", ctypes.c_int32),
                ("F", ctypes.c_int32), ("k", ctypes.c_int32), ("c", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("F_shared", ctypes.c_int32),
                ("score", ctypes.c_int32), ("select", ctypes.c_int32), ("gate", ctypes.c_int32),
                ("overflow", ctypes.c_int32), ("act", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("aux_alpha", ctypes.c_float),
                ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32)]


class MoeStats(ctypes.Structure):
    _fields_ = [("aux", ctypes.c_float), ("max_over_mean", ctypes.c_float),
                ("n_routes", ctypes.c_int32), ("n_kept", ctypes.c_int32),
                ("n_dropped", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("entropy", ctypes.c_float), ("count_p95", ctypes.c_float),
                ("count_p99", ctypes.c_float), ("reserved2", ctypes.c_float)]


class MoeLayerViews(ctypes.Structure):
    _fields_ = [("expert_ids", ctypes.c_void_p), ("gates", ctypes.c_void_p),
                ("logits", ctypes.c_void_p), ("importance", ctypes.c_void_p),
                ("entropy", ctypes.c_void_p),
                ("counts", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
                ("row_src", ctypes.c_void_p), ("inv", ctypes.c_void_p),
                ("x_perm", ctypes.c_void_p), ("h", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("y_shared", ctypes.c_void_p), ("h_shared", ctypes.c_void_p),
                ("shared_offsets", ctypes.c_void_p), ("f", ctypes.c_void_p),
                ("stats", ctypes.c_void_p), ("scratch", ctypes.c_void_p),
                ("scratch_bytes", ctypes.c_size_t), ("rows", ctypes.c_int64)]


class MoeBwdShared(ctypes.Structure):
    _fields_ = [("Ws_gate", ctypes.c_void_p), ("Ws_up", ctypes.c_void_p),
                ("Ws_down", ctypes.c_void_p), ("dWs_gate", ctypes.c_void_p),
                ("dWs_up", ctypes.c_void_p), ("dWs_down", ctypes.c_void_p)]


class MoeError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} (status {status})")


_LIB = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_DP = ctypes.POINTER(MoeDesc)

_SIGS = {
    "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "moe_version": ([], ctypes.c_char_p),
    "moe_rows_max": ([_DP, ctypes.POINTER(_I64)], ctypes.c_int),
    "moe_capacity": ([_DP, ctypes.POINTER(_I32)], ctypes.c_int),
    "moe_scratch_size": ([_DP, ctypes.POINTER(_SZ)], ctypes.c_int),
    "moe_workspace_size": ([_DP, ctypes.POINTER(_SZ)], ctypes.c_int),
    "moe_layer_views": ([_DP, _P, _SZ, ctypes.POINTER(MoeLayerViews)], ctypes.c_int),
    "moe_route": ([_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_permute": ([_DP, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_permute_noalloc": ([_DP, _P, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_expert_up": ([_DP, _I32, _I32, _P, _I64, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_expert_down": ([_DP, _I32, _I32, _P, _I64, _P, _P, _P, _P], ctypes.c_int),
    "moe_expert_ffn": ([_DP, _I32, _I32, _P, _I64, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_expert_up_gather": ([_DP, _I32, _I32, _P, _P, _I64, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_gather_fusion": ([_DP, ctypes.POINTER(_I32)], ctypes.c_int),
    "moe_expert_up_ws": ([_DP, _I32, _I32, _P, _I64, _P, _P, _P, _P, _P, _SZ, _P],
                         ctypes.c_int),
    "moe_expert_down_ws": ([_DP, _I32, _I32, _P, _I64, _P, _P, _P, _P, _SZ, _P], ctypes.c_int),
    "moe_combine": ([_DP, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_balance_stats": ([_DP, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_layer_forward": ([_DP, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P],
                          ctypes.c_int),
    "moe_backward_workspace_size": ([_DP, ctypes.POINTER(_SZ)], ctypes.c_int),
    "moe_layer_backward": ([_DP, _P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _SZ, _P, _P, _P,
                            _P, _P, _P, _SZ, _I32, _P], ctypes.c_int),
    "moe_layer_backward_ex": ([_DP, _P, _P, _P, _P, _P, ctypes.POINTER(MoeBwdShared), _P,
                               ctypes.c_float, _P, _SZ, _P, _P, _P, _P, _P, _P, _SZ, _I32, _P],
                              ctypes.c_int),
    "moe_layer_forward_train": ([_DP, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _SZ, _P],
                                ctypes.c_int),
    "moe_get_device_error": ([_P, ctypes.POINTER(_I32)], ctypes.c_int),
    "moe_debug_inject": ([_I32], ctypes.c_int),
    "moe_kernel_launches": ([], ctypes.c_int64),
}


def library_path() -> str:
    return os.path.join(_PKG, "libmoe.so")


def lib():
    """Loads libmoe.so (built in-tree by sparse_mixture_experts_warp_b200.build)."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"the CUDA library {path} is not built; run "
                               "`python -m sparse_mixture_experts_warp_b200.build`")
        L = ctypes.CDLL(path)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = L
    return _LIB


def header_functions(path: str = HEADER):
    """Names of the functions include/moe.h declares."""
    with open(path) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def _check(fn: str, status: int):
    if status != 0:
        raise MoeError(fn, status)


def desc_of(w, T=None) -> MoeDesc:
    """moe_desc_t of a workload (sparse_mixture_experts_warp_b200.workloads.Workload)."""
    return MoeDesc(
        T=w.T if T is None else T, D=w.D, E=w.E, F=w.F, k=w.k, c=w.c,
        n_shared=w.n_shared, F_shared=w.F_shared,
        score=SOFTMAX if w.score == "softmax" else SIGMOID,
        select=TOKEN_CHOICE if w.select == "token" else EXPERT_CHOICE,
        gate=RENORM if w.gate == "renorm" else RAW,
        overflow=DROPLESS if w.overflow == "dropless" else CAPACITY_DROP,
        act={"swiglu": SWIGLU, "relu": RELU, "gelu": GELU}[w.act],
        dtype=BF16 if w.dtype == "bf16" else F32,
        capacity_factor=w.capacity_factor, aux_alpha=w.aux_alpha,
        n_group=getattr(w, "n_group", 1), topk_group=getattr(w, "topk_group", 1))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors handed to the MoE library must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def rows_max(d: MoeDesc) -> int:
    v = _I64()
    _check("moe_rows_max", lib().moe_rows_max(ctypes.byref(d), ctypes.byref(v)))
    return v.value


def capacity(d: MoeDesc) -> int:
    v = _I32()
    _check("moe_capacity", lib().moe_capacity(ctypes.byref(d), ctypes.byref(v)))
    return v.value


def scratch_size(d: MoeDesc) -> int:
    v = _SZ()
    _check("moe_scratch_size", lib().moe_scratch_size(ctypes.byref(d), ctypes.byref(v)))
    return v.value


def workspace_size(d: MoeDesc) -> int:
    v = _SZ()
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(d), ctypes.byref(v)))
    return v.value


def empty_scratch(d: MoeDesc, device="cuda"):
    return torch.empty(scratch_size(d), dtype=torch.uint8, device=device)


def empty_workspace(d: MoeDesc, device="cuda"):
    return torch.empty(workspace_size(d), dtype=torch.uint8, device=device)


def layer_views(d: MoeDesc, ws: torch.Tensor) -> dict:
    """Torch views of the intermediates inside a moe_layer_forward workspace."""
    v = MoeLayerViews()
    _check("moe_layer_views", lib().moe_layer_views(ctypes.byref(d), _ptr(ws), ws.numel(),
                                                    ctypes.byref(v)))
    base = ws.data_ptr()
    dt = torch.bfloat16 if d.dtype == BF16 else torch.float32
    ec = d.select == EXPERT_CHOICE
    K = d.E if ec else d.k
    A = v.rows

    def view(addr, dtype, shape):
        if not addr:
            return None
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        off = addr - base
        return ws[off:off + nbytes].view(dtype).view(*shape)

    out = dict(
        expert_ids=view(v.expert_ids, torch.int32, (d.E, d.c) if ec else (d.T, K)),
        gates=view(v.gates, torch.float32, (d.T, K)),
        logits=view(v.logits, torch.float32, (d.T, d.E)),
        importance=view(v.importance, torch.float32, (d.E,)),
        entropy=view(v.entropy, torch.float32, (1,)),
        counts=view(v.counts, torch.int32, (d.E,)),
        offsets=view(v.offsets, torch.int32, (d.E + 1,)),
        row_src=view(v.row_src, torch.int32, (A,)),
        inv=view(v.inv, torch.int32, (d.T, K)),
        x_perm=view(v.x_perm, dt, (A, d.D)),
        h=view(v.h, dt, (A, d.F)),
        y=view(v.y, dt, (A, d.D)),
        y_shared=view(v.y_shared, dt, (d.n_shared, d.T, d.D)) if d.n_shared else None,
        f=view(v.f, torch.float32, (d.E,)),
        stats=view(v.stats, torch.uint8, (ctypes.sizeof(MoeStats),)),
        scratch=view(v.scratch, torch.uint8, (v.scratch_bytes,)),
        rows=A,
    )
    return out


def stats_of(raw: torch.Tensor) -> dict:
    """Decodes a moe_stats_t held in a uint8 tensor (device or host)."""
    b = bytes(raw.cpu().numpy().tobytes())
    s = MoeStats.from_buffer_copy(b)
    return dict(aux=s.aux, max_over_mean=s.max_over_mean, n_routes=s.n_routes,
                n_kept=s.n_kept, n_dropped=s.n_dropped, entropy=s.entropy,
                count_p95=s.count_p95, count_p99=s.count_p99)


# ---------------------------------------------------------------- steps ----

def moe_route(d, x, Wg, sel_bias, expert_ids, gates, logits=None, importance=None,
              scratch=None, stream=None, entropy=None):
    scratch = empty_scratch(d, x.device) if scratch is None else scratch
    _check("moe_route", lib().moe_route(
        ctypes.byref(d), _ptr(x), _ptr(Wg), _ptr(sel_bias), _ptr(expert_ids), _ptr(gates),
        _ptr(logits), _ptr(importance), _ptr(entropy), _ptr(scratch), scratch.numel(),
        _stream(stream)))


def moe_permute(d, expert_ids, x, x_perm, counts, offsets, row_src, inv, scratch=None,
                stream=None):
    scratch = empty_scratch(d, x.device) if scratch is None else scratch
    _check("moe_permute", lib().moe_permute(
        ctypes.byref(d), _ptr(expert_ids), _ptr(x), _ptr(x_perm), _ptr(counts), _ptr(offsets),
        _ptr(row_src), _ptr(inv), _ptr(scratch), scratch.numel(), _stream(stream)))


def moe_permute_noalloc(d, expert_ids, x, x_perm, counts, offsets, row_src, inv, stream=None):
    """moe_permute for callers that cannot allocate: its scratch is a fixed device array inside
    the library (see include/moe.h)."""
    _check("moe_permute_noalloc", lib().moe_permute_noalloc(
        ctypes.byref(d), _ptr(expert_ids), _ptr(x), _ptr(x_perm), _ptr(counts), _ptr(offsets),
        _ptr(row_src), _ptr(inv), _stream(stream)))


def moe_expert_up(d, n_groups, F, a, offsets, W_gate, W_up, h, stream=None):
    _check("moe_expert_up", lib().moe_expert_up(
        ctypes.byref(d), n_groups, F, _ptr(a), a.shape[0], _ptr(offsets), _ptr(W_gate),
        _ptr(W_up), _ptr(h), _stream(stream)))


def moe_expert_up_gather(d, n_groups, F, x, row_src, a_rows, offsets, W_gate, W_up, h,
                         stream=None):
    """moe_expert_up reading its rows from the tokens x through row_src (no x_perm)."""
    _check("moe_expert_up_gather", lib().moe_expert_up_gather(
        ctypes.byref(d), n_groups, F, _ptr(x), _ptr(row_src), int(a_rows), _ptr(offsets),
        _ptr(W_gate), _ptr(W_up), _ptr(h), _stream(stream)))


def gather_fusion(d: MoeDesc) -> bool:
    """Whether moe_layer_forward gathers the token rows inside the up projection."""
    v = _I32()
    _check("moe_gather_fusion", lib().moe_gather_fusion(ctypes.byref(d), ctypes.byref(v)))
    return bool(v.value)


def moe_expert_down(d, n_groups, F, h, offsets, W_down, y, stream=None):
    _check("moe_expert_down", lib().moe_expert_down(
        ctypes.byref(d), n_groups, F, _ptr(h), h.shape[0], _ptr(offsets), _ptr(W_down), _ptr(y),
        _stream(stream)))


def moe_expert_ffn(d, n_groups, F, a, offsets, W_gate, W_up, W_down, h, y, stream=None):
    _check("moe_expert_ffn", lib().moe_expert_ffn(
        ctypes.byref(d), n_groups, F, _ptr(a), a.shape[0], _ptr(offsets), _ptr(W_gate),
        _ptr(W_up), _ptr(W_down), _ptr(h), _ptr(y), _stream(stream)))


def moe_expert_up_ws(d, n_groups, F, a, offsets, W_gate, W_up, h, scratch, stream=None):
    _check("moe_expert_up_ws", lib().moe_expert_up_ws(
        ctypes.byref(d), n_groups, F, _ptr(a), a.shape[0], _ptr(offsets), _ptr(W_gate),
        _ptr(W_up), _ptr(h), _ptr(scratch), 0 if scratch is None else scratch.numel(),
        _stream(stream)))


def moe_expert_down_ws(d, n_groups, F, h, offsets, W_down, y, scratch, stream=None):
    _check("moe_expert_down_ws", lib().moe_expert_down_ws(
        ctypes.byref(d), n_groups, F, _ptr(h), h.shape[0], _ptr(offsets), _ptr(W_down), _ptr(y),
        _ptr(scratch), 0 if scratch is None else scratch.numel(), _stream(stream)))


def moe_combine(d, y, inv, gates, y_shared, out, stream=None):
    _check("moe_combine", lib().moe_combine(
        ctypes.byref(d), _ptr(y), _ptr(inv), _ptr(gates), _ptr(y_shared), _ptr(out),
        _stream(stream)))


def moe_balance_stats(d, counts, offsets, importance, f, stats, stream=None, entropy=None):
    _check("moe_balance_stats", lib().moe_balance_stats(
        ctypes.byref(d), _ptr(counts), _ptr(offsets), _ptr(importance), _ptr(entropy), _ptr(f),
        _ptr(stats), _stream(stream)))


def moe_layer_forward(d, x, Wg, sel_bias, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, out,
                      ws, stream=None):
    _check("moe_layer_forward", lib().moe_layer_forward(
        ctypes.byref(d), _ptr(x), _ptr(Wg), _ptr(sel_bias), _ptr(W_gate), _ptr(W_up),
        _ptr(W_down), _ptr(Ws_gate), _ptr(Ws_up), _ptr(Ws_down), _ptr(out), _ptr(ws),
        ws.numel(), _stream(stream)))


def backward_workspace_size(d: MoeDesc) -> int:
    n = _SZ()
    _check("moe_backward_workspace_size",
           lib().moe_backward_workspace_size(ctypes.byref(d), ctypes.byref(n)))
    return n.value


def empty_backward_workspace(d: MoeDesc, device="cuda"):
    return torch.empty(backward_workspace_size(d), dtype=torch.uint8, device=device)


BWD_PREACT_SAVED = 1


def moe_layer_backward(d, x, Wg, W_gate, W_up, W_down, dout, aux_grad, fwd_ws, dx, dWg, dW_gate,
                       dW_up, dW_down, bwd_ws, stream=None, flags=0):
    _check("moe_layer_backward", lib().moe_layer_backward(
        ctypes.byref(d), _ptr(x), _ptr(Wg), _ptr(W_gate), _ptr(W_up), _ptr(W_down), _ptr(dout),
        float(aux_grad), _ptr(fwd_ws), fwd_ws.numel(), _ptr(dx), _ptr(dWg), _ptr(dW_gate),
        _ptr(dW_up), _ptr(dW_down), _ptr(bwd_ws), bwd_ws.numel(), int(flags), _stream(stream)))


def moe_layer_backward_ex(d, x, Wg, W_gate, W_up, W_down, shared, dout, aux_grad, fwd_ws, dx,
                          dWg, dW_gate, dW_up, dW_down, bwd_ws, stream=None, flags=0):
    """moe_layer_backward for any layer; `shared` = (Ws_gate, Ws_up, Ws_down, dWs_gate, dWs_up,
    dWs_down) tensors, or None without shared experts."""
    sh = None
    if shared is not None:
        sh = MoeBwdShared(*[_ptr(t) for t in shared])
    _check("moe_layer_backward_ex", lib().moe_layer_backward_ex(
        ctypes.byref(d), _ptr(x), _ptr(Wg), _ptr(W_gate), _ptr(W_up), _ptr(W_down),
        ctypes.byref(sh) if sh is not None else None, _ptr(dout), float(aux_grad), _ptr(fwd_ws),
        fwd_ws.numel(), _ptr(dx), _ptr(dWg), _ptr(dW_gate), _ptr(dW_up), _ptr(dW_down),
        _ptr(bwd_ws), bwd_ws.numel(), int(flags), _stream(stream)))


def moe_layer_forward_train(d, x, Wg, sel_bias, W_gate, W_up, W_down, out, ws, bwd_ws,
                            stream=None):
    _check("moe_layer_forward_train", lib().moe_layer_forward_train(
        ctypes.byref(d), _ptr(x), _ptr(Wg), _ptr(sel_bias), _ptr(W_gate), _ptr(W_up),
        _ptr(W_down), _ptr(out), _ptr(ws), ws.numel(), _ptr(bwd_ws), bwd_ws.numel(),
        _stream(stream)))


def get_device_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the raw device error word."""
    code = _I32()
    lib().moe_get_device_error(_stream(stream), ctypes.byref(code))
    return code.value


def device_error_status(stream=None):
    """(moe_status_t, raw word) of moe_get_device_error."""
    code = _I32()
    st = lib().moe_get_device_error(_stream(stream), ctypes.byref(code))
    return st, code.value


def kernel_launches() -> int:
    """Kernels the library has enqueued since it was loaded."""
    return int(lib().moe_kernel_launches())


def debug_inject(fault: int):
    """Test hook of the bounded device waits (see moe_debug_inject in include/moe.h)."""
    _check("moe_debug_inject", lib().moe_debug_inject(fault))
