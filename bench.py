"""Throughput of the sparse MoE FFN layer forward pass on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixtral] [--impl cuda|reference]
                    [--tokens T] [--ffn F] [--no-graph] [--no-backward] [--no-cpu-baseline]

A step is one pass of the whole layer -- route, permute, expert up (gate/up + SiLU*up),
expert down, combine, balance statistics -- over one batch of synthetic tokens of the
Mixtral-8x7B layer shape (T=4096, D=4096, E=8, top-2, SwiGLU F=14336, bf16), with inputs and
weights resident in HBM.  The step calls the library's step entry points in the order
moe_layer_forward chains them, with CUDA events between them for the per-kernel times.
`e2e` times the public moe_layer_forward call with the step's tokens copied in from pinned
host memory and the layer output copied back, every step.

Multi-GPU: the layer does not shard (one GPU, no collectives); `--gpus N` under torchrun runs
N independent replicas, one per GPU, each on its own batch; value = all ranks' tokens / the
slowest rank's time (weak scaling).

`--impl reference` times the CPU oracle (fp64) on the host cores on bounded samples of the
same workload: each step routes the whole batch and evaluates a sample of its tokens.

After the forward, the same graph is replayed for about a second ("sustained": the clock the
1 kW power cap settles at, the GPU's joules per step from the NVML energy counter and the
expert GEMMs' TFLOP per joule), and a training step (moe_layer_forward_train + moe_layer_backward)
is timed, reported under "backward" (`--no-backward` skips it).  At one GPU the other layer
shapes the pages name -- Switch top-1, DeepSeek-V3, expert choice at the DeepSeekMoE-16B shape
and a one-token Mixtral decode step -- are then timed for a few graph-replayed steps each and
reported under "per_workload", each with its dominant stage and the fraction of its roofline.  `--tokens` and `--ffn` shrink the
batch or the expert width for profiling cases and the small-batch (decode) regime; the DRAM
traffic figure is then null (it is taken from an ncu capture of the full-size workload only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from sparse_mixture_experts_warp_b200.workloads import WORKLOADS, make_inputs, scaled  # noqa: E402

METRIC = "MoE-layer tokens/s at Mixtral-8x7B shape; % of tensor-core / HBM roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "grouped_gemm_traffic.json")
GEMM_SRC = os.path.join(ROOT, "sparse_mixture_experts_warp_b200", "csrc", "gemm_sm100.cu")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
STAGES = ["route", "permute", "expert_up", "expert_down", "combine", "stats"]
# "expert_down" includes the shared experts (both projections) when the workload has them.


# ------------------------------------------------------------------ helpers ----

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return ({k: float(p[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")},
                "measured")
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def file_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def load_traffic(workload, w):
    """DRAM bytes per launch of the gate/up grouped GEMM from a committed ncu capture of the
    full-size workload; null once the kernel source has changed since the capture, and for a
    shape that differs from the captured one (--tokens / --ffn overrides)."""
    if w != WORKLOADS.get(workload):
        return None
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        if t.get("kernel_sha") != file_sha(GEMM_SRC):
            return None
        return t.get("bytes_per_launch", {}).get(workload)
    except Exception:
        return None


class ClockSampler:
    """Samples the SM clock and clock-event reasons of one GPU in a thread (NVML, every 5 ms)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.error = None
        self._e0 = self._e1 = None     # NVML total energy (mJ) at start and end
        self._t0 = self._t1 = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - no NVML
            self.error = str(e)
            return self
        try:
            self._e0 = self._nvml.nvmlDeviceGetTotalEnergyConsumption(self._h)
            self._t0 = time.time()
        except Exception:  # pragma: no cover - no energy counter
            self._e0 = None
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def _run(self):
        p = self._nvml
        get_reasons = getattr(p, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(p, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(p.nvmlDeviceGetClockInfo(self._h, p.NVML_CLOCK_SM))
                r = get_reasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception as e:  # pragma: no cover
                self.error = str(e)
            self._stop.wait(0.005)

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()
        if self._e0 is not None:
            try:
                self._e1 = self._nvml.nvmlDeviceGetTotalEnergyConsumption(self._h)
                self._t1 = time.time()
            except Exception:  # pragma: no cover
                self._e1 = None

    def energy_j(self):
        """Joules the GPU drew while the sampler ran (NVML energy counter), or None."""
        if self._e0 is None or self._e1 is None:
            return None
        return (self._e1 - self._e0) / 1000.0

    def summary(self):
        med = statistics.median(self.samples) if self.samples else None
        out = {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
               "samples": len(self.samples)}
        e = self.energy_j()
        # the counter advances in steps: only a run of half a second or more gives a mean power
        if e is not None and e > 0 and self._t1 and self._t1 - self._t0 >= 0.5:
            out["avg_w"] = round(e / (self._t1 - self._t0), 1)
        if self.error:
            out["error"] = self.error
        return out

    def rejected(self):
        if self.reasons & {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}:
            return True
        s = self.summary()
        if s["sm_mhz"] and s["sm_max_mhz"] and not self.reasons:
            return s["sm_mhz"] < 0.7 * s["sm_max_mhz"]        # a leftover clock lock
        return False


def barrier(world):
    """Barrier across the replicas (no-op for one process)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device):
    """The largest value of x over all ranks (timings: the slowest replica sets the time)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank, world, steps, max_total_ms):
    """Whole-job tokens/s: every replica's tokens over the slowest replica's time."""
    return tokens_per_rank * world * steps / (max_total_ms / 1e3)


def stage_work(w, rows_exec, gather=False):
    """Algorithmic bytes (HBM-bound stages) or FLOPs (GEMMs) per launch; rows_exec = A_exec.
    With the gathering up projection the permutation moves indices only."""
    es = 2 if w.dtype == "bf16" else 4
    T, D, E, F = w.T, w.D, w.E, w.F
    K = w.E if w.select == "expert" else w.k
    A = rows_exec
    n_up = 2 if w.act == "swiglu" else 1
    return {
        # x and W_g read once; logits, ids and gates written
        "route": ("hbm", T * D * es + E * D * es + T * E * 4 + T * K * 8),
        # ids read; x read once; x_perm written; row_src and inv written
        "permute": ("hbm", T * K * 4 + (0 if gather else T * D * es + A * D * es) + A * 4
                    + T * K * 4),
        "expert_up": ("tensor", 2.0 * A * D * F * n_up),
        "expert_down": ("tensor", 2.0 * A * F * D + w.n_shared * 2.0 * T * D * w.F_shared * 3),
        # expert rows read once; out written once; inv and gates read
        "combine": ("hbm", A * D * es + (1 + w.n_shared) * T * D * es + T * K * 8),
        "stats": ("hbm", E * 16),
    }


def gemm_hbm_bytes(w, rows_exec, active_experts=None):
    """Bytes the expert GEMMs must move at least: the weights of every expert that has rows,
    once, the grouped rows in and out of each projection (x_perm read, h written and read, y
    written) and the shared experts' weights and activations."""
    es = 2 if w.dtype == "bf16" else 4
    n_up = 2 if w.act == "swiglu" else 1
    n_active = w.E if active_experts is None else active_experts
    weights = n_active * (n_up + 1) * w.F * w.D * es
    acts = rows_exec * (w.D + 2 * w.F + w.D) * es
    shared = w.n_shared * (3 * w.F_shared * w.D + w.T * (w.D + 2 * w.F_shared + w.D)) * es
    return weights + acts + shared


def workload_of(args):
    w = WORKLOADS[args.workload]
    if args.tokens:
        w = scaled(w, T=args.tokens)
    if getattr(args, "ffn", 0):
        w = scaled(w, F=args.ffn, description=w.description + f" (expert width F={args.ffn})")
    return w


# -------------------------------------------------------------- CUDA arm ----

def e2e_pipelined(M, d, inp, ws, stream, dev, steps, warmup, world):
    """Times `steps` calls of moe_layer_forward through host buffers.

    Returns (pipelined_ms, serial_ms).  Pipelined: step i's H2D copy (its own pinned host
    buffer) runs on a copy-in stream, the layer on `stream`, the D2H copy of its output on a
    copy-out stream; two device buffers of x and of out alternate, with events ordering each
    reuse.  Serial: the same copies and call back to back on one stream.
    """
    n_buf = 2
    x_host = [inp.x.cpu().pin_memory() for _ in range(n_buf)]
    out_host = [torch.empty(inp.x.shape, dtype=inp.x.dtype).pin_memory() for _ in range(n_buf)]
    x_dev = [torch.empty_like(inp.x) for _ in range(n_buf)]
    out_dev = [torch.empty_like(inp.x) for _ in range(n_buf)]
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=False)   # noqa: E731
    in_done = [ev() for _ in range(n_buf)]
    comp_done = [ev() for _ in range(n_buf)]
    out_done = [ev() for _ in range(n_buf)]

    def call(xd, od, st):
        M.moe_layer_forward(d, xd, inp.Wg, inp.bias, inp.W_gate, inp.W_up, inp.W_down,
                            inp.Ws_gate, inp.Ws_up, inp.Ws_down, od, ws, st)

    def pipelined(n, t0=None, t1=None):
        for i in range(n):
            b = i % n_buf
            with torch.cuda.stream(s_in):
                if i >= n_buf:
                    s_in.wait_event(comp_done[b])            # x_dev[b] no longer read
                if i == 0 and t0 is not None:
                    t0.record(s_in)
                x_dev[b].copy_(x_host[b], non_blocking=True)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if i >= n_buf:
                stream.wait_event(out_done[b])               # out_dev[b] already copied out
            call(x_dev[b], out_dev[b], stream)
            comp_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[b])
                out_host[b].copy_(out_dev[b], non_blocking=True)
                out_done[b].record(s_out)
                if i == n - 1 and t1 is not None:
                    t1.record(s_out)

    pipelined(warmup)
    torch.cuda.synchronize(dev)
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pipelined(steps, t0, t1)
    torch.cuda.synchronize(dev)
    barrier(world)
    pipelined_ms = t0.elapsed_time(t1)

    # the serial form, for reference
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(steps):
        x_dev[0].copy_(x_host[0], non_blocking=True)
        call(x_dev[0], out_dev[0], stream)
        out_host[0].copy_(out_dev[0], non_blocking=True)
    s1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    return pipelined_ms, s0.elapsed_time(s1)


def time_backward(M, w, d, inp, ws, stream, dev, steps, warmup, tc_peak, world):
    """Training step: moe_layer_forward_train (saves the expert pre-activations) then
    moe_layer_backward with the selection fixed.  Reports the backward's device time per call,
    its GEMM FLOPs (dgrad and wgrad: 2x the up and down projections) and their rate against the
    tensor peak, and the time of the whole forward + backward step."""
    bws = M.empty_backward_workspace(d, dev)
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    dout = torch.randn(w.T, w.D, generator=g, device=dev).to(torch.bfloat16)
    dx = torch.empty_like(inp.x)
    f32 = dict(dtype=torch.float32, device=dev)
    dWg = torch.empty(w.E, w.D, **f32)
    dWgate = torch.empty(w.E, w.F, w.D, **f32) if w.act == "swiglu" else None
    dWup = torch.empty(w.E, w.F, w.D, **f32)
    dWdown = torch.empty(w.E, w.D, w.F, **f32)

    out = torch.empty_like(inp.x)

    def fwd():
        M.moe_layer_forward_train(d, inp.x, inp.Wg, inp.bias, inp.W_gate, inp.W_up, inp.W_down,
                                  out, ws, bws, stream)

    def bwd():
        M.moe_layer_backward(d, inp.x, inp.Wg, inp.W_gate, inp.W_up, inp.W_down, dout, 1.0, ws,
                             dx, dWg, dWgate, dWup, dWdown, bws, stream,
                             flags=M.BWD_PREACT_SAVED)

    for _ in range(warmup):
        fwd()
        bwd()
    barrier(world)
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        fwd()
        ev[2 * i + 1].record(stream)
        bwd()
        ev[2 * i + 2].record(stream)
    torch.cuda.synchronize(dev)
    f_ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(steps)) / steps
    b_ms = sum(ev[2 * i + 1].elapsed_time(ev[2 * i + 2]) for i in range(steps)) / steps
    ms = max_over_ranks(b_ms, world, dev)
    train_ms = max_over_ranks(f_ms + b_ms, world, dev)
    rows = int(M.layer_views(d, ws)["offsets"][-1].item())
    n_up = 2 if w.act == "swiglu" else 1
    up, down = 2.0 * rows * w.D * w.F * n_up, 2.0 * rows * w.F * w.D
    flops = 2 * up + 2 * down          # dgrad and wgrad of both projections
    tf = flops / (ms * 1e-3) / 1e12
    return {"ms_per_step": round(ms, 4), "tokens_per_s": round(w.T * world / (ms * 1e-3), 1),
            "gemm_tflop_per_step": round(flops / 1e12, 3), "tflops": round(tf, 1),
            "frac_of_tensor_peak": round(tf / tc_peak, 3), "steps": steps,
            "train_step_ms": round(train_ms, 4),
            "train_tokens_per_s": round(w.T * world / (train_ms * 1e-3), 1),
            "what": "moe_layer_forward_train (saves the expert pre-activations) then "
                    "moe_layer_backward: dx, dW_g, dW_gate/up/down (fp32) with the selection "
                    "fixed; dout ~ N(0,1) bf16; ms_per_step is the backward alone"}


class LayerStep:
    """One step of the layer: `layer` is one moe_layer_forward call (the headline graph);
    calling the object runs the library's step entry points in the order moe_layer_forward
    chains them, with optional CUDA events between the stages (the eager and per-stage
    times)."""

    def __init__(self, M, w, inp, dev, stream):
        self.M, self.w, self.inp, self.dev, self.stream = M, w, inp, dev, stream
        self.d = M.desc_of(w)
        self.ws = M.empty_workspace(self.d, dev)
        self.v = M.layer_views(self.d, self.ws)
        self.out = torch.empty_like(inp.x)
        if w.n_shared:
            # shared experts: one group over all T tokens, SwiGLU of width F_shared
            self.d_sh = M.desc_of(w)
            self.d_sh.act = M.SWIGLU
            self.sh_off = torch.tensor([0, w.T], dtype=torch.int32, device=dev)
            self.h_sh = torch.empty(w.T, w.F_shared, dtype=inp.x.dtype, device=dev)
        self.graph, self.graph_launches, self.graph_error = None, 0, None
        # as in moe_layer_forward: with enough rows the up projection gathers the token rows
        # itself and the permutation writes indices only
        self.gather = M.gather_fusion(self.d)

    def layer(self, st=None):
        """The whole layer as one moe_layer_forward call."""
        M, w, inp = self.M, self.w, self.inp
        s = st if st is not None else self.stream
        sh = (inp.Ws_gate, inp.Ws_up, inp.Ws_down) if w.n_shared else (None, None, None)
        M.moe_layer_forward(self.d, inp.x, inp.Wg, inp.bias, inp.W_gate, inp.W_up, inp.W_down,
                            *sh, self.out, self.ws, s)

    def __call__(self, ev=None, st=None):
        M, w, inp, v = self.M, self.w, self.inp, self.v
        d, scratch = self.d, v["scratch"]
        s = st if st is not None else self.stream
        M.moe_route(d, inp.x, inp.Wg, inp.bias, v["expert_ids"], v["gates"], v["logits"],
                    v["importance"], scratch, s, entropy=v["entropy"])
        if ev is not None:
            ev[1].record(s)
        M.moe_permute(d, v["expert_ids"], inp.x, None if self.gather else v["x_perm"],
                      v["counts"], v["offsets"], v["row_src"], v["inv"], scratch, s)
        if ev is not None:
            ev[2].record(s)
        # (with a few executed rows the routed experts' products take the k-split schedule, its
        # partials in the step scratch, as in moe_layer_forward)
        if self.gather:
            M.moe_expert_up_gather(d, w.E, w.F, inp.x, v["row_src"], v["rows"], v["offsets"],
                                   inp.W_gate, inp.W_up, v["h"], s)
        else:
            M.moe_expert_up_ws(d, w.E, w.F, v["x_perm"], v["offsets"], inp.W_gate, inp.W_up,
                               v["h"], scratch, s)
        if ev is not None:
            ev[3].record(s)
        M.moe_expert_down_ws(d, w.E, w.F, v["h"], v["offsets"], inp.W_down, v["y"], scratch, s)
        for i in range(w.n_shared):
            M.moe_expert_ffn(self.d_sh, 1, w.F_shared, inp.x, self.sh_off, inp.Ws_gate[i],
                             inp.Ws_up[i], inp.Ws_down[i], self.h_sh, v["y_shared"][i], s)
        if ev is not None:
            ev[4].record(s)
        M.moe_combine(d, v["y"], v["inv"], v["gates"], v["y_shared"] if w.n_shared else None,
                      self.out, s)
        if ev is not None:
            ev[5].record(s)
        M.moe_balance_stats(d, v["counts"], v["offsets"], v["importance"], v["f"], v["stats"],
                            s, entropy=v["entropy"])
        if ev is not None:
            ev[6].record(s)

    def capture(self, warmup):
        """The layer (one moe_layer_forward call) captured once in a CUDA graph (the library
        allocates and synchronises nothing, so its calls capture as they are); replays remove
        the host launch gaps."""
        M, dev = self.M, self.dev
        try:
            cap = torch.cuda.Stream(dev)
            cap.wait_stream(self.stream)
            g = torch.cuda.CUDAGraph()
            n0 = M.kernel_launches()
            with torch.cuda.graph(g, stream=cap):
                self.layer(st=cap)
            self.graph_launches = M.kernel_launches() - n0
            self.stream.wait_stream(cap)
            for _ in range(max(warmup, 3)):
                g.replay()
            torch.cuda.synchronize(dev)
            self.graph = g
        except Exception as e:          # capture not possible here: time the eager calls
            self.graph_error = str(e).splitlines()[0][:200]

    def staged_times(self, steps):
        """Per-stage device times from replays of a second graph of the step that holds event
        record nodes between the stages (no host launch gaps); None if that capture fails."""
        M, dev = self.M, self.dev
        try:
            evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(7)]
            cap = torch.cuda.Stream(dev)
            cap.wait_stream(self.stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                evs[0].record(cap)
                self(evs, st=cap)
            self.stream.wait_stream(cap)
            g.replay()
            torch.cuda.synchronize(dev)
            acc = {s: 0.0 for s in STAGES}
            for _ in range(steps):
                g.replay()
                torch.cuda.synchronize(dev)
                for j, s in enumerate(STAGES):
                    acc[s] += evs[j].elapsed_time(evs[j + 1])
            del g
            return {s: acc[s] / steps for s in STAGES}
        except Exception:
            return None

    def timed(self, steps, use_graph, nvml_index, world):
        """(total ms, per-stage ms or None, clock sampler, kernel launches) of `steps` steps."""
        M, dev, stream = self.M, self.dev, self.stream
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(steps)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize(dev)
        with ClockSampler(nvml_index) as clk:
            n0 = M.kernel_launches()
            start.record(stream)
            for i in range(steps):
                if use_graph:
                    self.graph.replay()
                else:
                    evs[i][0].record(stream)
                    self(evs[i])
            end.record(stream)
            launches = self.graph_launches * steps if use_graph else M.kernel_launches() - n0
            torch.cuda.synchronize(dev)
        barrier(world)
        total = start.elapsed_time(end)
        if use_graph:
            return total, None, clk, launches
        per_stage = {s: 0.0 for s in STAGES}
        for i in range(steps):
            for j, s in enumerate(STAGES):
                per_stage[s] += evs[i][j].elapsed_time(evs[i][j + 1])
        return total, {s: per_stage[s] / steps for s in STAGES}, clk, launches

    def release(self):
        self.graph = None
        self.ws = self.v = self.out = None


def stage_rooflines(w, per_stage, rows_exec, active, peaks, tc_peak, gather=False):
    """Per stage: achieved rate and the fraction of its own roofline time (GEMM stages: the
    slower of FLOPs at the tensor peak and weight + activation bytes at the HBM peak; the
    others: bytes at the HBM peak), plus the whole layer's roofline."""
    work = stage_work(w, rows_exec, gather)
    es = 2 if w.dtype == "bf16" else 4
    n_up = 2 if w.act == "swiglu" else 1
    gemm_bytes = {
        "expert_up": active * n_up * w.F * w.D * es + rows_exec * (w.D + w.F) * es,
        "expert_down": active * w.F * w.D * es + rows_exec * (w.F + w.D) * es
        + w.n_shared * (3 * w.F_shared * w.D + w.T * (w.D + 2 * w.F_shared + w.D)) * es,
    }
    hbm = peaks["hbm_gbs"] * 1e9
    stages = {}
    for s in STAGES:
        kind, amount = work[s]
        t = per_stage[s] * 1e-3
        if kind == "tensor":
            roof = max(amount / (tc_peak * 1e12), gemm_bytes[s] / hbm)
            bound = "tensor" if amount / (tc_peak * 1e12) >= gemm_bytes[s] / hbm else "hbm"
            ach = amount / t / 1e12
            stages[s] = {"us": round(per_stage[s] * 1e3, 2), "tflops": round(ach, 1),
                         "gbs": round(gemm_bytes[s] / t / 1e9, 1), "bound": bound,
                         "frac": round(ach / tc_peak, 3), "roof_frac": round(roof / t, 3)}
        else:
            ach = amount / t / 1e9
            stages[s] = {"us": round(per_stage[s] * 1e3, 2), "gbs": round(ach, 1),
                         "bound": "hbm", "frac": round(ach / peaks["hbm_gbs"], 3),
                         "roof_frac": round(amount / hbm / t, 3)}
    gemm_flops = work["expert_up"][1] + work["expert_down"][1]
    hbm_bytes = sum(work[s][1] for s in ("route", "permute", "combine", "stats"))
    gemm_roof_s = max(gemm_flops / (tc_peak * 1e12),
                      gemm_hbm_bytes(w, rows_exec, active) / hbm)
    layer_roof_s = gemm_roof_s + hbm_bytes / hbm
    return stages, work, gemm_flops, layer_roof_s


def rows_and_active(v):
    offs = v["offsets"].cpu()
    return int(offs[-1].item()), int(((offs[1:] - offs[:-1]) > 0).sum().item())


def measure_workload(M, w, seed, dev, stream, steps, warmup, nvml_index, peaks):
    """A shorter measurement of another workload shape (graph replays for the step time,
    eager calls for the stage times), reported beside the headline."""
    inp = make_inputs(w, seed=seed, device=dev)
    st = LayerStep(M, w, inp, dev, stream)
    for _ in range(warmup):
        st()
    torch.cuda.synchronize(dev)
    st.capture(warmup)
    use_graph = st.graph is not None
    total, _, clk, launches = st.timed(steps, use_graph, nvml_index, 1)
    eager_total, per_stage, _, _ = st.timed(steps, False, nvml_index, 1)
    staged = st.staged_times(steps) if use_graph else None
    if staged is not None:
        per_stage = staged
    err = M.get_device_error(stream)
    if err:
        raise RuntimeError(f"device error word {err:#x} ({w.name})")
    ms = (total if use_graph else eager_total) / steps
    tc_key = "bf16_tflops_sustained" if "sw_power_cap" in clk.reasons else "bf16_tflops"
    rows_exec, active = rows_and_active(st.v)
    stages, work, gemm_flops, layer_roof_s = stage_rooflines(w, per_stage, rows_exec, active,
                                                             peaks, peaks[tc_key], st.gather)
    top = max(STAGES, key=lambda s: per_stage[s])
    res = {
        "shape": w.description, "T": w.T, "ms_per_step": round(ms, 4),
        "tokens_per_s": round(w.T / (ms * 1e-3), 1), "steps": steps,
        "timing": "CUDA-graph replay" if use_graph else "eager calls",
        "stage_timing": "graph replays, event nodes between stages" if staged is not None
        else "eager calls, events between stages",
        "rows_executed": rows_exec, "active_experts": active, "gather_fusion": st.gather,
        "dominant": {"stage": top, **stages[top]},
        "layer_frac_of_roofline": round(layer_roof_s / (ms * 1e-3), 3),
        "layer_roofline_ms": round(layer_roof_s * 1e3, 4),
        "stages": stages, "tc_peak": tc_key, "clocks": clk.summary(),
    }
    st.release()
    del inp
    torch.cuda.empty_cache()
    return res


# the other layer shapes timed beside the headline (name, batch override)
PER_WORKLOAD = [("switch", None), ("v3", None), ("ec", None), ("mixtral_T1", 1)]


def run_cuda(args, rank, world, local):
    import sparse_mixture_experts_warp_b200 as M

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = workload_of(args)
    inp = make_inputs(w, seed=rank, device=dev)
    stream = torch.cuda.current_stream(dev)
    step = LayerStep(M, w, inp, dev, stream)
    d, ws, v = step.d, step.ws, step.v

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if not args.no_graph:
        step.capture(args.warmup)
    nvml_index = local if "CUDA_VISIBLE_DEVICES" not in os.environ else \
        int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])

    # the headline from graph replays (timed first), per-stage times from the eager calls
    # (events between stages)
    use_graph = step.graph is not None
    total_ms, per_stage, clk, launches = step.timed(args.steps, use_graph, nvml_index, world)
    remeasured = False
    if clk.rejected():
        total_ms, per_stage, clk, launches = step.timed(args.steps, use_graph, nvml_index, world)
        remeasured = True
    if use_graph:
        eager_ms, eager_stage, _, _ = step.timed(args.steps, False, nvml_index, world)
        graph_stage = step.staged_times(args.steps)
        per_stage = graph_stage if graph_stage is not None else eager_stage
    else:
        eager_ms, eager_stage, graph_stage = total_ms, per_stage, None
    total_ms = max_over_ranks(total_ms, world, dev)
    eager_ms = max_over_ranks(eager_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(w.T, world, args.steps, total_ms)

    # sustained: the same graph replayed for about a second, where the 1 kW power cap sets the
    # clock, reported beside the headline
    sustained = None
    if use_graph and not args.no_sustained:
        n_sus = max(args.steps, int(math.ceil(1000.0 / max(ms_per_step, 1e-3))))
        sus_ms, _, sus_clk, _ = step.timed(n_sus, True, nvml_index, world)
        sus_ms = max_over_ranks(sus_ms, world, dev)
        sustained = {"steps": n_sus, "ms_per_step": round(sus_ms / n_sus, 4),
                     "value": round(job_throughput(w.T, world, n_sus, sus_ms), 1),
                     "clocks": sus_clk.summary()}
        e = sus_clk.energy_j()
        if e is not None and e > 0:
            # the GPU's energy over the replay (this rank's GPU), per step
            sustained["joules_per_step"] = round(e / n_sus, 4)

    # e2e: the public call with host buffers; every step copies its own tokens in from pinned
    # host memory and its output back, inside the timed region.  Copies run on their own
    # streams, double-buffered, so step i's copies overlap the compute of steps i-1 and i+1.
    e2e_ms, e2e_serial_ms = e2e_pipelined(M, d, inp, ws, stream, dev, args.steps, args.warmup,
                                          world)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    e2e_serial_ms = max_over_ranks(e2e_serial_ms, world, dev)
    e2e_value = job_throughput(w.T, world, args.steps, e2e_ms)
    x_bytes = inp.x.numel() * inp.x.element_size()
    err = M.get_device_error(stream)
    if err:
        raise RuntimeError(f"device error word {err:#x}")

    # roofline of the dominant kernel (gate/up grouped GEMM launch)
    rows_exec, active = rows_and_active(v)
    peaks, peaks_kind = load_peaks()
    power_capped = "sw_power_cap" in clk.reasons
    tc_key = "bf16_tflops_sustained" if power_capped else "bf16_tflops"
    tc_peak = peaks[tc_key]
    stages, work, gemm_flops, layer_roof_s = stage_rooflines(w, per_stage, rows_exec, active,
                                                             peaks, tc_peak, step.gather)
    up_flops = work["expert_up"][1]
    if sustained and sustained.get("joules_per_step"):
        sustained["gemm_tflop_per_joule"] = round(gemm_flops / 1e12 / sustained["joules_per_step"], 3)
    achieved = up_flops / (per_stage["expert_up"] * 1e-3) / 1e12
    gemm_tflops = gemm_flops / ((per_stage["expert_up"] + per_stage["expert_down"]) * 1e-3) / 1e12
    roofline = {
        "bound": "tensor",
        "kernel": "grouped_gemm_kernel<EPI_SWIGLU> (expert up: gate+up, SiLU*up epilogue)",
        "achieved": round(achieved, 1), "peak": tc_peak, "unit": "TFLOP/s",
        "frac": round(achieved / tc_peak, 3),
        "traffic": load_traffic(args.workload, w),
        "peak_source": f"{peaks_kind} {tc_key} (MEASURED_PEAKS.json)",
        "flops_per_launch": up_flops,
        "grouped_gemm_up_down_tflops": round(gemm_tflops, 1),
        "layer_frac_of_roofline": round(layer_roof_s / (ms_per_step * 1e-3), 3),
        "layer_roofline_ms": round(layer_roof_s * 1e3, 4),
    }
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) weights, random-init)",
        "config": {"workload": w.name, "shape": w.description, "T": w.T,
                   "D": w.D, "E": w.E, "k": w.k, "F": w.F, "tokens_per_step": w.T * world,
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "rows_executed": rows_exec, "gather_fusion": step.gather,
                   "l2": "inputs larger than L2: %.2f GB of expert weights stream per step"
                         % ((w.E * 3 * w.F * w.D * 2) / 1e9)},
        "roofline": roofline, "stages": stages,
        "stage_timing": ("graph replays with event record nodes between the stages"
                         if graph_stage is not None else "eager calls, events between stages")
                        + "; each stage is its step entry point (moe_layer_forward computes the"
                          " statistics inside the combine's launch and, under a capacity"
                          " limit, sums the down projection's k-split there too)",
        "eager_stage_us": {s: round(eager_stage[s] * 1e3, 2) for s in STAGES},
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                "ms_per_step": round(e2e_ms / args.steps, 4),
                "h2d_bytes_per_step": x_bytes, "d2h_bytes_per_step": x_bytes,
                "pipelined": "copy-in, compute and copy-out on three streams, double-buffered",
                "serial_value": round(job_throughput(w.T, world, args.steps, e2e_serial_ms), 1)},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "timing": ("CUDA-graph replay of one moe_layer_forward call (%d library kernels per "
                   "step); per-stage times from the step entry points" % step.graph_launches)
                  if use_graph else
                  ("eager calls" + (" (graph capture failed: %s)" % step.graph_error
                                    if step.graph_error else "")),
        "eager_value": round(job_throughput(w.T, world, args.steps, eager_ms), 1),
    }
    if sustained:
        res["sustained"] = sustained
    if remeasured:
        res["clocks"]["remeasured"] = True
    if (not args.no_backward and w.dtype == "bf16" and w.select == "token"
            and not w.n_shared):
        res["backward"] = time_backward(M, w, d, inp, ws, stream, dev, min(args.steps, 20),
                                        max(args.warmup, 3), tc_peak, world)
    step.release()
    del inp
    torch.cuda.empty_cache()
    if world == 1 and not args.no_per_workload and args.workload == "mixtral" \
            and not args.tokens and not args.ffn:
        per = {}
        for name, T in PER_WORKLOAD:
            wk = WORKLOADS[name.split("_")[0]]
            if T:
                wk = scaled(wk, T=T)
            per[name] = measure_workload(M, wk, rank, dev, stream, min(args.steps, 20), 3,
                                         nvml_index, peaks)
        res["per_workload"] = per
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        w_cpu = workload_of(args)
        inp_cpu = make_inputs(w_cpu, seed=rank, device=dev)
        res["cpu_baseline"] = cpu_baseline(w_cpu, inp_cpu, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(res), flush=True)


# ---------------------------------------------------------- oracle arm ----

def _host_inputs(inp):
    """The workload's tensors copied to host memory once (bf16/fp32 as generated)."""
    def h(t):
        return None if t is None else t.cpu()
    return dict(x=h(inp.x), Wg=h(inp.Wg), bias=h(inp.bias), W_gate=h(inp.W_gate),
                W_up=h(inp.W_up), W_down=h(inp.W_down), Ws_gate=h(inp.Ws_gate),
                Ws_up=h(inp.Ws_up), Ws_down=h(inp.Ws_down))


def oracle_step(w, host, tokens):
    """One bounded oracle step: route the whole batch, evaluate the sampled tokens."""
    from oracle import moe_oracle as O

    def f64(t):
        return None if t is None else t.float().double().numpy()

    def weights_of(e):
        g = f64(host["W_gate"][e]) if host["W_gate"] is not None else None
        return g, f64(host["W_up"][e]), f64(host["W_down"][e])

    wd = dict(T=w.T, D=w.D, E=w.E, F=w.F, k=w.k, c=w.c, score=w.score, select=w.select,
              gate=w.gate, overflow=w.overflow, capacity_factor=w.capacity_factor, act=w.act,
              n_shared=w.n_shared, F_shared=w.F_shared, aux_alpha=w.aux_alpha)
    r = O.layer_forward_rows(wd, tokens, f64(host["x"]), f64(host["Wg"]), f64(host["bias"]),
                             None, None, None, f64(host["Ws_gate"]), f64(host["Ws_up"]),
                             f64(host["Ws_down"]), weights_of=weights_of)
    return r["out_rows"]


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(w, inp, budget_s=15.0, sample=128):
    import numpy as np
    host = _host_inputs(inp)
    rng = np.random.default_rng(0)
    done, reps, t0 = 0, 0, time.perf_counter()
    while True:
        tokens = sorted(rng.choice(w.T, size=sample, replace=False).tolist())
        oracle_step(w, host, tokens)
        done += len(tokens)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(done / dt, 2), "unit": "tokens/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{reps} x {sample} random tokens of one {w.name} batch (T={w.T}); each "
                      f"repetition routes the whole batch and evaluates the sampled tokens' "
                      f"experts in fp64 ({dt:.1f} s of CPU work)"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import numpy as np
    w = workload_of(args)
    device = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(w, seed=0, device=device)
    host = _host_inputs(inp)
    del inp
    if device == "cuda":
        torch.cuda.empty_cache()
    rng = np.random.default_rng(0)
    probe = sorted(rng.choice(w.T, size=16, replace=False).tolist())
    t0 = time.perf_counter()
    oracle_step(w, host, probe)
    fixed = time.perf_counter() - t0
    # per-step sample sized so that warm-up + steps take about args.ref_budget seconds
    per_step = max(fixed, args.ref_budget / max(1, args.steps + args.warmup))
    sample = int(max(8, min(w.T, 16 * per_step / max(fixed, 1e-3))))
    for _ in range(args.warmup):
        oracle_step(w, host, sorted(rng.choice(w.T, size=sample, replace=False).tolist()))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(w, host, sorted(rng.choice(w.T, size=sample, replace=False).tolist()))
    dt = time.perf_counter() - t0
    value = sample * args.steps / dt
    desc = (f"each step routes one whole {w.name} batch (T={w.T}) and evaluates {sample} "
            f"random tokens' experts in fp64")
    res = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) weights, random-init)",
        "config": {"workload": w.name, "shape": w.description, "T": w.T,
                   "D": w.D, "E": w.E, "k": w.k, "F": w.F, "tokens_per_step": w.T,
                   "parallelism": "CPU oracle (rank 0)"},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="mixtral", choices=["mixtral", "switch", "v3", "ec"])
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the batch size T (smaller cases for profiling)")
    ap.add_argument("--ffn", type=int, default=0,
                    help="override the expert width F (smaller cases for profiling)")
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager calls instead of a CUDA-graph replay of the step")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward-pass timing that follows the forward measurement")
    ap.add_argument("--no-sustained", action="store_true",
                    help="skip the one-second replay of the step reported as 'sustained'")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the shorter measurements of the other layer shapes")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=90.0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        run_cuda(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
