"""Benchmark of the multi-LoRA shrink + expand hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step = one pass of the whole path over one batch: for a per-token (BGMV)
batch the public one-call entry point (group-by-slot, shrink into the fp32
intermediate, expand into the output slices); for a segment (SGMV) batch the
segment shrink and expand.  At N=1 the headline workload is the largest
single-GPU one, the large mixed batch (T=4096 single tokens, D=D_out=8192,
128 slots, rank 32, Zipf(1.1) adapter popularity with 10 % of tokens on the
base model only, unsorted, bf16), unless --config picks another.  Inputs are
seeded synthetic tensors of that shape; adapter weights are random, not
trained.

Timing: the K steps are captured in CUDA graphs, replayed once untimed (with
the warm-up steps) and then timed; each step runs on the next of several
input sets whose total size is more than three times the L2 cache, so every
step reads cold HBM.  CUDA events on the launching stream, barrier +
synchronize on both sides, max over ranks.  Every kernel's own time comes from
a separate graph of at least 256 launches, also replayed once before timing.
The end-to-end figure times at least 100 ms of steps through the public call
with the inputs copied from pinned host memory and the result read back.
The line carries a per-workload block ("configs") with every workload's step
and kernel times and their fractions of the HBM and tensor rooflines.
Multi-GPU runs are independent data-parallel replicas (each rank its own token
batch, adapters replicated; no collective on the data path): weak scaling.

Rank 0 prints one JSON line.  --impl reference times the CPU oracle (the
plain fp64 definition) on bounded samples of the same workload instead.
"""
import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gather_matmul_b200 import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
# the source files each kernel is built from: a DRAM-traffic figure taken
# with ncu stays valid until one of them changes
_CSRC = os.path.join(ROOT, "gather_matmul_b200", "csrc")
_COMMON = ("common.cuh", "ptx.cuh", "internal.h")
KERNEL_SOURCES = {
    "bgmv_fused_kernel": ("bgmv_fused.cu", "tmap.cu") + _COMMON,
    "sgmv_shrink_tc_kernel": ("sgmv_tc.cu", "tmap.cu") + _COMMON,
    "sgmv_expand_tc_kernel": ("sgmv_tc.cu", "tmap.cu") + _COMMON,
    "shrink_items_kernel": ("bgmv.cu",) + _COMMON,
    "expand_items_kernel": ("bgmv.cu",) + _COMMON,
    "group_kernel": ("group.cu",) + _COMMON,
    "segment_items_kernel": ("group.cu",) + _COMMON,
}


# --------------------------------------------------------------------------
# host logic (unit-tested on CPU)
# --------------------------------------------------------------------------
def active_stats(p: W.Problem):
    """(active tokens, distinct slots used) of a problem."""
    if p.segmented:
        ss, sa = p.seg_starts, p.seg_adapter
        lens = np.diff(ss)
        act = (sa >= 0) & (sa < p.S)
        return int(lens[act].sum()), len(set(sa[act & (lens > 0)].tolist()))
    a = p.idx[(p.idx >= 0) & (p.idx < p.S)]
    return int(a.size), int(np.unique(a).size)


def algorithmic_bytes(p: W.Problem, with_group=True):
    """Bytes the path must move at minimum: active x rows, the used slots'
    A and B once each, the fp32 intermediate written then read, y read and
    written for active rows, the indices (and the grouping's permutation)."""
    xb = 2
    Ta, U = active_stats(p)
    nA = len(p.A)
    shrink = Ta * p.D * xb + nA * U * p.r * p.D * xb + 4 * p.T + 4 * nA * p.T * p.r
    expand = 4 * p.T
    for o in p.d_out:
        expand += 4 * Ta * p.r + U * o * p.r * xb + 2 * Ta * o * xb
    group = 8 * p.T if (with_group and not p.segmented) else 0
    return {"shrink": shrink, "expand": expand, "group": group,
            "step": shrink + expand + group}


def algorithmic_flops(p: W.Problem):
    Ta, _ = active_stats(p)
    return 2 * Ta * p.r * p.D * len(p.A) + 2 * Ta * p.r * sum(p.d_out)


def rotation_sets(working_set_bytes, l2_bytes=L2_BYTES, factor=3, cap=64):
    """Input sets to rotate through so that consecutive reuse of a set is more
    than factor * L2 bytes apart."""
    n = -(-factor * l2_bytes // max(int(working_set_bytes), 1))
    return int(max(2, min(cap, n)))


def aggregate(values_per_rank_tokens, elapsed_max_s):
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return float(sum(values_per_rank_tokens)) / elapsed_max_s


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        path = os.path.join(_CSRC, f)
        if os.path.exists(path):
            h.update(open(path, "rb").read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_tflops():
    """Dense bf16 tensor peak (burst cuBLAS GEMM) of this machine's B200s."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"])
    return FALLBACK_BF16_TFLOPS


def profile_traffic(kernel, workload=None):
    """DRAM bytes per launch from the committed ncu summary, or None when it
    is missing, was taken on another workload, or on other sources of that
    kernel."""
    if not os.path.exists(PROFILE_TRAFFIC) or kernel not in KERNEL_SOURCES:
        return None
    k = json.load(open(PROFILE_TRAFFIC)).get("kernels", {}).get(kernel)
    if k is None or k.get("source_hash") != kernel_source_hash(kernel):
        return None
    if workload is not None and k.get("workload") != workload:
        return None
    return k.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(ws, backend):
    if ws > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=120))


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(v, ws, device):
    if ws == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v, ws, device):
    if ws == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# --------------------------------------------------------------------------
# clocks
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "utilization.gpu",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [s.strip() for s in line.split(",")]
            if len(parts) == len(self.FIELDS):
                self.rows.append(parts)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return self.summary()

    def summary(self):
        def num(s):
            try:
                return float(s)
            except ValueError:
                return None
        busy = [r for r in self.rows if num(r[3]) is not None and num(r[3]) > 0] or self.rows
        sm = [num(r[0]) for r in busy if num(r[0]) is not None]
        mx = [num(r[1]) for r in self.rows if num(r[1]) is not None]
        reasons = set()
        for r in busy:
            for k, name in enumerate(self.REASONS):
                if r[4 + k].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(self.rows),
                "samples_busy": len(busy)}


# --------------------------------------------------------------------------
# which kernels each call launches (mirrors the library's dispatch rules)
# --------------------------------------------------------------------------
def grouped_tc(p):
    """Per-token batches with r >= 16 and at least 16 tokens per slot on
    average run their slot groups through the tensor-core kernels."""
    return p.r >= 16 and p.T >= 16 * p.S and p.D % 8 == 0


def kernels_of(p, what, fused_fits):
    """Kernel names behind one timed call of a step."""
    if what == "fused":
        return ["bgmv_fused_kernel"]
    if what == "group":
        return ["group_kernel"]
    if p.segmented:
        if p.r >= 16 and len(p.seg_adapter) <= 2048:
            return ["sgmv_%s_tc_kernel" % what]
        return ["segment_items_kernel", "%s_items_kernel" % what]
    return ["sgmv_%s_tc_kernel" % what] if grouped_tc(p) else ["%s_items_kernel" % what]


def kernel_calls(p, fused_fits):
    """The separately timed calls that make one step."""
    if p.segmented:
        return ["shrink", "expand"]
    return ["fused"] if fused_fits else ["group", "shrink", "expand"]


def call_bytes(p, what):
    by = algorithmic_bytes(p)
    if what == "fused":
        return by["shrink"] + by["expand"]
    return by[what]


def call_flops(p, what):
    Ta, _ = active_stats(p)
    sh = 2 * Ta * p.r * p.D * len(p.A)
    ex = 2 * Ta * p.r * sum(p.d_out)
    return {"fused": sh + ex, "shrink": sh, "expand": ex, "group": 0}[what]


def e2e_steps_for(step_s, steps, min_s=0.1, cap=20000):
    """Steps of the end-to-end loop: at least `steps`, and enough for
    min_s seconds at the estimated time per step."""
    need = math.ceil(round(min_s / max(step_s, 1e-9), 6))
    return int(max(steps, min(cap, need)))


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
class DeviceSet:
    """One independent copy of a problem's tensors on the device."""

    def __init__(self, p: W.Problem, src=None):
        from gather_matmul_b200 import ops
        td = W.TORCH_DTYPE[p.dtype]
        if src is None:
            mk = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(td).cuda()
            self.x = mk(p.x)
            self.A = [mk(a) for a in p.A]
            self.B = [mk(b) for b in p.B]
            self.y = mk(p.y)
            self.idx = torch.from_numpy(p.idx).cuda() if not p.segmented else None
            self.ss = torch.from_numpy(p.seg_starts).cuda() if p.segmented else None
            self.sa = torch.from_numpy(p.seg_adapter).cuda() if p.segmented else None
        else:
            self.x = src.x.clone()
            self.A = [a.clone() for a in src.A]
            self.B = [b.clone() for b in src.B]
            self.y = src.y.clone()
            self.idx = src.idx.clone() if src.idx is not None else None
            self.ss = src.ss.clone() if src.ss is not None else None
            self.sa = src.sa.clone() if src.sa is not None else None
        self.buf = torch.zeros((len(p.A), p.T, p.r), dtype=torch.float32, device="cuda")
        self.meta = ops.workspace(p.T, p.S)

    def nbytes(self):
        ts = [self.x, self.y, self.buf, self.meta] + self.A + self.B
        return sum(t.numel() * t.element_size() for t in ts)


def fused(p):
    from gather_matmul_b200 import ops
    return (not p.segmented) and ops.bgmv_launches(W.TORCH_DTYPE[p.dtype], p.T, p.D, p.r, p.S,
                                                   p.d_out) == 1


def step_calls(p, d, what="step"):
    """Enqueue one step (or one call of it) on the current stream."""
    from gather_matmul_b200 import ops
    shared = p.shared_A and p.n_slices > 1
    buf = d.buf[0] if shared else d.buf
    if p.segmented:
        if what == "step":       # the public one-call segment path: shrink + expand
            ops.sgmv(d.x, d.A, d.B, d.ss, d.sa, d.y, d.buf, d.meta, p.scale, y_col_off=p.col_off)
        if what == "shrink":
            ops.shrink_segment(d.x, d.A, d.ss, d.sa, d.buf, d.meta)
        if what == "expand":
            ops.expand_segment(buf, d.B, d.ss, d.sa, d.y, d.meta, p.scale, y_col_off=p.col_off)
        return
    if what in ("step", "fused"):
        # the public one-call per-token path: one fused launch when the shape
        # fits (plain stream order), else group + shrink + expand with
        # LORA_FLAG_PDL_EARLY, whose promise holds here: the launch before a
        # step is the previous step's expand, which writes y only (in a model
        # it is the base GEMM, which writes y as well)
        ops.bgmv(d.x, d.A, d.B, d.idx, d.y, d.buf, d.meta, p.scale, y_col_off=p.col_off,
                 pdl_early=not fused(p))
        return
    if what == "group":
        ops.group(d.idx, p.S, d.meta)
    if what == "shrink":
        ops.shrink(d.x, d.A, d.idx, d.buf, d.meta)
    if what == "expand":
        ops.expand(buf, d.B, d.idx, d.y, d.meta, p.scale, y_col_off=p.col_off)


class GraphRunner:
    """Calls over rotating sets, as replays of captured CUDA graphs of up to
    G calls each."""

    def __init__(self, p, sets, stream, what="step", G=64):
        self.p, self.sets, self.stream, self.what = p, sets, stream, what
        self.G = G
        self.graphs = {}

    def _graph(self, n, start):
        key = (n, start % len(self.sets))
        if key not in self.graphs:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                for k in range(n):
                    step_calls(self.p, self.sets[(start + k) % len(self.sets)], self.what)
            self.graphs[key] = g
        return self.graphs[key]

    def prepare(self, K):
        full, rem = divmod(K, self.G)
        plan = []
        pos = 0
        for _ in range(full):
            plan.append(self._graph(self.G, pos))
            pos += self.G
        if rem:
            plan.append(self._graph(rem, pos))
        return plan

    def run(self, plan):
        with torch.cuda.stream(self.stream):
            for g in plan:
                g.replay()


def time_plan(runner, plan):
    """Device time of one replay of `plan`, measured with CUDA events on the
    launching stream, synchronized on both sides."""
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(runner.stream)
    runner.run(plan)
    e1.record(runner.stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3


def warm_then_time(runner, K, warm_calls=0):
    """Capture K calls, replay that exact plan untimed (at least once, and for
    at least warm_calls calls), then time one replay of it."""
    plan = runner.prepare(K)
    for _ in range(max(1, -(-warm_calls // max(K, 1)))):
        runner.run(plan)
    torch.cuda.synchronize()
    return time_plan(runner, plan)


def make_sets(p):
    base = DeviceSet(p)
    n = rotation_sets(base.nbytes())
    return [base] + [DeviceSet(p, src=base) for _ in range(n - 1)]


def launches_per_step(p, d, stream):
    """Kernels one step launches, counted by the library while one step is
    recorded into a (discarded) graph."""
    from gather_matmul_b200 import ops
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    before = ops.launch_count()
    with torch.cuda.graph(g, stream=stream):
        step_calls(p, d, "step")
    n = ops.launch_count() - before
    del g
    return n


def kernel_times(p, sets, stream, reps, fused_fits):
    """Average device time of each call of the step, from graphs of `reps`
    calls each replayed once before timing."""
    out = {}
    if not p.segmented and not fused_fits:
        # the grouping must exist on each set before its shrink / expand
        with torch.cuda.stream(stream):
            for d in sets:
                step_calls(p, d, "group")
        torch.cuda.synchronize()
    for what in kernel_calls(p, fused_fits):
        r = GraphRunner(p, sets, stream, what)
        out[what] = warm_then_time(r, reps) / reps
    return out


def e2e_measure(p, dsets, steps, warmup, stream):
    """The same metric through the public API with host buffers: per step,
    pinned host -> device copies of x, idx and y, the call(s), and a device ->
    host copy of the updated y.  Each step's inputs sit in one pinned host
    block and one device block (x, y and idx as views of it), so they cross
    PCIe as one copy.  Steps are double-buffered over two device sets and
    three streams (copy in, compute, copy out), as a serving loop would
    overlap one batch's transfers with another's compute; every step still
    moves all of its bytes.  The loop runs at least `steps` steps and at least
    100 ms."""
    import types
    nb = min(2, len(dsets))
    d0 = dsets[0]
    xb = d0.x.numel() * d0.x.element_size()
    yb = d0.y.numel() * d0.y.element_size()
    ib = d0.idx.numel() * 4 if d0.idx is not None else 0
    h2d, d2h = xb + yb + ib, yb
    hin = torch.empty(h2d, dtype=torch.uint8, pin_memory=True)
    hin[:xb].copy_(d0.x.cpu().view(-1).view(torch.uint8))
    hin[xb:xb + yb].copy_(d0.y.cpu().view(-1).view(torch.uint8))
    if ib:
        hin[xb + yb:].copy_(d0.idx.cpu().view(torch.uint8))
    hout = [torch.empty(yb, dtype=torch.uint8, pin_memory=True) for _ in range(nb)]
    io, views = [], []
    for i in range(nb):
        blk = torch.empty(h2d, dtype=torch.uint8, device="cuda")
        v = types.SimpleNamespace(**vars(dsets[i]))
        v.x = blk[:xb].view(d0.x.dtype).view(d0.x.shape)
        v.y = blk[xb:xb + yb].view(d0.y.dtype).view(d0.y.shape)
        v.idx = blk[xb + yb:].view(torch.int32) if ib else None
        io.append(blk)
        views.append(v)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    done_in = [torch.cuda.Event() for _ in range(nb)]
    done_step = [torch.cuda.Event() for _ in range(nb)]
    done_out = [torch.cuda.Event() for _ in range(nb)]
    used = [False] * nb

    def one(k):
        i = k % nb
        with torch.cuda.stream(s_in):
            if used[i]:
                s_in.wait_event(done_out[i])          # set i's previous result has left
            io[i].copy_(hin, non_blocking=True)
            done_in[i].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(done_in[i])
            step_calls(p, views[i])
            done_step[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done_step[i])
            hout[i].copy_(io[i][xb:xb + yb], non_blocking=True)
            done_out[i].record(s_out)
        used[i] = True

    def timed(n):
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for k in range(n):
            one(k)
        s_in.wait_stream(s_out)
        e1.record(s_in)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3

    for k in range(warmup):
        one(k)
    est = timed(max(warmup, 3)) / max(warmup, 3)
    n = e2e_steps_for(est, steps)
    return timed(n), n, h2d, d2h


def cpu_baseline(p, budget_s=10.0):
    """The oracle as it stands, on this host's cores, over a bounded sample
    of the workload: whole passes over the first n tokens, repeated until
    about budget_s seconds have been spent."""
    import oracle
    cores = oracle.set_threads(os.cpu_count() or 1)
    n = p.T
    idx = p.idx if not p.segmented else oracle.segments_to_idx(p.T, p.seg_starts, p.seg_adapter)
    x, y = p.x, p.y

    def one(n):
        buf, _ = oracle.shrink(p.dtype, x[:n], p.A, idx[:n], p.S)
        shared = p.shared_A and p.n_slices > 1
        oracle.expand(p.dtype, buf[0] if shared else buf, p.B, idx[:n], p.S, p.scale, y[:n],
                      p.col_off, shared_buf=shared)

    t0 = time.perf_counter()
    one(min(n, 8))
    t_probe = max(time.perf_counter() - t0, 1e-6)
    per_tok = t_probe / min(n, 8)
    n = int(max(1, min(p.T, budget_s / 3 / per_tok)))
    reps, done, t0 = 0, 0, time.perf_counter()
    while True:
        one(n)
        reps += 1
        done += n
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 100000:
            break
    return {"value": done / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} passes of shrink+expand over the first {n} of {p.T} tokens "
                      f"({el:.1f} s, fp64, OpenMP over tokens)"}


def roofline_entry(p, ktimes, peak, peak_kind, fused_fits):
    """Roofline of the dominant (longest) call of the step."""
    dom = max((k for k in ktimes if k != "group"), key=lambda k: ktimes[k])
    ach = call_bytes(p, dom) / ktimes[dom] / 1e9
    names = kernels_of(p, dom, fused_fits)
    return {"bound": "hbm", "kernel": "+".join(names), "achieved": round(ach, 1), "peak": peak,
            "peak_kind": peak_kind, "unit": "GB/s", "frac": round(ach / peak, 4),
            "traffic": profile_traffic(names[-1], p.name) if len(names) == 1 else None,
            "algorithmic_bytes": call_bytes(p, dom),
            "us_per_launch": round(ktimes[dom] * 1e6, 3)}


def config_label(p):
    return (f"{p.name}: T={p.T} D={p.D} r={p.r} S={p.S} slices={p.d_out} "
            f"{W.DTYPE_NAME[p.dtype]} scale={p.scale}")


def workload_numbers(p, t_step, kt, peak, tf_peak, fused_fits, launches):
    """Step and per-call figures of one projection: times, throughput, and the
    fractions of the HBM roofline (algorithmic bytes / time / measured copy
    bandwidth), of the tensor roofline (contraction FLOPs / time / bf16
    peak), and of the slower of the two."""
    by = algorithmic_bytes(p)
    fl = algorithmic_flops(p)
    Ta, U = active_stats(p)
    return {
        "workload": config_label(p),
        "us_per_step": round(t_step * 1e6, 3),
        "tokens_per_s": round(p.T / t_step, 1),
        "active_tokens": Ta, "slots_used": U,
        "launches_per_step": launches,
        "gbs_step": round(by["step"] / t_step / 1e9, 1),
        "frac_step": round(by["step"] / t_step / 1e9 / peak, 4),
        "calls": {k: {"kernels": kernels_of(p, k, fused_fits),
                      "us": round(v * 1e6, 3),
                      "bytes": call_bytes(p, k),
                      "gbs": round(call_bytes(p, k) / v / 1e9, 1),
                      "frac_hbm": round(call_bytes(p, k) / v / 1e9 / peak, 4),
                      "tensor_frac": round(call_flops(p, k) / v / 1e12 / tf_peak, 4)}
                  for k, v in kt.items()},
        "tflops_step": round(fl / t_step / 1e12, 2),
        "tensor_frac_step": round(fl / t_step / 1e12 / tf_peak, 4),
        "roofline_frac_step": round(max(fl / (tf_peak * 1e12), by["step"] / (peak * 1e9))
                                    / t_step, 4),
        "frac_step_vs_8tbs": round(by["step"] / t_step / 8e12, 4),
        "bytes": by,
    }


def copy_floor(nbytes, stream, reps=256):
    """Device time of ONE plain copy kernel (torch's) that reads nbytes / 2 and
    writes nbytes / 2, timed like the steps (graph replay over rotating buffers
    larger than L2): the speed a single launch moving the step's bytes reaches
    at this size, launch and ramp included.  A reference for the fractions,
    not part of the path."""
    half = max(4096, (nbytes // 2) // 4096 * 4096)
    n = rotation_sets(2 * half)
    bufs = [(torch.ones(half, dtype=torch.uint8, device="cuda"),
             torch.empty(half, dtype=torch.uint8, device="cuda")) for _ in range(n)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for k in range(reps):
            src, dst = bufs[k % n]
            dst.copy_(src)
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / reps
    del g, bufs
    torch.cuda.empty_cache()
    return t, 2 * half


def measure_workload(p, stream, reps, peak, tf_peak):
    sets = make_sets(p)
    ff = fused(p)
    launches = launches_per_step(p, sets[0], stream)
    kt = kernel_times(p, sets, stream, reps, ff)
    t = warm_then_time(GraphRunner(p, sets, stream, "step"), reps) / reps
    out = workload_numbers(p, t, kt, peak, tf_peak, ff, launches)
    out["l2"] = f"{len(sets)} rotating input sets, {sum(s.nbytes() for s in sets) / 1e6:.0f} MB"
    del sets
    torch.cuda.empty_cache()
    tc, cb = copy_floor(algorithmic_bytes(p)["step"], stream, reps)
    out["one_launch_copy"] = {"bytes": cb, "us": round(tc * 1e6, 3),
                              "gbs": round(cb / tc / 1e9, 1),
                              "frac_hbm": round(cb / tc / 1e9 / peak, 4),
                              "step_time_ratio": round(tc / t, 4)}
    return out


def configs_block(stream, peak, tf_peak, reps=256):
    """Every workload: each projection's numbers, plus the three fused-slice
    projections of one decoder layer summed."""
    out = {}
    layer = []
    for n in (1, 2, 3, 4, 5):
        for p in W.config(n):
            r = measure_workload(p, stream, reps, peak, tf_peak)
            out[f"cfg{n}:{p.name}"] = r
            if n == 3:
                layer.append((r["us_per_step"] * 1e-6, r["bytes"]["step"], p.T))
    t3 = sum(v[0] for v in layer)
    b3 = sum(v[1] for v in layer)
    out["cfg3:layer_sum"] = {"us_per_layer": round(t3 * 1e6, 3),
                             "tokens_per_s": round(layer[0][2] / t3, 1),
                             "gbs": round(b3 / t3 / 1e9, 1),
                             "frac_hbm": round(b3 / t3 / 1e9 / peak, 4)}
    out["cfg3:layer_one_grouping"] = layer_one_grouping(stream, peak, reps)
    return out


def layer_one_grouping(stream, peak, reps):
    """The three fused-slice projections of one decoder layer as a decode
    step runs them: the batch's grouping built once (lora_group) and shared by
    every projection (the projections of one batch carry the same indices),
    each projection one lora_bgmv call with LORA_FLAG_GROUPED (shrink, then
    the chained expand)."""
    from gather_matmul_b200 import ops
    probs = W.config(3)
    sets = [make_sets(p) for p in probs]
    n = min(len(s) for s in sets)

    def one(k):
        d0 = sets[0][k % n]
        ops.group(d0.idx, probs[0].S, d0.meta)
        for p, ss in zip(probs, sets):
            d = ss[k % n]
            ops.bgmv(d.x, d.A, d.B, d0.idx, d.y, d.buf, d0.meta, p.scale, y_col_off=p.col_off,
                     grouped=True)

    graphs = []
    G = 32
    for start in range(0, reps, G):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for k in range(start, min(reps, start + G)):
                one(k)
        graphs.append(g)

    def run():
        with torch.cuda.stream(stream):
            for g in graphs:
                g.replay()
    run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run()
    e1.record(stream)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / reps
    by = algorithmic_bytes(probs[0])["group"] + sum(
        algorithmic_bytes(p, with_group=False)["step"] for p in probs)
    del graphs, sets
    torch.cuda.empty_cache()
    return {"us_per_layer": round(t * 1e6, 3), "tokens_per_s": round(probs[0].T / t, 1),
            "gbs": round(by / t / 1e9, 1), "frac_hbm": round(by / t / 1e9 / peak, 4),
            "launches_per_layer": 1 + 2 * len(probs)}


def idle_call_us(calls=2000):
    """Host time of a per-token call when no token has an adapter (has_active
    = 0): the library returns before any launch, so this is the whole cost of
    LoRA being enabled but idle.  Through the Python binding, and through the
    C ABI with the arguments marshalled once."""
    import ctypes
    from gather_matmul_b200 import _lib, ops
    p = W.config(2)[0]
    d = DeviceSet(p)
    out = {}
    for _ in range(10):
        ops.bgmv(d.x, d.A, d.B, d.idx, d.y, d.buf, d.meta, p.scale, has_active=False)
    t0 = time.perf_counter()
    for _ in range(calls):
        ops.bgmv(d.x, d.A, d.B, d.idx, d.y, d.buf, d.meta, p.scale, has_active=False)
    out["python_op"] = round((time.perf_counter() - t0) / calls * 1e6, 3)
    vp = ctypes.c_void_p
    ptrs = lambda ts: (vp * len(ts))(*[t.data_ptr() for t in ts])
    n = len(d.B)
    args = (_lib.LORA_F16 if p.dtype == W.F16 else _lib.LORA_BF16, p.T, p.D, p.r, p.S, n,
            vp(d.x.data_ptr()), p.D, ptrs(d.A), 0, ptrs(d.B),
            (ctypes.c_int32 * n)(*[b.shape[1] for b in d.B]), ctypes.c_float(p.scale),
            vp(d.y.data_ptr()), d.y.stride(0), (ctypes.c_int64 * n)(*[int(o) for o in p.col_off]),
            vp(d.buf.data_ptr()), vp(d.idx.data_ptr()), 0, 0, vp(d.meta.data_ptr()),
            d.meta.numel(), vp(torch.cuda.current_stream().cuda_stream))
    fn = _lib.load().lora_bgmv
    assert fn(*args) == 0
    t0 = time.perf_counter()
    for _ in range(calls):
        fn(*args)
    out["c_abi"] = round((time.perf_counter() - t0) / calls * 1e6, 3)
    return out


def graph_specialization(stream, reps=200, T=256, S=32, r=16):
    """LoRA enabled but idle, with one graph set and with graphs specialised
    on has_lora ("[LoRA] LoRA cuda graph specialization": two graph sets,
    dispatch on the batch's flag; its latency logs: 10.5 % -> 1.4 %).

    Stand-in for one decoder layer of a decode step at Llama-3-8B shapes:
    the base projections qkv (4096 -> 4096+1024+1024), o (4096 -> 4096),
    gate_up (4096 -> 14336+14336) and down (14336 -> 4096) as torch matmuls
    (the base model, not this library), each followed by its LoRA update
    through lora_bgmv; T tokens, S slots, rank r, bf16, random weights.
    Device times per step from CUDA events around `reps` graph replays."""
    from gather_matmul_b200 import ops
    from gather_matmul_b200.graphs import LoraGraphSet
    g = torch.Generator(device="cuda").manual_seed(80)
    td = torch.bfloat16
    rnd = lambda *shape, std=1.0: (torch.randn(*shape, generator=g, device="cuda") * std).to(td)
    projs = [(4096, [4096, 1024, 1024]), (4096, [4096]), (4096, [14336, 14336]), (14336, [4096])]
    layers = []
    for D, d_out in projs:
        n = sum(d_out)
        layers.append(dict(
            D=D, d_out=d_out, off=list(np.concatenate([[0], np.cumsum(d_out)[:-1]]).astype(int)),
            x=rnd(T, D), W=rnd(n, D, std=0.02), y=torch.empty(T, n, dtype=td, device="cuda"),
            A=[rnd(S, r, D, std=0.02) for _ in d_out], B=[rnd(S, o, r, std=0.02) for o in d_out],
            buf=torch.empty(len(d_out), T, r, dtype=torch.float32, device="cuda"),
            meta=ops.workspace(T, S)))
    idx = torch.empty(T, dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(81)
    idx_active = rng.integers(0, S, size=T).astype(np.int32)
    idx_idle = np.full(T, -1, dtype=np.int32)

    def step(has_lora):
        for L in layers:
            torch.matmul(L["x"], L["W"].t(), out=L["y"])
            if has_lora:
                ops.bgmv(L["x"], L["A"], L["B"], idx, L["y"], L["buf"], L["meta"], 1.0,
                         y_col_off=L["off"])

    idx.copy_(torch.from_numpy(idx_active))
    gs = LoraGraphSet(step, stream).capture()

    def timed(body):
        for _ in range(3):
            body()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        t0 = time.perf_counter()
        for _ in range(reps):
            body()
        host = time.perf_counter() - t0
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3 / reps, host / reps

    with torch.cuda.stream(stream):
        t_base, _ = timed(lambda: gs.replay(False))
        idx.copy_(torch.from_numpy(idx_idle))
        t_idle_one, _ = timed(lambda: gs.replay(True))
        t_idle_spec, host_spec = timed(lambda: gs.replay_for(idx_idle, S))
        idx.copy_(torch.from_numpy(idx_active))
        t_active, _ = timed(lambda: gs.replay_for(idx_active, S))
    t0 = time.perf_counter()
    for _ in range(1000):
        ops.active_from_host(idx_idle, S)
    decide = (time.perf_counter() - t0) / 1000
    launches = {"without_lora": gs.lora_launches[False], "with_lora": gs.lora_launches[True]}
    del gs
    return {
        "stand_in": f"decode layer, T={T}, Llama-3-8B qkv/o/gate_up/down base matmuls + "
                    f"lora_bgmv per projection, S={S} r={r} bf16",
        "us_base_graph": round(t_base * 1e6, 2),
        "us_idle_one_graph_set": round(t_idle_one * 1e6, 2),
        "us_idle_specialized": round(t_idle_spec * 1e6, 2),
        "us_lora_active": round(t_active * 1e6, 2),
        "overhead_idle_one_graph_set": round(t_idle_one / t_base - 1, 4),
        "overhead_idle_specialized": round(t_idle_spec / t_base - 1, 4),
        "host_us_per_dispatch": round(host_spec * 1e6, 2),
        "host_us_has_lora_from_indices": round(decide * 1e6, 2),
        "library_launches_per_step": launches,
    }


def laning_block(stream, peak, reps=256):
    """The laned shrink (every slot's A as one [S*r, D] matrix on tensor
    cores, each token keeping its own lanes, no grouping) against the grouped
    shrink (group-by-slot, then the shrink over the grouping), on the
    small-rank per-token workloads.  Same algorithmic bytes, so the HBM
    fractions compare directly."""
    from gather_matmul_b200 import ops
    out = {}
    for n in (1, 2):
        p = W.config(n)[0]
        sets = make_sets(p)
        res = {}
        calls = {
            "laned_shrink": lambda d: ops.shrink_laned(d.x, d.A, d.idx, d.buf, d.meta),
            "group_then_shrink": lambda d: (ops.group(d.idx, p.S, d.meta),
                                            ops.shrink(d.x, d.A, d.idx, d.buf, d.meta)),
        }
        for name, fn in calls.items():
            graphs = []
            for start in range(0, reps, 64):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for k in range(start, min(reps, start + 64)):
                        fn(sets[k % len(sets)])
                graphs.append(g)
            with torch.cuda.stream(stream):
                for g in graphs:
                    g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            with torch.cuda.stream(stream):
                for g in graphs:
                    g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) / 1e3 / reps
            by = algorithmic_bytes(p)["shrink"] + (algorithmic_bytes(p)["group"]
                                                   if name == "group_then_shrink" else 0)
            res[name] = {"us": round(t * 1e6, 3), "gbs": round(by / t / 1e9, 1),
                         "frac_hbm": round(by / t / 1e9 / peak, 4)}
            del graphs
        res["lane_flops_per_useful"] = p.S
        out[f"cfg{n}:{p.name}"] = res
        del sets
        torch.cuda.empty_cache()
    return out


def pick_workload(args):
    ps = W.config(args.config)
    if args.workload is None:
        return ps[0]
    for p in ps:
        if p.name == args.workload:
            return p
    raise SystemExit(f"config {args.config} has no workload {args.workload!r} "
                     f"(it has {', '.join(q.name for q in ps)})")


def run_ours(args):
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    init_dist(ws, "nccl")
    dev = torch.device("cuda", local)
    from gather_matmul_b200 import ops
    ops.build_info()   # loads the library or fails loudly

    p = pick_workload(args)
    if rank:   # data parallel: every rank serves its own batch of the same shape
        p = W.make_problem(p.name, p.dtype, p.T, p.D, p.r, p.S, p.d_out, p.scale,
                           seed=1000 * rank + args.config,
                           idx_kind={2: "uniform", 1: "uniform_neg", 5: "zipf"}.get(args.config, "frac_neg"),
                           frac_neg=0.25 if args.config == 3 else 0.10,
                           segments=(p.seg_starts, p.seg_adapter) if p.segmented else None)
    stream = torch.cuda.Stream(device=dev)
    peak, peak_kind = measured_peaks()
    tf_peak = measured_bf16_tflops()
    sets = make_sets(p)
    l2_desc = (f"inputs larger than L2: step k runs on input set k mod {len(sets)}, "
               f"{sum(d.nbytes() for d in sets) / 1e6:.0f} MB in all > {L2_BYTES / 1e6:.0f} MB")
    ff = fused(p)
    launches = launches_per_step(p, sets[0], stream)
    runner = GraphRunner(p, sets, stream, "step")
    plan = runner.prepare(args.steps)
    # warm-up: W untimed steps, and the exact timed graphs replayed once
    runner.run(runner.prepare(args.warmup))
    runner.run(plan)
    torch.cuda.synchronize()

    sampler = ClockSampler(local).start() if rank == 0 else None
    time.sleep(0.2)
    barrier(ws)
    torch.cuda.synchronize()
    elapsed = time_plan(runner, plan)
    barrier(ws)
    torch.cuda.synchronize()
    reps = max(256, args.steps)
    kt = kernel_times(p, sets, stream, reps, ff)

    el_max = max_over_ranks(elapsed, ws, dev)
    tokens_all = sum_over_ranks(p.T * args.steps, ws, dev)
    value = tokens_all / el_max
    by = algorithmic_bytes(p)

    e2e_t, e2e_n, h2d, d2h = e2e_measure(p, sets, args.steps, 3, stream)
    e2e_t = max_over_ranks(e2e_t, ws, dev)
    e2e_val = sum_over_ranks(p.T * e2e_n, ws, dev) / e2e_t
    del sets, runner, plan
    torch.cuda.empty_cache()
    blocks = None
    if ws == 1 and not args.no_configs:
        blocks = configs_block(stream, peak, tf_peak)
    clocks = sampler.stop() if sampler is not None else None

    if rank != 0:
        barrier(ws)
        return
    line = {
        "metric": "LoRA shrink+expand tokens/s (achieved HBM GB/s and % of B200 roofline alongside)",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(el_max / args.steps * 1e3, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": W.DTYPE_NAME[p.dtype], "data": "synthetic (seeded normal inputs, random adapters)",
        "config": {"workload": config_label(p),
                   "step": ("one lora_sgmv call: segment shrink + expand, 2 launches" if p.segmented else
                            "one lora_bgmv call: group-by-slot + shrink + expand, "
                            + ("one fused launch" if ff else
                               f"{launches} launches, LORA_FLAG_PDL_EARLY (the launch before "
                               "a step writes none of A, B, idx)")),
                   "l2": l2_desc,
                   "graph": "K steps replayed from CUDA graphs of up to 64 steps, "
                            "the same graphs replayed once untimed first",
                   "parallelism": f"dp{ws} independent replicas"},
        "active_tokens_per_s": round(active_stats(p)[0] * args.steps * ws / el_max, 1),
        "achieved_gbs_step": round(by["step"] * args.steps * ws / el_max / 1e9, 1),
        "frac_step": round(by["step"] * args.steps * ws / el_max / 1e9 / peak, 4),
        "roofline": roofline_entry(p, kt, peak, peak_kind, ff),
        "kernel_us": {k: round(v * 1e6, 3) for k, v in kt.items()},
        "kernel_reps": reps,
        "gpu_launches": launches * args.steps,
        "e2e": {"value": round(e2e_val, 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_n,
                "seconds": round(e2e_t, 4)},
        "clocks": clocks,
    }
    if ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(p, budget_s=args.cpu_seconds)
    if blocks is not None:
        blocks["idle_call_us"] = idle_call_us()
        line["configs"] = blocks
        line["graph_specialization"] = graph_specialization(stream)
        line["laning"] = laning_block(stream, peak)
    print(json.dumps(line), flush=True)
    barrier(ws)


# --------------------------------------------------------------------------
# reference arm: the CPU oracle
# --------------------------------------------------------------------------
def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    p = pick_workload(args)
    cores = oracle.set_threads(os.cpu_count() or 1)
    idx = p.idx if not p.segmented else oracle.segments_to_idx(p.T, p.seg_starts, p.seg_adapter)
    shared = p.shared_A and p.n_slices > 1

    def one(n, off):
        sl = slice(off, off + n)
        buf, _ = oracle.shrink(p.dtype, p.x[sl], p.A, idx[sl], p.S)
        oracle.expand(p.dtype, buf[0] if shared else buf, p.B, idx[sl], p.S, p.scale, p.y[sl],
                      p.col_off, shared_buf=shared)

    t0 = time.perf_counter()
    one(min(p.T, 4), 0)
    per_tok = max(time.perf_counter() - t0, 1e-6) / min(p.T, 4)
    budget = args.reference_seconds
    n = int(max(1, min(p.T, budget / max(args.steps + args.warmup, 1) / per_tok)))
    for k in range(args.warmup):
        one(n, (k * n) % max(p.T - n + 1, 1))
    t0 = time.perf_counter()
    for k in range(args.steps):
        one(n, (k * n) % max(p.T - n + 1, 1))
    el = time.perf_counter() - t0
    value = n * args.steps / el
    sample = (f"each step: shrink+expand of {n} of the batch's {p.T} tokens "
              f"(fp64 oracle, OpenMP over tokens)")
    line = {
        "impl": "reference",
        "metric": "LoRA shrink+expand tokens/s (achieved HBM GB/s and % of B200 roofline alongside)",
        "value": round(value, 3), "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded normal inputs, random adapters)",
        "config": {"workload": config_label(p), "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=5, choices=[1, 2, 3, 4, 5],
                    help="headline workload (default 5: the large mixed batch)")
    ap.add_argument("--workload", default=None,
                    help="one workload of the config by name (default: its first), e.g. "
                         "decode_gate_up of config 3")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-configs", action="store_true",
                    help="leave out the per-workload block")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-seconds", type=float, default=60.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
