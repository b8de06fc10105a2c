"""Benchmark of the multi-LoRA shrink + expand hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step = one pass of the whole per-token (BGMV) path over one batch:
group-by-slot metadata, shrink into the fp32 intermediate, expand into the
output slices.  At N=1 the workload is the decode batch at a Llama-3-8B
q_proj shape (T=256 tokens, D=D_out=4096, 32 slots, rank 16, fp16, scale 2),
unless --config picks another.  Inputs are seeded synthetic tensors of that
shape; adapter weights are random, not trained.

Timing: K steps are captured in CUDA graphs and replayed, each step on the
next of several input sets whose total size is more than three times the L2
cache, so every step reads cold HBM.  CUDA events on the launching stream,
barrier + synchronize on both sides, max over ranks.  Multi-GPU runs are
independent data-parallel replicas (each rank its own token batch, adapters
replicated; no collective on the data path): weak scaling.

Rank 0 prints one JSON line.  --impl reference times the CPU oracle (the
plain fp64 definition) on bounded samples of the same workload instead.
"""
import argparse
import datetime
import hashlib
import json
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


def profile_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, or None when it
    is missing or was taken on other sources of that kernel."""
    if not os.path.exists(PROFILE_TRAFFIC) or kernel not in KERNEL_SOURCES:
        return None
    k = json.load(open(PROFILE_TRAFFIC)).get("kernels", {}).get(kernel)
    if k is None or k.get("source_hash") != kernel_source_hash(kernel):
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


def kernel_list(p):
    if p.segmented:
        return ["shrink", "expand"]
    return ["fused"] if fused(p) else ["group", "shrink", "expand"]


def step_calls(p, d, what="step"):
    """Enqueue one step (or one kernel of it) on the current stream."""
    from gather_matmul_b200 import ops
    shared = p.shared_A and p.n_slices > 1
    buf = d.buf[0] if shared else d.buf
    if p.segmented:
        if what in ("step", "shrink"):
            ops.shrink_segment(d.x, d.A, d.ss, d.sa, d.buf, d.meta)
        if what in ("step", "expand"):
            ops.expand_segment(buf, d.B, d.ss, d.sa, d.y, d.meta, p.scale, y_col_off=p.col_off)
        return
    if what in ("step", "fused"):
        # the whole per-token path in one call (one launch when it fits), in
        # plain stream order (no early start of the next launch)
        ops.bgmv(d.x, d.A, d.B, d.idx, d.y, d.buf, d.meta, p.scale, y_col_off=p.col_off)
        return
    if what == "group":
        ops.group(d.idx, p.S, d.meta)
    if what == "shrink":
        ops.shrink(d.x, d.A, d.buf, d.meta)
    if what == "expand":
        ops.expand(buf, d.B, d.y, d.meta, p.scale, y_col_off=p.col_off)


def launches_per(p, what="step"):
    if what != "step":
        return 1
    return 2 if p.segmented else (1 if fused(p) else 3)


class GraphRunner:
    """K calls over rotating sets, as replays of captured CUDA graphs of up to
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

    @staticmethod
    def run(plan):
        for g in plan:
            g.replay()


def time_plan(plan, stream):
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    with torch.cuda.stream(stream):
        GraphRunner.run(plan)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3


def make_sets(p, extra_copies):
    base = DeviceSet(p)
    n = rotation_sets(base.nbytes())
    sets = [base] + [DeviceSet(p, src=base) for _ in range(n - 1)] if extra_copies else [base]
    return sets


def e2e_measure(p, dsets, steps, warmup, stream):
    """The same metric through the public API with host buffers: per step,
    pinned host -> device copies of x, idx and y, the call(s), and a device ->
    host copy of the updated y.  Each step's inputs sit in one pinned host
    block and one device block (x, y and idx as views of it), so they cross
    PCIe as one copy.  Steps are double-buffered over two device sets and
    three streams (copy in, compute, copy out), as a serving loop would
    overlap one batch's transfers with another's compute; every step still
    moves all of its bytes."""
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

    for k in range(warmup):
        one(k)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(steps):
        one(k)
    e1.record(s_out)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3, h2d, d2h


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


def measure_config(p, steps, warmup, stream, detail=False):
    sets = make_sets(p, extra_copies=True)
    runner = GraphRunner(p, sets, stream, "step")
    plan_w = runner.prepare(max(warmup, 1))
    with torch.cuda.stream(stream):
        GraphRunner.run(plan_w)
    torch.cuda.synchronize()
    plan = runner.prepare(steps)
    return sets, runner, plan


def kernel_times(p, sets, stream, reps):
    out = {}
    if not p.segmented and not fused(p):
        # the group kernel must have run on each set before shrink / expand
        for d in sets:
            with torch.cuda.stream(stream):
                step_calls(p, d, "group")
        torch.cuda.synchronize()
    for what in kernel_list(p):
        r = GraphRunner(p, sets, stream, what)
        plan = r.prepare(reps)
        with torch.cuda.stream(stream):
            GraphRunner.run(r.prepare(min(reps, 64)))
        torch.cuda.synchronize()
        t = time_plan(plan, stream)
        out[what] = t / reps
    return out


KERNEL_NAMES = {"fused": "bgmv_fused_kernel", "group": "group_kernel",
                "shrink": "shrink_items_kernel", "expand": "expand_items_kernel"}
SEG_KERNEL_NAMES = {"shrink": "sgmv_shrink", "expand": "sgmv_expand"}


def kernel_bytes(p, what):
    by = algorithmic_bytes(p)
    if what == "fused":
        return by["shrink"] + by["expand"]
    return by[what]


def roofline_entry(p, ktimes, peak, peak_kind):
    dom = max((k for k in ktimes if k != "group"), key=lambda k: ktimes[k])
    ach = kernel_bytes(p, dom) / ktimes[dom] / 1e9
    name = (SEG_KERNEL_NAMES if p.segmented else KERNEL_NAMES)[dom]
    return {"bound": "hbm", "kernel": name, "achieved": round(ach, 1), "peak": peak,
            "peak_kind": peak_kind, "unit": "GB/s", "frac": round(ach / peak, 4),
            "traffic": profile_traffic(name),
            "algorithmic_bytes": kernel_bytes(p, dom),
            "us_per_launch": round(ktimes[dom] * 1e6, 3)}


def config_label(p):
    return (f"{p.name}: T={p.T} D={p.D} r={p.r} S={p.S} slices={p.d_out} "
            f"{W.DTYPE_NAME[p.dtype]} scale={p.scale}")


def run_ours(args):
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    init_dist(ws, "nccl")
    dev = torch.device("cuda", local)
    from gather_matmul_b200 import ops
    ops.build_info()   # loads the library or fails loudly

    probs = W.config(args.config)
    p = probs[0]
    if rank:   # data parallel: every rank serves its own batch of the same shape
        p = W.make_problem(p.name, p.dtype, p.T, p.D, p.r, p.S, p.d_out, p.scale,
                           seed=1000 * rank + args.config,
                           idx_kind={2: "uniform", 1: "uniform_neg", 5: "zipf"}.get(args.config, "frac_neg"),
                           frac_neg=0.25 if args.config == 3 else 0.10,
                           segments=(p.seg_starts, p.seg_adapter) if p.segmented else None)
    stream = torch.cuda.Stream(device=dev)
    sets, runner, plan = measure_config(p, args.steps, args.warmup, stream)
    peak, peak_kind = measured_peaks()

    sampler = ClockSampler(local).start() if rank == 0 else None
    time.sleep(0.2)
    barrier(ws)
    torch.cuda.synchronize()
    elapsed = time_plan(plan, stream)
    barrier(ws)
    torch.cuda.synchronize()
    kt = kernel_times(p, sets, stream, reps=min(args.steps, 2048))
    clocks = sampler.stop() if sampler is not None else None

    el_max = max_over_ranks(elapsed, ws, dev)
    tokens_all = sum_over_ranks(p.T * args.steps, ws, dev)
    value = tokens_all / el_max
    by = algorithmic_bytes(p)

    e2e_steps = max(3, min(args.steps, 2000))
    e2e_t, h2d, d2h = e2e_measure(p, sets, e2e_steps, 3, stream)
    e2e_t = max_over_ranks(e2e_t, ws, dev)
    e2e_val = sum_over_ranks(p.T * e2e_steps, ws, dev) / e2e_t

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
                   "step": ("segment shrink + expand" if p.segmented else
                            "group-by-slot + shrink + expand in one fused launch" if fused(p)
                            else "group-by-slot + shrink + expand (3 launches)"),
                   "l2": f"inputs larger than L2: {len(sets)} rotating input sets, "
                         f"{sum(s.nbytes() for s in sets) / 1e6:.0f} MB > {L2_BYTES / 1e6:.0f} MB",
                   "graph": "K steps replayed from CUDA graphs of up to 64 steps",
                   "parallelism": f"dp{ws} independent replicas"},
        "achieved_gbs_step": round(by["step"] * args.steps * ws / el_max / 1e9, 1),
        "roofline": roofline_entry(p, kt, peak, peak_kind),
        "kernel_us": {k: round(v * 1e6, 3) for k, v in kt.items()},
        "gpu_launches": launches_per(p) * args.steps,
        "e2e": {"value": round(e2e_val, 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "clocks": clocks,
    }
    if ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(p, budget_s=args.cpu_seconds)
    if args.detail:
        line["detail"] = detail_all(args, stream, peak, peak_kind)
    print(json.dumps(line), flush=True)
    barrier(ws)


def detail_all(args, stream, peak, peak_kind):
    """Per-projection numbers of every workload (not the headline line)."""
    out = {}
    layer = []
    tf_peak = measured_bf16_tflops()
    for n in (1, 2, 3, 4, 5):
        for p in W.config(n):
            sets = make_sets(p, extra_copies=True)
            reps = 256
            kt = kernel_times(p, sets, stream, reps)
            r = GraphRunner(p, sets, stream, "step")
            plan = r.prepare(reps)
            with torch.cuda.stream(stream):
                GraphRunner.run(r.prepare(min(reps, 64)))
            t = time_plan(plan, stream) / reps
            by = algorithmic_bytes(p)
            fl = algorithmic_flops(p)
            out[f"cfg{n}:{p.name}"] = {
                "us_per_step": round(t * 1e6, 3),
                "tokens_per_s": round(p.T / t, 1),
                "gbs_step": round(by["step"] / t / 1e9, 1),
                "frac_step": round(by["step"] / t / 1e9 / peak, 4),
                "kernel_us": {k: round(v * 1e6, 3) for k, v in kt.items()},
                "kernel_gbs": {k: round(kernel_bytes(p, k) / v / 1e9, 1) for k, v in kt.items()},
                "kernel_frac": {k: round(kernel_bytes(p, k) / v / 1e9 / peak, 4)
                                for k, v in kt.items()},
                "tflops_step": round(fl / t / 1e12, 2),
                # fraction of the tensor roofline, and of the slower of the two
                # rooflines (contraction FLOPs at the bf16 peak, bytes at HBM)
                "tensor_frac_step": round(fl / t / 1e12 / tf_peak, 4),
                "roofline_frac_step": round(max(fl / (tf_peak * 1e12), by["step"] / (peak * 1e9))
                                            / t, 4),
                "frac_step_vs_8tbs": round(by["step"] / t / 8e12, 4),
                "bytes": by,
            }
            if n == 3:
                layer.append((t, by["step"], p.T))
            del sets
            torch.cuda.empty_cache()
    # the three fused-slice projections of one decoder layer, back to back
    t3 = sum(v[0] for v in layer)
    b3 = sum(v[1] for v in layer)
    out["cfg3:layer_sum"] = {"us_per_layer": round(t3 * 1e6, 3),
                             "tokens_per_s": round(layer[0][2] / t3, 1),
                             "gbs": round(b3 / t3 / 1e9, 1), "frac": round(b3 / t3 / 1e9 / peak, 4)}
    out["idle_call_us"] = idle_call_us()
    return out


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


# --------------------------------------------------------------------------
# reference arm: the CPU oracle
# --------------------------------------------------------------------------
def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    p = W.config(args.config)[0]
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
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--detail", action="store_true", help="add every workload's numbers")
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
