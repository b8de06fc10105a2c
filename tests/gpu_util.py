"""Helpers shared by the GPU parity tests: move a seeded problem to the
device, run the CUDA path through the C ABI binding, run the oracle on the
same bits, and compare under the stated tolerances."""
import os

import numpy as np
import torch

import oracle
from gather_matmul_b200 import ops
from gather_matmul_b200 import workloads as W

# buf: |g - o| <= 1e-3 |o| + 1e-5 sum_d |x_d A_jd|   (fp32 intermediate)
BUF_REL, BUF_ABS_COND = 1e-3, 1e-5
# y:   |g - o| <= 1e-2 (1 + |o|)
Y_TOL = 1e-2

oracle.set_threads(os.cpu_count() or 1)


def dev_bits(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(W.TORCH_DTYPE[dtype])
    return t.cuda()


def host_bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


class Dev:
    def __init__(self, p: W.Problem):
        self.p = p
        self.x = dev_bits(p.x, p.dtype)
        self.A = [dev_bits(a, p.dtype) for a in p.A]
        self.B = [dev_bits(b, p.dtype) for b in p.B]
        self.y = dev_bits(p.y, p.dtype)
        self.buf = torch.full((len(p.A), p.T, p.r), float("nan"), dtype=torch.float32,
                              device="cuda")
        self.meta = ops.workspace(p.T, p.S)
        if p.segmented:
            self.ss = torch.from_numpy(p.seg_starts).cuda()
            self.sa = torch.from_numpy(p.seg_adapter).cuda()
        else:
            self.idx = torch.from_numpy(p.idx).cuda()

    def shrink(self, path=None):
        p = self.p
        if path == "sgmv" or (path is None and p.segmented):
            ops.shrink_segment(self.x, self.A, self.ss, self.sa, self.buf, self.meta)
        else:
            ops.group(self.idx, p.S, self.meta)
            ops.shrink(self.x, self.A, self.idx, self.buf, self.meta)
        return self.buf

    def expand(self, buf=None, path=None):
        p = self.p
        buf = self.buf if buf is None else buf
        shared = p.shared_A and p.n_slices > 1
        b = buf[0] if shared else buf
        if path == "sgmv" or (path is None and p.segmented):
            ops.expand_segment(b, self.B, self.ss, self.sa, self.y, self.meta, p.scale,
                               y_col_off=p.col_off)
        else:
            ops.expand(b, self.B, self.idx, self.y, self.meta, p.scale, y_col_off=p.col_off)
        return self.y


def run_bgmv(d: "Dev", pdl_early=False):
    """The one-call per-token path (fused kernel when the shape fits)."""
    p = d.p
    ops.bgmv(d.x, d.A, d.B, d.idx, d.y, d.buf, d.meta, p.scale, y_col_off=p.col_off,
             pdl_early=pdl_early)
    return d.buf, d.y


def problem_idx(p):
    if p.segmented:
        return oracle.segments_to_idx(p.T, p.seg_starts, p.seg_adapter)
    return p.idx


def oracle_shrink(p):
    buf, cabs, _ = oracle.shrink(p.dtype, p.x, p.A, problem_idx(p), p.S, want_cabs=True)
    return buf, cabs


def oracle_expand(p, buf64):
    shared = p.shared_A and p.n_slices > 1
    y, _ = oracle.expand(p.dtype, buf64[0] if shared else buf64, p.B, problem_idx(p), p.S,
                         p.scale, p.y, p.col_off, shared_buf=shared)
    return y


def assert_buf_close(g, o, cabs, what="buf"):
    g = g.detach().cpu().double().numpy()
    assert np.all(np.isfinite(g)), f"{what}: non-finite values (unwritten rows?)"
    err = np.abs(g - o)
    bound = BUF_REL * np.abs(o) + BUF_ABS_COND * cabs
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; "
                           f"worst err {err.max():.3e} at {np.unravel_index(err.argmax(), err.shape)}")


def assert_y_close(p, y_dev, y_ref, what="y"):
    g = oracle.decode(p.dtype, host_bits(y_dev))
    idx = problem_idx(p)
    neg = ~((idx >= 0) & (idx < p.S))
    # rows without an adapter: bit-identical to the input
    assert np.array_equal(host_bits(y_dev)[neg], p.y[neg]), f"{what}: a -1 row changed"
    err = np.abs(g - y_ref)
    bound = Y_TOL * (1.0 + np.abs(y_ref))
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; "
                           f"worst err {err.max():.3e}")
