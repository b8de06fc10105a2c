"""The allocation-free shrink entry point (lora_shrink_noalloc).

Some callers cannot allocate device memory (they run where cudaMalloc is not
available or not allowed and only hold the input and output buffers), so they
cannot pass the workspace that lora_group + lora_shrink use.  This entry
point keeps that workspace in a fixed device array inside the library.  The
test calls it through the C ABI twice in a row, on two different batches,
and checks each result against the workspace-based entry points on the same
inputs, within the tolerance the other parity tests use, and against the fp64
oracle element by element.  The second batch carries indices outside [-1, S),
which the entry point treats as -1 (it has no caller workspace to report them
in).  The file sorts last so that a run that stops at the first failure has
run every other test.
"""
import dataclasses

import numpy as np
import pytest
import torch

from gather_matmul_b200 import _lib, ops
from gather_matmul_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _gpu_tensors(p):
    td = W.TORCH_DTYPE[p.dtype]
    mk = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(td).cuda()
    return mk(p.x), [mk(a) for a in p.A], torch.from_numpy(p.idx).cuda()


def test_noalloc_matches_workspace_entry_points_on_two_calls():
    import oracle
    probs = [
        W.make_problem("na1", W.BF16, T=300, D=2048, r=32, S=12, d_out=[8, 8], seed=31,
                       idx_kind="uniform_neg"),
        # second call: fewer tokens, more slots, another dtype and rank; any
        # state left by the first call would show here
        W.make_problem("na2", W.F16, T=77, D=4096, r=16, S=40, d_out=[8], seed=32,
                       idx_kind="frac_neg", frac_neg=0.3),
    ]
    # out-of-range indices in the second batch: treated as -1 (zero buf rows)
    bad = probs[1].idx.copy()
    bad[[4, 50]] = [40, -3]
    probs[1] = dataclasses.replace(probs[1], idx=bad)
    for p in probs:
        x, A, idx = _gpu_tensors(p)
        buf_ref = torch.full((len(A), p.T, p.r), float("nan"), device="cuda")
        meta = ops.workspace(p.T, p.S)
        ops.group(idx, p.S, meta)
        ops.shrink(x, A, idx, buf_ref, meta)
        buf = torch.full((len(A), p.T, p.r), float("nan"), device="cuda")
        ops.shrink_noalloc(x, A, idx, buf)
        torch.cuda.synchronize()
        # the oracle reads an index outside [0, S) as "no adapter"
        clean = np.where((p.idx >= 0) & (p.idx < p.S), p.idx, -1).astype(np.int32)
        o, cabs, _ = oracle.shrink(p.dtype, p.x, p.A, clean, p.S, want_cabs=True)
        g = buf.cpu().double().numpy()
        ref = buf_ref.cpu().double().numpy()
        assert np.all(np.isfinite(g)), "rows left unwritten"
        assert np.all(np.abs(g - ref) <= 1e-3 * np.abs(ref) + 1e-5 * cabs)
        assert np.all(np.abs(g - o) <= 1e-3 * np.abs(o) + 1e-5 * cabs)
        assert np.all(g[:, clean < 0] == 0.0)


def test_noalloc_rejects_sizes_beyond_its_array():
    p = W.make_problem("na3", W.BF16, T=8, D=64, r=16, S=4, d_out=[8], seed=33)
    x, A, idx = _gpu_tensors(p)
    buf = torch.zeros((1, p.T, p.r), device="cuda")
    big_T = _lib.LORA_NOALLOC_MAX_TOKENS + 1
    L = _lib.load()
    import ctypes
    arr = (ctypes.c_void_p * 1)(A[0].data_ptr())
    st = L.lora_shrink_noalloc(_lib.LORA_BF16, big_T, p.D, p.r, p.S, 1, x.data_ptr(), p.D, arr,
                               idx.data_ptr(), buf.data_ptr(), 1, None)
    assert st == _lib.LORA_ERR_UNSUPPORTED
