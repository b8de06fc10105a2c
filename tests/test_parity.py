"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.

Tolerances (fixed by the target): fp32 intermediate within
|g - o| <= 1e-3 |o| + 1e-5 sum_d |x_d A_jd|, fp16/bf16 outputs within
|g - o| <= 1e-2 (1 + |o|), rows of tokens without an adapter bit-identical.
Expand is checked twice: alone (fed the GPU's own buf, oracle expand of that
same fp32 buf) and end to end (GPU shrink then expand vs oracle in fp64).
"""
import numpy as np
import pytest
import torch

from gather_matmul_b200 import workloads as W

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from gpu_util import (Dev, assert_buf_close, assert_y_close, oracle_expand,
                          oracle_shrink)


def _run_and_check(p, path=None):
    d = Dev(p)
    buf_ref, cabs = oracle_shrink(p)
    buf = d.shrink(path)
    torch.cuda.synchronize()
    assert_buf_close(buf, buf_ref, cabs)
    # expand alone: the oracle expands the GPU's own fp32 intermediate
    y_alone = oracle_expand(p, buf.detach().cpu().double().numpy())
    y = d.expand(path=path)
    torch.cuda.synchronize()
    assert_y_close(p, y, y_alone, "y (expand alone)")
    # end to end against the fp64 oracle
    y_e2e = oracle_expand(p, buf_ref)
    assert_y_close(p, y, y_e2e, "y (end to end)")
    return d


CONFIG_CASES = [(n, k) for n in (1, 2, 3, 4, 5) for k in range(3 if n == 3 else 1)]


@pytest.mark.parametrize("cfg,proj", CONFIG_CASES,
                         ids=[f"cfg{n}-{k}" for n, k in CONFIG_CASES])
def test_config_full_size(cfg, proj):
    """Every workload at its full size, every output element compared."""
    p = W.config(cfg)[proj]
    _run_and_check(p)


SHAPES = [
    # dtype, T, D, r, S, d_out, idx_kind, shared_A
    (W.F16, 1, 8, 8, 1, [8], "uniform", False),
    (W.F16, 37, 1032, 8, 5, [264], "uniform_neg", False),
    (W.BF16, 50, 2056, 16, 7, [1024, 136], "frac_neg", False),
    (W.F16, 129, 4104, 32, 3, [512, 256, 128], "uniform_neg", True),
    (W.BF16, 77, 3000, 64, 4, [96, 1000], "uniform_neg", False),
    (W.BF16, 300, 520, 64, 2, [4096], "single", False),
    (W.F16, 16, 11264, 16, 33, [8], "uniform", False),
    (W.BF16, 257, 64, 32, 300, [1024], "uniform_neg", False),
]


@pytest.mark.parametrize("case", SHAPES, ids=[f"{W.DTYPE_NAME[c[0]]}-T{c[1]}-D{c[2]}-r{c[3]}-S{c[4]}"
                                               for c in SHAPES])
def test_bgmv_ragged_shapes(case):
    dt, T, D, r, S, d_out, kind, shared = case
    p = W.make_problem("ragged", dt, T=T, D=D, r=r, S=S, d_out=d_out, scale=0.625, seed=T + D,
                       idx_kind=kind, frac_neg=0.3, shared_A=shared)
    _run_and_check(p)


SEGMENTS = [
    # dtype, D, r, S, d_out, seg_starts, seg_adapter
    (W.BF16, 4096, 64, 8, [4096], [0, 1024, 2048], [3, 5]),
    (W.BF16, 520, 16, 4, [264, 8], [0, 5, 5, 200, 333, 334, 500], [1, 2, -1, 0, 3, 1]),
    (W.F16, 1024, 32, 3, [512], [0, 129, 130, 383, 384], [0, 1, 2, 0]),
    (W.F16, 256, 8, 2, [64], [0, 7, 19], [1, -1]),
    (W.BF16, 2048, 64, 6, [1024, 512], [0, 640, 700, 1500], [5, 4, 5]),
]


@pytest.mark.parametrize("case", SEGMENTS, ids=[f"seg{i}" for i in range(len(SEGMENTS))])
def test_sgmv_segments(case):
    dt, D, r, S, d_out, ss, sa = case
    T = ss[-1]
    p = W.make_problem("segments", dt, T=T, D=D, r=r, S=S, d_out=d_out, scale=1.25,
                       seed=len(ss) * 7 + D, segments=(np.array(ss), np.array(sa)))
    _run_and_check(p)
