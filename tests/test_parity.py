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

from gather_matmul_b200 import _lib, ops
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


@pytest.mark.parametrize("cfg", [4, 5], ids=["cfg4-prefill-f16", "cfg5-large-mixed-f16"])
def test_tensor_core_workloads_full_size_fp16(cfg):
    """The two workloads that run on the tcgen05 kernels (prefill segments and
    the large mixed per-token batch through the grouping), drawn in fp16: the
    fp16 instruction descriptors, the fp16 hi + lo split of the intermediate
    and fp16 rounding of y, at full size."""
    p = W.config(cfg, dtype=W.F16)[0]
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


def _many_segments(n_seg, seg_len, S, every_neg):
    ss = np.arange(n_seg + 1, dtype=np.int64) * seg_len
    sa = np.array([-1 if (i % every_neg) == every_neg - 1 else i % S for i in range(n_seg)])
    return ss, sa


def test_sgmv_many_tiles_per_cta():
    """2048 segments of 8 tokens over 8 output slices of 128 columns: about
    a hundred tile runs per CTA of the persistent expand, more than one run
    list holds, so the lists are rebuilt mid-kernel."""
    ss, sa = _many_segments(2048, 8, 16, 7)
    p = W.make_problem("many_tiles", W.BF16, T=int(ss[-1]), D=64, r=16, S=16,
                       d_out=[128] * 8, scale=0.75, seed=11, segments=(ss, sa))
    _run_and_check(p)


def test_sgmv_long_segment_list_item_kernels():
    """More than 2048 segments: the segment calls take the item kernels."""
    ss, sa = _many_segments(2050, 2, 5, 4)
    p = W.make_problem("long_list", W.F16, T=int(ss[-1]), D=256, r=32, S=5,
                       d_out=[256], scale=1.5, seed=12, segments=(ss, sa))
    _run_and_check(p)


def test_sgmv_many_mixed_segments():
    """Forty segments of mixed lengths (1 to 513 tokens, some without an
    adapter, adapters repeated): more tiles than the GPU has SMs, full and
    partial tiles interleaved."""
    rng = np.random.default_rng(13)
    lens = rng.choice([1, 37, 128, 200, 256, 300, 513], size=40)
    ss = np.concatenate([[0], np.cumsum(lens)])
    sa = rng.integers(-1, 6, size=40)
    p = W.make_problem("mixed_segments", W.BF16, T=int(ss[-1]), D=1024, r=32, S=6,
                       d_out=[512], scale=0.5, seed=13, segments=(ss, sa))
    _run_and_check(p)


RANDOM_SEGMENT_SEEDS = list(range(8))


@pytest.mark.parametrize("seed", RANDOM_SEGMENT_SEEDS)
def test_sgmv_random_segment_layouts(seed):
    """Random segment lists (empty segments, repeats, no-adapter runs, lengths
    around the 64- and 128-row tile boundaries) over 1-3 slices whose widths
    are not multiples of 128: every tile shape and schedule split of the
    tensor-core kernels against the oracle."""
    rng = np.random.default_rng(100 + seed)
    n_seg = int(rng.integers(1, 60))
    lens = rng.choice([0, 1, 3, 8, 31, 63, 64, 65, 127, 128, 129, 200, 257], size=n_seg)
    if lens.sum() == 0:
        lens[0] = 5
    ss = np.concatenate([[0], np.cumsum(lens)])
    S = int(rng.integers(1, 9))
    sa = rng.integers(-1, S, size=n_seg)
    r = int(rng.choice([16, 32, 64]))
    d_out = [int(rng.choice([8, 136, 256, 392])) for _ in range(int(rng.integers(1, 4)))]
    dt = W.BF16 if seed % 2 else W.F16
    p = W.make_problem("random_segments", dt, T=int(ss[-1]), D=int(rng.choice([64, 264, 1024])),
                       r=r, S=S, d_out=d_out, scale=0.75, seed=200 + seed, segments=(ss, sa))
    _run_and_check(p)


@pytest.mark.parametrize("seed", list(range(6)))
def test_grouped_random_batches(seed):
    """Random per-token batches with at least 16 tokens per slot on average,
    so the grouping feeds the tensor-core kernels: skewed and uniform slot
    popularity, tokens without an adapter, slot groups of every size."""
    rng = np.random.default_rng(300 + seed)
    S = int(rng.integers(1, 24))
    T = int(16 * S + rng.integers(0, 700))
    kind = ["uniform", "uniform_neg", "zipf", "frac_neg", "single", "uniform"][seed]
    r = [16, 32, 64][seed % 3]
    d_out = [int(rng.choice([64, 200, 512])) for _ in range(1 + seed % 3)]
    p = W.make_problem("grouped_random", W.BF16 if seed % 2 else W.F16, T=T,
                       D=int(rng.choice([128, 776, 2048])), r=r, S=S, d_out=d_out, scale=1.25,
                       seed=400 + seed, idx_kind=kind, frac_neg=0.2)
    _run_and_check(p)


def _sgmv_case(name):
    if name == "prefill-full-size":
        return W.config(4)[0]
    if name == "mixed":
        rng = np.random.default_rng(21)
        lens = rng.choice([0, 1, 37, 64, 65, 128, 200, 513], size=30)
        ss = np.concatenate([[0], np.cumsum(lens)])
        sa = rng.integers(-1, 6, size=30)
        return W.make_problem("sgmv_mixed", W.BF16, T=int(ss[-1]), D=1024, r=32, S=6,
                              d_out=[512, 136], scale=0.5, seed=21, segments=(ss, sa))
    if name == "long-list":                     # > 2048 segments: CUDA-core item kernels
        ss, sa = _many_segments(2050, 2, 5, 4)
        return W.make_problem("sgmv_long", W.F16, T=int(ss[-1]), D=256, r=32, S=5,
                              d_out=[256], scale=1.5, seed=22, segments=(ss, sa))
    ss, sa = np.array([0, 100, 300, 301, 700]), np.array([2, -1, 0, 3])
    return W.make_problem("sgmv_shared", W.F16, T=700, D=512, r=64, S=4,
                          d_out=[256, 128, 128], scale=2.0, seed=23, segments=(ss, sa),
                          shared_A=True)


@pytest.mark.parametrize("name", ["prefill-full-size", "mixed", "long-list", "shared-A"])
def test_sgmv_one_call(name):
    """lora_sgmv (segment shrink + expand in one call, the expand started
    while the shrink finishes) against the oracle."""
    p = _sgmv_case(name)
    d = Dev(p)
    buf_ref, cabs = oracle_shrink(p)
    ops.sgmv(d.x, d.A, d.B, d.ss, d.sa, d.y, d.buf, d.meta, p.scale, y_col_off=p.col_off)
    torch.cuda.synchronize()
    assert_buf_close(d.buf, buf_ref, cabs)
    assert_y_close(p, d.y, oracle_expand(p, buf_ref), "y (end to end)")
    assert ops.check_errors(d.meta) == _lib.LORA_OK


def test_sgmv_one_call_idle_writes_nothing():
    p = _sgmv_case("mixed")
    d = Dev(p)
    y0 = d.y.clone()
    ops.sgmv(d.x, d.A, d.B, d.ss, d.sa, d.y, d.buf, d.meta, p.scale, y_col_off=p.col_off,
             has_active=False)
    torch.cuda.synchronize()
    assert torch.equal(d.y, y0)
    assert torch.isnan(d.buf).all()


@pytest.mark.parametrize("seed", list(range(4)))
def test_grouped_many_slots(seed):
    """Per-token batches over 64 or more slots: the shrink cuts tiles at 96
    rows (a slot's tokens then span full 96-row tiles and a short last one,
    of every length), with skewed, uniform and one-hot popularity and tokens
    without an adapter."""
    rng = np.random.default_rng(500 + seed)
    S = int(rng.integers(64, 200))
    T = int(16 * S + rng.integers(0, 900))
    kind = ["zipf", "uniform_neg", "frac_neg", "single"][seed]
    r = [32, 16, 64, 32][seed]
    d_out = [[512], [136, 64], [256], [392, 8]][seed]
    p = W.make_problem("many_slots", W.BF16 if seed % 2 else W.F16, T=T,
                       D=int(rng.choice([512, 1032, 4096])), r=r, S=S, d_out=d_out, scale=0.75,
                       seed=600 + seed, idx_kind=kind, frac_neg=0.15)
    _run_and_check(p)
