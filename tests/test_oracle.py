"""Pins for the fp64 CPU oracle (no GPU).

Each check ties the oracle to something other than itself: exact element
decoding checked against numpy / torch over every bit pattern, a worked example
computed by hand (tests/golden), a dense special case computed by
torch.matmul, the ref_bgmv gather-then-batched-matmul formulation run through
numpy einsum, closed forms, and invariants (-1 rows untouched, linearity in
scale, permutation equivariance).  The mutation test at the end plants
plausible mistakes in copies of the oracle source and checks that some pin
catches every one of them.
"""
import json
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest
import torch

import oracle
from gather_matmul_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ref_bgmv_tiny.json")


def _bits(vals, dtype):
    return W._round_bits(np.asarray(vals, dtype=np.float64), dtype)


def _dec(p, a):
    return oracle.decode(p.dtype, a)


def _small(seed, dtype=W.F16, T=9, D=24, r=8, S=3, d_out=(16, 8), idx_kind="uniform_neg",
           shared_A=False, values="normal", scale=1.5):
    return W.make_problem("small", dtype, T=T, D=D, r=r, S=S, d_out=list(d_out),
                          scale=scale, seed=seed, idx_kind=idx_kind, shared_A=shared_A,
                          values=values)


# ---------------------------------------------------------------- checks
# Plain functions so that the mutation test can run them against broken
# copies of the oracle.

def check_decode_f16():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.decode(oracle.F16, bits)
    want = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


def check_decode_bf16():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.decode(oracle.BF16, bits)
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


def check_golden():
    g = json.load(open(GOLDEN))
    dt = oracle.F16
    x = _bits(g["x"], dt)
    A = _bits(g["A"], dt)
    B = _bits(g["B"], dt)
    yo = _bits(g["y_old"], dt)
    idx = np.array(g["idx"], dtype=np.int32)
    buf, bad = oracle.shrink(dt, x, [A], idx, g["S"])
    assert bad == 0
    assert np.array_equal(buf[0], np.array(g["buf"], dtype=np.float64))
    y, _ = oracle.expand(dt, buf, [B], idx, g["S"], g["scale"], yo, [0])
    assert np.array_equal(y, np.array(g["y"], dtype=np.float64))
    sg = g["segments"]
    buf, rc = oracle.shrink_segment(dt, x, [A], sg["seg_starts"], sg["seg_adapter"], g["S"])
    assert rc == 0
    assert np.array_equal(buf[0], np.array(sg["buf"], dtype=np.float64))
    y, rc = oracle.expand_segment(dt, buf, [B], sg["seg_starts"], sg["seg_adapter"], g["S"],
                                  g["scale"], yo, [0])
    assert rc == 0
    assert np.array_equal(y, np.array(sg["y"], dtype=np.float64))


def check_minus_one_rows_untouched():
    for dt in (W.F16, W.BF16):
        p = _small(11, dtype=dt, T=17)
        buf, _ = oracle.shrink(dt, p.x, p.A, p.idx, p.S)
        y, _ = oracle.expand(dt, buf, p.B, p.idx, p.S, p.scale, p.y, p.col_off)
        neg = p.idx == -1
        assert neg.any() and (~neg).any()
        assert np.all(buf[:, neg, :] == 0.0)
        yo = _dec(p, p.y)
        assert np.array_equal(y[neg], yo[neg])
        # tokens with an adapter do change
        assert not np.array_equal(y[~neg], yo[~neg])


def check_single_adapter_equals_dense():
    # one adapter for the whole batch: y = y_old + scale * (x A^T) B^T per slice
    for dt in (W.F16, W.BF16):
        p = _small(12, dtype=dt, T=7, D=40, r=16, S=4, d_out=(24, 16), idx_kind="single")
        x = torch.from_numpy(_dec(p, p.x))
        y0 = torch.from_numpy(_dec(p, p.y))
        buf, _ = oracle.shrink(dt, p.x, p.A, p.idx, p.S)
        y, _ = oracle.expand(dt, buf, p.B, p.idx, p.S, p.scale, p.y, p.col_off)
        want = y0.clone()
        for i in range(p.n_slices):
            Ai = torch.from_numpy(_dec(p, p.A[i])[0])          # [r, D]
            Bi = torch.from_numpy(_dec(p, p.B[i])[0])          # [D_out, r]
            h = torch.matmul(x, Ai.T)
            np.testing.assert_allclose(buf[i], h.numpy(), rtol=1e-12, atol=1e-12)
            c0 = p.col_off[i]
            want[:, c0:c0 + p.d_out[i]] += p.scale * torch.matmul(h, Bi.T)
        np.testing.assert_allclose(y, want.numpy(), rtol=1e-12, atol=1e-12)


def check_gather_einsum_formulation():
    # ref_bgmv's own shape of the computation: gather the per-token matrices,
    # then one batched contraction (numpy einsum), with -1 masked out.
    for dt, shared in ((W.F16, False), (W.BF16, True)):
        p = _small(13, dtype=dt, T=13, D=32, r=8, S=5, d_out=(8, 24, 16), shared_A=shared)
        x = _dec(p, p.x)
        idx = p.idx
        act = (idx >= 0).astype(np.float64)
        safe = np.where(idx >= 0, idx, 0)
        buf, _ = oracle.shrink(dt, p.x, p.A, idx, p.S)
        for i, Ab in enumerate(p.A):
            sel = _dec(p, Ab)[safe]                              # [T, r, D]
            want = np.einsum("trd,td->tr", sel, x) * act[:, None]
            np.testing.assert_allclose(buf[i], want, rtol=1e-12, atol=1e-12)
        y, _ = oracle.expand(dt, buf[0] if shared else buf, p.B, idx, p.S, p.scale, p.y,
                             p.col_off, shared_buf=shared)
        want = _dec(p, p.y).copy()
        for i, Bb in enumerate(p.B):
            sel = _dec(p, Bb)[safe]                              # [T, D_out, r]
            bi = buf[0] if shared else buf[i]
            c0 = p.col_off[i]
            want[:, c0:c0 + p.d_out[i]] += p.scale * np.einsum("tor,tr->to", sel, bi) * act[:, None]
        np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)


def check_linear_in_scale():
    p = _small(14, T=11)
    buf, _ = oracle.shrink(p.dtype, p.x, p.A, p.idx, p.S)
    yo = _dec(p, p.y)
    y1, _ = oracle.expand(p.dtype, buf, p.B, p.idx, p.S, 0.75, p.y, p.col_off)
    y2, _ = oracle.expand(p.dtype, buf, p.B, p.idx, p.S, 1.5, p.y, p.col_off)
    y0, _ = oracle.expand(p.dtype, buf, p.B, p.idx, p.S, 0.0, p.y, p.col_off)
    assert np.array_equal(y0, yo)
    np.testing.assert_allclose(y2 - yo, 2.0 * (y1 - yo), rtol=1e-12, atol=1e-14)
    assert np.abs(y1 - yo).max() > 0


def check_permutation_equivariance():
    p = _small(15, T=12)
    rng = np.random.default_rng(0)
    perm = rng.permutation(p.T)
    buf, _ = oracle.shrink(p.dtype, p.x, p.A, p.idx, p.S)
    y, _ = oracle.expand(p.dtype, buf, p.B, p.idx, p.S, p.scale, p.y, p.col_off)
    bufp, _ = oracle.shrink(p.dtype, p.x[perm], p.A, p.idx[perm], p.S)
    yp, _ = oracle.expand(p.dtype, bufp, p.B, p.idx[perm], p.S, p.scale, p.y[perm], p.col_off)
    assert np.array_equal(bufp, buf[:, perm, :])
    assert np.array_equal(yp, y[perm])


def check_one_hot_closed_form():
    # x = e_d  =>  buf[t] = A[idx[t]][:, d]
    p = _small(16, T=6, D=16, r=8, S=3, d_out=(8,), idx_kind="uniform")
    D = p.D
    ds = np.arange(p.T) % D * 3 % D
    xv = np.zeros((p.T, D))
    xv[np.arange(p.T), ds] = 1.0
    x = _bits(xv, p.dtype)
    buf, _ = oracle.shrink(p.dtype, x, p.A, p.idx, p.S)
    Ad = _dec(p, p.A[0])
    for t in range(p.T):
        assert np.array_equal(buf[0, t], Ad[p.idx[t], :, ds[t]])


def check_segments():
    p = _small(17, T=10, idx_kind="uniform")
    ss = np.array([0, 3, 3, 7, 10], dtype=np.int32)      # includes an empty segment
    sa = np.array([2, 0, -1, 1], dtype=np.int32)
    idx = oracle.segments_to_idx(p.T, ss, sa)
    assert idx.tolist() == [2, 2, 2, -1, -1, -1, -1, 1, 1, 1]
    b1, rc = oracle.shrink_segment(p.dtype, p.x, p.A, ss, sa, p.S)
    b2, _ = oracle.shrink(p.dtype, p.x, p.A, idx, p.S)
    assert rc == 0 and np.array_equal(b1, b2)
    y1, rc = oracle.expand_segment(p.dtype, b1, p.B, ss, sa, p.S, p.scale, p.y, p.col_off)
    y2, _ = oracle.expand(p.dtype, b2, p.B, idx, p.S, p.scale, p.y, p.col_off)
    assert rc == 0 and np.array_equal(y1, y2)
    # malformed segment lists are rejected
    for bad in ([1, 3, 3, 7, 10], [0, 3, 2, 7, 10], [0, 3, 3, 7, 9]):
        assert oracle.segments_to_idx(p.T, np.array(bad), sa) is None


def check_group_by_slot():
    rng = np.random.default_rng(1)
    for T, S in ((1, 1), (37, 4), (500, 16), (64, 300)):
        idx = rng.integers(-1, S, size=T).astype(np.int32)
        perm, off, bad = oracle.group_by_slot(idx, S)
        act = np.nonzero(idx >= 0)[0]
        want = act[np.argsort(idx[act], kind="stable")]
        assert bad == 0
        assert np.array_equal(perm, want)
        assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(idx[act], minlength=S))]))


def check_bad_index_is_no_adapter():
    p = _small(18, T=8, idx_kind="uniform")
    idx = p.idx.copy()
    idx[1] = p.S          # out of range high
    idx[5] = -7           # out of range low
    ref = idx.copy()
    ref[[1, 5]] = -1
    b1, bad = oracle.shrink(p.dtype, p.x, p.A, idx, p.S)
    b2, bad2 = oracle.shrink(p.dtype, p.x, p.A, ref, p.S)
    assert bad == 2 and bad2 == 0 and np.array_equal(b1, b2)
    y1, bad = oracle.expand(p.dtype, b1, p.B, idx, p.S, p.scale, p.y, p.col_off)
    y2, _ = oracle.expand(p.dtype, b2, p.B, ref, p.S, p.scale, p.y, p.col_off)
    assert bad == 2 and np.array_equal(y1, y2)
    perm, off, bad = oracle.group_by_slot(idx, p.S)
    assert bad == 2 and 1 not in perm and 5 not in perm


def check_columns_and_shared_buf():
    # slices write only their own columns; a shared intermediate equals the
    # same intermediate replicated per slice
    p = _small(19, T=8, d_out=(8, 16), shared_A=True)
    buf, _ = oracle.shrink(p.dtype, p.x, p.A, p.idx, p.S)
    assert buf.shape[0] == 1
    ldy = p.y.shape[1] + 8
    yo = np.zeros((p.T, ldy), dtype=np.uint16)
    yo[:, :p.y.shape[1]] = p.y
    yo[:, p.y.shape[1]:] = _bits(np.full((p.T, 8), 3.0), p.dtype)
    off = [p.y.shape[1] - 8 - 16 + 8, 0]           # slice 0 at col 8, slice 1 at col 0 .. 15
    B = [p.B[0], p.B[1]]
    ys, _ = oracle.expand(p.dtype, buf[0], B, p.idx, p.S, p.scale, yo, off, shared_buf=True)
    yr, _ = oracle.expand(p.dtype, np.repeat(buf, 2, axis=0), B, p.idx, p.S, p.scale, yo, off)
    assert np.array_equal(ys, yr)
    assert np.all(ys[:, p.y.shape[1]:] == 3.0)
    # with the slices reversed, slice 1 (16 wide) covers cols 0..15, slice 0 cols 16..23
    act = p.idx >= 0
    assert not np.array_equal(ys[act, 0:16], _dec(p, yo)[act, 0:16])


def check_cabs_bounds():
    p = _small(20, T=9)
    buf, cabs, _ = oracle.shrink(p.dtype, p.x, p.A, p.idx, p.S, want_cabs=True)
    assert np.all(np.abs(buf) <= cabs + 0.0)
    act = p.idx >= 0
    assert np.all(cabs[:, act, :] > 0)


def check_integer_values_exact():
    # x, A, B in {-1,0,1}, y in [-8, 8]: every intermediate is a small integer
    p = _small(21, T=10, D=64, r=8, d_out=(16,), values="int", scale=1.0)
    buf, _ = oracle.shrink(p.dtype, p.x, p.A, p.idx, p.S)
    assert np.array_equal(buf, np.round(buf)) and np.abs(buf).max() <= 64
    y, _ = oracle.expand(p.dtype, buf, p.B, p.idx, p.S, 1.0, p.y, p.col_off)
    assert np.array_equal(y, np.round(y))


CHECKS = [check_decode_f16, check_decode_bf16, check_golden, check_minus_one_rows_untouched,
          check_single_adapter_equals_dense, check_gather_einsum_formulation,
          check_linear_in_scale, check_permutation_equivariance, check_one_hot_closed_form,
          check_segments, check_group_by_slot, check_bad_index_is_no_adapter,
          check_columns_and_shared_buf, check_cabs_bounds, check_integer_values_exact]


@pytest.mark.parametrize("check", CHECKS, ids=[c.__name__ for c in CHECKS])
def test_oracle_pin(check):
    check()


# ---------------------------------------------------------------- mutations
# Each entry replaces one snippet of the oracle source with a plausible
# mistake; at least one pin above must then fail.
MUTANTS = {
    "f16_subnormal_exponent": ("ldexp((double)f, -24)", "ldexp((double)f, -25)"),
    "bf16_bias": ("ldexp((double)(128 + f), e - 134)", "ldexp((double)(128 + f), e - 133)"),
    "minus_one_wraps_to_last_slot": ("return (a >= 0 && a < S) ? a : -1;",
                                     "return (a >= 0 && a < S) ? a : (a == -1 ? S - 1 : -1);"),
    "dropped_first_term": ("            s += p;", "            s += (d == 0 ? 0.0 : p);"),
    "wrong_row_of_A": ("Ai + ((int64_t)a * r + j) * D", "Ai + ((int64_t)a * r + (j + 1) % r) * D"),
    "expand_wrong_sign": ("y_out[(int64_t)t * ldy + y_col_off[i] + o] += scale * s;",
                          "y_out[(int64_t)t * ldy + y_col_off[i] + o] -= scale * s;"),
    "scale_dropped": ("y_out[(int64_t)t * ldy + y_col_off[i] + o] += scale * s;",
                      "y_out[(int64_t)t * ldy + y_col_off[i] + o] += s;"),
    "slice_offset_dropped": ("y_out[(int64_t)t * ldy + y_col_off[i] + o]",
                             "y_out[(int64_t)t * ldy + o]"),
    "slice_stride_dropped": ("buf + (int64_t)i * buf_slice_stride", "buf + 0 * buf_slice_stride"),
    "B_transposed": ("s += bt[j] * dec(dtype, row[j]);",
                     "s += bt[j] * dec(dtype, Bi[((int64_t)a * r + j) * D_out[i] + o]);"),
    "unstable_grouping": ("if (a >= 0) perm[fill[a]++] = t;",
                          "if (a >= 0) perm[slot_off[a + 1] - 1 - (fill[a]++ - slot_off[a])] = t;"),
    "segment_off_by_one": ("for (int t = seg_starts[s]; t < seg_starts[s + 1]; ++t)",
                           "for (int t = seg_starts[s]; t < seg_starts[s + 1] && t + 1 < T; ++t)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    old, new = MUTANTS[name]
    src = open(oracle._build.SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    with tempfile.TemporaryDirectory() as d:
        msrc = os.path.join(d, "mutant.c")
        open(msrc, "w").write(src.replace(old, new))
        mlib = os.path.join(d, "libmutant.so")
        oracle._build.build(force=True, src=msrc, out=mlib)
        failed = []
        with oracle.use_library(mlib):
            for c in CHECKS:
                try:
                    c()
                except (AssertionError, ValueError, IndexError):
                    failed.append(c.__name__)
        assert failed, f"no pin caught the planted mistake {name}"
