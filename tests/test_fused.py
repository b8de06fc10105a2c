"""GPU parity of the one-call per-token path (lora_bgmv): grouping, shrink and
expand in one fused launch when the shape fits, otherwise the three-launch
path; both against the fp64 oracle under the same tolerances as
test_parity.py, plus determinism, error counting and graph capture with
programmatic dependent launch."""
import dataclasses

import numpy as np
import pytest
import torch

from gather_matmul_b200 import _lib, ops
from gather_matmul_b200 import workloads as W

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from gpu_util import (Dev, assert_buf_close, assert_y_close, oracle_expand, oracle_shrink,
                          run_bgmv)


def _check(p, pdl_early=False):
    d = Dev(p)
    buf_ref, cabs = oracle_shrink(p)
    buf, y = run_bgmv(d, pdl_early)
    torch.cuda.synchronize()
    assert_buf_close(buf, buf_ref, cabs)
    assert_y_close(p, y, oracle_expand(p, buf.detach().cpu().double().numpy()), "y (own buf)")
    assert_y_close(p, y, oracle_expand(p, buf_ref), "y (end to end)")
    assert ops.check_errors(d.meta) == _lib.LORA_OK
    return d


CASES = [(n, k) for n in (1, 2, 3, 5) for k in range(3 if n == 3 else 1)]


@pytest.mark.parametrize("cfg,proj", CASES, ids=[f"cfg{n}-{k}" for n, k in CASES])
def test_bgmv_workloads_full_size(cfg, proj):
    _check(W.config(cfg)[proj], pdl_early=True)


RAGGED = [
    # dtype, T, D, r, S, d_out, idx_kind, shared_A
    (W.F16, 1, 16, 8, 1, [8], "uniform", False),
    (W.F16, 33, 1032, 8, 5, [264], "uniform_neg", False),
    (W.BF16, 70, 2056, 16, 3, [1024, 136], "frac_neg", False),
    (W.F16, 129, 4104, 32, 3, [512, 256, 128], "uniform_neg", True),
    (W.BF16, 300, 3000, 64, 4, [96, 1000], "uniform_neg", False),   # > 16 tokens per slot
    (W.BF16, 600, 520, 16, 2, [4096], "single", False),              # one hot slot, many chunks
    (W.F16, 17, 8, 16, 40, [24, 8], "uniform", False),                # tiny D, unused slots
    (W.BF16, 257, 64, 32, 300, [1024], "uniform_neg", False),
]


@pytest.mark.parametrize("case", RAGGED, ids=[f"{W.DTYPE_NAME[c[0]]}-T{c[1]}-D{c[2]}-r{c[3]}-S{c[4]}"
                                              for c in RAGGED])
def test_bgmv_ragged(case):
    dt, T, D, r, S, d_out, kind, shared = case
    p = W.make_problem("ragged", dt, T=T, D=D, r=r, S=S, d_out=d_out, scale=0.375, seed=T * 3 + D,
                       idx_kind=kind, frac_neg=0.3, shared_A=shared)
    assert ops.bgmv_launches(W.TORCH_DTYPE[dt], T, D, r, S, d_out) == 1
    _check(p)


def test_fused_matches_three_launch_path():
    p = W.make_problem("cmp", W.BF16, T=200, D=4096, r=16, S=12, d_out=[4096, 1024], seed=11,
                       idx_kind="uniform_neg")
    d1, d2 = Dev(p), Dev(p)
    run_bgmv(d1)
    d2.shrink()
    d2.expand()
    torch.cuda.synchronize()
    _, cabs = oracle_shrink(p)
    assert_buf_close(d1.buf, d2.buf.cpu().double().numpy(), cabs)
    assert_y_close(p, d1.y, oracle_expand(p, d2.buf.cpu().double().numpy()))


def test_fused_integer_inputs_bitwise():
    # x, A, B in {-1,0,1}, y in [-8,8]: every sum is an exact small integer,
    # also through the two-term split of the intermediate.
    import oracle
    from gpu_util import host_bits
    for dt, D in ((W.F16, 64), (W.BF16, 16)):
        p = W.make_problem("int", dt, T=40, D=D, r=16, S=3, d_out=[32, 16], scale=1.0, seed=5,
                           idx_kind="uniform_neg", values="int")
        d = Dev(p)
        buf, y = run_bgmv(d)
        torch.cuda.synchronize()
        buf_ref, _ = oracle_shrink(p)
        assert np.array_equal(buf.cpu().double().numpy(), buf_ref)
        assert np.array_equal(oracle.decode(p.dtype, host_bits(y)), oracle_expand(p, buf_ref))


def test_fused_deterministic_and_counts_bad_indices():
    p = W.make_problem("det", W.F16, T=256, D=4096, r=16, S=32, d_out=[4096], scale=2.0, seed=2,
                       idx_kind="uniform")
    idx = p.idx.copy()
    idx[5] = 99
    idx[9] = -4
    q = dataclasses.replace(p, idx=idx)
    d1, d2 = Dev(q), Dev(q)
    run_bgmv(d1)
    run_bgmv(d2)
    torch.cuda.synchronize()
    assert torch.equal(d1.buf, d2.buf) and torch.equal(d1.y, d2.y)
    assert ops.check_errors(d1.meta) == _lib.LORA_ERR_BAD_INDEX
    r = dataclasses.replace(p, idx=np.where((idx >= 0) & (idx < p.S), idx, -1).astype(np.int32))
    buf_ref, cabs = oracle_shrink(r)
    assert_buf_close(d1.buf, buf_ref, cabs)


def test_fused_graph_with_pdl_chain():
    # several consecutive calls on different batches, captured in one graph
    # with programmatic dependent launch, replayed: same as eager
    probs = [W.make_problem(f"g{k}", W.F16, T=256, D=4096, r=16, S=32, d_out=[4096], scale=2.0,
                            seed=40 + k, idx_kind="uniform") for k in range(4)]
    devs = [Dev(p) for p in probs]
    y_in = [d.y.clone() for d in devs]
    for d in devs:
        run_bgmv(d)
    torch.cuda.synchronize()
    y_eager = [d.y.clone() for d in devs]
    for d, y0 in zip(devs, y_in):
        d.y.copy_(y0)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        for d in devs:
            run_bgmv(d, pdl_early=True)
    for d, y0 in zip(devs, y_in):
        d.y.copy_(y0)
    g.replay()
    torch.cuda.synchronize()
    for d, ye in zip(devs, y_eager):
        assert torch.equal(d.y, ye)


def test_fused_no_active_does_nothing():
    p = W.make_problem("none", W.BF16, T=64, D=1024, r=16, S=4, d_out=[512], seed=1,
                       idx_kind="none")
    d = Dev(p)
    d.buf.fill_(7.0)
    y0 = d.y.clone()
    ops.bgmv(d.x, d.A, d.B, d.idx, d.y, d.buf, d.meta, p.scale, has_active=False)
    torch.cuda.synchronize()
    assert torch.all(d.buf == 7.0) and torch.equal(d.y, y0)
    run_bgmv(d)     # the kernel itself: zero intermediate rows, y untouched
    torch.cuda.synchronize()
    assert torch.all(d.buf == 0) and torch.equal(d.y, y0)


def test_grouped_flag_shares_one_grouping_across_projections():
    # One lora_group for the batch, then the three fused-slice decode
    # projections (the same indices) as lora_bgmv calls with LORA_FLAG_GROUPED
    # on that workspace: two launches each, no grouping.  Each against the
    # oracle.
    probs = W.config(3)
    for p in probs[1:]:
        assert np.array_equal(p.idx, probs[0].idx)
    devs = [Dev(p) for p in probs]
    meta = devs[0].meta
    ops.group(devs[0].idx, probs[0].S, meta)
    before = _lib.load().lora_launch_count()
    for p, d in zip(probs, devs):
        ops.bgmv(d.x, d.A, d.B, devs[0].idx, d.y, d.buf, meta, p.scale, y_col_off=p.col_off,
                 grouped=True)
    torch.cuda.synchronize()
    assert _lib.load().lora_launch_count() - before == 2 * len(probs)
    for p, d in zip(probs, devs):
        buf_ref, cabs = oracle_shrink(p)
        assert_buf_close(d.buf, buf_ref, cabs)
        assert_y_close(p, d.y, oracle_expand(p, buf_ref), "y (end to end)")
    assert ops.check_errors(meta) == _lib.LORA_OK


def test_grouped_flag_with_a_stale_grouping_is_reported():
    # The workspace grouped from another batch of the same size: the call
    # reports it (LORA_ERR_BAD_INDEX) instead of using it silently.
    p1 = W.config(3)[0]
    p2 = W.make_problem(p1.name, p1.dtype, p1.T, p1.D, p1.r, p1.S, p1.d_out, p1.scale,
                        seed=79, idx_kind="frac_neg", frac_neg=0.25)
    assert not np.array_equal(p1.idx, p2.idx)
    d1, d2 = Dev(p1), Dev(p2)
    ops.group(d1.idx, p1.S, d1.meta)
    ops.bgmv(d2.x, d2.A, d2.B, d2.idx, d2.y, d2.buf, d1.meta, p2.scale, y_col_off=p2.col_off,
             grouped=True)
    assert ops.check_errors(d1.meta) == _lib.LORA_ERR_BAD_INDEX


def test_early_grouping_right_after_a_grouping_on_the_same_workspace():
    # A stand-alone grouping of one batch, then at once a three-launch
    # lora_bgmv call of another batch with LORA_FLAG_PDL_EARLY on the same
    # workspace: the second grouping's CTAs exchange their counts through the
    # workspace before waiting for the first grouping, which must have
    # finished its own exchange before the second one can start.  Batches of
    # 4096 tokens use several grouping CTAs.  Result against the oracle.
    p1 = W.config(5)[0]
    p2 = W.make_problem(p1.name, p1.dtype, p1.T, p1.D, p1.r, p1.S, p1.d_out, p1.scale,
                        seed=78, idx_kind="uniform_neg")
    d1, d2 = Dev(p1), Dev(p2)
    d2.meta = d1.meta
    y0 = d2.y.clone()
    for _ in range(3):
        d2.y.copy_(y0)
        ops.group(d1.idx, p1.S, d1.meta)
        run_bgmv(d2, pdl_early=True)
    torch.cuda.synchronize()
    buf_ref, cabs = oracle_shrink(p2)
    assert_buf_close(d2.buf, buf_ref, cabs)
    assert_y_close(p2, d2.y, oracle_expand(p2, buf_ref), "y (end to end)")
    assert ops.check_errors(d1.meta) == _lib.LORA_OK


def test_back_to_back_calls_share_a_workspace_with_early_grouping():
    # Two three-launch lora_bgmv calls (grouping, shrink, expand) on ONE
    # workspace, different batches, LORA_FLAG_PDL_EARLY: the second call's
    # grouping reads and counts its indices while the first call's expand may
    # still be reading the grouping held in the workspace; it must write the
    # workspace only after that expand has finished.  Both results against the
    # oracle.
    p1 = W.config(5)[0]
    p2 = W.make_problem(p1.name, p1.dtype, p1.T, p1.D, p1.r, p1.S, p1.d_out, p1.scale,
                        seed=77, idx_kind="uniform_neg")
    assert ops.bgmv_launches(W.TORCH_DTYPE[p1.dtype], p1.T, p1.D, p1.r, p1.S, p1.d_out) == 3
    d1, d2 = Dev(p1), Dev(p2)
    d2.meta = d1.meta
    for _ in range(2):             # the second round also follows a call on the same stream
        d1.y.copy_(Dev(p1).y)
        d2.y.copy_(Dev(p2).y)
        run_bgmv(d1, pdl_early=True)
        run_bgmv(d2, pdl_early=True)
    torch.cuda.synchronize()
    for p, d in ((p1, d1), (p2, d2)):
        buf_ref, cabs = oracle_shrink(p)
        assert_buf_close(d.buf, buf_ref, cabs)
        assert_y_close(p, d.y, oracle_expand(p, buf_ref), "y (end to end)")
    assert ops.check_errors(d1.meta) == _lib.LORA_OK
