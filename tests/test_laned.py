"""GPU parity of the laned shrink (lora_shrink_laned): every slot's adapter
as one [S*r, D] matrix in a dense tensor-core contraction, each token keeping
its own slot's lanes, with no grouping ("[Hardware][TPU][V1] Better tpu
multilora compilation", the LoRA laning of the TPU kernels).  Against the
fp64 oracle under the buf tolerance of the other parity tests, at the decode
and tiny workloads' full sizes and on ragged shapes (token and lane tiles
with tails, K not a multiple of the 64-wide stage, several slices), plus
integer-exact bitwise agreement, bad-index counting and determinism."""
import dataclasses

import numpy as np
import pytest
import torch

from gather_matmul_b200 import _lib, ops
from gather_matmul_b200 import workloads as W

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from gpu_util import Dev, assert_buf_close, oracle_shrink


def _laned(d):
    ops.shrink_laned(d.x, d.A, d.idx, d.buf, d.meta)
    torch.cuda.synchronize()
    return d.buf


@pytest.mark.parametrize("cfg", [1, 2], ids=["cfg1-tiny", "cfg2-decode-q-proj"])
def test_laned_workloads_full_size(cfg):
    p = W.config(cfg)[0]
    d = Dev(p)
    buf_ref, cabs = oracle_shrink(p)
    assert_buf_close(_laned(d), buf_ref, cabs)
    assert ops.check_errors(d.meta) == _lib.LORA_OK


CASES = [
    # dtype, T, D, r, S, n_slices, idx_kind
    (W.BF16, 300, 1032, 64, 5, 1, "uniform_neg"),    # 3 token tiles, 320 lanes, K tail
    (W.F16, 1, 64, 8, 40, 1, "uniform"),             # one token, 320 lanes of rank 8
    (W.BF16, 129, 4104, 32, 9, 3, "frac_neg"),       # three slices, one-row token tail
    (W.F16, 520, 2048, 16, 12, 2, "zipf"),
    (W.BF16, 64, 8, 16, 3, 1, "uniform_neg"),        # D smaller than one stage
]


@pytest.mark.parametrize("case", CASES, ids=[f"{W.DTYPE_NAME[c[0]]}-T{c[1]}-D{c[2]}-r{c[3]}-S{c[4]}-n{c[5]}"
                                             for c in CASES])
def test_laned_ragged_shapes(case):
    dt, T, D, r, S, n, kind = case
    p = W.make_problem("laned", dt, T=T, D=D, r=r, S=S, d_out=[8] * n, scale=1.0, seed=T + D + r,
                       idx_kind=kind, frac_neg=0.3)
    d = Dev(p)
    buf_ref, cabs = oracle_shrink(p)
    assert_buf_close(_laned(d), buf_ref, cabs)


def test_laned_matches_grouped_path():
    p = W.make_problem("cmp", W.BF16, T=256, D=4096, r=16, S=32, d_out=[8], seed=91,
                       idx_kind="uniform_neg")
    d1, d2 = Dev(p), Dev(p)
    b1 = _laned(d1)
    b2 = d2.shrink()
    torch.cuda.synchronize()
    _, cabs = oracle_shrink(p)
    assert_buf_close(b1, b2.detach().cpu().double().numpy(), cabs)


def test_laned_integer_inputs_bitwise():
    # x, A in {-1,0,1}: every lane sum is a small integer, exact in fp32
    import oracle  # noqa: F401
    for dt, D in ((W.F16, 64), (W.BF16, 1024)):
        p = W.make_problem("int", dt, T=200, D=D, r=16, S=9, d_out=[8], scale=1.0, seed=D,
                           idx_kind="uniform_neg", values="int")
        d = Dev(p)
        buf_ref, _ = oracle_shrink(p)
        assert np.array_equal(_laned(d).cpu().double().numpy(), buf_ref)


def test_laned_bad_indices_and_determinism():
    p = W.make_problem("bad", W.F16, T=150, D=2048, r=16, S=20, d_out=[8], seed=92,
                       idx_kind="uniform")
    idx = p.idx.copy()
    idx[[7, 140]] = [20, -5]
    q = dataclasses.replace(p, idx=idx)
    d1, d2 = Dev(q), Dev(q)
    b1, b2 = _laned(d1).clone(), _laned(d2).clone()
    assert torch.equal(b1, b2)
    assert ops.check_errors(d1.meta) == _lib.LORA_ERR_BAD_INDEX
    clean = dataclasses.replace(p, idx=np.where((idx >= 0) & (idx < p.S), idx, -1).astype(np.int32))
    buf_ref, cabs = oracle_shrink(clean)
    assert_buf_close(b1, buf_ref, cabs)
    assert torch.all(b1[:, [7, 140]] == 0)


def test_laned_no_active_enqueues_nothing():
    p = W.make_problem("none", W.BF16, T=64, D=1024, r=16, S=4, d_out=[8], seed=93,
                       idx_kind="none")
    d = Dev(p)
    d.buf.fill_(3.0)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ops.shrink_laned(d.x, d.A, d.idx, d.buf, d.meta, idx_host=p.idx)
    assert s.query()
    torch.cuda.synchronize()
    assert torch.all(d.buf == 3.0)
