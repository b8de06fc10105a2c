"""GPU boundary behaviour: the no-active short-circuit, unread-data probes,
device-flagged bad indices, determinism, integer-exact (bitwise) agreement
with the oracle, and SGMV == BGMV on the expanded indices."""
import numpy as np
import pytest
import torch

import oracle
from gather_matmul_b200 import _lib
from gather_matmul_b200 import ops
from gather_matmul_b200 import workloads as W

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from gpu_util import Dev, assert_buf_close, assert_y_close, host_bits, oracle_expand, oracle_shrink


def _p(seed=3, dt=W.BF16, T=70, D=1032, r=16, S=5, d_out=(256, 64), kind="uniform_neg", **kw):
    return W.make_problem("b", dt, T=T, D=D, r=r, S=S, d_out=list(d_out), scale=0.5, seed=seed,
                          idx_kind=kind, **kw)


def test_no_active_launches_nothing_and_writes_nothing():
    # "[LoRA] LoRA cuda graph specialization": with no active adapter the LoRA
    # ops do no work at all, not even zeroing the intermediate.
    p = _p(kind="none")
    d = Dev(p)
    sentinel = torch.full_like(d.buf, 12345.0)
    d.buf.copy_(sentinel)
    y0 = d.y.clone()
    ops.group(d.idx, p.S, d.meta)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ops.shrink(d.x, d.A, d.idx, d.buf, d.meta, has_active=False)
        ops.expand(d.buf, d.B, d.idx, d.y, d.meta, p.scale, has_active=False)
    # a call with has_active=0 enqueues nothing: the stream has no pending work
    assert s.query()
    torch.cuda.synchronize()
    assert torch.equal(d.buf, sentinel)
    assert torch.equal(d.y, y0)


def test_all_minus_one_with_has_active_true():
    # the kernels themselves also leave every row alone and write zeros to buf
    p = _p(kind="none")
    d = Dev(p)
    d.shrink()
    y0 = d.y.clone()
    d.expand()
    torch.cuda.synchronize()
    assert torch.all(d.buf == 0)
    assert torch.equal(d.y, y0)


def test_empty_batch():
    p = _p(T=0)
    d = Dev(p)
    d.shrink()
    d.expand()
    torch.cuda.synchronize()
    p = W.make_problem("e", W.BF16, T=0, D=64, r=16, S=2, d_out=[64], seed=0,
                       segments=(np.array([0]), np.array([], dtype=np.int32)))
    d = Dev(p)
    d.shrink()
    d.expand()
    torch.cuda.synchronize()


@pytest.mark.parametrize("shape", [dict(T=64, S=6, r=16, D=1032, d_out=(256, 64)),
                                   dict(T=160, S=5, r=32, D=2056, d_out=(384, 136))],
                         ids=["cuda-core-items", "tensor-core-grouped"])
def test_unread_data_is_not_read(shape):
    # x rows and y rows of -1 tokens, and the weights of slots nobody uses,
    # are poisoned with NaN; results must not change.
    p = _p(seed=9, kind="uniform_neg", **shape)
    if shape["S"] == 5:   # leave slot 3 unused
        idx = p.idx.copy()
        idx[idx == 3] = 2
        import dataclasses
        p = dataclasses.replace(p, idx=idx)
    used = set(int(v) for v in p.idx if v >= 0)
    unused = [g for g in range(p.S) if g not in used]
    nan_bits = np.uint16(0x7FC0 if p.dtype == W.BF16 else 0x7E00)
    neg = p.idx < 0
    x = p.x.copy()
    x[neg] = nan_bits
    y = p.y.copy()
    y[neg] = nan_bits
    A = [a.copy() for a in p.A]
    B = [b.copy() for b in p.B]
    for a in A:
        a[unused] = nan_bits
    for b in B:
        b[unused] = nan_bits
    import dataclasses
    q = dataclasses.replace(p, x=x, y=y, A=A, B=B)
    d = Dev(q)
    buf_ref, cabs = oracle_shrink(p)
    buf = d.shrink()
    yd = d.expand()
    torch.cuda.synchronize()
    assert_buf_close(buf, buf_ref, cabs)
    assert np.array_equal(host_bits(yd)[neg], y[neg])      # NaN rows untouched, bit for bit
    y_ref = oracle_expand(p, buf_ref)
    g = oracle.decode(p.dtype, host_bits(yd))
    act = ~neg
    assert np.all(np.abs(g[act] - y_ref[act]) <= 1e-2 * (1 + np.abs(y_ref[act])))


def test_bad_indices_are_flagged_and_treated_as_none():
    p = _p(seed=4, T=40, kind="uniform")
    idx = p.idx.copy()
    idx[3] = p.S
    idx[17] = -9
    import dataclasses
    q = dataclasses.replace(p, idx=idx)
    d = Dev(q)
    assert ops.check_errors(d.meta) == _lib.LORA_OK
    d.shrink()
    d.expand()
    assert ops.check_errors(d.meta) == _lib.LORA_ERR_BAD_INDEX
    assert ops.check_errors(d.meta) == _lib.LORA_OK          # cleared by the check
    ref = idx.copy()
    ref[[3, 17]] = -1
    r = dataclasses.replace(p, idx=ref)
    buf_ref, cabs = oracle_shrink(r)
    assert_buf_close(d.buf, buf_ref, cabs)
    assert np.array_equal(host_bits(d.y)[[3, 17]], p.y[[3, 17]])


@pytest.mark.parametrize("T,S,r", [(70, 5, 16), (400, 6, 32)],
                         ids=["cuda-core-items", "tensor-core-grouped"])
def test_stale_grouping_is_flagged_never_silently_wrong(T, S, r):
    # The workspace is grouped from batch k's indices, then the compute calls
    # get batch k+1 (same sizes, a third of the tokens on another slot or
    # none).  Every token whose index changed must be left unwritten (buf
    # keeps its NaN sentinel, y its input bits) and counted; every other row
    # must still be right.
    import dataclasses
    pk = _p(seed=50, T=T, S=S, r=r, D=1032, d_out=(256, 64), kind="uniform_neg")
    rng = np.random.default_rng(51)
    idx2 = pk.idx.copy()
    moved = rng.choice(T, size=T // 3, replace=False)
    shift = 1 + rng.integers(0, S, size=moved.size)          # never a multiple of S + 1
    idx2[moved] = (idx2[moved] + 1 + shift) % (S + 1) - 1
    assert np.all(idx2[moved] != pk.idx[moved])
    q = dataclasses.replace(pk, idx=idx2.astype(np.int32))
    d = Dev(q)
    ops.group(torch.from_numpy(pk.idx).cuda(), S, d.meta)     # batch k's grouping
    ops.shrink(d.x, d.A, d.idx, d.buf, d.meta)                # batch k+1's data
    ops.expand(d.buf, d.B, d.idx, d.y, d.meta, q.scale, y_col_off=q.col_off)
    assert ops.check_errors(d.meta) == _lib.LORA_ERR_BAD_INDEX
    keep = np.ones(T, dtype=bool)
    keep[moved] = False
    g = d.buf.detach().cpu().double().numpy()
    assert np.all(np.isnan(g[:, moved])), "a row of a moved token was written"
    assert np.array_equal(host_bits(d.y)[moved], q.y[moved]), "y of a moved token changed"
    buf_ref, cabs = oracle_shrink(q)
    assert_buf_close(torch.from_numpy(g[:, keep]), buf_ref[:, keep], cabs[:, keep])
    y_ref = oracle_expand(q, buf_ref)
    gy = oracle.decode(q.dtype, host_bits(d.y))
    assert np.all(np.abs(gy[keep] - y_ref[keep]) <= 1e-2 * (1 + np.abs(y_ref[keep])))
    # grouped from the right batch, the same calls are clean
    d2 = Dev(q)
    d2.shrink()
    d2.expand()
    assert ops.check_errors(d2.meta) == _lib.LORA_OK


def test_malformed_segments_are_flagged():
    p = W.make_problem("s", W.BF16, T=64, D=256, r=16, S=3, d_out=[64], seed=1,
                       segments=(np.array([0, 40, 30, 64]), np.array([0, 1, 2])))
    d = Dev(p)
    d.shrink()
    assert ops.check_errors(d.meta) == _lib.LORA_ERR_BAD_INDEX


def test_deterministic_bitwise():
    p = _p(seed=5, T=200, D=4096, r=32, S=9, d_out=(1024,))
    d1, d2 = Dev(p), Dev(p)
    for d in (d1, d2):
        d.shrink()
        d.expand()
    torch.cuda.synchronize()
    assert torch.equal(d1.buf, d2.buf)
    assert torch.equal(d1.y, d2.y)


@pytest.mark.parametrize("dt,D,r", [(W.F16, 64, 8), (W.BF16, 16, 8), (W.F16, 64, 16)])
def test_integer_inputs_match_oracle_bitwise(dt, D, r):
    # x, A, B in {-1,0,1}, y in [-8,8]: all sums are small integers, exact in
    # fp32 and in the output type, so GPU == oracle bit for bit.
    for segmented in (False, True):
        seg = (np.array([0, 5, 5, 19, 33]), np.array([1, 0, -1, 2])) if segmented else None
        p = W.make_problem("int", dt, T=33, D=D, r=r, S=3, d_out=[16, 8], scale=1.0, seed=D + r,
                           idx_kind="uniform_neg", values="int", segments=seg)
        d = Dev(p)
        buf_ref, _ = oracle_shrink(p)
        buf = d.shrink()
        y = d.expand()
        torch.cuda.synchronize()
        assert np.array_equal(buf.cpu().double().numpy(), buf_ref)
        y_ref = oracle_expand(p, buf_ref)
        assert np.array_equal(oracle.decode(p.dtype, host_bits(y)), y_ref)


@pytest.mark.parametrize("dt,D,T,S", [(W.F16, 64, 200, 3), (W.F16, 64, 300, 2),
                                      (W.BF16, 8, 200, 3), (W.BF16, 8, 300, 2),
                                      (W.F16, 64, 200, 8), (W.BF16, 8, 260, 12)],
                         ids=["f16-small-groups", "f16-full-tiles", "bf16-small-groups",
                              "bf16-full-tiles", "f16-many-slots", "bf16-many-slots"])
def test_integer_inputs_grouped_tensor_cores_bitwise(dt, D, T, S):
    # T >= 16 S with r = 16: the per-token batch runs through the grouping on
    # the tcgen05 kernels (groups of about 66 rows take the 128-row layout,
    # about 150 rows a full tile and a 22-row one, 21-25 rows the
    # operand-swapped tile).  x, A, B in {-1,0,1},
    # y in [-8,8]: |buf| <= D and |y| <= 8 + 16 D stay exact (fp16: <= 1032
    # < 2048; bf16: <= 136 < 256), through the hi + lo split as well, so the
    # GPU equals the oracle bit for bit.
    p = W.make_problem("int_tc", dt, T=T, D=D, r=16, S=S, d_out=[136, 64], scale=1.0,
                       seed=T + S, idx_kind="uniform_neg", values="int")
    d = Dev(p)
    buf_ref, _ = oracle_shrink(p)
    buf = d.shrink()
    y = d.expand()
    torch.cuda.synchronize()
    assert np.array_equal(buf.cpu().double().numpy(), buf_ref)
    assert np.array_equal(oracle.decode(p.dtype, host_bits(y)), oracle_expand(p, buf_ref))


def test_sgmv_equals_bgmv_on_expanded_indices():
    ss, sa = np.array([0, 100, 100, 260, 300]), np.array([2, 0, -1, 1])
    p = W.make_problem("s", W.BF16, T=300, D=2048, r=64, S=3, d_out=[512, 256], scale=0.75,
                       seed=8, segments=(ss, sa))
    import dataclasses
    q = dataclasses.replace(p, seg_starts=None, seg_adapter=None,
                            idx=oracle.segments_to_idx(p.T, ss, sa))
    ds, dq = Dev(p), Dev(q)
    bs = ds.shrink()
    bq = dq.shrink()
    ys = ds.expand()
    yq = dq.expand()
    torch.cuda.synchronize()
    buf_ref, cabs = oracle_shrink(q)
    assert_buf_close(bs, buf_ref, cabs)
    assert_buf_close(bq, buf_ref, cabs)
    y_ref = oracle_expand(q, buf_ref)
    assert_y_close(q, ys, y_ref)
    assert_y_close(q, yq, y_ref)


def test_stream_and_graph_capture():
    # the calls are stream-ordered and capturable: replaying a captured
    # group + shrink + expand gives the eager result
    p = _p(seed=6, T=96, D=2048, r=16, S=4, d_out=(512,))
    d = Dev(p)
    y_in = d.y.clone()
    d.shrink()
    d.expand()
    torch.cuda.synchronize()
    y_eager = d.y.clone()
    d.y.copy_(y_in)
    d.buf.fill_(float("nan"))
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        ops.group(d.idx, p.S, d.meta)
        ops.shrink(d.x, d.A, d.idx, d.buf, d.meta)
        ops.expand(d.buf, d.B, d.idx, d.y, d.meta, p.scale)
    d.y.copy_(y_in)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(d.y, y_eager)


@pytest.mark.parametrize("path", ["grouped", "fused", "segments"])
def test_power_of_two_scale_scales_y_exactly(path):
    # With y_old = 0, y = rn(scale * acc): a power-of-two scale commutes with
    # the rounding, so scale 4 gives exactly 4x the scale-1 result, element for
    # element (no value here comes near the fp16/bf16 range limits).
    if path == "segments":
        ss, sa = np.array([0, 64, 200, 330]), np.array([1, -1, 0])
        p = W.make_problem("s", W.BF16, T=330, D=1024, r=32, S=2, d_out=[384], scale=1.0,
                           seed=21, segments=(ss, sa))
    else:
        # bf16: fp32's exponent range, so no result is subnormal (in fp16 a
        # subnormal would round at a fixed absolute step and break the identity)
        p = W.make_problem("s", W.BF16, T=256, D=1024, r=16, S=4, d_out=[512], scale=1.0, seed=22,
                           idx_kind="uniform_neg")
    ys = []
    for scale in (1.0, 4.0):
        d = Dev(p)
        d.y.zero_()
        if path == "fused":
            ops.bgmv(d.x, d.A, d.B, d.idx, d.y, d.buf, d.meta, scale, y_col_off=p.col_off)
        else:
            d.shrink()
            b = d.buf
            if p.segmented:
                ops.expand_segment(b, d.B, d.ss, d.sa, d.y, d.meta, scale, y_col_off=p.col_off)
            else:
                ops.expand(b, d.B, d.idx, d.y, d.meta, scale, y_col_off=p.col_off)
        torch.cuda.synchronize()
        ys.append(oracle.decode(p.dtype, host_bits(d.y)))
    assert np.any(ys[0] != 0)
    assert np.array_equal(ys[1], 4.0 * ys[0])
