"""Python face of the fp64 CPU oracle for multi-LoRA shrink / expand.

TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the benchmark's
CPU-baseline leg may import this package.  It never imports the CUDA package
(gather_matmul_b200) and the CUDA package never imports it.

Every function takes plain numpy arrays (fp16 / bf16 elements passed as their
uint16 bit patterns, indices as int32) and returns numpy float64 results:

  shrink(...)   buf[i][t][j] = sum_d x[t][d] * A_i[idx[t]][j][d]
  expand(...)   y[t][off_i+o] = y_old[t][off_i+o]
                                + scale * sum_j buf_i[t][j] * B_i[idx[t]][o][j]

This is the ref_bgmv definition from "[Hardware][TPU][V1] Better tpu
multilora compilation" (vllm-project/vllm pull 16989, the baseline function in
the discussion) with index -1 meaning "no adapter" (the "base model only"
requests of "Add multi-LoRA support", vllm pull 1804, Features list).  The
arithmetic lives in lora_oracle.c; this module only marshals arguments.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F16 = 0
BF16 = 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        vp = ctypes.c_void_p
        L.lo_set_threads.argtypes = [i32]
        L.lo_set_threads.restype = i32
        L.lo_decode.argtypes = [i32, ctypes.c_uint16]
        L.lo_decode.restype = dbl
        L.lo_decode_array.argtypes = [i32, vp, vp, i64]
        L.lo_group_by_slot.argtypes = [i32, i32, vp, vp, vp, vp]
        L.lo_group_by_slot.restype = i32
        L.lo_shrink.argtypes = [i32, i32, i32, i32, i32, i32, vp, i64, vp, vp, vp, vp]
        L.lo_shrink.restype = i32
        L.lo_expand.argtypes = [i32, i32, i32, i32, i32, vp, i64, vp, vp, vp, dbl,
                                vp, i64, vp, vp]
        L.lo_expand.restype = i32
        L.lo_segments_to_idx.argtypes = [i32, i32, vp, vp, vp]
        L.lo_segments_to_idx.restype = i32
        L.lo_shrink_segment.argtypes = [i32, i32, i32, i32, i32, i32, vp, i64, vp,
                                        vp, vp, i32, vp, vp]
        L.lo_shrink_segment.restype = i32
        L.lo_expand_segment.argtypes = [i32, i32, i32, i32, i32, vp, i64, vp, vp,
                                        vp, vp, i32, dbl, vp, i64, vp, vp]
        L.lo_expand_segment.restype = i32
        _lib = L
    return _lib


class use_library:
    """Context manager that points this module at another build of the oracle
    source (the mutation tests load deliberately broken copies this way)."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = lib()
        _lib = None
        saved_build = _build.build
        _build.build = lambda *a, **k: self.path
        try:
            lib()
        finally:
            _build.build = saved_build
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def set_threads(n: int) -> int:
    """Host threads for the per-token loops; returns the count in effect."""
    return lib().lo_set_threads(int(n))


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("fp16/bf16 arrays are passed as uint16 bit patterns")
    return a


def _ptr_array(arrs):
    return (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])


def decode(dtype: int, bits: np.ndarray) -> np.ndarray:
    """Exact fp16/bf16 -> float64 decoding of uint16 bit patterns."""
    b = _bits(bits)
    out = np.empty(b.shape, dtype=np.float64)
    lib().lo_decode_array(dtype, _p(b), _p(out), b.size)
    return out


def group_by_slot(idx: np.ndarray, S: int):
    """Stable counting sort of active tokens by slot.

    Returns (perm[n_active], slot_off[S+1], n_bad)."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T = idx.shape[0]
    perm = np.full(max(T, 1), -1, dtype=np.int32)
    off = np.zeros(S + 1, dtype=np.int32)
    na = np.zeros(1, dtype=np.int32)
    bad = lib().lo_group_by_slot(T, S, _p(idx), _p(perm), _p(off), _p(na))
    return perm[: int(na[0])].copy(), off, bad


def shrink(dtype, x_bits, A_bits_list, idx, S, want_cabs=False, ldx=None):
    """buf[n_slices, T, r] (and optionally the |x*A| sums) in float64."""
    x = _bits(x_bits)
    T = x.shape[0]
    A = [_bits(a) for a in A_bits_list]
    n = len(A)
    _, r, D = A[0].shape
    ldx = x.shape[1] if ldx is None else ldx
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    buf = np.zeros((n, T, r), dtype=np.float64)
    cabs = np.zeros((n, T, r), dtype=np.float64) if want_cabs else None
    bad = lib().lo_shrink(dtype, T, D, r, S, n, _p(x), ldx, _ptr_array(A), _p(idx),
                          _p(buf), _p(cabs) if want_cabs else None)
    return (buf, cabs, bad) if want_cabs else (buf, bad)


def expand(dtype, buf, B_bits_list, idx, S, scale, y_old_bits, col_off,
           shared_buf=False):
    """y (float64, [T, ldy]) = y_old + scale * per-token buf . B^T per slice.

    buf is float64 [n_slices, T, r], or [T, r] with shared_buf=True (one
    intermediate for every slice)."""
    B = [_bits(b) for b in B_bits_list]
    n = len(B)
    r = B[0].shape[2]
    yo = _bits(y_old_bits)
    T, ldy = yo.shape
    buf = np.ascontiguousarray(buf, dtype=np.float64)
    stride = 0 if shared_buf else T * r
    d_out = np.array([b.shape[1] for b in B], dtype=np.int32)
    off = np.ascontiguousarray(col_off, dtype=np.int64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    y = np.empty((T, ldy), dtype=np.float64)
    bad = lib().lo_expand(dtype, T, r, S, n, _p(buf), stride, _ptr_array(B), _p(d_out),
                          _p(idx), float(scale), _p(yo), ldy, _p(off), _p(y))
    return y, bad


def segments_to_idx(T, seg_starts, seg_adapter):
    """Per-token adapter indices from CSR segments; None if malformed."""
    ss = np.ascontiguousarray(seg_starts, dtype=np.int32)
    sa = np.ascontiguousarray(seg_adapter, dtype=np.int32)
    n_seg = sa.shape[0]
    if ss.shape[0] != n_seg + 1:
        return None
    idx = np.zeros(max(T, 1), dtype=np.int32)
    rc = lib().lo_segments_to_idx(T, n_seg, _p(ss), _p(sa), _p(idx))
    return None if rc != 0 else idx[:T].copy()


def shrink_segment(dtype, x_bits, A_bits_list, seg_starts, seg_adapter, S,
                   want_cabs=False):
    x = _bits(x_bits)
    T = x.shape[0]
    A = [_bits(a) for a in A_bits_list]
    n = len(A)
    _, r, D = A[0].shape
    ss = np.ascontiguousarray(seg_starts, dtype=np.int32)
    sa = np.ascontiguousarray(seg_adapter, dtype=np.int32)
    buf = np.zeros((n, T, r), dtype=np.float64)
    cabs = np.zeros((n, T, r), dtype=np.float64) if want_cabs else None
    rc = lib().lo_shrink_segment(dtype, T, D, r, S, n, _p(x), x.shape[1], _ptr_array(A),
                                 _p(ss), _p(sa), sa.shape[0], _p(buf),
                                 _p(cabs) if want_cabs else None)
    return (buf, cabs, rc) if want_cabs else (buf, rc)


def expand_segment(dtype, buf, B_bits_list, seg_starts, seg_adapter, S, scale,
                   y_old_bits, col_off, shared_buf=False):
    B = [_bits(b) for b in B_bits_list]
    n = len(B)
    r = B[0].shape[2]
    yo = _bits(y_old_bits)
    T, ldy = yo.shape
    buf = np.ascontiguousarray(buf, dtype=np.float64)
    stride = 0 if shared_buf else T * r
    d_out = np.array([b.shape[1] for b in B], dtype=np.int32)
    off = np.ascontiguousarray(col_off, dtype=np.int64)
    ss = np.ascontiguousarray(seg_starts, dtype=np.int32)
    sa = np.ascontiguousarray(seg_adapter, dtype=np.int32)
    y = np.empty((T, ldy), dtype=np.float64)
    rc = lib().lo_expand_segment(dtype, T, r, S, n, _p(buf), stride, _ptr_array(B),
                                 _p(d_out), _p(ss), _p(sa), sa.shape[0], float(scale),
                                 _p(yo), ldy, _p(off), _p(y))
    return y, rc
