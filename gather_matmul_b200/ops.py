"""Python binding of the multi-LoRA shrink / expand C ABI.

Argument marshalling only: each function reads shapes, strides and device
pointers off torch tensors, passes them to liblora_b200.so on the current
torch CUDA stream, and raises LoraError on a non-OK status.  Every step of the
computation runs in the library's CUDA kernels; torch supplies device memory
and streams.

  group(idx, S, meta)                          per-batch group-by-slot metadata
  shrink(x, A, idx, buf, meta)                 buf[i] = per-token x . A_i[idx]^T
  expand(buf, B, idx, y, meta, scale)          y[:, slice_i] += scale buf_i . B_i[idx]^T
  bgmv(x, A, B, idx, y, buf, meta, scale)      group + shrink + expand in one call
  shrink_segment / expand_segment              the same with segments
  check_errors(meta)                           device-side bad-index report

has_active: the per-token calls take the host flag of the C ABI.  Left as
None, it is derived from `idx_host` (a host copy of the batch's indices, as a
serving loop has before it moves them to the device) when one is given: no
index in [0, S) means no LoRA work at all, so nothing is enqueued.  Without a
host copy the call runs, and the kernels skip tokens without an adapter.
"""
import ctypes
from typing import Optional, Sequence

import torch

from . import _lib

_DT = {torch.float16: _lib.LORA_F16, torch.bfloat16: _lib.LORA_BF16}


class LoraError(RuntimeError):
    def __init__(self, call, status):
        self.status = status
        super().__init__(f"{call} failed: {_lib.status_string(status)} ({status})")


def _check(call, status):
    if status != _lib.LORA_OK:
        raise LoraError(call, status)


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _ptrs(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


def _dtype(t):
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}; fp16 or bf16")
    return _DT[t.dtype]


def active_from_host(idx_host, S: int) -> bool:
    """Whether any index of a host copy of a batch's indices selects a slot
    in [0, S)."""
    if isinstance(idx_host, torch.Tensor):
        if idx_host.is_cuda:
            raise ValueError("idx_host must be a host tensor or array")
        idx_host = idx_host.numpy()
    import numpy as np
    a = np.asarray(idx_host)
    return bool(np.any((a >= 0) & (a < S)))


def _active(has_active, idx_host, S):
    if has_active is not None:
        return int(bool(has_active))
    if idx_host is not None:
        return int(active_from_host(idx_host, S))
    return 1


def _check_idx(idx, T):
    if idx.dtype != torch.int32 or not idx.is_contiguous() or idx.numel() != T:
        raise TypeError("idx must be a contiguous int32 tensor of one index per token")


def workspace_bytes(T: int, S: int) -> int:
    return _lib.load().lora_workspace_bytes(int(T), int(S))


def workspace(T: int, S: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace ("meta") for batches of up to T tokens over S slots."""
    n = workspace_bytes(T, S)
    if n == 0:
        raise LoraError("lora_workspace_bytes", _lib.LORA_ERR_UNSUPPORTED)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def set_slot_ranks(ranks: Optional[torch.Tensor], S: int, meta: torch.Tensor, stream=None):
    """Record each slot's own rank (device int32 [S]; None clears) in the
    workspace: the kernels then skip the zero padding of smaller-rank slots."""
    if ranks is not None:
        if ranks.dtype != torch.int32 or not ranks.is_contiguous() or ranks.numel() != S:
            raise TypeError("ranks must be a contiguous int32 tensor of one rank per slot")
    _check("lora_set_slot_ranks", _lib.load().lora_set_slot_ranks(
        int(S), _ptr(ranks), _ptr(meta), meta.numel(), _stream(stream)))


def group(idx: torch.Tensor, S: int, meta: torch.Tensor, stream=None):
    """Group-by-slot metadata of one batch's int32 adapter indices (-1 = none)."""
    _check_idx(idx, idx.numel())
    _check("lora_group", _lib.load().lora_group(idx.numel(), int(S), _ptr(idx), _ptr(meta),
                                                meta.numel(), _stream(stream)))


def _xinfo(x):
    if x.dim() != 2 or (x.numel() > 0 and x.stride(1) != 1):
        raise ValueError("x must be [T, D] with unit column stride")
    return x.shape[0], x.shape[1], (x.stride(0) if x.numel() > 0 else x.shape[1])


def shrink(x: torch.Tensor, A: Sequence[torch.Tensor], idx: torch.Tensor, buf: torch.Tensor,
           meta: torch.Tensor, has_active: Optional[bool] = None, idx_host=None,
           stream=None) -> torch.Tensor:
    """buf[i, t, :] = x[t] . A[i][idx[t]]^T (0 for tokens without an adapter).

    A: list of [S, r, D] stacks; idx: the device int32 indices that group()
    grouped into meta; buf: float32 [len(A), T, r]."""
    T, D, ldx = _xinfo(x)
    S, r, _ = A[0].shape
    _check_idx(idx, T)
    _check("lora_shrink", _lib.load().lora_shrink(
        _dtype(x), T, D, r, S, len(A), _ptr(x), ldx, _ptrs(A), _ptr(idx), _ptr(buf),
        _active(has_active, idx_host, S), _ptr(meta), meta.numel(), _stream(stream)))
    return buf


def shrink_laned(x: torch.Tensor, A: Sequence[torch.Tensor], idx: torch.Tensor,
                 buf: torch.Tensor, meta: torch.Tensor, has_active: Optional[bool] = None,
                 idx_host=None, stream=None) -> torch.Tensor:
    """shrink() without a grouping: every slot's lanes in one dense tensor-core
    contraction, each token keeping its own slot's r lanes.  meta only
    collects the error counters (group() is not needed)."""
    T, D, ldx = _xinfo(x)
    S, r, _ = A[0].shape
    _check_idx(idx, T)
    _check("lora_shrink_laned", _lib.load().lora_shrink_laned(
        _dtype(x), T, D, r, S, len(A), _ptr(x), ldx, _ptrs(A), _ptr(idx), _ptr(buf),
        _active(has_active, idx_host, S), _ptr(meta), meta.numel(), _stream(stream)))
    return buf


def _expand_common(buf, B, y, y_col_off, buf_slice_stride):
    if y.dim() != 2 or (y.numel() > 0 and y.stride(1) != 1):
        raise ValueError("y must be [T, ldy] with unit column stride")
    T, ldy = y.shape[0], (y.stride(0) if y.numel() > 0 else y.shape[1])
    S, _, r = B[0].shape
    n = len(B)
    d_out = (ctypes.c_int32 * n)(*[b.shape[1] for b in B])
    if y_col_off is None:
        offs, c = [], 0
        for b in B:
            offs.append(c)
            c += b.shape[1]
        y_col_off = offs
    off = (ctypes.c_int64 * n)(*[int(v) for v in y_col_off])
    if buf_slice_stride is None:
        buf_slice_stride = 0 if buf.dim() == 2 else buf.stride(0)
    return T, ldy, S, r, n, d_out, off, int(buf_slice_stride)


def expand(buf: torch.Tensor, B: Sequence[torch.Tensor], idx: torch.Tensor, y: torch.Tensor,
           meta: torch.Tensor, scale: float = 1.0, y_col_off=None, buf_slice_stride=None,
           has_active: Optional[bool] = None, idx_host=None, stream=None) -> torch.Tensor:
    """y[t, off_i:off_i+D_out_i] += scale * buf[i, t] . B[i][idx[t]]^T, in place.

    B: list of [S, D_out_i, r]; idx as for shrink(); buf: float32 [n, T, r]
    (or [T, r] shared by every slice); y: [T, >= sum D_out] fp16/bf16."""
    T, ldy, S, r, n, d_out, off, stride = _expand_common(buf, B, y, y_col_off, buf_slice_stride)
    _check_idx(idx, T)
    _check("lora_expand", _lib.load().lora_expand(
        _dtype(y), T, r, S, n, _ptr(buf), stride, _ptrs(B), d_out, _ptr(idx),
        ctypes.c_float(scale), _ptr(y), ldy, off, _active(has_active, idx_host, S), _ptr(meta),
        meta.numel(), _stream(stream)))
    return y


def bgmv(x: torch.Tensor, A: Sequence[torch.Tensor], B: Sequence[torch.Tensor], idx: torch.Tensor,
         y: torch.Tensor, buf: torch.Tensor, meta: torch.Tensor, scale: float = 1.0,
         y_col_off=None, has_active: Optional[bool] = None, idx_host=None,
         pdl_early: bool = False, grouped: bool = False, stream=None):
    """group + shrink + expand of one batch in one call (one launch when the
    shape fits the fused kernel).  A: one stack per slice of B, or a single
    stack shared by every slice; buf: float32 [len(A), T, r] receives the
    intermediate; y is updated in place.  pdl_early=True promises that A, B
    and idx are not written by the kernel launched just before on the stream;
    grouped=True that meta already holds this idx's grouping (group(), or an
    earlier bgmv of the batch): no grouping launch."""
    T, D, ldx = _xinfo(x)
    S, r, _ = A[0].shape
    n = len(B)
    shared = len(A) == 1 and n > 1
    if not shared and len(A) != n:
        raise ValueError("A must hold one stack per slice, or one shared stack")
    _, ldy, _, _, _, d_out, off, _ = _expand_common(buf, B, y, y_col_off, None)
    _check_idx(idx, T)
    flags = (_lib.LORA_FLAG_PDL_EARLY if pdl_early else 0) | \
        (_lib.LORA_FLAG_GROUPED if grouped else 0)
    _check("lora_bgmv", _lib.load().lora_bgmv(
        _dtype(x), T, D, r, S, n, _ptr(x), ldx, _ptrs(A), int(shared), _ptrs(B), d_out,
        ctypes.c_float(scale), _ptr(y), ldy, off, _ptr(buf), _ptr(idx),
        _active(has_active, idx_host, S), flags, _ptr(meta), meta.numel(), _stream(stream)))
    return y


def bgmv_launches(dtype, T: int, D: int, r: int, S: int, d_out) -> int:
    """Kernel launches bgmv() makes for this shape: 1 (fused) or 3."""
    dt = _DT[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    arr = (ctypes.c_int32 * len(d_out))(*[int(v) for v in d_out])
    return _lib.load().lora_bgmv_launches(dt, int(T), int(D), int(r), int(S), len(d_out), arr)


def shrink_segment(x, A, seg_starts, seg_adapter, buf, meta, has_active=True, stream=None):
    """shrink() with adapters given by segments (int32 CSR starts [n+1], adapters [n])."""
    T, D, ldx = _xinfo(x)
    S, r, _ = A[0].shape
    _check("lora_shrink_segment", _lib.load().lora_shrink_segment(
        _dtype(x), T, D, r, S, len(A), _ptr(x), ldx, _ptrs(A), _ptr(seg_starts),
        _ptr(seg_adapter), seg_adapter.numel(), _ptr(buf), int(bool(has_active)), _ptr(meta),
        meta.numel(), _stream(stream)))
    return buf


def expand_segment(buf, B, seg_starts, seg_adapter, y, meta, scale=1.0, y_col_off=None,
                   buf_slice_stride=None, has_active=True, stream=None):
    """expand() with adapters given by segments."""
    T, ldy, S, r, n, d_out, off, stride = _expand_common(buf, B, y, y_col_off, buf_slice_stride)
    _check("lora_expand_segment", _lib.load().lora_expand_segment(
        _dtype(y), T, r, S, n, _ptr(buf), stride, _ptrs(B), d_out, _ptr(seg_starts),
        _ptr(seg_adapter), seg_adapter.numel(), ctypes.c_float(scale), _ptr(y), ldy, off,
        int(bool(has_active)), _ptr(meta), meta.numel(), _stream(stream)))
    return y


def sgmv(x: torch.Tensor, A: Sequence[torch.Tensor], B: Sequence[torch.Tensor],
         seg_starts: torch.Tensor, seg_adapter: torch.Tensor, y: torch.Tensor, buf: torch.Tensor,
         meta: torch.Tensor, scale: float = 1.0, y_col_off=None, has_active: bool = True,
         stream=None):
    """shrink_segment() + expand_segment() of one prefill batch in one call
    (the expand starts while the shrink finishes).  A: one stack per slice of
    B, or a single stack shared by every slice; buf: float32 [len(A), T, r]."""
    T, D, ldx = _xinfo(x)
    S, r, _ = A[0].shape
    n = len(B)
    shared = len(A) == 1 and n > 1
    if not shared and len(A) != n:
        raise ValueError("A must hold one stack per slice, or one shared stack")
    _, ldy, _, _, _, d_out, off, _ = _expand_common(buf, B, y, y_col_off, None)
    _check("lora_sgmv", _lib.load().lora_sgmv(
        _dtype(x), T, D, r, S, n, _ptr(x), ldx, _ptrs(A), int(shared), _ptrs(B), d_out,
        ctypes.c_float(scale), _ptr(y), ldy, off, _ptr(buf), _ptr(seg_starts), _ptr(seg_adapter),
        seg_adapter.numel(), int(bool(has_active)), _ptr(meta), meta.numel(), _stream(stream)))
    return y


def shrink_noalloc(x: torch.Tensor, A: Sequence[torch.Tensor], idx: torch.Tensor,
                   buf: torch.Tensor, has_active: bool = True, stream=None) -> torch.Tensor:
    """group() + shrink() in one call that needs no workspace: the library keeps
    the grouping scratch in a fixed device array.  For callers that cannot
    allocate; calls that overlap on the GPU race on that array."""
    T, D, ldx = _xinfo(x)
    S, r, _ = A[0].shape
    _check_idx(idx, T)
    _check("lora_shrink_noalloc", _lib.load().lora_shrink_noalloc(
        _dtype(x), T, D, r, S, len(A), _ptr(x), ldx, _ptrs(A), _ptr(idx), _ptr(buf),
        int(bool(has_active)), _stream(stream)))
    return buf


def check_errors(meta: torch.Tensor, stream=None) -> int:
    """Synchronise and return the library status for device-detected bad
    indices / segments since the last check (0 = LORA_OK); clears them."""
    return _lib.load().lora_check_errors(_ptr(meta), meta.numel(), _stream(stream))


def build_info() -> str:
    return _lib.load().lora_build_info().decode()


def launch_count() -> int:
    """Kernel launches the library has made in this process (a launch recorded
    into a stream capture counts once)."""
    return int(_lib.load().lora_launch_count())
