"""The C-ABI library on the CPU: it loads, exports every symbol include/lora.h
declares, sizes workspaces as documented, and rejects bad arguments on the
host before touching the GPU (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from gather_matmul_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lora.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lora_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("lora_group", "lora_shrink", "lora_expand", "lora_shrink_segment",
              "lora_expand_segment", "lora_workspace_bytes", "lora_check_errors"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for n in declared_functions():
        assert hasattr(L, n), f"{n} declared in lora.h but not exported"
        assert n in _lib.SIGNATURES, f"{n} has no binding signature"


def test_build_info_and_status_strings(L):
    assert "sm_100a" in L.lora_build_info().decode()
    for code, name in [(0, "LORA_OK"), (-1, "LORA_ERR_INVALID_ARG"), (-2, "LORA_ERR_UNSUPPORTED"),
                       (-3, "LORA_ERR_MISALIGNED"), (-4, "LORA_ERR_CUDA"),
                       (-5, "LORA_ERR_BAD_INDEX")]:
        assert _lib.status_string(code) == name


def a256(v):
    return (v + 255) // 256 * 256


@pytest.mark.parametrize("T,S", [(0, 1), (1, 1), (32, 4), (256, 32), (4096, 128), (8192, 8),
                                 (100000, 1024)])
def test_workspace_bytes_formula(L, T, S):
    tt = max(T, 1)
    max_items = T // 16 + max(S + 1, T + 1) + 2
    ctas = min(64, max(1, -(-T // 512)))      # grouping CTAs, one per 512 tokens
    want = (256 + a256(4 * (S + 2)) + a256(4 * S) + a256(4 * tt) + a256(16 * max_items)
            + a256(4 * ctas * (S + 1)))
    assert L.lora_workspace_bytes(T, S) == want


def test_noalloc_array_holds_the_largest_workspace(L):
    assert L.lora_workspace_bytes(_lib.LORA_NOALLOC_MAX_TOKENS, _lib.LORA_MAX_SLOTS) <= 246784


def test_workspace_bytes_rejects_out_of_range(L):
    assert L.lora_workspace_bytes(-1, 4) == 0
    assert L.lora_workspace_bytes(16, 0) == 0
    assert L.lora_workspace_bytes(16, _lib.LORA_MAX_SLOTS + 1) == 0
    assert L.lora_workspace_bytes(_lib.LORA_MAX_TOKENS + 1, 4) == 0


FAKE = 0x10000  # a 16-byte aligned non-null address; never dereferenced


def _shrink(L, dt=0, T=16, D=64, r=16, S=4, n=1, x=FAKE, ldx=64, A=(FAKE,), buf=FAKE, meta=FAKE,
            meta_bytes=None, idx=FAKE):
    arr = (ctypes.c_void_p * max(len(A), 1))(*A)
    mb = L.lora_workspace_bytes(T, S) if meta_bytes is None else meta_bytes
    return L.lora_shrink(dt, T, D, r, S, n, x, ldx, arr, idx, buf, 1, meta, mb, None)


@pytest.mark.parametrize("kw,status", [
    (dict(dt=7), _lib.LORA_ERR_INVALID_ARG),
    (dict(T=-1), _lib.LORA_ERR_INVALID_ARG),
    (dict(r=12), _lib.LORA_ERR_UNSUPPORTED),
    (dict(r=128), _lib.LORA_ERR_UNSUPPORTED),
    (dict(S=0), _lib.LORA_ERR_UNSUPPORTED),
    (dict(n=9, A=(FAKE,) * 9), _lib.LORA_ERR_UNSUPPORTED),
    (dict(n=0), _lib.LORA_ERR_UNSUPPORTED),
    (dict(D=60, ldx=64), _lib.LORA_ERR_MISALIGNED),
    (dict(ldx=60, D=56), _lib.LORA_ERR_MISALIGNED),
    (dict(ldx=32), _lib.LORA_ERR_INVALID_ARG),
    (dict(x=FAKE + 2), _lib.LORA_ERR_MISALIGNED),
    (dict(A=(FAKE + 8,)), _lib.LORA_ERR_MISALIGNED),
    (dict(A=(0,)), _lib.LORA_ERR_INVALID_ARG),
    (dict(x=0), _lib.LORA_ERR_INVALID_ARG),
    (dict(meta=0), _lib.LORA_ERR_INVALID_ARG),
    (dict(meta_bytes=64), _lib.LORA_ERR_INVALID_ARG),
    (dict(idx=0), _lib.LORA_ERR_INVALID_ARG),                # the batch's indices are required
])
def test_shrink_host_validation(L, kw, status):
    assert _shrink(L, **kw) == status


def _expand(L, T=16, r=16, S=4, B=(FAKE, FAKE), d_out=(64, 32), off=(0, 64), ldy=96,
            stride=16 * 16, buf=FAKE, y=FAKE, idx=FAKE):
    n = len(B)
    arr = (ctypes.c_void_p * n)(*B)
    do = (ctypes.c_int32 * n)(*d_out)
    of = (ctypes.c_int64 * n)(*off)
    return L.lora_expand(0, T, r, S, n, buf, stride, arr, do, idx, ctypes.c_float(1.0), y, ldy,
                         of, 1, FAKE, L.lora_workspace_bytes(T, S), None)


@pytest.mark.parametrize("kw,status", [
    (dict(off=(0, 32)), _lib.LORA_ERR_INVALID_ARG),          # overlapping slices
    (dict(off=(0, 68)), _lib.LORA_ERR_MISALIGNED),           # offset not a multiple of 8
    (dict(ldy=64), _lib.LORA_ERR_INVALID_ARG),               # slice past the row
    (dict(d_out=(64, 36)), _lib.LORA_ERR_MISALIGNED),
    (dict(stride=100), _lib.LORA_ERR_INVALID_ARG),           # stride smaller than T*r
    (dict(stride=258), _lib.LORA_ERR_MISALIGNED),
    (dict(y=FAKE + 4), _lib.LORA_ERR_MISALIGNED),
    (dict(B=(FAKE, 0)), _lib.LORA_ERR_INVALID_ARG),
    (dict(idx=0), _lib.LORA_ERR_INVALID_ARG),
])
def test_expand_host_validation(L, kw, status):
    assert _expand(L, **kw) == status


def test_segment_host_validation(L):
    arr = (ctypes.c_void_p * 1)(FAKE)
    mb = L.lora_workspace_bytes(16, 4)
    # n_seg > T + 1 and n_seg == 0 with T > 0 are rejected on the host
    assert L.lora_shrink_segment(0, 16, 64, 16, 4, 1, FAKE, 64, arr, FAKE, FAKE, 18, FAKE, 1,
                                 FAKE, mb, None) == _lib.LORA_ERR_INVALID_ARG
    assert L.lora_shrink_segment(0, 16, 64, 16, 4, 1, FAKE, 64, arr, FAKE, FAKE, 0, FAKE, 1,
                                 FAKE, mb, None) == _lib.LORA_ERR_INVALID_ARG
    assert L.lora_shrink_segment(0, 16, 64, 16, 4, 1, FAKE, 64, arr, 0, FAKE, 2, FAKE, 1,
                                 FAKE, mb, None) == _lib.LORA_ERR_INVALID_ARG


def test_group_host_validation(L):
    assert L.lora_group(-1, 4, FAKE, FAKE, 4096, None) == _lib.LORA_ERR_INVALID_ARG
    assert L.lora_group(16, 2000, FAKE, FAKE, 1 << 20, None) == _lib.LORA_ERR_UNSUPPORTED
    assert L.lora_group(16, 4, 0, FAKE, 4096, None) == _lib.LORA_ERR_INVALID_ARG
    assert L.lora_group(16, 4, FAKE, FAKE + 4, 4096, None) == _lib.LORA_ERR_MISALIGNED
    assert L.lora_group(16, 4, FAKE, FAKE, 16, None) == _lib.LORA_ERR_INVALID_ARG


def test_launch_count_starts_at_zero_without_launches(L):
    # nothing in this process has launched a kernel: the counter only moves
    # on successful launches, and host-side rejections launch nothing
    before = L.lora_launch_count()
    assert _shrink(L, r=12) == _lib.LORA_ERR_UNSUPPORTED
    assert L.lora_launch_count() == before == 0


def test_has_active_from_host_indices():
    import numpy as np
    import torch
    from gather_matmul_b200 import ops
    assert not ops.active_from_host(np.array([-1, -1, 4, -7]), 4)   # 4 is outside [0, 4)
    assert ops.active_from_host(np.array([-1, 3]), 4)
    assert not ops.active_from_host(torch.full((5,), -1, dtype=torch.int32), 2)
    assert not ops.active_from_host(np.array([], dtype=np.int32), 2)
    assert ops._active(None, None, 4) == 1          # no host copy: the device decides
    assert ops._active(None, np.array([-1]), 4) == 0
    assert ops._active(False, np.array([0]), 4) == 0   # an explicit flag wins


def test_binding_constants_match_the_header():
    # the flag and size constants of the Python binding are the header's own
    import os
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "include", "lora.h")).read()
    defines = {m.group(1): int(m.group(2))
               for m in re.finditer(r"#define\s+(LORA_FLAG_\w+)\s+(\d+)u", src)}
    assert defines == {"LORA_FLAG_PDL_EARLY": 1, "LORA_FLAG_GROUPED": 2}
    for name, value in defines.items():
        assert getattr(_lib, name) == value, name
