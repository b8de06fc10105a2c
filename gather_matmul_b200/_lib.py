"""ctypes loader for liblora_b200.so (the C ABI declared in include/lora.h).

Loading fails loudly when the library has not been built: there is no
fallback implementation behind this module.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblora_b200.so")

LORA_OK = 0
LORA_ERR_INVALID_ARG = -1
LORA_ERR_UNSUPPORTED = -2
LORA_ERR_MISALIGNED = -3
LORA_ERR_CUDA = -4
LORA_ERR_BAD_INDEX = -5
LORA_F16 = 0
LORA_BF16 = 1
LORA_MAX_SLICES = 8
LORA_MAX_SLOTS = 1024
LORA_MAX_TOKENS = 1 << 22
LORA_NOALLOC_MAX_TOKENS = 8192
LORA_FLAG_PDL_EARLY = 1
LORA_FLAG_GROUPED = 2

# Every symbol the header declares, with (restype, argtypes).
_i32, _i64, _sz, _f32, _vp = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p
SIGNATURES = {
    "lora_workspace_bytes": (_sz, [_i32, _i32]),
    "lora_workspace_reset": (_i32, [_vp, _sz, _vp]),
    "lora_group": (_i32, [_i32, _i32, _vp, _vp, _sz, _vp]),
    "lora_shrink": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp, _vp, _i32,
                           _vp, _sz, _vp]),
    "lora_expand": (_i32, [_i32, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp, _vp, _f32, _vp,
                           _i64, _vp, _i32, _vp, _sz, _vp]),
    "lora_shrink_segment": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp, _vp,
                                   _i32, _vp, _i32, _vp, _sz, _vp]),
    "lora_expand_segment": (_i32, [_i32, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp, _vp, _vp,
                                   _i32, _f32, _vp, _i64, _vp, _i32, _vp, _sz, _vp]),
    "lora_bgmv": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _i32, _vp, _vp, _f32,
                         _vp, _i64, _vp, _vp, _vp, _i32, ctypes.c_uint, _vp, _sz, _vp]),
    "lora_bgmv_launches": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _vp]),
    "lora_sgmv": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _i32, _vp, _vp, _f32,
                         _vp, _i64, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _sz, _vp]),
    "lora_check_errors": (_i32, [_vp, _sz, _vp]),
    "lora_shrink_noalloc": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp,
                                   _vp, _i32, _vp]),
    "lora_shrink_laned": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp, _vp,
                                 _i32, _vp, _sz, _vp]),
    "lora_set_slot_ranks": (_i32, [_i32, _vp, _vp, _sz, _vp]),
    "lora_status_string": (ctypes.c_char_p, [_i32]),
    "lora_build_info": (ctypes.c_char_p, []),
    "lora_launch_count": (ctypes.c_ulonglong, []),
}

_lib = None


def load(path: str = LIB_PATH):
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m gather_matmul_b200.build` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    L = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    if path == LIB_PATH:
        _lib = L
    return L


def status_string(code: int) -> str:
    return load().lora_status_string(code).decode()
