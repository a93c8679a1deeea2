"""ctypes view of the C ABI declared in include/vsa.h.

Loads the in-tree libvsa_b200.so.  There is no fallback: if the library is
missing, importing the package raises.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvsa_b200.so")

VSA_OK = 0
STATUS_NAMES = {
    0: "VSA_OK", 1: "VSA_ERR_INVALID_ARGUMENT", 2: "VSA_ERR_UNSUPPORTED", 3: "VSA_ERR_MISALIGNED",
    4: "VSA_ERR_WORKSPACE", 5: "VSA_ERR_CUDA", 6: "VSA_ERR_TIMEOUT",
}

# Every symbol the header declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_F32 = ctypes.c_float
_SZ = ctypes.c_size_t
_I64 = ctypes.c_int64


class VsaShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("grid_t", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32)]


_SP = ctypes.POINTER(VsaShape)

SIGNATURES = {
    "vsa_abi_version": (ctypes.c_int32, []),
    "vsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "vsa_last_error": (ctypes.c_char_p, []),
    "vsa_shape_info": (ctypes.c_int, [_SP, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int32)]),
    "vsa_tile": (ctypes.c_int, [_SP, _P, _P, _P]),
    "vsa_untile": (ctypes.c_int, [_SP, _P, _P, _P]),
    "vsa_pool": (ctypes.c_int, [_SP, _P, _P, _P]),
    "vsa_coarse_workspace_bytes": (_SZ, [_SP]),
    "vsa_coarse": (ctypes.c_int, [_SP, _P, _P, _P, _F32, _P, _P, _P, _SZ, _P]),
    "vsa_topk": (ctypes.c_int, [_SP, _P, _I32, _P, _P]),
    "vsa_group": (ctypes.c_int, [_SP, _P, _P, _P]),
    "vsa_fine": (ctypes.c_int, [_SP, _P, _P, _P, _P, _I32, _P, _F32, _P, _P, _P]),
    "vsa_combine": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _P]),
    "vsa_pool_qkv": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _P, _P]),
    "vsa_topk_order": (ctypes.c_int, [_SP, _P, _I32, _P, _P, _P, _P]),
    "vsa_fine_fused": (ctypes.c_int, [_SP, _P, _P, _P, _P, _I32, _P, _P, _F32, _P, _P, _P, _P, _P, _P]),
    "vsa_schedule_bytes": (_SZ, [_SP, _I32]),
    "vsa_schedule": (ctypes.c_int, [_SP, _P, _I32, _P, _P, _P]),
    "vsa_qk_norm_rope": (ctypes.c_int, [_SP, _P, _P, _P, _P, _F32, _F32, _I64, _I64, _P, _P, _P]),
    "vsa_workspace_bytes": (_SZ, [_SP, _I32]),
    "vsa_forward": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _I32, _F32, _P, _SZ, _P, _P]),
    "vsa_forward_rerun": (ctypes.c_int, [_SP, _I32, _I32, _P, ctypes.POINTER(ctypes.c_int32), _P]),
    "vsa_workspace_bytes_host": (_SZ, [_SP, _I32]),
    "vsa_forward_host": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _I32, _F32, _P, _SZ, _P, _P]),
    "vsa_forward_noalloc": (ctypes.c_int, [_SP, _P, _P, _P, _P, _P, _I32, _F32, _P, _P]),
    "vsa_device_status": (ctypes.c_int, [_P]),
    "vsa_debug_wait_probe": (ctypes.c_int, [ctypes.c_uint64, _P]),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"CUDA library {path} is missing; build it with "
            "`python block_sparse_attention_cube_b200/build_lib.py` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
