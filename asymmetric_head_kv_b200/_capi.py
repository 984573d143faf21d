"""ctypes declarations of the libdiffqkv.so C ABI (include/diffqkv.h).

Loading fails loudly when the library has not been built: there is no
fallback implementation of any entry point.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
# DIFFQKV_BOUNDS_CHECK=1 selects the checked build (device-side index checks that skip an out-of-range
# access and report DIFFQKV_ERR_DEVICE_BOUNDS); both are built in-tree by asymmetric_head_kv_b200.build
CHECKED = os.environ.get("DIFFQKV_BOUNDS_CHECK", "") not in ("", "0")
LIB_PATH = os.path.join(PKG, "libdiffqkv_checked.so" if CHECKED else "libdiffqkv.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "diffqkv.h")

STATUS = {
    0: "DIFFQKV_OK",
    1: "DIFFQKV_ERR_INVALID_ARG",
    2: "DIFFQKV_ERR_UNSUPPORTED",
    3: "DIFFQKV_ERR_MISALIGNED",
    4: "DIFFQKV_ERR_WORKSPACE",
    5: "DIFFQKV_ERR_CUDA",
    6: "DIFFQKV_ERR_DEVICE_TIMEOUT",
    7: "DIFFQKV_ERR_DEVICE_SEQLEN",
    8: "DIFFQKV_ERR_NO_DEVICE",
    9: "DIFFQKV_ERR_SCRATCH_LIMIT",
    10: "DIFFQKV_ERR_DEVICE_PAGE",
    11: "DIFFQKV_ERR_DEVICE_BOUNDS",
}
(OK, INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA_ERR, DEVICE_TIMEOUT, DEVICE_SEQLEN, NO_DEVICE,
 SCRATCH_LIMIT, DEVICE_PAGE, DEVICE_BOUNDS) = range(12)
TOPV_FULL_SOFTMAX_WEIGHTS = 1  # flag of diffqkv_decode_topv_ex (include/diffqkv.h)


class Dims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("n_q", ctypes.c_int32),
        ("n_k", ctypes.c_int32),
        ("n_v", ctypes.c_int32),
        ("d_k", ctypes.c_int32),
        ("d_v", ctypes.c_int32),
        ("scale", ctypes.c_float),
    ]


class DecodeTuning(ctypes.Structure):
    _fields_ = [("grid_ctas", ctypes.c_int32), ("stages", ctypes.c_int32), ("ctas_per_sm", ctypes.c_int32)]


class DecodePlan(ctypes.Structure):
    _fields_ = [
        ("tile_tokens", ctypes.c_int32),
        ("stages", ctypes.c_int32),
        ("grid_ctas", ctypes.c_int32),
        ("threads", ctypes.c_int32),
        ("v_heads_per_tile", ctypes.c_int32),
        ("smem_bytes", ctypes.c_int64),
        ("workspace_bytes", ctypes.c_int64),
    ]


class DiffqkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


_lib = None

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_DIMS = ctypes.POINTER(Dims)

SIGNATURES = {
    "diffqkv_status_string": ([_I32], ctypes.c_char_p),
    "diffqkv_version": ([], _I32),
    "diffqkv_decode_workspace_size": ([_DIMS], _SZ),
    "diffqkv_workspace_init": ([_P, _SZ, _P], _I32),
    "diffqkv_decode": ([_DIMS, _P, _P, _P, _P, _I32, _I32, _P, _P, _SZ, _P], _I32),
    "diffqkv_decode_ex": ([_DIMS, _P, _P, _P, _P, _I32, _I32, _P, _P, _SZ, ctypes.POINTER(DecodeTuning), _P], _I32),
    "diffqkv_decode_append": ([_DIMS, _P, _P, _P, _P, _P, _P, _I32, _I32, _P, _P, _SZ, _P], _I32),
    "diffqkv_decode_paged": ([_DIMS, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _P, _I32, _P, _P, _SZ, _P], _I32),
    "diffqkv_decode_plan": ([_DIMS, _I32, _I32, _I32, ctypes.POINTER(DecodeTuning), ctypes.POINTER(DecodePlan)],
                            _I32),
    "diffqkv_decode_from_host": ([_DIMS, _P, _P, _P, _P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], _I32),
    "diffqkv_decode_topv_workspace_size": ([_DIMS, _I32, _I32], _SZ),
    "diffqkv_decode_topv": ([_DIMS, _P, _P, _P, _P, _I32, _I32, _I32, _P, _P, _P, _SZ, _P], _I32),
    "diffqkv_decode_topv_ex": ([_DIMS, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _SZ, _P], _I32),
    "diffqkv_decode_topv_paged": ([_DIMS, _P, _P, _P, _P, _I32, _I32, _I32, _P, _I32, _I32, _I32, _P, _P, _P, _SZ,
                                   _P], _I32),
    "diffqkv_prefill_causal": ([_DIMS, _P, _P, _P, _I32, _P, _P], _I32),
    "diffqkv_prefill_causal_prefix": ([_DIMS, _P, _P, _P, _I32, _I32, _P, _P], _I32),
    "diffqkv_prefill_causal_ex": ([_DIMS, _P, _P, _P, _I32, _I32, _P, _P, _P], _I32),
    "diffqkv_prefill_causal_paged": ([_DIMS, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _P, _P, _P], _I32),
    "diffqkv_augq_project": ([_P, _P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _P], _I32),
    "diffqkv_workspace_status": ([_P, _SZ, _P, ctypes.POINTER(_I32)], _I32),
    "diffqkv_get_device_status": ([_P, ctypes.POINTER(_I32)], _I32),
    "diffqkv_selftest_wait_timeout": ([_I64, _P], _I32),
    "diffqkv_decode_noalloc": ([_DIMS, _P, _P, _P, _P, _I32, _I32, _P, _P], _I32),
    "diffqkv_fold_query": ([_DIMS, _I32, _I32, _P, _P, _P, _P], _I32),
}


def header_symbols() -> list:
    """Names of every function include/diffqkv.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(diffqkv_[a-z0-9_]+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m asymmetric_head_kv_b200.build` "
                "(there is no fallback implementation)")
        h = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.argtypes = args
            fn.restype = res
        _lib = h
    return _lib


def check(status: int, what: str):
    if status != OK:
        raise DiffqkvError(status, what)
