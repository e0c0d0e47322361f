"""ctypes binding of libtl_nvfp4.so: argument marshalling only.

Every function here forwards to the C ABI declared in include/tl_nvfp4.h. Raises
RuntimeError with the library's status and message on any non-OK status. There is no
fallback: if the shared library cannot be loaded, importing a function fails loudly.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtl_nvfp4.so")

TL_OK = 0
STATUS = {
    0: "TL_OK", 1: "TL_ERR_INVALID_VALUE", 2: "TL_ERR_MISALIGNED", 3: "TL_ERR_UNSUPPORTED",
    4: "TL_ERR_CUDA", 5: "TL_ERR_TIMEOUT", 6: "TL_ERR_NOT_INITIALIZED", 7: "TL_ERR_NONFINITE",
    8: "TL_ERR_DEVICE_FAULT",
}

# Every symbol include/tl_nvfp4.h declares.
EXPORTS = (
    "tl_init", "tl_shutdown", "tl_nvfp4_verify_gemm", "tl_nvfp4_verify_gemm_simt", "tl_nvfp4_verify_gemm_noalloc",
    "tl_nvfp4_verify_stack", "tl_nvfp4_verify_stack_host", "tl_nvfp4_plan_create",
    "tl_nvfp4_plan_run", "tl_nvfp4_plan_run_host", "tl_nvfp4_plan_destroy", "tl_nvfp4_dequant",
    "tl_nvfp4_quantize", "tl_check_device_error", "tl_selftest_bounded_wait", "tl_num_sms", "tl_status_string",
    "tl_last_error_message", "tl_set_gemm_path", "tl_get_gemm_path", "tl_noalloc_check_error", "tl_fp8_head",
    "tl_gdn_commit",
)

# Tensor-core paths (tl_set_gemm_path).
TL_PATH_BLOCK_SCALED = 0
TL_PATH_BF16_EXACT = 1
TL_PATH_EXACT = 2


class HeadTop2(ctypes.Structure):
    """tl_head_top2."""
    _fields_ = [("token", ctypes.c_int), ("top1", ctypes.c_float), ("top2", ctypes.c_float), ("gap_ulp", ctypes.c_float)]


class TlError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class Matrix(ctypes.Structure):
    """tl_nvfp4_matrix."""
    _fields_ = [
        ("w_codes", ctypes.c_void_p), ("w_scales", ctypes.c_void_p),
        ("x", ctypes.c_void_p), ("y", ctypes.c_void_p),
        ("global_scale", ctypes.c_float), ("N", ctypes.c_int), ("K", ctypes.c_int),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m nvfp4_weight_gemm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        sig = {
            "tl_init": [i],
            "tl_shutdown": [],
            "tl_nvfp4_verify_gemm": [vp, i, vp, vp, f, vp, i, i, vp],
            "tl_nvfp4_verify_gemm_simt": [vp, i, vp, vp, f, vp, i, i, vp],
            "tl_nvfp4_verify_gemm_noalloc": [vp, i, vp, vp, f, vp, i, i, vp],
            "tl_nvfp4_verify_stack": [ctypes.POINTER(Matrix), i, i, vp],
            "tl_nvfp4_verify_stack_host": [ctypes.POINTER(Matrix), i, i, vp, vp, vp, vp, vp],
            "tl_nvfp4_plan_create": [ctypes.POINTER(Matrix), i, i, ctypes.POINTER(vp)],
            "tl_nvfp4_plan_run": [vp, vp],
            "tl_nvfp4_plan_run_host": [vp, vp, vp, vp],
            "tl_nvfp4_plan_destroy": [vp],
            "tl_nvfp4_dequant": [vp, vp, f, vp, i, i, vp],
            "tl_nvfp4_quantize": [vp, i, i, vp, vp, ctypes.POINTER(f), vp],
            "tl_check_device_error": [vp],
            "tl_noalloc_check_error": [vp],
            "tl_fp8_head": [vp, i, vp, i, i, f, vp, vp, vp, vp],
            "tl_gdn_commit": [vp, i, i, i, vp, vp, vp, vp, i, ctypes.POINTER(i), i, vp],
            "tl_selftest_bounded_wait": [ctypes.c_uint, vp],
            "tl_num_sms": [i],
            "tl_status_string": [i],
            "tl_last_error_message": [],
            "tl_set_gemm_path": [i],
            "tl_get_gemm_path": [],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = i
        L.tl_shutdown.restype = None
        L.tl_status_string.restype = ctypes.c_char_p
        L.tl_last_error_message.restype = ctypes.c_char_p
        _lib = L
    return _lib


def check(status: int) -> None:
    if status != TL_OK:
        raise TlError(status, lib().tl_last_error_message().decode())


def call(name: str, *args) -> int:
    """Call an entry point and return its raw status (tests of the error paths use this)."""
    return getattr(lib(), name)(*args)
