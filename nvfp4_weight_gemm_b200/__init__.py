"""NVFP4 verify GEMM for B200: Y[M,N] = X[M,K] . dequant(W)[N,K]^T, M <= 128.

Thin Python layer over libtl_nvfp4.so (the C ABI in include/tl_nvfp4.h). Torch tensors
are used for device memory and streams only; every step of the computation runs in the
library's CUDA kernels. There is no CPU path.
"""

from __future__ import annotations

import ctypes

from . import _lib
from ._lib import Matrix, TlError, check

__all__ = ["verify_gemm", "verify_gemm_simt", "set_gemm_path", "get_gemm_path", "gemm_path", "PATH_BLOCK_SCALED",
           "PATH_BF16_EXACT", "PATH_EXACT", "verify_stack", "verify_stack_host", "Plan", "dequant",
           "quantize", "check_device_error", "noalloc_check_error", "fp8_head", "gdn_commit", "init", "num_sms", "Matrix", "TlError"]


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def init(device: int = 0) -> None:
    check(_lib.lib().tl_init(device))


def num_sms(device: int = 0) -> int:
    return _lib.lib().tl_num_sms(device)


PATH_BLOCK_SCALED = _lib.TL_PATH_BLOCK_SCALED
PATH_BF16_EXACT = _lib.TL_PATH_BF16_EXACT
PATH_EXACT = _lib.TL_PATH_EXACT


def set_gemm_path(path: int) -> None:
    """Select the tensor-core path of verify_gemm, verify_stack(_host) and new plans:
    PATH_EXACT (default; exact f16 operands: hardware E2M1 decode, X prepared per row),
    PATH_BF16_EXACT (exact bf16 operands, integer decode; slower) or PATH_BLOCK_SCALED
    (approximate: X split into FP4 pieces for the block-scaled MMA)."""
    check(_lib.lib().tl_set_gemm_path(path))


def get_gemm_path() -> int:
    return _lib.lib().tl_get_gemm_path()


class gemm_path:
    """Context manager: `with gemm_path(PATH_BF16_EXACT): ...` restores the previous path on exit."""

    def __init__(self, path: int):
        self.path = path
        self.prev = None

    def __enter__(self):
        self.prev = get_gemm_path()
        set_gemm_path(self.path)
        return self

    def __exit__(self, *exc):
        set_gemm_path(self.prev)
        return False


def _gemm(name, x, codes, scales, global_scale, y=None, stream=None):
    import torch
    M, K = x.shape
    N = codes.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    check(getattr(_lib.lib(), name)(_ptr(x), M, _ptr(codes), _ptr(scales), ctypes.c_float(global_scale),
                                    _ptr(y), N, K, _stream(stream)))
    return y


def verify_gemm(x, codes, scales, global_scale, y=None, stream=None):
    """Tensor-core path. x: bf16 [M, K]; codes: uint8 [N, K/2]; scales: uint8 [N, K/16]."""
    return _gemm("tl_nvfp4_verify_gemm", x, codes, scales, global_scale, y, stream)


def verify_gemm_simt(x, codes, scales, global_scale, y=None, stream=None):
    """CUDA-core path (cross-check)."""
    return _gemm("tl_nvfp4_verify_gemm_simt", x, codes, scales, global_scale, y, stream)


def make_matrices(entries):
    """entries: iterable of (codes, scales, global_scale, x, y) tensors -> ctypes array of Matrix."""
    entries = list(entries)
    arr = (Matrix * len(entries))()
    for i, (c, s, g, x, y) in enumerate(entries):
        arr[i] = Matrix(c.data_ptr(), s.data_ptr(), x.data_ptr() if x is not None else None,
                        y.data_ptr() if y is not None else None, float(g), c.shape[0], c.shape[1] * 2)
    return arr


def verify_stack(mats, M: int, stream=None):
    """mats: ctypes array from make_matrices (x and y set)."""
    check(_lib.lib().tl_nvfp4_verify_stack(mats, len(mats), M, _stream(stream)))


def verify_stack_host(mats, M: int, x_host, x_dev, y_host, y_dev, stream=None):
    """End-to-end stack call: X from host memory in, Y to host memory out (contiguous buffers)."""
    check(_lib.lib().tl_nvfp4_verify_stack_host(mats, len(mats), M, _ptr(x_host), _ptr(x_dev),
                                                _ptr(y_host), _ptr(y_dev), _stream(stream)))


class Plan:
    """A stack whose descriptors are built once (tl_nvfp4_plan_create); run() only launches.

    Keeps the ctypes matrix table and the tensors it points to alive while the plan lives."""

    def __init__(self, entries, M: int):
        self._entries = list(entries)
        self._mats = make_matrices(self._entries)
        self.M = M
        h = ctypes.c_void_p()
        check(_lib.lib().tl_nvfp4_plan_create(self._mats, len(self._mats), M, ctypes.byref(h)))
        self._h = h

    def run(self, stream=None):
        check(_lib.lib().tl_nvfp4_plan_run(self._h, _stream(stream)))

    def run_host(self, x_host, y_host, stream=None):
        check(_lib.lib().tl_nvfp4_plan_run_host(self._h, _ptr(x_host), _ptr(y_host), _stream(stream)))

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            _lib.lib().tl_nvfp4_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def dequant(codes, scales, global_scale, out=None, stream=None):
    import torch
    N, K = codes.shape[0], codes.shape[1] * 2
    if out is None:
        out = torch.empty((N, K), dtype=torch.float32, device=codes.device)
    check(_lib.lib().tl_nvfp4_dequant(_ptr(codes), _ptr(scales), ctypes.c_float(global_scale), _ptr(out), N, K,
                                      _stream(stream)))
    return out


def quantize(w, stream=None):
    """fp32 [N, K] device tensor -> (codes uint8 [N, K/2], scales uint8 [N, K/16], g). Synchronises."""
    import torch
    N, K = w.shape
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((N, K // 16), dtype=torch.uint8, device=w.device)
    g = ctypes.c_float(0.0)
    check(_lib.lib().tl_nvfp4_quantize(_ptr(w), N, K, _ptr(codes), _ptr(scales), ctypes.byref(g), _stream(stream)))
    return codes, scales, g.value


def check_device_error(stream=None) -> None:
    check(_lib.lib().tl_check_device_error(_stream(stream)))


def noalloc_check_error(stream=None) -> None:
    """Status word of the no-allocation entry point's static scratch (allocation-free)."""
    check(_lib.lib().tl_noalloc_check_error(_stream(stream)))


def fp8_head(x, w_fp8, scale, logits=None, stream=None):
    """FP8 output head: x bf16 [M, K]; w_fp8 uint8 [N, K] (E4M3 bytes); scale a float (per tensor)
    or a float32 device tensor [N] (per row). Returns (logits float32 [M, N], top2 int32/float32
    tensor [M, 4] viewed as (token, top1, top2, gap_ulp): the token as int32 bits in column 0)."""
    import torch
    M, K = x.shape
    N = w_fp8.shape[0]
    if logits is None:
        logits = torch.empty((M, N), dtype=torch.float32, device=x.device)
    top2 = torch.empty((M, 4), dtype=torch.int32, device=x.device)
    if isinstance(scale, (float, int)):
        ts, rs = float(scale), None
    else:
        ts, rs = 0.0, ctypes.c_void_p(scale.data_ptr())
    check(_lib.lib().tl_fp8_head(_ptr(x), M, _ptr(w_fp8), N, K, ctypes.c_float(ts), rs, _ptr(logits), _ptr(top2),
                                 _stream(stream)))
    return logits, top2


def head_top2_fields(top2):
    """(token int64[M], top1, top2, gap float64[M]) from fp8_head's top2 tensor (on the host)."""
    import numpy as np
    t = top2.cpu().numpy()
    return (t[:, 0].astype(np.int64), t[:, 1].view(np.float32).astype(np.float64),
            t[:, 2].view(np.float32).astype(np.float64), t[:, 3].view(np.float32).astype(np.float64))


def gdn_commit(state, k, v, alpha, beta, path, stream=None):
    """Closed-form commit of an accepted draft path through Gated DeltaNet states, in place.

    state float32 [H, d_v, d_k] (device); k float32 [n_nodes, H, d_k]; v float32 [n_nodes, H, d_v];
    alpha, beta float32 [n_nodes, H]; path: the accepted node indices in order (a host sequence
    of at most 32 ints). Returns `state`."""
    H, d_v, d_k = state.shape
    n_nodes = k.shape[0]
    p = [int(t) for t in path]
    arr = (ctypes.c_int * max(1, len(p)))(*p)
    check(_lib.lib().tl_gdn_commit(_ptr(state), H, d_k, d_v, _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), n_nodes, arr,
                                   len(p), _stream(stream)))
    return state
