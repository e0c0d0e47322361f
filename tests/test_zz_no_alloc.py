"""The entry point that allocates nothing, checked against the regular entry point.

tl_nvfp4_verify_gemm_noalloc() serves callers that cannot allocate device memory at call
time (a serving engine that gave all free HBM to its KV-cache pool, or a host runtime that
forbids libraries from calling cudaMalloc). It keeps its split-K scratch in a static device
array. This file sorts last so that a run stopping at the first failure has run every other
test already; it also passes on its own in a fresh process (the first call does the
one-time set-up).
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _call(name, x, codes, scales, g, y):
    from nvfp4_weight_gemm_b200 import _lib
    M, K = x.shape
    N = codes.shape[0]
    st = getattr(_lib.lib(), name)(ctypes.c_void_p(x.data_ptr()), M, ctypes.c_void_p(codes.data_ptr()),
                                   ctypes.c_void_p(scales.data_ptr()), ctypes.c_float(g),
                                   ctypes.c_void_p(y.data_ptr()), N, K,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    _lib.check(st)


@pytest.mark.parametrize("N,K,M", [(677, 2304, 24), (5120, 5120, 32), (256, 512, 5)])
def test_no_alloc_matches_regular_entry_point_twice_in_a_row(N, K, M):
    from nvfp4_weight_gemm_b200 import build
    build.build()
    oracle.build()
    w = synth.w_f32(N, K, seed=4, tensor_id=N)
    codes, scales, g = oracle.quantize(w)
    x_bits = synth.x_bf16(M, K, seed=4, tensor_id=synth.X_ID_BASE + N)
    _, a_ref = oracle.gemm(x_bits, codes, scales, g)
    x, c, s = _dev_bf16(x_bits), _dev_u8(codes), _dev_u8(scales)
    y_reg = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    _call("tl_nvfp4_verify_gemm", x, c, s, g, y_reg)
    ref = y_reg.float().cpu().numpy().astype(np.float64)
    for _ in range(2):  # two calls in a row share the static scratch
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        _call("tl_nvfp4_verify_gemm_noalloc", x, c, s, g, y)
        torch.cuda.synchronize()
        got = y.float().cpu().numpy().astype(np.float64)
        tol = 1e-3 * a_ref + 2.0 ** -8 * np.abs(ref)
        assert np.all(np.abs(got - ref) <= tol), "no-alloc entry point differs from tl_nvfp4_verify_gemm"


def test_no_alloc_rejects_too_many_rows():
    from nvfp4_weight_gemm_b200 import _lib
    A = 1 << 20
    st = _lib.lib().tl_nvfp4_verify_gemm_noalloc(A, 33, A, A, ctypes.c_float(1.0), A + (1 << 16), 256, 512, None)
    assert st == 3
    assert "32" in _lib.lib().tl_last_error_message().decode()
