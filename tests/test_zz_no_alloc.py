"""The entry point that allocates nothing, checked against the oracle and the regular entry point.

tl_nvfp4_verify_gemm_noalloc() serves callers that cannot allocate device memory at call
time (a serving engine that gave all free HBM to its KV-cache pool, or a host runtime that
forbids libraries from calling cudaMalloc). It keeps its split-K scratch in a static device
array and always runs the TL_PATH_BF16_EXACT kernel, with the same grid on this GPU, so its
output must equal tl_nvfp4_verify_gemm() under that path bit for bit, and the oracle within
the per-element tolerance. This file sorts last so that a run stopping at the first failure
has run every other test already; it also passes on its own in a fresh process (the first
call does the one-time set-up).
"""

import ctypes
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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
def test_no_alloc_matches_oracle_and_exact_path_twice_in_a_row(N, K, M):
    from nvfp4_weight_gemm_b200 import build, _lib
    import nvfp4_weight_gemm_b200 as tl
    build.build()
    oracle.build()
    w = synth.w_f32(N, K, seed=4, tensor_id=N)
    codes, scales, g = oracle.quantize(w)
    x_bits = synth.x_bf16(M, K, seed=4, tensor_id=synth.X_ID_BASE + N)
    y_ref, a_ref = oracle.gemm(x_bits, codes, scales, g)
    tol = 1e-3 * a_ref + 2.0 ** -8 * np.abs(y_ref)
    x, c, s = _dev_bf16(x_bits), _dev_u8(codes), _dev_u8(scales)
    y_reg = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with tl.gemm_path(tl.PATH_BF16_EXACT):   # the kernel the no-allocation entry point runs
        _call("tl_nvfp4_verify_gemm", x, c, s, g, y_reg)
    for _ in range(2):  # two calls in a row share the static scratch
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        _call("tl_nvfp4_verify_gemm_noalloc", x, c, s, g, y)
        torch.cuda.synchronize()
        _lib.check(_lib.lib().tl_noalloc_check_error(None))
        assert torch.equal(y, y_reg), "no-allocation entry point differs from the bf16-exact path"
        got = y.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - y_ref) <= tol), "no-allocation entry point outside the oracle's tolerance"


def test_no_alloc_rejects_too_many_rows():
    from nvfp4_weight_gemm_b200 import _lib
    A = 1 << 20
    st = _lib.lib().tl_nvfp4_verify_gemm_noalloc(A, 33, A, A, ctypes.c_float(1.0), A + (1 << 16), 256, 512, None)
    assert st == 3
    assert "32" in _lib.lib().tl_last_error_message().decode()


_FRESH = textwrap.dedent("""
    import ctypes, sys
    import numpy as np
    import torch
    sys.path.insert(0, {root!r})
    import oracle, synth
    from nvfp4_weight_gemm_b200 import _lib
    N, K, M = 1024, 2048, 16
    codes, scales, g = oracle.quantize(synth.w_f32(N, K, seed=7, tensor_id=7))
    xb = synth.x_bf16(M, K, seed=7)
    y_ref, a_ref = oracle.gemm(xb, codes, scales, g)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    c, s = torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda()
    ys = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    torch.cuda.synchronize()
    L = _lib.lib()
    def call(y):
        _lib.check(L.tl_nvfp4_verify_gemm_noalloc(ctypes.c_void_p(x.data_ptr()), M, ctypes.c_void_p(c.data_ptr()),
                                                  ctypes.c_void_p(s.data_ptr()), ctypes.c_float(g),
                                                  ctypes.c_void_p(y.data_ptr()), N, K, None))
        torch.cuda.synchronize()
        return torch.cuda.mem_get_info()[0]
    free0 = torch.cuda.mem_get_info()[0]
    free1 = call(ys[0])      # loads the module (static scratch, code): the one call that takes memory
    free2 = call(ys[1])
    free3 = call(ys[2])
    _lib.check(L.tl_noalloc_check_error(None))
    tol = 1e-3 * a_ref + 2.0 ** -8 * np.abs(y_ref)
    for y in ys:
        got = y.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - y_ref) <= tol)
        assert torch.equal(y, ys[0])
    print("FREE", free0, free1, free2, free3)
    assert free2 == free1 and free3 == free1, (free0, free1, free2, free3)
""")


def test_no_alloc_in_a_fresh_process_takes_memory_only_at_its_first_call():
    # a process whose only library call is the no-allocation entry point, with lazy module
    # loading: the first call's set-up loads the module (and with it the static scratch); the
    # calls after it must leave the device's free memory unchanged
    from nvfp4_weight_gemm_b200 import build
    build.build()
    oracle.build()
    env = dict(os.environ, CUDA_MODULE_LOADING="LAZY")
    r = subprocess.run([sys.executable, "-c", _FRESH.format(root=ROOT)], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "FREE" in r.stdout
