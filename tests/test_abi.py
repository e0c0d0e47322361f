"""The C ABI on the host: the library loads, exports every declared symbol, and rejects
invalid arguments before touching the GPU (these calls never reach CUDA)."""

import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "tl_nvfp4.h")


@pytest.fixture(scope="module")
def L():
    from nvfp4_weight_gemm_b200 import build, _lib
    build.build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tl_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("tl_nvfp4_verify_gemm", "tl_nvfp4_verify_stack", "tl_nvfp4_dequant", "tl_init",
                 "tl_check_device_error", "tl_status_string", "tl_last_error_message"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    from nvfp4_weight_gemm_b200 import _lib
    for name in declared_functions():
        assert hasattr(L, name), name
    assert sorted(_lib.EXPORTS) == declared_functions()


def test_status_strings(L):
    from nvfp4_weight_gemm_b200._lib import STATUS
    for code, name in STATUS.items():
        assert L.tl_status_string(code).decode() == name


A = 1 << 20  # a fake, 16-byte aligned address: never dereferenced on these paths


def _gemm(L, x=A, M=8, c=A + 4096, s=A + 8192, g=1.0, y=A + (1 << 16), N=256, K=512):
    return L.tl_nvfp4_verify_gemm(x, M, c, s, ctypes.c_float(g), y, N, K, None)


@pytest.mark.parametrize("kw,status", [
    (dict(M=129), 3), (dict(M=-1), 1), (dict(K=100), 1), (dict(K=0), 1), (dict(K=128), 1),
    (dict(N=0), 1), (dict(c=A + 8), 2), (dict(s=A + 4), 2), (dict(x=A + 2), 2), (dict(y=A + 6), 2),
    (dict(c=0), 1), (dict(g=float("nan")), 1), (dict(g=float("inf")), 1), (dict(y=A), 1),
])
def test_verify_gemm_rejects(L, kw, status):
    assert _gemm(L, **kw) == status
    assert L.tl_last_error_message().decode() != ""


def test_simt_path_validates_the_same_way(L):
    assert L.tl_nvfp4_verify_gemm_simt(A, 129, A, A, ctypes.c_float(1.0), A, 8, 256, None) == 3
    assert L.tl_nvfp4_verify_gemm_simt(A, 4, A, A, ctypes.c_float(1.0), A + 1, 8, 256, None) == 2


def test_stack_rejects_bad_counts(L):
    from nvfp4_weight_gemm_b200._lib import Matrix
    arr = (Matrix * 1)()
    assert L.tl_nvfp4_verify_stack(arr, 0, 8, None) == 1
    assert L.tl_nvfp4_verify_stack(arr, 5000, 8, None) == 1
    assert L.tl_nvfp4_verify_stack(arr, 1, 129, None) == 3
    arr[0] = Matrix(A + 8, A, A, A + (1 << 16), 1.0, 256, 512)
    assert L.tl_nvfp4_verify_stack(arr, 1, 8, None) == 2


def test_dequant_and_quantize_validate(L):
    assert L.tl_nvfp4_dequant(A, A, ctypes.c_float(1.0), A + 4, 16, 256, None) == 2
    assert L.tl_nvfp4_dequant(A, A, ctypes.c_float(1.0), A, 16, 100, None) == 1
    g = ctypes.c_float()
    assert L.tl_nvfp4_quantize(A, 0, 256, A, A, ctypes.byref(g), None) == 1
    assert L.tl_nvfp4_quantize(A, 4, 24, A, A, ctypes.byref(g), None) == 1


def test_gdn_commit_validates(L):
    path = (ctypes.c_int * 4)(0, 1, 2, 3)
    def call(H=4, dk=128, dv=128, state=A, n_nodes=8, p=path, n=4):
        # fake, disjoint 16-byte aligned addresses; never dereferenced on these paths
        return L.tl_gdn_commit(state, H, dk, dv, A + (1 << 24), A + (1 << 25), A + (1 << 26), A + (1 << 27),
                               n_nodes, p, n, None)
    assert call(H=0) == 1
    assert call(dk=96) == 3 and call(dv=32) == 3
    assert call(n=33) == 1 and call(n=-1) == 1
    assert call(n_nodes=3) == 1                 # node index 3 is outside 0..2
    assert call(state=A + 4) == 2
    assert L.tl_gdn_commit(A, 4, 128, 128, A + (1 << 24) + 4, A + (1 << 25), A + (1 << 26), A + (1 << 27), 8, path, 4,
                           None) == 2   # misaligned keys
    assert call(state=0) == 1
    assert call(n=0) == 0                       # an empty path is a no-op and never reaches CUDA
    # the state may not overlap the per-node inputs (state = keys)
    assert L.tl_gdn_commit(A, 4, 128, 128, A, A + (1 << 24), A + (1 << 25), A + (1 << 26), 8, path, 4, None) == 1


def test_fp8_head_validates(L):
    def call(x=A, M=8, w=A + (1 << 24), N=1000, K=512, ts=1.0, rs=None, lg=A + (1 << 26), t2=A + (1 << 27)):
        return L.tl_fp8_head(x, M, w, N, K, ctypes.c_float(ts), rs, lg, t2, None)
    assert call(M=33) == 3 and call(M=-1) == 1
    assert call(N=1) == 1 and call(K=100) == 1
    assert call(x=A + 4) == 2 and call(lg=A + (1 << 26) + 4) == 2
    assert call(ts=float("nan")) == 1
    assert call(lg=A) == 1                       # logits over x
    assert call(t2=A + (1 << 26)) == 1           # top2 over logits
    assert call(M=0) == 0                        # no rows: a no-op before any CUDA call
