"""CPU oracle for the NVFP4 verify GEMM: Python bindings to ``nvfp4_oracle.c``.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package. The GPU library never
imports it and shares no code with it.

It also holds, in numpy fp64, the oracles of two next rows: the FP8 output head's logits and the
greedy top-2 / near-tie statistic, and the closed-form commit of an accepted draft path through a
Gated DeltaNet state (end of this file; that one's parity against the pages is unpinned, as they
print no equation).

The C source computes everything in fp64 from the format definitions:
E2M1 codes (two per byte, low nibble = even k), one E4M3 scale per 16-element
K block, one FP32 tensor scale; Y = X . dequant(W)^T. See the header of
``nvfp4_oracle.c`` for the definitions and their sources.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_nvfp4.so")

OR_OK = 0


def build(force: bool = False) -> str:
    """Compile the oracle into a host shared library (gcc, OpenMP, strict IEEE fp64)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.or_e2m1_decode.restype = ctypes.c_double
        L.or_e2m1_decode.argtypes = [ctypes.c_uint32]
        L.or_e4m3_decode.restype = ctypes.c_double
        L.or_e4m3_decode.argtypes = [ctypes.c_uint32]
        L.or_e4m3_encode.restype = ctypes.c_uint32
        L.or_e4m3_encode.argtypes = [ctypes.c_double]
        L.or_e2m1_encode.restype = ctypes.c_uint32
        L.or_e2m1_encode.argtypes = [ctypes.c_double]
        L.or_quantize.restype = ctypes.c_int
        L.or_quantize.argtypes = [p, i64, i64, p, p, p]
        L.or_dequant.restype = ctypes.c_int
        L.or_dequant.argtypes = [p, p, ctypes.c_float, i64, i64, p, p]
        L.or_gemm.restype = ctypes.c_int
        L.or_gemm.argtypes = [p, i64, p, p, ctypes.c_float, i64, i64, p, p]
        L.or_gemm_sampled.restype = ctypes.c_int
        L.or_gemm_sampled.argtypes = [p, i64, p, p, ctypes.c_float, i64, i64, p, p, i64, p, p]
        L.or_num_threads.restype = ctypes.c_int
        L.or_set_num_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def e2m1_decode(code: int) -> float:
    return lib().or_e2m1_decode(code)


def e4m3_decode(byte: int) -> float:
    return lib().or_e4m3_decode(byte)


def e4m3_encode(t: float) -> int:
    return lib().or_e4m3_encode(float(t))


def e2m1_encode(q: float) -> int:
    return lib().or_e2m1_encode(float(q))


def quantize(w: np.ndarray):
    """fp32 W[N, K] -> (codes uint8[N, K/2], scales uint8[N, K/16], g float)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros((N, K // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    rc = lib().or_quantize(_ptr(w), N, K, _ptr(codes), _ptr(scales), _ptr(g))
    if rc != OR_OK:
        raise ValueError(f"or_quantize failed with code {rc}")
    return codes, scales, float(g[0])


def dequant(codes: np.ndarray, scales: np.ndarray, g: float, want_wq: bool = False):
    """-> w32 float32[N, K] = fp32(e2m1*e4m3*g), and optionally wq float64[N, K] = e2m1*e4m3."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    N, K = codes.shape[0], codes.shape[1] * 2
    w32 = np.zeros((N, K), dtype=np.float32)
    wq = np.zeros((N, K), dtype=np.float64) if want_wq else None
    rc = lib().or_dequant(_ptr(codes), _ptr(scales), ctypes.c_float(g), N, K, _ptr(w32),
                          _ptr(wq) if wq is not None else None)
    if rc != OR_OK:
        raise ValueError(f"or_dequant failed with code {rc}")
    return (w32, wq) if want_wq else w32


def gemm(x_bits: np.ndarray, codes: np.ndarray, scales: np.ndarray, g: float):
    """x_bits: bf16 bits uint16[M, K]. -> (y_ref float64[M, N], a_ref float64[M, N])."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    M, K = x_bits.shape
    N = codes.shape[0]
    if codes.shape[1] * 2 != K:
        raise ValueError("K of X and W differ")
    y = np.zeros((M, N), dtype=np.float64)
    a = np.zeros((M, N), dtype=np.float64)
    rc = lib().or_gemm(_ptr(x_bits), M, _ptr(codes), _ptr(scales), ctypes.c_float(g), N, K,
                       _ptr(y), _ptr(a))
    if rc != OR_OK:
        raise ValueError(f"or_gemm failed with code {rc}")
    return y, a


def gemm_sampled(x_bits, codes, scales, g, m_idx, n_idx):
    """Oracle outputs at the (m_idx[i], n_idx[i]) positions only."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    m_idx = np.ascontiguousarray(m_idx, dtype=np.int64)
    n_idx = np.ascontiguousarray(n_idx, dtype=np.int64)
    M, K = x_bits.shape
    N = codes.shape[0]
    y = np.zeros(len(m_idx), dtype=np.float64)
    a = np.zeros(len(m_idx), dtype=np.float64)
    rc = lib().or_gemm_sampled(_ptr(x_bits), M, _ptr(codes), _ptr(scales), ctypes.c_float(g), N, K,
                               _ptr(m_idx), _ptr(n_idx), len(m_idx), _ptr(y), _ptr(a))
    if rc != OR_OK:
        raise ValueError(f"or_gemm_sampled failed with code {rc}")
    return y, a


def num_threads() -> int:
    return lib().or_num_threads()


def set_num_threads(n: int) -> None:
    lib().or_set_num_threads(int(n))


# ---------------------------------------------------------------- FP8 output head (next row)
#
# The served weights keep the output head in FP8 (TandemLLM docs v0.12.0, "What TandemLLM is",
# the paragraph on cutting the bytes a step reads), and the greedy output is exact up to near
# ties, where the two best tokens are within one unit in the last place (same page, "the first
# rule is agreement with greedy decoding"). Parity pinned by tests/test_oracle_pins.py.

def fp8_head_logits(x_bits: np.ndarray, w_fp8: np.ndarray, scale) -> np.ndarray:
    """Logits of an FP8 output head in fp64: L[m, n] = (sum_k x[m, k] * e4m3(w[n, k])) * s_n.

    x_bits: bf16 bits uint16[M, K]; w_fp8: uint8[N, K] E4M3 bytes (0x7F / 0xFF decode to NaN,
    which gives NaN logits); scale: one float (per tensor) or N floats (per output row): the
    pages do not say which, so both are accepted. The sum is a library fp64 matrix product."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    w_fp8 = np.ascontiguousarray(w_fp8, dtype=np.uint8)
    if x_bits.ndim != 2 or w_fp8.ndim != 2 or x_bits.shape[1] != w_fp8.shape[1]:
        raise ValueError("x is [M, K] and w is [N, K]")
    table = np.array([e4m3_decode(b) for b in range(256)], dtype=np.float64)
    w = table[w_fp8]
    x = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    logits = x @ w.T
    s = np.asarray(scale, dtype=np.float64)
    if s.ndim == 0:
        return logits * s
    if s.shape != (w_fp8.shape[0],):
        raise ValueError("a per-row scale has one value per output row")
    return logits * s[None, :]


def bf16_ulp(v: float) -> float:
    """Spacing of bf16 values at |v|: 2^(e - 7) for 2^e <= |v| < 2^(e + 1) with e >= -126 (eight
    significand bits), the subnormal spacing 2^-133 below 2^-126; NaN for a non-finite v."""
    a = abs(float(v))
    if not np.isfinite(a):
        return float("nan")
    if a < 2.0 ** -126:
        return 2.0 ** -133
    e = int(np.floor(np.log2(a)))
    # guard the floor of log2 at exact powers of two and just below them
    if 2.0 ** e > a:
        e -= 1
    elif 2.0 ** (e + 1) <= a:
        e += 1
    return 2.0 ** (e - 7)


def greedy_top2(logits: np.ndarray):
    """Per row of logits[M, N] (N >= 2): the greedy token (largest logit, lowest index among
    equal ones), the largest and second largest values, and their gap in bf16 units in the last
    place at the largest value. The pages report near ties as gaps below one ulp (0.04 to 0.76
    ulp measured), so the gap is read on logits finer than the ulp's format: here fp64 logits
    against the bf16 spacing. A row with a NaN gives index -1 and NaN values."""
    L = np.asarray(logits, dtype=np.float64)
    if L.ndim != 2 or L.shape[1] < 2:
        raise ValueError("logits is [M, N] with N >= 2")
    M = L.shape[0]
    idx = np.full(M, -1, dtype=np.int64)
    top1 = np.full(M, np.nan)
    top2 = np.full(M, np.nan)
    gap = np.full(M, np.nan)
    for m in range(M):
        row = L[m]
        if np.isnan(row).any():
            continue
        i = int(np.argmax(row))            # the first of equal maxima
        rest = np.delete(row, i)
        idx[m] = i
        top1[m] = row[i]
        top2[m] = rest.max()
        gap[m] = (top1[m] - top2[m]) / bf16_ulp(top1[m])
    return idx, top1, top2, gap


# ---------------------------------------------------------------- GDN closed-form commit (next row)
#
# 48 of the served model's 64 layers are Gated DeltaNet layers whose recurrent state cannot step
# back after a wrong guess, so the engine commits the state of the accepted path in closed form
# (TandemLLM docs v0.12.0, "What TandemLLM is", section 1.7; the author's "Research" page,
# StairCut abstract). The pages give no equations. Reading taken here: the state of one head is
# S (d_v x d_k) and one token with key k, value v, gate alpha in (0, 1] and step beta in [0, 1]
# updates it by the gated delta rule
#
#     S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
#
# and "committing the accepted path" means producing S_L, the state after the path's L tokens
# (taken in order from the draft tree's nodes), from S_0 in one batched step instead of L
# sequential updates. PARITY UNPINNED against the pages (they print no equation or value); the
# functions below are pinned against each other, against exact rational arithmetic and against
# the properties of the rule in tests/test_oracle_pins.py.

def gdn_sequential(S0: np.ndarray, K: np.ndarray, V: np.ndarray, alpha: np.ndarray, beta: np.ndarray) -> np.ndarray:
    """The definition: L sequential gated-delta updates of S0 (d_v x d_k) in fp64, token t with
    key K[t] (d_k), value V[t] (d_v), gate alpha[t], step beta[t]."""
    S = np.array(S0, dtype=np.float64)
    for k, v, a, b in zip(np.asarray(K, np.float64), np.asarray(V, np.float64), np.asarray(alpha, np.float64),
                          np.asarray(beta, np.float64)):
        S = a * (S - b * np.outer(S @ k, k)) + b * np.outer(v, k)
    return S


def gdn_commit_closed_form(S0: np.ndarray, K: np.ndarray, V: np.ndarray, alpha: np.ndarray,
                           beta: np.ndarray) -> np.ndarray:
    """The same state in closed form, in fp64.

    Write the rule as S_t = alpha_t S_{t-1} + u_t k_t^T with u_t = beta_t (v_t - alpha_t S_{t-1} k_t),
    and let g_t = alpha_1 ... alpha_t (g_0 = 1). Unrolling S_{t-1} gives, for the columns u_t of U:
        u_t + sum_{s<t} beta_t (g_t / g_s) (k_s . k_t) u_s = beta_t (v_t - g_t S_0 k_t),
    a unit lower-triangular system (I + A) in the path's order, so
        U = ((V^T - S_0 K^T G) B) (I + A)^-T,      S_L = g_L S_0 + U diag(g_L / g_t) K
    with G = diag(g), B = diag(beta) and K holding one key per row. The triangular solve is a
    library routine; everything else is written out."""
    S0 = np.asarray(S0, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    a = np.asarray(alpha, np.float64)
    b = np.asarray(beta, np.float64)
    L = K.shape[0]
    if L == 0:
        return S0.copy()
    g = np.cumprod(a)                                   # g_t, t = 1..L
    A = np.zeros((L, L))
    for t in range(L):
        for s in range(t):
            A[t, s] = b[t] * (np.prod(a[s + 1:t + 1])) * float(K[s] @ K[t])
    R = (V.T - (S0 @ K.T) * g[None, :]) * b[None, :]    # d_v x L: beta_t (v_t - g_t S0 k_t)
    # U (I + A)^T = R  <=>  (I + A) U^T = R^T
    U = np.linalg.solve(np.eye(L) + A, R.T).T
    decay = np.array([np.prod(a[t + 1:]) for t in range(L)])   # g_L / g_t
    return g[-1] * S0 + (U * decay[None, :]) @ K


def gdn_path_inputs(K_nodes, V_nodes, alpha_nodes, beta_nodes, path):
    """Gather one head's path inputs from per-node arrays of a draft tree (node-major)."""
    p = np.asarray(path, dtype=np.int64)
    return (np.asarray(K_nodes)[p], np.asarray(V_nodes)[p], np.asarray(alpha_nodes)[p], np.asarray(beta_nodes)[p])
