"""Pins for the CPU oracle: checks against facts that do not come from the oracle itself.

Each test pins one part of the oracle to something independent of its code:
hand-worked values from the format definitions (tests/golden), library
decoders/encoders (torch float8_e4m3fn, ml_dtypes float4_e2m1fn), closed forms,
brute force with exact rationals, and special cases whose result is known
exactly (identity, one-hot and small-integer weights, M-invariance).
A plausible mistake (a dropped term, a wrong sign or nibble order, a transposed
operand, a tie broken the wrong way) fails at least one of them.
"""

import math
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import synth
from conftest import read_golden


def _f(s):
    return float("nan") if s == "nan" else float(s)


def _same(a, b):
    if math.isnan(b):
        return math.isnan(a)
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


# ---------------------------------------------------------------- E2M1 / E4M3 decode

def test_e2m1_decode_hand_worked(orc):
    rows = read_golden("e2m1_decode.txt")
    assert len(rows) == 16
    for code, val in rows:
        assert _same(orc.e2m1_decode(int(code, 16)), _f(val)), code


def test_e2m1_decode_matches_ml_dtypes(orc):
    lib_vals = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for c in range(16):
        assert _same(orc.e2m1_decode(c), float(lib_vals[c])), c


def test_e4m3_decode_hand_worked(orc):
    for byte, val in read_golden("e4m3_decode.txt"):
        assert _same(orc.e4m3_decode(int(byte, 16)), _f(val)), byte


def test_e4m3_decode_all_bytes_match_torch(orc):
    lib_vals = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for b in range(256):
        assert _same(orc.e4m3_decode(b), float(lib_vals[b])), hex(b)


def test_e4m3_decode_invariants(orc):
    pos = [orc.e4m3_decode(b) for b in range(0x7F)]
    assert all(pos[i] < pos[i + 1] for i in range(len(pos) - 1))  # strictly increasing
    assert pos[-1] == 448.0 and pos[1] == 2.0 ** -9
    for b in range(0x7F):
        assert orc.e4m3_decode(0x80 | b) == -orc.e4m3_decode(b)


# ---------------------------------------------------------------- encoders

def test_e2m1_round_hand_worked(orc):
    for q, code in read_golden("e2m1_round.txt"):
        assert orc.e2m1_encode(float(q)) == int(code, 16), q


def test_e2m1_round_matches_ml_dtypes(orc):
    # Every multiple of 1/64 in [-6, 6]: ml_dtypes rounds to nearest even (it is a library RNE).
    qs = np.arange(-384, 385, dtype=np.float64) / 64.0
    lib = qs.astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    for q, c in zip(qs, lib):
        want = int(c) & 0xF
        if want == 0x8:
            want = 0x0  # the weight format never stores -0
        assert orc.e2m1_encode(float(q)) == want, q


def test_e2m1_round_brute_force_nearest(orc):
    grid = [Fraction(v) for v in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
    for i in range(-900, 901):
        q = Fraction(i, 128)
        a = min(abs(q), Fraction(6))
        d = [abs(a - g) for g in grid]
        best = min(d)
        cands = [c for c in range(8) if d[c] == best]
        c = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
        if c and q < 0:
            c |= 8
        assert orc.e2m1_encode(float(q)) == c, q


def test_e4m3_round_hand_worked(orc):
    for t, b in read_golden("e4m3_round.txt"):
        assert orc.e4m3_encode(float(t)) == int(b, 16), t


def test_e4m3_round_matches_torch(orc):
    rng = np.random.default_rng(1)
    ts = np.concatenate([
        rng.uniform(0, 448, 3000), np.exp(rng.uniform(math.log(2.0 ** -12), math.log(448.0), 3000)),
    ]).astype(np.float32)
    # every midpoint between adjacent finite codes is a tie; all are exact in fp32
    vals = [float(v) for v in torch.arange(0x7F, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)]
    mids = np.array([(vals[i] + vals[i + 1]) / 2 for i in range(len(vals) - 1)], dtype=np.float32)
    ts = np.concatenate([ts, mids])
    lib = torch.from_numpy(ts).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for t, b in zip(ts, lib):
        assert orc.e4m3_encode(float(t)) == int(b), float(t)


def test_e4m3_round_saturates(orc):
    for t in (448.0, 448.5, 464.0, 480.0, 1e30, float("inf")):
        assert orc.e4m3_encode(t) == 0x7E


# ---------------------------------------------------------------- packed decode

def test_dequant_hand_worked_bytes(orc):
    for cb, sb, g, w0, w1 in read_golden("nvfp4_packed.txt"):
        codes = np.zeros((1, 8), dtype=np.uint8)
        codes[0, 0] = int(cb, 16)
        scales = np.array([[int(sb, 16)]], dtype=np.uint8)
        w32 = orc.dequant(codes, scales, float(g))
        assert _same(float(w32[0, 0]), float(w0)), (cb, sb, g)
        assert _same(float(w32[0, 1]), float(w1)), (cb, sb, g)


def test_dequant_scale_index_per_16_block(orc):
    # scale b covers k in [16b, 16b+16): give each block a distinct power-of-two scale
    K = 64
    codes = np.full((1, K // 2), 0x22, dtype=np.uint8)  # every weight code 2 -> 1.0
    scales = np.array([[0x38, 0x40, 0x48, 0x30]], dtype=np.uint8)  # 1, 2, 4, 0.5
    w = orc.dequant(codes, scales, 1.0)[0]
    want = np.repeat([1.0, 2.0, 4.0, 0.5], 16)
    assert np.array_equal(w, want)


def test_dequant_fp32_single_rounding(orc):
    # g with a full 24-bit mantissa: the fp32 result must be the correctly rounded exact product
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, (4, 32), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, (4, 4), dtype=np.uint8)
    g = float(np.float32(0.1234567))
    w32, wq = orc.dequant(codes, scales, g, want_wq=True)
    for n in range(4):
        for k in range(64):
            exact = Fraction(float(wq[n, k])) * Fraction(g)
            assert Fraction(float(w32[n, k])) == Fraction(float(np.float32(float(exact)))) or \
                abs(Fraction(float(w32[n, k])) - exact) <= abs(exact) * Fraction(1, 2 ** 24)


# ---------------------------------------------------------------- quantiser

def _grid_tensor(rng, N, K, g):
    """A tensor whose blocks are exactly on the NVFP4 grid: returns (w, codes, scales)."""
    nb = K // 16
    codes = rng.integers(0, 16, (N, K))
    codes[codes == 8] = 0  # -0 is never produced
    # one element of every block has magnitude 6 so the block max is 6*dec(s)*g
    pos = rng.integers(0, 16, (N, nb))
    for n in range(N):
        for b in range(nb):
            codes[n, 16 * b + pos[n, b]] = 7 if rng.random() < 0.5 else 15
    scales = rng.integers(0x08, 0x7E, (N, nb))
    scales[0, 0] = 0x7E  # the tensor's absmax block carries 448
    mag = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    e2m1 = np.where(codes & 8, -1.0, 1.0) * mag[codes & 7]
    dec = np.array([float(v) for v in torch.arange(256, dtype=torch.int32).to(torch.uint8)
                    .view(torch.float8_e4m3fn).to(torch.float64)])
    w = e2m1 * np.repeat(dec[scales], 16, axis=1) * g
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return w.astype(np.float32), packed, scales.astype(np.uint8)


def test_quantize_round_trips_grid_tensors(orc):
    rng = np.random.default_rng(7)
    for g in (2.0 ** -8, 2.0 ** -3, 1.0):
        w, codes, scales = _grid_tensor(rng, 8, 64, g)
        c2, s2, g2 = orc.quantize(w)
        assert g2 == g
        assert np.array_equal(s2, scales)
        assert np.array_equal(c2, codes)


def test_quantize_recipe_invariants(orc):
    w = synth.w_f32(64, 256, seed=3, tensor_id=0)
    codes, scales, g = orc.quantize(w)
    amax = float(np.max(np.abs(w)))
    assert g == float(np.float32(amax / 2688.0))
    w32, wq = orc.dequant(codes, scales, g, want_wq=True)
    dec = np.array([orc.e4m3_decode(int(b)) for b in range(256)])
    sv = np.repeat(dec[scales], 16, axis=1)
    # the block holding the tensor's absmax has scale 448 (0x7E)
    n0, k0 = np.unravel_index(np.argmax(np.abs(w)), w.shape)
    assert scales[n0, k0 // 16] == 0x7E
    # every element is within one grid step of the scaled value, sign is kept
    err = np.abs(w.astype(np.float64) - wq * g)
    assert np.all(err <= sv * g * 1.0 + 1e-30)
    assert np.all((wq == 0) | (np.sign(wq) == np.sign(w)))
    # block max maps to at most 6*(1 + 2^-4) on the E2M1 grid (E4M3 rounding bound, normal scales)
    bmax = np.abs(w.astype(np.float64)).reshape(64, 16, 16).max(axis=2)
    dv = dec[scales]
    normal = dv >= 2.0 ** -6
    assert np.all(bmax[normal] / (dv[normal] * g) <= 6.0 * (1 + 2.0 ** -4))


def test_quantize_zero_tensor(orc):
    codes, scales, g = orc.quantize(np.zeros((4, 32), dtype=np.float32))
    assert g == 0.0 and not codes.any() and not scales.any()


def test_quantize_rejects_nonfinite(orc):
    w = np.zeros((2, 16), dtype=np.float32)
    w[1, 3] = np.inf
    with pytest.raises(ValueError):
        orc.quantize(w)


# ---------------------------------------------------------------- GEMM

def test_gemm_hand_worked(orc):
    rows = {r[0]: r[1:] for r in read_golden("gemm_worked.txt")}
    codes = np.array([[int(b, 16) for b in rows["codes"]]], dtype=np.uint8)
    scales = np.array([[int(rows["scale"][0], 16)]], dtype=np.uint8)
    g = float(rows["g"][0])
    x = np.array([[float(v) for v in rows["x0"]], [float(v) for v in rows["x1"]]], dtype=np.float32)
    y, a = orc.gemm(synth.f32_to_bf16_bits(x), codes, scales, g)
    assert y[:, 0].tolist() == [float(v) for v in rows["y"]]


def _exact_y(x_bits, wq, g):
    xf = synth.bf16_bits_to_f32(x_bits).astype(np.float64)
    M, K = xf.shape
    N = wq.shape[0]
    out = []
    for m in range(M):
        row = []
        for n in range(N):
            s = sum(Fraction(float(xf[m, k])) * Fraction(float(wq[n, k])) for k in range(K))
            row.append(s * Fraction(g))
        out.append(row)
    return out


def test_gemm_brute_force_2x16x16_exact(orc):
    for trial in range(4):
        w = synth.w_f32(16, 16, seed=trial, tensor_id=1)
        codes, scales, g = orc.quantize(w)
        x = synth.x_bf16(2, 16, seed=trial, tensor_id=2)
        y, a = orc.gemm(x, codes, scales, g)
        _, wq = orc.dequant(codes, scales, g, want_wq=True)
        ex = _exact_y(x, wq, g)
        for m in range(2):
            for n in range(16):
                # sum of 16 exact products: within one fp64 rounding of the product with g
                assert abs(Fraction(y[m, n]) - ex[m][n]) <= Fraction(a[m, n]) * Fraction(1, 2 ** 50)


def test_gemm_matches_numpy_matmul(orc):
    w = synth.w_f32(48, 512, seed=0, tensor_id=3, dist="t4")
    codes, scales, g = orc.quantize(w)
    x = synth.x_bf16(5, 512, seed=0, tensor_id=4)
    y, a = orc.gemm(x, codes, scales, g)
    _, wq = orc.dequant(codes, scales, g, want_wq=True)
    ref = (synth.bf16_bits_to_f32(x).astype(np.float64) @ wq.T) * g
    assert np.all(np.abs(y - ref) <= a * 1e-12)
    assert np.all(a >= np.abs(y) * (1 - 1e-12))


def test_gemm_identity_weight_returns_x(orc):
    K = 64
    codes = np.zeros((K, K // 2), dtype=np.uint8)
    for n in range(K):
        codes[n, n // 2] = 0x02 if n % 2 == 0 else 0x20  # code 2 = 1.0 on the diagonal
    scales = np.full((K, K // 16), 0x38, dtype=np.uint8)
    x = synth.x_bf16(7, K, seed=1, tensor_id=5)
    y, _ = orc.gemm(x, codes, scales, 1.0)
    assert np.array_equal(y, synth.bf16_bits_to_f32(x).astype(np.float64))


def test_gemm_one_hot_weight_is_permuted_scaled_copy(orc):
    rng = np.random.default_rng(2)
    K = N = 128
    perm = rng.permutation(K)
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    for n in range(N):
        k = perm[n]
        codes[n, k // 2] |= (0xD if k % 2 == 0 else 0xD0)  # code 0xD = -3.0
    scales = np.full((N, K // 16), 0x30, dtype=np.uint8)  # 0.5
    x = synth.x_bf16(3, K, seed=2, tensor_id=6)
    y, _ = orc.gemm(x, codes, scales, 0.25)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    assert np.array_equal(y, xf[:, perm] * (-3.0 * 0.5 * 0.25))


def test_gemm_small_integer_exact(orc):
    rng = np.random.default_rng(4)
    M, N, K = 4, 32, 256
    x = rng.integers(-4, 5, (M, K)).astype(np.float32)
    codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = np.full((N, K // 16), 0x38, dtype=np.uint8)
    g = 2.0 ** -3
    y, _ = orc.gemm(synth.f32_to_bf16_bits(x), codes, scales, g)
    mag = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    lo, hi = codes & 15, codes >> 4
    c = np.empty((N, K), dtype=np.int64)
    c[:, 0::2], c[:, 1::2] = lo, hi
    wv = np.where(c & 8, -1.0, 1.0) * mag[c & 7]
    want = (x.astype(np.float64) @ wv.T) * g  # integers and halves: exact in fp64
    assert np.array_equal(y, want)


def test_gemm_row_independent_of_M(orc):
    w = synth.w_f32(40, 1024, seed=9, tensor_id=7)
    codes, scales, g = orc.quantize(w)
    x = synth.x_bf16(8, 1024, seed=9, tensor_id=8)
    y8, _ = orc.gemm(x, codes, scales, g)
    for i in range(8):
        y1, _ = orc.gemm(x[i:i + 1], codes, scales, g)
        assert np.array_equal(y1[0], y8[i])


def test_gemm_sampled_equals_full(orc):
    w = synth.w_f32(64, 256, seed=1, tensor_id=9)
    codes, scales, g = orc.quantize(w)
    x = synth.x_bf16(6, 256, seed=1, tensor_id=10)
    y, a = orc.gemm(x, codes, scales, g)
    rng = np.random.default_rng(0)
    mi, ni = rng.integers(0, 6, 50), rng.integers(0, 64, 50)
    ys, as_ = orc.gemm_sampled(x, codes, scales, g, mi, ni)
    assert np.array_equal(ys, y[mi, ni]) and np.array_equal(as_, a[mi, ni])


# ---------------------------------------------------------------- FP8 output head (next row)

def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_head_one_hot_rows_pick_x_columns(orc):
    # W row n holds the E4M3 code of +1 (0x38) or -1 (0xB8) at column k_n, zeros elsewhere:
    # logits[m, n] = +-x[m, k_n] * s_n exactly; catches a transposed W or a scale on the wrong axis
    M, N, K = 3, 5, 7
    rng = np.random.default_rng(3)
    x = rng.integers(-8, 9, size=(M, K)).astype(np.float32) / 4.0
    cols = [6, 0, 3, 3, 1]
    signs = [1, -1, 1, -1, 1]
    w = np.zeros((N, K), dtype=np.uint8)
    for n, (k, sg) in enumerate(zip(cols, signs)):
        w[n, k] = 0x38 if sg > 0 else 0xB8
    s = np.array([1.0, 0.5, 2.0, 0.25, 8.0])
    got = orc.fp8_head_logits(_bf16_bits(x), w, s)
    for m in range(M):
        for n in range(N):
            assert got[m, n] == signs[n] * x[m, cols[n]] * s[n]
    got1 = orc.fp8_head_logits(_bf16_bits(x), w, 0.5)
    assert np.array_equal(got1, orc.fp8_head_logits(_bf16_bits(x), w, np.full(N, 0.5)))


def test_head_brute_force_exact_rationals(orc):
    # tiny random case against exact rational sums, E4M3 decoded by torch's float8_e4m3fn
    M, N, K = 2, 3, 5
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((M, K)) * 3).astype(np.float32)
    xb = _bf16_bits(x)
    w = rng.integers(0, 256, size=(N, K)).astype(np.uint8)
    w[(w & 0x7F) == 0x7F] = 0x3A                      # no NaN codes here
    wv = torch.from_numpy(w).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    xv = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    s = np.array([0.75, 1.0 / 3.0, 5.0])
    got = orc.fp8_head_logits(xb, w, s)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(xv[m, k])) * Fraction(float(wv[n, k])) for k in range(K)) * Fraction(float(s[n]))
            assert abs(Fraction(float(got[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 200)


def test_head_nan_codes_give_nan_logits(orc):
    w = np.array([[0x38, 0x7F], [0x38, 0x38]], dtype=np.uint8)
    got = orc.fp8_head_logits(_bf16_bits(np.array([[1.0, 1.0]])), w, 1.0)
    assert math.isnan(got[0, 0]) and got[0, 1] == 2.0


def test_bf16_ulp_matches_torch_nextafter(orc):
    vals = [1.0, 1.5, 2.0, 3.0, -3.0, 0.1, 1e-3, 448.0, 65504.0, 3.0e38, 2.0 ** -126, 2.0 ** -130]
    for v in vals:
        b = torch.tensor(v, dtype=torch.bfloat16)
        up = torch.nextafter(b.abs(), torch.tensor(float("inf"), dtype=torch.bfloat16))
        assert orc.bf16_ulp(float(b)) == float(up.double() - b.abs().double()), v
    assert orc.bf16_ulp(0.0) == 2.0 ** -133
    assert math.isnan(orc.bf16_ulp(float("inf")))


def test_greedy_top2_hand_worked(orc):
    logits = np.array([
        [1.0, 1.0 + 2.0 ** -9, 0.5],      # best is index 1; gap 2^-9 in ulps of 2^-7: 0.25
        [2.0, 2.0, 1.0],                  # equal maxima: the lower index, gap 0
        [-1.0, -2.0, -5.0],               # gap 1 in ulps of 2^-7 at -1: 128
        [0.0, 3.0, 2.9375],               # gap 0.0625 in ulps of 2^-6 at 3: 4
        [1.0, float("nan"), 0.0],         # a NaN row
    ])
    idx, t1, t2, gap = orc.greedy_top2(logits)
    assert list(idx) == [1, 0, 0, 1, -1]
    assert list(t1[:4]) == [1.0 + 2.0 ** -9, 2.0, -1.0, 3.0]
    assert list(t2[:4]) == [1.0, 2.0, -2.0, 2.9375]
    assert list(gap[:4]) == [0.25, 0.0, 128.0, 4.0]
    assert math.isnan(gap[4]) and math.isnan(t1[4])
    with pytest.raises(ValueError):
        orc.greedy_top2(np.zeros((2, 1)))


# ---------------------------------------------------------------- GDN closed-form commit

def _gdn_cases():
    rows = read_golden("gdn_worked.txt")
    cases, cur = [], None
    for r in rows:
        if r[0] == "case":
            cur = {"alpha": float(r[2]), "beta": float(r[3])}
            cases.append(cur)
        else:
            cur[r[0]] = np.array([float(x) for x in r[1:]])
    return cases


def test_gdn_one_token_hand_worked(orc):
    for c in _gdn_cases():
        S0 = c["S0"].reshape(2, 2)
        K, V = c["k"][None, :], c["v"][None, :]
        for fn in (orc.gdn_sequential, orc.gdn_commit_closed_form):
            S1 = fn(S0, K, V, [c["alpha"]], [c["beta"]])
            assert np.allclose(S1.reshape(-1), c["S1"], rtol=0, atol=1e-12), (fn.__name__, S1)


def _gdn_exact(S0, K, V, alpha, beta):
    # the rule token by token in exact rational arithmetic
    S = [[Fraction(x) for x in row] for row in S0]
    for k, v, a, b in zip(K, V, alpha, beta):
        k = [Fraction(x) for x in k]
        Sk = [sum(S[i][j] * k[j] for j in range(len(k))) for i in range(len(S))]
        S = [[Fraction(a) * (S[i][j] - Fraction(b) * Sk[i] * k[j]) + Fraction(b) * Fraction(v[i]) * k[j]
              for j in range(len(k))] for i in range(len(S))]
    return np.array([[float(x) for x in row] for row in S])


def test_gdn_closed_form_matches_exact_rationals(orc):
    # small dyadic inputs: every step is exact in rationals; the closed form (a triangular solve
    # in fp64) must land on the same state
    rng = np.random.default_rng(11)
    for L, dk, dv in ((1, 2, 2), (3, 3, 2), (4, 2, 3), (6, 4, 4)):
        S0 = rng.integers(-4, 5, (dv, dk)) / 4.0
        K = rng.integers(-2, 3, (L, dk)) / 2.0
        V = rng.integers(-4, 5, (L, dv)) / 4.0
        alpha = rng.choice([0.5, 0.75, 1.0], L)
        beta = rng.choice([0.0, 0.25, 0.5, 1.0], L)
        ref = _gdn_exact(S0, K, V, alpha, beta)
        got = orc.gdn_commit_closed_form(S0, K, V, alpha, beta)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12 * max(1.0, np.abs(ref).max()))
        assert np.allclose(orc.gdn_sequential(S0, K, V, alpha, beta), ref, rtol=0, atol=1e-12 * max(1.0, np.abs(ref).max()))


def test_gdn_special_cases(orc):
    rng = np.random.default_rng(12)
    dk, dv, L = 16, 8, 7
    S0 = rng.standard_normal((dv, dk))
    K = rng.standard_normal((L, dk))
    V = rng.standard_normal((L, dv))
    alpha = rng.uniform(0.5, 1.0, L)
    # beta = 0: only the gates act, S_L = (alpha_1 ... alpha_L) S_0
    got = orc.gdn_commit_closed_form(S0, K, V, alpha, np.zeros(L))
    assert np.allclose(got, np.prod(alpha) * S0, rtol=1e-14, atol=0)
    # beta = 0 and alpha = 1: nothing changes; an empty path changes nothing either
    assert np.array_equal(orc.gdn_commit_closed_form(S0, K, V, np.ones(L), np.zeros(L)), S0)
    assert np.array_equal(orc.gdn_commit_closed_form(S0, K[:0], V[:0], alpha[:0], alpha[:0]), S0)


def test_gdn_orthonormal_keys_write_their_values(orc):
    # alpha = beta = 1 with orthonormal keys: the delta rule stores v_t at k_t exactly and leaves
    # every direction orthogonal to the keys as it was
    rng = np.random.default_rng(13)
    dk, dv, L = 32, 16, 12
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    K = Q[:, :L].T
    V = rng.standard_normal((L, dv))
    S0 = rng.standard_normal((dv, dk))
    SL = orc.gdn_commit_closed_form(S0, K, V, np.ones(L), np.ones(L))
    assert np.allclose(SL @ K.T, V.T, atol=1e-12)
    q = Q[:, L]
    assert np.allclose(SL @ q, S0 @ q, atol=1e-12)


def test_gdn_commit_composes_and_matches_the_recurrence(orc):
    rng = np.random.default_rng(14)
    dk, dv, L = 128, 128, 32
    S0 = rng.standard_normal((dv, dk)) * 0.1
    K = rng.standard_normal((L, dk))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    V = rng.standard_normal((L, dv))
    alpha = rng.uniform(0.9, 1.0, L)
    beta = rng.uniform(0.0, 1.0, L)
    full = orc.gdn_commit_closed_form(S0, K, V, alpha, beta)
    seq = orc.gdn_sequential(S0, K, V, alpha, beta)
    assert np.allclose(full, seq, rtol=0, atol=1e-12)
    a = 13
    first = orc.gdn_commit_closed_form(S0, K[:a], V[:a], alpha[:a], beta[:a])
    both = orc.gdn_commit_closed_form(first, K[a:], V[a:], alpha[a:], beta[a:])
    assert np.allclose(both, full, rtol=0, atol=1e-12)


def test_gdn_path_gather(orc):
    # a draft tree of 5 nodes; the accepted path 0 -> 2 -> 4 takes those nodes' inputs in order
    rng = np.random.default_rng(15)
    Kn, Vn = rng.standard_normal((5, 4)), rng.standard_normal((5, 3))
    an, bn = rng.uniform(0.5, 1, 5), rng.uniform(0, 1, 5)
    K, V, a, b = orc.gdn_path_inputs(Kn, Vn, an, bn, [0, 2, 4])
    assert np.array_equal(K, Kn[[0, 2, 4]]) and np.array_equal(b, bn[[0, 2, 4]])
    S0 = rng.standard_normal((3, 4))
    assert np.allclose(orc.gdn_commit_closed_form(S0, K, V, a, b), orc.gdn_sequential(S0, K, V, a, b), atol=1e-13)


def test_gdn_closed_form_matches_transition_matrices(orc):
    # a third formulation, written out with explicit d_k x d_k matrices: with
    # T_t = a_t (I - b_t k_t k_t^T), S_L = S_0 T_1 ... T_L + sum_t b_t v_t k_t^T T_{t+1} ... T_L
    rng = np.random.default_rng(16)
    dk, dv, L = 12, 7, 9
    S0 = rng.standard_normal((dv, dk))
    K = rng.standard_normal((L, dk))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    V = rng.standard_normal((L, dv))
    a = rng.uniform(0.6, 1.0, L)
    b = rng.uniform(0.0, 1.0, L)
    T = [a[t] * (np.eye(dk) - b[t] * np.outer(K[t], K[t])) for t in range(L)]

    def chain(lo):
        P = np.eye(dk)
        for t in range(lo, L):
            P = P @ T[t]
        return P

    ref = S0 @ chain(0) + sum(b[t] * np.outer(V[t], K[t]) @ chain(t + 1) for t in range(L))
    assert np.allclose(orc.gdn_commit_closed_form(S0, K, V, a, b), ref, rtol=0, atol=1e-12)
