"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Bars (all written here):
  * dequantised weights and quantiser output: bit-exact;
  * Y: |y - y_ref| <= 1e-3 * sum_k |x_k w_k| + 2^-8 * |y_ref| per element (fp32 accumulation,
    one bf16 rounding: the 2^-8 term covers the output rounding); NaN only where the reference
    is NaN. The exact paths (the default f16 tensor-core path, the bf16 tensor-core path and
    the CUDA-core path) are held to it on every input, including single-nonzero weights and
    activation outliers. The approximate block-scaled path (X as FP4 pieces) is held to the
    same bar, unwidened, on the dense weights of the workload only: it does not claim the bar
    for every input;
  * cases whose exact result is representable (identity, one-hot, small integers, f16-subnormal
    activations, rows recomputed by the fallback): bit-exact against bf16(y_ref) on the exact
    paths;
  * determinism: repeated runs bit-identical on every path.
"""

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU hosts, skipped there
    pytest.skip("needs a CUDA device", allow_module_level=True)

import nvfp4_weight_gemm_b200 as tl  # noqa: E402

DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _init():
    from nvfp4_weight_gemm_b200 import build
    build.build()
    oracle.build()
    tl.init(0)
    yield
    tl.check_device_error()


# ------------------------------------------------------------------ helpers

def dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def host_f64(y):
    return y.float().cpu().numpy().astype(np.float64)


def bf16_round(a):
    """bf16(a) for fp64 values that are exact in fp32 (no double rounding then)."""
    return torch.from_numpy(np.asarray(a, dtype=np.float64)).float().to(torch.bfloat16).double().numpy()


def assert_within_tol(y, y_ref, a_ref, what=""):
    """The per-element bar; a NaN (or infinity) passes only where the reference has the same."""
    y, y_ref, a_ref = np.asarray(y), np.asarray(y_ref), np.asarray(a_ref)
    tol = 1e-3 * a_ref + 2.0 ** -8 * np.abs(y_ref)
    with np.errstate(invalid="ignore"):
        err = np.abs(y - y_ref)
        same_special = (np.isnan(y) & np.isnan(y_ref)) | (np.isinf(y) & (y == y_ref))
        bad = ~((err <= tol) | same_special)
    if bad.any():
        excess = np.where(bad, np.nan_to_num(err - tol, nan=np.inf), -np.inf)
        at = np.unravel_index(np.argmax(excess), excess.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst at {at}: "
                             f"y={y[at]!r} ref={y_ref[at]!r} tol={tol[at]!r}")


def make_weight(N, K, seed, tid, dist="normal"):
    w = synth.w_f32(N, K, seed=seed, tensor_id=tid, dist=dist)
    codes, scales, g = oracle.quantize(w)
    return w, codes, scales, g


TC_PATHS = {"exact": tl.PATH_EXACT, "bf16-exact": tl.PATH_BF16_EXACT, "block-scaled": tl.PATH_BLOCK_SCALED}
EXACT = ("exact", "bf16-exact", "simt")   # every path whose products are exact


def gemm_on(path, x, c, s, g):
    with tl.gemm_path(TC_PATHS[path]):
        return tl.verify_gemm(x, c, s, g)


def run_paths(x_bits, codes, scales, g, paths=None):
    """Y from every path (or those named): {"exact", "bf16-exact", "block-scaled", "simt"} -> fp64."""
    x = dev_bf16(x_bits)
    c, s = dev_u8(codes), dev_u8(scales)
    out = {p: gemm_on(p, x, c, s, g) for p in TC_PATHS if paths is None or p in paths}
    if paths is None or "simt" in paths:
        out["simt"] = tl.verify_gemm_simt(x, c, s, g)
    torch.cuda.synchronize()
    tl.check_device_error()
    return {k: host_f64(v) for k, v in out.items()}


def assert_all_within_tol(ys, y_ref, a_ref, what=""):
    for path, y in ys.items():
        assert_within_tol(y, y_ref, a_ref, f"{what} [{path}]")


# ------------------------------------------------------------------ format kernels

def test_dequant_bit_exact_tiny():
    _, codes, scales, g = make_weight(256, 512, 0, 0)
    w_ref = oracle.dequant(codes, scales, g)
    w_gpu = tl.dequant(dev_u8(codes), dev_u8(scales), g).cpu().numpy()
    assert np.array_equal(w_gpu.view(np.uint32), w_ref.view(np.uint32))


def test_dequant_bit_exact_all_bytes():
    rng = np.random.default_rng(3)
    N, K = 64, 4096
    codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = np.tile(np.arange(256, dtype=np.uint8), N * (K // 16) // 256).reshape(N, K // 16)
    for g in (1.0, float(np.float32(0.0123)), float(np.float32(3.7e-39))):
        w_ref = oracle.dequant(codes, scales, g)
        w_gpu = tl.dequant(dev_u8(codes), dev_u8(scales), g).cpu().numpy()
        same = (w_gpu.view(np.uint32) == w_ref.view(np.uint32)) | (np.isnan(w_gpu) & np.isnan(w_ref))
        assert same.all(), g


@pytest.mark.parametrize("N,K,dist", [(256, 512, "normal"), (677, 2304, "normal"), (640, 4096, "t4"),
                                      (5120, 5120, "normal")])
def test_quantize_bit_exact(N, K, dist):
    w = synth.w_f32(N, K, seed=1, tensor_id=N + K, dist=dist)
    codes, scales, g = oracle.quantize(w)
    c2, s2, g2 = tl.quantize(torch.from_numpy(w).to(DEV))
    assert g2 == g
    assert np.array_equal(s2.cpu().numpy(), scales)
    assert np.array_equal(c2.cpu().numpy(), codes)


def test_quantize_special_tensors():
    c, s, g = tl.quantize(torch.zeros((16, 256), device=DEV))
    assert g == 0.0 and not c.any() and not s.any()
    w = torch.ones((16, 256), device=DEV)
    w[3, 17] = float("nan")
    with pytest.raises(tl.TlError):
        tl.quantize(w)


# ------------------------------------------------------------------ GEMM parity

def test_tiny_config_both_paths():
    _, codes, scales, g = make_weight(256, 512, 0, 0)
    x = synth.x_bf16(8, 512, seed=0)
    y_ref, a_ref = oracle.gemm(x, codes, scales, g)
    assert_all_within_tol(run_paths(x, codes, scales, g), y_ref, a_ref, "tiny")


@pytest.mark.parametrize("M", [1, 2, 7, 8, 15, 16, 17, 24, 31, 32])
def test_ragged_split_k_all_row_counts(M):
    # 6 n-tiles (last one 37 rows), 9 k-tiles: every n-tile is split over several CTAs
    _, codes, scales, g = make_weight(677, 2304, 2, 1)
    x = synth.x_bf16(M, 2304, seed=2, tensor_id=synth.X_ID_BASE + M)
    y_ref, a_ref = oracle.gemm(x, codes, scales, g)
    assert_all_within_tol(run_paths(x, codes, scales, g), y_ref, a_ref, f"M={M}")


@pytest.mark.parametrize("M", [33, 48, 64, 65, 100, 128])
def test_more_rows_than_one_launch(M):
    # above 32 rows: one 64-row launch on the block-scaled path (two 128-line MMAs per chunk),
    # groups of rows beyond that; groups of 32 rows on the exact and CUDA-core paths
    _, codes, scales, g = make_weight(677, 2304, 2, 1)
    x = synth.x_bf16(M, 2304, seed=22, tensor_id=synth.X_ID_BASE + 300 + M)
    y_ref, a_ref = oracle.gemm(x, codes, scales, g)
    assert_all_within_tol(run_paths(x, codes, scales, g), y_ref, a_ref, f"M={M}")


@pytest.mark.parametrize("path", list(TC_PATHS))
@pytest.mark.parametrize("M", [1, 8, 16, 24, 32])
def test_attention_projection_full(M, path):
    _, codes, scales, g = make_weight(5120, 5120, 0, 2)
    x = synth.x_bf16(M, 5120, seed=0, tensor_id=synth.X_ID_BASE + 2)
    y_ref, a_ref = oracle.gemm(x, codes, scales, g)
    y = host_f64(gemm_on(path, dev_bf16(x), dev_u8(codes), dev_u8(scales), g))
    tl.check_device_error()
    assert_within_tol(y, y_ref, a_ref, f"attn M={M} [{path}]")


def _sampled_check(N, K, dist, Ms, tid, path):
    _, codes, scales, g = make_weight(N, K, 0, tid, dist)
    c, s = dev_u8(codes), dev_u8(scales)
    rng = np.random.default_rng(tid)
    for M in Ms:
        x = synth.x_bf16(M, K, seed=0, tensor_id=synth.X_ID_BASE + tid)
        y = host_f64(gemm_on(path, dev_bf16(x), c, s, g))
        tl.check_device_error()
        mi = rng.integers(0, M, 4096)
        ni = np.concatenate([rng.integers(0, N, 4000), np.arange(N - 96, N)])
        y_ref, a_ref = oracle.gemm_sampled(x, codes, scales, g, mi, ni)
        assert_within_tol(y[mi, ni], y_ref, a_ref, f"{N}x{K} M={M} [{path}]")
        assert np.isfinite(y).all()


@pytest.mark.parametrize("path", list(TC_PATHS))
def test_mlp_gate_up_sampled(path):
    _sampled_check(34816, 5120, "normal", [1, 13, 32], 10, path)


@pytest.mark.parametrize("path", list(TC_PATHS))
def test_mlp_down_heavy_tail_sampled(path):
    _sampled_check(5120, 17408, "t4", [1, 19, 32], 11, path)


# ------------------------------------------------------------------ exact special cases

def identity_weight(K):
    codes = np.zeros((K, K // 2), dtype=np.uint8)
    for n in range(K):
        codes[n, n // 2] = 0x02 if n % 2 == 0 else 0x20    # +1.0
    return codes, np.full((K, K // 16), 0x38, dtype=np.uint8)


def test_default_path_is_exact():
    assert tl.get_gemm_path() == tl.PATH_EXACT


def test_identity_weight_returns_x_exactly():
    K = 512
    codes, scales = identity_weight(K)
    for M in (3, 32):
        x = synth.x_bf16(M, K, seed=5, tensor_id=M)
        ys = run_paths(x, codes, scales, 1.0, paths=EXACT)
        xf = synth.bf16_bits_to_f32(x).astype(np.float64)
        for p in EXACT:
            assert np.array_equal(ys[p], xf), p


def test_one_hot_weight_exact():
    rng = np.random.default_rng(8)
    K = N = 1024
    perm = rng.permutation(K)
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    for n in range(N):
        k = perm[n]
        codes[n, k // 2] |= (0xD if k % 2 == 0 else 0xD0)   # -3.0
    scales = np.full((N, K // 16), 0x30, dtype=np.uint8)    # 0.5
    x = synth.x_bf16(20, K, seed=6)
    y_ref, a_ref = oracle.gemm(x, codes, scales, 0.25)
    ys = run_paths(x, codes, scales, 0.25, paths=EXACT)
    want = bf16_round(y_ref)
    for p in EXACT:
        assert np.array_equal(ys[p], want), p


def test_small_integer_exact():
    rng = np.random.default_rng(9)
    M, N, K = 32, 384, 1024
    x = synth.f32_to_bf16_bits(rng.integers(-4, 5, (M, K)).astype(np.float32))
    codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = np.full((N, K // 16), 0x38, dtype=np.uint8)
    g = 2.0 ** -3
    y_ref, a_ref = oracle.gemm(x, codes, scales, g)
    ys = run_paths(x, codes, scales, g)
    want = bf16_round(y_ref)
    for p in EXACT:
        assert np.array_equal(ys[p], want), p
    assert_within_tol(ys["block-scaled"], y_ref, a_ref, "small integers [block-scaled]")


def test_f16_subnormal_activations_exact():
    # the exact path prepares X row m as f16(x * 2^-e_m) with the row's largest element in
    # [2^15, 2^16): elements 2^-26 .. 2^-31 of the largest land on f16 subnormals, which the
    # tensor core must take exactly (identity weight: y = x bit for bit, no fallback needed)
    K = 512
    codes, scales = identity_weight(K)
    rng = np.random.default_rng(23)
    xf = synth.bf16_bits_to_f32(synth.x_bf16(4, K, seed=23)).astype(np.float64)
    xf[:, 0] = 1.5                                        # the largest |x| of every row
    xf[:, 1:] = np.clip(np.abs(xf[:, 1:]), 0.5, 1.0) * np.sign(xf[:, 1:] + 1e-9)
    xf[:, 1:] *= 2.0 ** -rng.integers(26, 32, (4, K - 1))  # 2^-26 .. 2^-32 of 1.5
    x = synth.f32_to_bf16_bits(xf.astype(np.float32))
    want = synth.bf16_bits_to_f32(x).astype(np.float64)
    ys = run_paths(x, codes, scales, 1.0, paths=("exact",))
    assert np.array_equal(ys["exact"], want)


@pytest.mark.parametrize("case", ["wide-range", "huge", "tiny", "inf", "nan"])
def test_rows_outside_f16_take_the_fp64_fallback(case):
    # rows the X preparation cannot hold exactly in f16 are recomputed from the bf16 X in fp64:
    # exact (identity weight) where the result is representable, IEEE special values as the
    # oracle gives them otherwise; the other rows are untouched
    K = 512
    codes, scales = identity_weight(K)
    x = synth.x_bf16(6, K, seed=24)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    if case == "wide-range":
        xf[2, 7] = 2.0 ** -45 * np.abs(xf[2]).max()      # 45 binades below the row's largest
    elif case == "huge":
        xf[2] *= 2.0 ** 90                                # largest |x| above 2^75
    elif case == "tiny":
        xf[2] *= 2.0 ** -80                               # largest |x| below 2^-45
    elif case == "inf":
        xf[2, 7] = np.inf
    else:
        xf[2, 7] = np.nan
    x = synth.f32_to_bf16_bits(xf.astype(np.float32))
    y_ref, a_ref = oracle.gemm(x, codes, scales, 1.0)
    ys = run_paths(x, codes, scales, 1.0, paths=EXACT)
    for p in EXACT:
        assert_within_tol(ys[p], y_ref, a_ref, f"{case} [{p}]")
    fin = np.isfinite(y_ref)
    assert np.array_equal(ys["exact"][fin], bf16_round(y_ref[fin]))
    assert np.array_equal(np.isnan(ys["exact"]), np.isnan(y_ref))


@pytest.mark.parametrize("K,ratio", [(512, 1e4), (5120, 3e5)])
def test_single_outlier_channel(K, ratio):
    # one activation channel far above the rest, on a dense RTN weight: the rows of W whose code
    # at that channel is 0 see the small elements of the outlier's 16-block alone, so each X
    # element must be carried exactly (the tolerance is per element of the exact sum)
    N = 2048 if K == 512 else 5120
    _, codes, scales, g = make_weight(N, K, 25, 25 + K)
    rng = np.random.default_rng(25)
    xf = synth.bf16_bits_to_f32(synth.x_bf16(8, K, seed=25, tensor_id=K)).astype(np.float64)
    ch = int(rng.integers(0, K))
    xf[:, ch] *= ratio
    x = synth.f32_to_bf16_bits(xf.astype(np.float32))
    nib = (codes[:, ch // 2] >> (4 * (ch % 2))) & 0xF
    zero_rows = np.flatnonzero((nib & 7) == 0)
    assert zero_rows.size > 10
    y_ref, a_ref = oracle.gemm(x, codes, scales, g)
    ys = run_paths(x, codes, scales, g, paths=EXACT)
    for p in EXACT:
        assert_within_tol(ys[p][:, zero_rows], y_ref[:, zero_rows], a_ref[:, zero_rows], f"zero-code rows [{p}]")
        assert_within_tol(ys[p], y_ref, a_ref, f"all rows [{p}]")


def test_subnormal_scales_and_zero_blocks():
    # scales across the whole E4M3 range, including subnormals and zero, with random codes
    rng = np.random.default_rng(12)
    M, N, K = 9, 256, 2048
    codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, (N, K // 16), dtype=np.uint8)
    scales[:, ::7] = rng.integers(0, 8, scales[:, ::7].shape)
    x = synth.x_bf16(M, K, seed=12)
    y_ref, a_ref = oracle.gemm(x, codes, scales, 0.5)
    assert_all_within_tol(run_paths(x, codes, scales, 0.5), y_ref, a_ref, "subnormal scales")


def test_negative_scales():
    # E4M3 scale bytes with the sign bit set (0x80..0xFE): the block's weights change sign
    rng = np.random.default_rng(13)
    M, N, K = 17, 384, 1536
    codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = rng.integers(0x28, 0x48, (N, K // 16), dtype=np.uint8)
    neg = rng.random((N, K // 16)) < 0.4
    scales[neg] |= 0x80
    scales[5, :] |= 0x80                   # a whole row of negative scales
    scales[7, 3] = 0x80                    # -0
    x = synth.x_bf16(M, K, seed=13)
    y_ref, a_ref = oracle.gemm(x, codes, scales, 0.125)
    assert_all_within_tol(run_paths(x, codes, scales, 0.125), y_ref, a_ref, "negative scales")


def test_nan_scale_gives_nan_column():
    # a NaN scale (0x7F or 0xFF) makes every output of that weight row NaN, as in the reference
    rng = np.random.default_rng(14)
    M, N, K = 8, 256, 1024
    codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = rng.integers(0x30, 0x40, (N, K // 16), dtype=np.uint8)
    scales[3, 10] = 0x7F
    scales[200, 63] = 0xFF
    codes[200, 63 * 8:64 * 8] = 0          # NaN times zero codes is still NaN
    x = synth.x_bf16(M, K, seed=14)
    y_ref, a_ref = oracle.gemm(x, codes, scales, 1.0)
    assert np.isnan(y_ref[:, [3, 200]]).all() and np.isfinite(np.delete(y_ref, [3, 200], axis=1)).all()
    assert_all_within_tol(run_paths(x, codes, scales, 1.0), y_ref, a_ref, "NaN scale")


def test_nonfinite_x_row():
    # a NaN in X makes that row NaN on every path; the other rows are unaffected
    _, codes, scales, g = make_weight(256, 512, 15, 15)
    x = synth.x_bf16(5, 512, seed=15)
    x[2, 100] = 0x7FC0                     # bf16 NaN
    y_ref, a_ref = oracle.gemm(x, codes, scales, g)
    assert np.isnan(y_ref[2]).all()
    assert_all_within_tol(run_paths(x, codes, scales, g), y_ref, a_ref, "NaN in X")


@pytest.mark.parametrize("ratio", [1e2, 1e4, 1e6])
def test_outlier_channels_in_x(ratio):
    # a few channels far larger than the rest (large activation outliers), and rows at the
    # extremes of the bf16 range
    _, codes, scales, g = make_weight(640, 4096, 16, 16)
    rng = np.random.default_rng(16)
    xf = synth.bf16_bits_to_f32(synth.x_bf16(12, 4096, seed=16)).astype(np.float64)
    cols = rng.choice(4096, 6, replace=False)
    xf[:, cols] *= ratio
    xf[10] *= 2.0 ** -100
    xf[11] *= 2.0 ** 100
    x = synth.f32_to_bf16_bits(xf.astype(np.float32))
    y_ref, a_ref = oracle.gemm(x, codes, scales, g)
    assert_all_within_tol(run_paths(x, codes, scales, g, paths=EXACT), y_ref, a_ref, f"outliers x{ratio:g}")


# ------------------------------------------------------------------ determinism, stack, host path

@pytest.mark.parametrize("path", list(TC_PATHS))
def test_repeat_runs_bit_identical(path):
    _, codes, scales, g = make_weight(677, 2304, 2, 1)
    x = dev_bf16(synth.x_bf16(32, 2304, seed=4))
    c, s = dev_u8(codes), dev_u8(scales)
    first = gemm_on(path, x, c, s, g).clone()
    for _ in range(5):
        assert torch.equal(gemm_on(path, x, c, s, g), first)
    tl.check_device_error()


@pytest.mark.parametrize("path", list(TC_PATHS))
def test_rows_do_not_depend_on_M(path):
    # row i of a call with M rows equals the same row computed alone, bit for bit
    _, codes, scales, g = make_weight(677, 2304, 2, 1)
    x = synth.x_bf16(48, 2304, seed=17)
    c, s = dev_u8(codes), dev_u8(scales)
    alone = [gemm_on(path, dev_bf16(x[i:i + 1]), c, s, g) for i in (0, 5, 15, 16, 31, 40)]
    for M in (16, 17, 32, 48):
        y = gemm_on(path, dev_bf16(x[:M]), c, s, g)
        for j, i in enumerate((0, 5, 15, 16, 31, 40)):
            if i < M:
                assert torch.equal(y[i:i + 1], alone[j]), (M, i)
    tl.check_device_error()


def _small_stack(M, n_layers=3):
    shapes = [(384, 1024), (256, 1024), (1280, 1024), (256, 2560)]
    ents, refs = [], []
    for layer in range(n_layers):
        for j, (N, K) in enumerate(shapes):
            tid = 100 + 4 * layer + j
            _, codes, scales, g = make_weight(N, K, 3, tid, "t4" if j == 3 else "normal")
            x = synth.x_bf16(M, K, seed=3, tensor_id=synth.X_ID_BASE + tid)
            y_ref, a_ref = oracle.gemm(x, codes, scales, g)
            ents.append((dev_u8(codes), dev_u8(scales), g, dev_bf16(x),
                         torch.empty((M, N), dtype=torch.bfloat16, device=DEV)))
            refs.append((y_ref, a_ref, x))
    return ents, refs


@pytest.mark.parametrize("path", list(TC_PATHS))
@pytest.mark.parametrize("M", [8, 24])
def test_stack_matches_oracle_and_single_calls(M, path):
    ents, refs = _small_stack(M)
    mats = tl.make_matrices(ents)
    with tl.gemm_path(TC_PATHS[path]):
        tl.verify_stack(mats, M)
    torch.cuda.synchronize()
    tl.check_device_error()
    for (c, s, g, x, y), (y_ref, a_ref, _) in zip(ents, refs):
        assert_within_tol(host_f64(y), y_ref, a_ref, "stack")
    # the cached descriptor table is reused on the second call: same results
    ys = [e[4].clone() for e in ents]
    with tl.gemm_path(TC_PATHS[path]):
        tl.verify_stack(mats, M)
    for e, y0 in zip(ents, ys):
        assert torch.equal(e[4], y0)
    # a single call gives the same rows as the stack
    c, s, g, x, y = ents[5]
    assert torch.equal(gemm_on(path, x, c, s, g), y)


def test_large_stack_schedule_matches_oracle_and_repeats():
    # enough n-tiles (more than 4 per SM) that the block-scaled schedule deals whole n-tiles
    # round-robin before its stream-K tail, with several K and a ragged last n-tile; results
    # must match the oracle and be bit-identical from run to run
    M = 24
    units = 4 * tl.num_sms(0) + 40
    Ks = [256, 512, 768, 512]
    per = (units + len(Ks) - 1) // len(Ks)
    ents, refs = [], []
    for j, K in enumerate(Ks):
        N = per * 128 - (37 if j == 1 else 0)   # one ragged last n-tile
        _, codes, scales, g = make_weight(N, K, 21, 200 + j)
        x = synth.x_bf16(M, K, seed=21, tensor_id=synth.X_ID_BASE + 200 + j)
        ents.append((dev_u8(codes), dev_u8(scales), g, dev_bf16(x), torch.empty((M, N), dtype=torch.bfloat16, device=DEV)))
        refs.append((codes, scales, g, x))
    mats = tl.make_matrices(ents)
    with tl.gemm_path(tl.PATH_BLOCK_SCALED):
        tl.verify_stack(mats, M)
        torch.cuda.synchronize()
        first = [e[4].clone() for e in ents]
        for _ in range(3):
            tl.verify_stack(mats, M)
            for e, y0 in zip(ents, first):
                assert torch.equal(e[4], y0)
    tl.check_device_error()
    rng = np.random.default_rng(21)
    for (c, s, g, x, y), (codes, scales, gg, xb) in zip(ents, refs):
        N = y.shape[1]
        mi = rng.integers(0, M, 3000)
        ni = np.concatenate([rng.integers(0, N, 2900), np.arange(N - 100, N)])
        y_ref, a_ref = oracle.gemm_sampled(xb, codes, scales, gg, mi, ni)
        assert_within_tol(host_f64(y)[mi, ni], y_ref, a_ref, "large stack")


@pytest.mark.parametrize("path", list(TC_PATHS))
def test_plan_matches_stack(path):
    M = 24
    ents, refs = _small_stack(M, n_layers=2)
    mats = tl.make_matrices(ents)
    with tl.gemm_path(TC_PATHS[path]):
        tl.verify_stack(mats, M)
        ys = [e[4].clone() for e in ents]
        plan = tl.Plan(ents, M)
    for e in ents:
        e[4].fill_(0)
    with tl.gemm_path((TC_PATHS[path] + 1) % 3):   # a plan keeps the path it was made with
        plan.run()
        plan.run()
    torch.cuda.synchronize()
    tl.check_device_error()
    for e, y0 in zip(ents, ys):
        assert torch.equal(e[4], y0)
    plan.close()


def test_plan_row_limits():
    # a plan is one launch: up to 64 rows on the block-scaled path, 32 on the exact one
    ents, _ = _small_stack(48, n_layers=1)
    with tl.gemm_path(tl.PATH_BLOCK_SCALED):
        plan = tl.Plan(ents, 48)
        plan.run()
        torch.cuda.synchronize()
        plan.close()
    tl.check_device_error()
    for path in (tl.PATH_BF16_EXACT, tl.PATH_EXACT):
        with tl.gemm_path(path):
            with pytest.raises(tl.TlError) as ei:
                tl.Plan(ents, 48)
        assert ei.value.status == 3


@pytest.mark.parametrize("path", list(TC_PATHS))
@pytest.mark.parametrize("M", [8, 48])
def test_stack_rows_above_32(M, path):
    ents, refs = _small_stack(M, n_layers=1)
    mats = tl.make_matrices(ents)
    with tl.gemm_path(TC_PATHS[path]):
        tl.verify_stack(mats, M)
    torch.cuda.synchronize()
    tl.check_device_error()
    for (c, s, g, x, y), (y_ref, a_ref, _) in zip(ents, refs):
        assert_within_tol(host_f64(y), y_ref, a_ref, f"stack M={M} [{path}]")


@pytest.mark.parametrize("path", list(TC_PATHS))
def test_stack_host_buffers_end_to_end(path):
    M = 16
    ents, refs = _small_stack(M, n_layers=2)
    xs = torch.cat([e[3].reshape(-1) for e in ents]).cpu().pin_memory()
    ytot = sum(e[4].numel() for e in ents)
    x_dev = torch.empty_like(xs, device=DEV)
    y_dev = torch.empty(ytot, dtype=torch.bfloat16, device=DEV)
    y_host = torch.empty(ytot, dtype=torch.bfloat16).pin_memory()
    mats = tl.make_matrices([(c, s, g, None, None) for c, s, g, _, _ in ents])
    with tl.gemm_path(TC_PATHS[path]):
        tl.verify_stack_host(mats, M, xs, x_dev, y_host, y_dev)
    torch.cuda.synchronize()
    tl.check_device_error()
    off = 0
    for (c, s, g, x, y), (y_ref, a_ref, _) in zip(ents, refs):
        n = y.numel()
        got = y_host[off:off + n].view(y.shape).float().numpy().astype(np.float64)
        assert_within_tol(got, y_ref, a_ref, "stack host")
        off += n


@pytest.mark.parametrize("path", list(TC_PATHS))
@pytest.mark.parametrize("M", [3, 17])
def test_plan_host_buffers_pipelined(M, path):
    # a plan's host-buffer run copies X in, computes and copies Y out in overlapping chunks of
    # matrices (each chunk its own launch, scheduled on its own): within tolerance of the oracle,
    # like the plan's device run, and the same bits on every run
    ents, refs = _small_stack(M, n_layers=3)
    xtot = sum(e[3].numel() for e in ents)
    ytot = sum(e[4].numel() for e in ents)
    x_dev = torch.empty(xtot, dtype=torch.bfloat16, device=DEV)
    y_dev = torch.empty(ytot, dtype=torch.bfloat16, device=DEV)
    packed, xo, yo = [], 0, 0
    for (c, s, g, x, y) in ents:
        xv = x_dev[xo:xo + x.numel()].view(x.shape)
        xv.copy_(x)
        packed.append((c, s, g, xv, y_dev[yo:yo + y.numel()].view(y.shape)))
        xo += x.numel()
        yo += y.numel()
    x_host = x_dev.cpu().pin_memory()
    y_host = torch.empty(ytot, dtype=torch.bfloat16).pin_memory()
    with tl.gemm_path(TC_PATHS[path]):
        plan = tl.Plan(packed, M)
    try:
        plan.run()
        torch.cuda.synchronize()
        y_dev_run = y_dev.cpu()
        y_dev.zero_()
        x_dev.zero_()
        first = None
        for _ in range(2):
            y_host.zero_()
            plan.run_host(x_host, y_host)
            torch.cuda.synchronize()
            tl.check_device_error()
            if first is None:
                first = y_host.clone()
            assert torch.equal(y_host, first), "host-buffer runs differ"
        off = 0
        for (c, s, g, x, y), (y_ref, a_ref, _) in zip(ents, refs):
            n = y.numel()
            for name, buf in (("host", y_host), ("device", y_dev_run)):
                got = buf[off:off + n].view(y.shape).float().numpy().astype(np.float64)
                assert_within_tol(got, y_ref, a_ref, f"plan {name} M={M} [{path}]")
            off += n
    finally:
        plan.close()


# ------------------------------------------------------------------ failure path

def test_bounded_wait_reports_timeout_and_context_survives():
    from nvfp4_weight_gemm_b200 import _lib
    tl.check_device_error()
    _lib.check(_lib.lib().tl_selftest_bounded_wait(1000, None))
    with pytest.raises(tl.TlError) as ei:
        tl.check_device_error()
    assert ei.value.status == 5
    tl.check_device_error()  # cleared
    _, codes, scales, g = make_weight(256, 512, 0, 0)
    x = synth.x_bf16(8, 512, seed=0)
    y_ref, a_ref = oracle.gemm(x, codes, scales, g)
    assert_all_within_tol(run_paths(x, codes, scales, g), y_ref, a_ref, "after timeout")


def test_zero_rows_is_a_no_op():
    y = torch.full((1, 256), 7.0, dtype=torch.bfloat16, device=DEV)
    from nvfp4_weight_gemm_b200 import _lib
    import ctypes
    st = _lib.lib().tl_nvfp4_verify_gemm(ctypes.c_void_p(y.data_ptr()), 0, ctypes.c_void_p(y.data_ptr() + 4096),
                                         ctypes.c_void_p(y.data_ptr() + 8192), ctypes.c_float(1.0),
                                         ctypes.c_void_p(y.data_ptr()), 256, 512, None)
    assert st == 0 and bool((y == 7.0).all())


def test_unplanned_calls_stop_allocating_after_warm_up():
    # more distinct pointer sets than the descriptor cache has slots (8), alternated through
    # tl_nvfp4_verify_stack: once every slot and the path scratch have grown (the first round),
    # no call allocates device memory; every round still matches the oracle
    M = 8
    sets = [(_small_stack(M, n_layers=1)) for _ in range(10)]
    mats = [tl.make_matrices(ents) for ents, _ in sets]
    for m in mats:
        tl.verify_stack(m, M)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        for m in mats:
            tl.verify_stack(m, M)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    tl.check_device_error()
    for ents, refs in sets:
        for (c, s, g, x, y), (y_ref, a_ref, _) in zip(ents, refs):
            assert_within_tol(host_f64(y), y_ref, a_ref, "alternating stacks")
