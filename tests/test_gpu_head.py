"""FP8 output head on the GPU (tl_fp8_head through the C ABI) against the fp64 oracle.

Bars (written here):
  * logits: |L - L_ref| <= 1e-3 * sum_k |x_k w_k s_n| + 2^-22 |L_ref| per element (exact f16
    products, fp32 accumulation, one fp32 rounding of the scaled sum); NaN exactly where the
    reference is NaN;
  * greedy top-2: the kernel's token, top1 and top2 equal those of its own logits exactly (fixed
    order of comparisons), and its gap matches them to float rounding; against the oracle the
    token must be the oracle's wherever the oracle's best logit beats every other by more than
    twice the bar, and otherwise one of the logits within twice the bar of the best (a near tie:
    several answers are right).
"""

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
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


def make_head(N, K, seed, per_row):
    """Synthetic FP8 head: W ~ N(0, 0.02) drawn on the device, scale = absmax / 448 per row (or per
    tensor), bytes = E4M3 round-to-nearest of W / scale (torch's float8_e4m3fn cast)."""
    w = synth.w_f32_torch(N, K, seed, 9000 + N, DEV)
    if per_row:
        s = (w.abs().amax(dim=1) / 448.0).clamp_min(1e-30)
        q = (w / s[:, None]).to(torch.float8_e4m3fn)
        scale = s.float().contiguous()
    else:
        s = float(w.abs().max()) / 448.0
        q = (w / s).to(torch.float8_e4m3fn)
        scale = s
    del w
    return q.view(torch.uint8).contiguous(), scale


def scale_np(scale, N):
    return np.full(N, float(np.float32(scale))) if isinstance(scale, float) else scale.cpu().numpy().astype(np.float64)


def bound(x_bits, wq, s):
    """Per-element bar: 1e-3 * sum_k |x w s| + 2^-22 |L_ref| (the second term added by the caller)."""
    xa = np.abs(synth.bf16_bits_to_f32(x_bits).astype(np.float64))
    table = np.array([oracle.e4m3_decode(b) for b in range(256)], dtype=np.float64)
    wa = np.abs(np.nan_to_num(table[wq], nan=0.0))
    return 1e-3 * (xa @ wa.T) * np.abs(s)[None, :]


def check_logits(got, ref, a):
    tol = a + 2.0 ** -22 * np.abs(ref)
    with np.errstate(invalid="ignore"):
        ok = (np.abs(got - ref) <= tol) | (np.isnan(got) & np.isnan(ref))
    assert ok.all(), f"{(~ok).sum()} of {ok.size} logits outside the bar"
    return tol


def check_top2(top2, logits_gpu, ref, tol):
    tok, t1, t2, gap = tl.head_top2_fields(top2)
    # against the kernel's own logits: exact
    idx, v1, v2, g = oracle.greedy_top2(logits_gpu.astype(np.float64))
    assert np.array_equal(tok, idx)
    fin = idx >= 0
    assert np.array_equal(t1[fin], v1[fin]) and np.array_equal(t2[fin], v2[fin])
    assert np.allclose(gap[fin], g[fin], rtol=1e-6, atol=1e-6)
    assert np.isnan(t1[~fin]).all()
    # against the oracle: the unique answer where the margin is clear, a near-tied one otherwise
    ridx, r1, r2, _ = oracle.greedy_top2(ref)
    for m in range(ref.shape[0]):
        if ridx[m] < 0:
            assert tok[m] == -1
            continue
        margin = r1[m] - r2[m]
        if margin > 2.0 * (tol[m, ridx[m]] + tol[m].max()):
            assert tok[m] == ridx[m], (m, tok[m], ridx[m], margin)
        else:
            assert ref[m, tok[m]] >= r1[m] - 2.0 * (tol[m, tok[m]] + tol[m, ridx[m]]), (m, tok[m], ridx[m])


@pytest.mark.parametrize("per_row", [True, False])
@pytest.mark.parametrize("M", [1, 5, 16, 17, 32])
def test_head_matches_oracle(M, per_row):
    N, K = 3001, 1024                      # a ragged last n-tile, split-K over the CTAs
    wq, scale = make_head(N, K, 3, per_row)
    x = synth.x_bf16(M, K, seed=31, tensor_id=synth.X_ID_BASE + 31)
    logits, top2 = tl.fp8_head(torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16), wq, scale)
    torch.cuda.synchronize()
    tl.check_device_error()
    w_host = wq.cpu().numpy()
    s = scale_np(scale, N)
    ref = oracle.fp8_head_logits(x, w_host, s)
    got = logits.cpu().numpy().astype(np.float64)
    tol = check_logits(got, ref, bound(x, w_host, s))
    check_top2(top2, logits.cpu().numpy(), ref, tol)


def test_head_repeat_runs_bit_identical():
    wq, scale = make_head(2048, 2048, 4, True)
    x = torch.from_numpy(synth.x_bf16(24, 2048, seed=32).view(np.int16)).to(DEV).view(torch.bfloat16)
    l0, t0 = tl.fp8_head(x, wq, scale)
    for _ in range(3):
        l1, t1 = tl.fp8_head(x, wq, scale)
        assert torch.equal(l0, l1) and torch.equal(t0, t1)


def test_head_nan_weight_and_ties():
    # a NaN byte (0x7F) in one weight row makes that logit NaN in every row, and the rows' top-2
    # report no token; two equal best logits resolve to the lower index with a zero gap
    N, K, M = 512, 256, 4
    wq, scale = make_head(N, K, 5, False)
    w = wq.cpu().numpy()
    w[:, :] = 0x30                         # every weight 0.5
    w[100, :] = 0x38                       # rows 100 and 300: 1.0, tied best
    w[300, :] = 0x38
    x = np.full((M, K), 0x3F80, dtype=np.uint16)   # x = 1.0
    w_nan = w.copy()
    w_nan[7, 5] = 0x7F
    xd = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    for wb, expect_nan in ((w, False), (w_nan, True)):
        logits, top2 = tl.fp8_head(xd, torch.from_numpy(wb).to(DEV), 1.0)
        torch.cuda.synchronize()
        tok, t1, t2, gap = tl.head_top2_fields(top2)
        ref = oracle.fp8_head_logits(x, wb, 1.0)
        ridx, r1, r2, rg = oracle.greedy_top2(ref)
        assert np.array_equal(tok, ridx)
        if expect_nan:
            assert (tok == -1).all() and np.isnan(logits.cpu().numpy()[:, 7]).all()
        else:
            assert (tok == 100).all() and np.array_equal(t1, r1) and (gap == 0.0).all()


def test_head_row_outside_f16_takes_the_fp64_fallback():
    N, K, M = 1000, 512, 3
    wq, scale = make_head(N, K, 6, True)
    xf = synth.bf16_bits_to_f32(synth.x_bf16(M, K, seed=33)).astype(np.float64)
    xf[1, 3] = 2.0 ** -50 * np.abs(xf[1]).max()      # 50 binades below the row's largest
    xf[2] *= 2.0 ** 90
    x = synth.f32_to_bf16_bits(xf.astype(np.float32))
    logits, top2 = tl.fp8_head(torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16), wq, scale)
    torch.cuda.synchronize()
    w_host = wq.cpu().numpy()
    s = scale_np(scale, N)
    ref = oracle.fp8_head_logits(x, w_host, s)
    tol = check_logits(logits.cpu().numpy().astype(np.float64), ref, bound(x, w_host, s))
    check_top2(top2, logits.cpu().numpy(), ref, tol)


def test_head_vocabulary_sized():
    # a vocabulary-sized head (151,936 rows x 5,120): logits of sampled rows against the oracle,
    # the top-2 against the kernel's own logits, and the token against the oracle over the
    # kernel's 64 best candidates of every row
    N, K, M = 151936, 5120, 8
    wq, scale = make_head(N, K, 7, True)
    x = synth.x_bf16(M, K, seed=34)
    logits, top2 = tl.fp8_head(torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16), wq, scale)
    torch.cuda.synchronize()
    tl.check_device_error()
    lg = logits.cpu().numpy()
    s_all = scale.cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(35)
    cols = np.unique(np.concatenate([rng.integers(0, N, 2048), np.arange(N - 64, N)]))
    w_s = wq[torch.from_numpy(cols).to(DEV)].cpu().numpy()
    ref_s = oracle.fp8_head_logits(x, w_s, s_all[cols])
    check_logits(lg[:, cols].astype(np.float64), ref_s, bound(x, w_s, s_all[cols]))
    tok, t1, t2, gap = tl.head_top2_fields(top2)
    idx, v1, v2, g = oracle.greedy_top2(lg.astype(np.float64))
    assert np.array_equal(tok, idx) and np.array_equal(t1, v1) and np.array_equal(t2, v2)
    for m in range(M):
        cand = np.argsort(-lg[m])[:64]
        w_c = wq[torch.from_numpy(cand).to(DEV)].cpu().numpy()
        ref_c = oracle.fp8_head_logits(x[m:m + 1], w_c, s_all[cand])[0]
        tol_c = bound(x[m:m + 1], w_c, s_all[cand])[0] + 2.0 ** -22 * np.abs(ref_c)
        best = int(np.argmax(ref_c))
        second = np.max(np.delete(ref_c, best))
        if ref_c[best] - second > 2.0 * (tol_c[best] + tol_c.max()):
            assert cand[best] == tok[m]
        else:
            j = int(np.flatnonzero(cand == tok[m])[0])
            assert ref_c[j] >= ref_c[best] - 2.0 * (tol_c[j] + tol_c[best])
