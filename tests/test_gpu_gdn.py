"""Closed-form commit of an accepted draft path through Gated DeltaNet states (tl_gdn_commit
through the C ABI) against the fp64 oracle.

Bar (written here): per element |S - S_ref| <= 1e-4 * max(1, max |S_ref| of the head). The kernel
works in fp32: dot products of at most 128 terms, a forward substitution of at most 32 steps on
unit-length keys with steps in [0, 1] and gates in (0, 1], and sums of at most 32 rank-one terms,
which stay near 1e-6 relative on these inputs; the bar leaves room for ill-conditioned paths.
The oracle's own parity with the pages is unpinned (they print no equation).
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
    tl.init(0)
    yield
    tl.check_device_error()


def run(S0, K, V, a, b, path):
    st = torch.from_numpy(np.ascontiguousarray(S0)).to(DEV)
    args = [torch.from_numpy(np.ascontiguousarray(t)).to(DEV) for t in (K, V, a, b)]
    tl.gdn_commit(st, *args, path)
    torch.cuda.synchronize()
    return st.cpu().numpy().astype(np.float64)


def reference(S0, K, V, a, b, path, heads):
    out = {}
    for h in heads:
        Kp, Vp, ap, bp = oracle.gdn_path_inputs(K[:, h], V[:, h], a[:, h], b[:, h], path)
        out[h] = oracle.gdn_commit_closed_form(S0[h], Kp, Vp, ap, bp)
    return out


def check(got, ref):
    for h, r in ref.items():
        bar = 1e-4 * max(1.0, float(np.abs(r).max()))
        err = float(np.abs(got[h] - r).max())
        assert err <= bar, (h, err, bar)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("path", [[5], [0, 3, 7, 11, 19], list(range(31, -1, -1))])
def test_commit_matches_oracle(dk, dv, path):
    H, n_nodes = 6, 32
    S0, K, V, a, b = synth.gdn_inputs(H, dk, dv, n_nodes, seed=1)
    got = run(S0, K, V, a, b, path)
    check(got, reference(S0, K, V, a, b, path, range(H)))


def test_empty_path_and_special_cases():
    H, dk, dv, n = 4, 128, 128, 8
    S0, K, V, a, b = synth.gdn_inputs(H, dk, dv, n, seed=2)
    assert np.array_equal(run(S0, K, V, a, b, []), S0.astype(np.float64))
    # steps 0: only the gates act
    got = run(S0, K, V, a, np.zeros_like(b), [1, 2, 3])
    decay = a[1] * a[2] * a[3]
    assert np.allclose(got, S0 * decay[:, None, None], rtol=1e-6, atol=1e-7)
    # orthonormal keys, gates and steps 1: v_t is stored at k_t
    rng = np.random.default_rng(3)
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    Ko = np.repeat(Q[:, :n].T[:, None, :], H, axis=1).astype(np.float32)
    got = run(S0, Ko, V, np.ones_like(a), np.ones_like(b), list(range(n)))
    for h in range(H):
        assert np.allclose(got[h] @ Ko[:, h].T.astype(np.float64), V[:, h].T, atol=2e-5)


def test_two_commits_equal_one_and_runs_repeat_bit_for_bit():
    H, dk, dv, n = 8, 128, 128, 32
    S0, K, V, a, b = synth.gdn_inputs(H, dk, dv, n, seed=4)
    path = [2, 9, 4, 17, 30, 1, 6, 22, 13, 8]
    once = run(S0, K, V, a, b, path)
    assert np.array_equal(once, run(S0, K, V, a, b, path))
    st = torch.from_numpy(S0).to(DEV)
    args = [torch.from_numpy(t).to(DEV) for t in (K, V, a, b)]
    tl.gdn_commit(st, *args, path[:4])
    tl.gdn_commit(st, *args, path[4:])
    torch.cuda.synchronize()
    twice = st.cpu().numpy().astype(np.float64)
    assert np.allclose(twice, once, rtol=0, atol=1e-4 * max(1.0, float(np.abs(once).max())))


def test_full_model_sized_commit_sampled():
    # 48 layers x 32 heads of 128 x 128 states, a 32-node tree, the longest path; 12 heads checked
    H, dk, dv, n = 1536, 128, 128, 32
    S0, K, V, a, b = synth.gdn_inputs_torch(H, dk, dv, n, 5, DEV)
    path = [0, 1, 3, 7, 8, 12, 15, 16, 20, 21, 25, 26, 27, 29, 30, 31]
    S_host = S0.cpu().numpy()
    tl.gdn_commit(S0, K, V, a, b, path)
    torch.cuda.synchronize()
    got = S0.cpu().numpy().astype(np.float64)
    heads = list(np.random.default_rng(6).integers(0, H, 10)) + [0, H - 1]
    ref = reference(S_host, K.cpu().numpy(), V.cpu().numpy(), a.cpu().numpy(), b.cpu().numpy(), path, heads)
    check(got, ref)
