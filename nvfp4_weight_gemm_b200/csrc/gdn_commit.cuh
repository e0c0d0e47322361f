// gdn_commit.cuh -- closed-form commit of an accepted draft path through Gated DeltaNet states.
//
// 48 of the served model's 64 layers carry a recurrent Gated DeltaNet state that cannot step back
// after a wrong guess; after each verify pass the engine commits the state of the accepted path
// in closed form (TandemLLM docs v0.12.0, "What TandemLLM is", section 1.7; the author's
// "Research" page, StairCut abstract). The pages print no equation. The rule taken here is the
// gated delta rule: one token with key k, value v, gate a and step b updates a head's state
// S (DV x DK) to
//
//     S' = a S (I - b k k^T) + b v k^T.
//
// For the L tokens of the path (L <= 32), with g_t = a_1 ... a_t and u_t = b_t (v_t - a_t S_{t-1} k_t):
//
//     u_t + sum_{s<t} b_t (a_{s+1} ... a_t) (k_s . k_t) u_s = b_t (v_t - g_t S_0 k_t)
//     S_L = g_L S_0 + sum_t (a_{t+1} ... a_L) u_t k_t^T
//
// so one launch forms the right-hand sides R = B (V^T - S_0 K^T G), solves the unit
// lower-triangular system for U by forward substitution (one thread per state row), and writes
// S_L = g_L S_0 + U' K, all in fp32 on CUDA cores. One CTA per head (about 106 KB of shared memory
// at d_k = d_v = 128, two per SM); S_0 is read once from HBM into shared memory and S_L written
// back in place, coalesced. Bound: HBM for the state (2 * DV * DK * 4 bytes per head) against the
// fp32 FMA pipe for the 2 * DV * DK * L multiply-adds per head.
#pragma once
#include <cstdint>

namespace tl {

constexpr int GDN_THREADS = 256;
constexpr int GDN_MAX_L = 32;

// The accepted path: node indices into the per-node inputs, in path order (passed by value).
struct GdnPath {
    int idx[GDN_MAX_L];
};

template <int DK, int DV>
struct GdnCfg {
    static constexpr int SP = DK + 4;                    // padded row (16-byte steps, conflict-free float4)
    static constexpr int G = GDN_THREADS / DV;           // thread groups over the rows of S
    static constexpr int PL = GDN_MAX_L + 1;
    static constexpr int SMEM_FLOATS = DV * SP           // S_0, then S_L
                                     + GDN_MAX_L * SP    // keys of the path
                                     + DV * PL           // R, then U
                                     + GDN_MAX_L * PL    // A
                                     + 4 * GDN_MAX_L;    // g, decay, beta, alpha
    static constexpr int SMEM_BYTES = SMEM_FLOATS * 4;
    static_assert(GDN_THREADS % DV == 0 && DK % (4 * G) == 0, "thread layout");
};

// One CTA per head; LMAX (8, 16 or 32) bounds the path length, so the substitution's unrolled
// loops run no further than needed.
template <int DK, int DV, int LMAX>
__global__ void __launch_bounds__(GDN_THREADS) gdn_commit_kernel(float* __restrict__ state, int H,
                                                                 const float* __restrict__ k,
                                                                 const float* __restrict__ v,
                                                                 const float* __restrict__ alpha,
                                                                 const float* __restrict__ beta,
                                                                 const GdnPath path, int L) {
    using C = GdnCfg<DK, DV>;
    constexpr int SP = C::SP, PL = C::PL;
    extern __shared__ float sm[];
    float* Ss = sm;                                  // [DV][SP]
    float* Ks = Ss + DV * SP;                        // [L][SP]
    float* Rs = Ks + GDN_MAX_L * SP;                 // [DV][PL]: R, then U (in place)
    float* As = Rs + DV * PL;                        // [L][PL]
    float* gs = As + GDN_MAX_L * PL;                 // g_t
    float* ds = gs + GDN_MAX_L;                      // a_{t+1} ... a_L
    float* bs = ds + GDN_MAX_L;                      // beta_t
    float* as = bs + GDN_MAX_L;                      // alpha_t

    const int h = blockIdx.x;
    const int tid = threadIdx.x;
    float* S = state + (size_t)h * DV * DK;

    // S_0 into shared memory (coalesced; a thread's loads all in flight at once), the path's keys,
    // gates and steps
    constexpr int NQ = DV * DK / 4 / GDN_THREADS;
    {
        float4 q[NQ];
#pragma unroll
        for (int u = 0; u < NQ; ++u) q[u] = __ldcs(reinterpret_cast<const float4*>(S) + tid + u * GDN_THREADS);
#pragma unroll
        for (int u = 0; u < NQ; ++u) {
            const int e = tid + u * GDN_THREADS;
            *reinterpret_cast<float4*>(Ss + ((4 * e) / DK) * SP + (4 * e) % DK) = q[u];
        }
    }
    for (int e = tid; e < L * DK / 4; e += GDN_THREADS) {
        const int t = (4 * e) / DK, j = (4 * e) % DK;
        *reinterpret_cast<float4*>(Ks + t * SP + j) =
            __ldg(reinterpret_cast<const float4*>(k + ((size_t)path.idx[t] * H + h) * DK + j));
    }
    if (tid < L) {
        as[tid] = alpha[(size_t)path.idx[tid] * H + h];
        bs[tid] = beta[(size_t)path.idx[tid] * H + h];
    }
    __syncthreads();
    if (tid == 0) {
        float g = 1.0f;
        for (int t = 0; t < L; ++t) { g *= as[t]; gs[t] = g; }
        float d = 1.0f;
        for (int t = L - 1; t >= 0; --t) { ds[t] = d; d *= as[t]; }
    }
    // A[t][s] = b_t (a_{s+1} ... a_t) (k_s . k_t), s < t
    for (int p = tid; p < L * L; p += GDN_THREADS) {
        const int t = p / L, s = p % L;
        if (s >= t) continue;
        float dot = 0.0f;
#pragma unroll 4
        for (int j = 0; j < DK; j += 4) {
            const float4 x = *reinterpret_cast<const float4*>(Ks + s * SP + j);
            const float4 y = *reinterpret_cast<const float4*>(Ks + t * SP + j);
            dot = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, dot))));
        }
        float decay = 1.0f;
        for (int r = s + 1; r <= t; ++r) decay *= as[r];
        As[t * PL + s] = bs[t] * decay * dot;
    }
    __syncthreads();
    // R = B (V^T - S_0 K^T G): thread (row i, group gi) takes t = gi, gi + G, ..., four at a time;
    // the values are loaded before the dot products so their latency overlaps them
    const int i = tid % DV, gi = tid / DV;
    {
        const float* srow = Ss + i * SP;
        for (int t0 = gi; t0 < L; t0 += 4 * C::G) {
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f}, vv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int t = t0 + C::G * u;
                vv[u] = (t < L) ? __ldg(v + ((size_t)path.idx[t] * H + h) * DV + i) : 0.0f;
            }
#pragma unroll 4
            for (int j = 0; j < DK; j += 4) {
                const float4 sv = *reinterpret_cast<const float4*>(srow + j);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int t = t0 + C::G * u;
                    if (t < L) {
                        const float4 kk = *reinterpret_cast<const float4*>(Ks + t * SP + j);
                        acc[u] = fmaf(sv.x, kk.x, fmaf(sv.y, kk.y, fmaf(sv.z, kk.z, fmaf(sv.w, kk.w, acc[u]))));
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int t = t0 + C::G * u;
                if (t < L) Rs[i * PL + t] = bs[t] * (vv[u] - gs[t] * acc[u]);
            }
        }
    }
    __syncthreads();
    // forward substitution, one thread per row, in registers: u_t = r_t - sum_{s<t} A[t][s] u_s
    // (the sum in four interleaved partial sums, added in a fixed order, to shorten the chain)
    if (tid < DV) {
        float* row = Rs + i * PL;
        float u[LMAX];
#pragma unroll
        for (int t = 0; t < LMAX; ++t) u[t] = (t < L) ? row[t] : 0.0f;
#pragma unroll
        for (int t = 1; t < LMAX; ++t) {
            if (t < L) {
                float p0 = 0.0f, p1 = 0.0f, p2 = 0.0f, p3 = 0.0f;
#pragma unroll
                for (int s = 0; s < t; ++s) {
                    const float term = As[t * PL + s] * u[s];
                    if ((s & 3) == 0) p0 += term;
                    else if ((s & 3) == 1) p1 += term;
                    else if ((s & 3) == 2) p2 += term;
                    else p3 += term;
                }
                u[t] -= (p0 + p1) + (p2 + p3);
            }
        }
#pragma unroll
        for (int t = 0; t < LMAX; ++t)
            if (t < L) row[t] = u[t];
    }
    __syncthreads();
    // S_L = g_L S_0 + sum_t (a_{t+1} ... a_L) u_t k_t^T: thread (row i, group gi) takes columns
    // [gi * DK / G, (gi + 1) * DK / G)
    {
        constexpr int NC = DK / C::G;
        const int j0 = gi * NC;
        float acc[NC];
        const float gL = (L > 0) ? gs[L - 1] : 1.0f;
        float* srow = Ss + i * SP + j0;
#pragma unroll
        for (int c = 0; c < NC; c += 4) {
            const float4 sv = *reinterpret_cast<const float4*>(srow + c);
            acc[c] = gL * sv.x; acc[c + 1] = gL * sv.y; acc[c + 2] = gL * sv.z; acc[c + 3] = gL * sv.w;
        }
        for (int t = 0; t < L; ++t) {
            const float ut = ds[t] * Rs[i * PL + t];
            const float* kr = Ks + t * SP + j0;
#pragma unroll
            for (int c = 0; c < NC; c += 4) {
                const float4 kk = *reinterpret_cast<const float4*>(kr + c);
                acc[c] = fmaf(ut, kk.x, acc[c]);
                acc[c + 1] = fmaf(ut, kk.y, acc[c + 1]);
                acc[c + 2] = fmaf(ut, kk.z, acc[c + 2]);
                acc[c + 3] = fmaf(ut, kk.w, acc[c + 3]);
            }
        }
        // each thread rewrites only the elements it read
#pragma unroll
        for (int c = 0; c < NC; c += 4)
            *reinterpret_cast<float4*>(srow + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
        const int e = tid + u * GDN_THREADS;
        __stcs(reinterpret_cast<float4*>(S) + e,
               *reinterpret_cast<const float4*>(Ss + ((4 * e) / DK) * SP + (4 * e) % DK));
    }
}

}  // namespace tl
