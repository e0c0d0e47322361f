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
// so one launch computes P = S_0 K^T, solves the unit lower-triangular system for U by forward
// substitution (one thread per state row), and writes S_L = g_L S_0 + U' K, all in fp32 on CUDA
// cores. One CTA per head; S_0 is read once from HBM into shared memory and S_L written back in
// place, coalesced. Bound: HBM for the state (2 * DV * DK * 4 bytes per head) against the fp32
// FMA pipe for the 2 * DV * DK * L multiply-adds per head.
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
    static constexpr int SP = DK + 1;                    // padded row of S in shared memory
    static constexpr int G = GDN_THREADS / DV;           // thread groups over the rows of S
    static constexpr int SMEM_FLOATS = DV * SP           // S_0, then S_L
                                     + GDN_MAX_L * DK    // keys of the path
                                     + DV * (GDN_MAX_L + 1)   // P, then U'
                                     + GDN_MAX_L * (GDN_MAX_L + 1)   // A
                                     + 4 * GDN_MAX_L;    // g, decay, beta, alpha
    static constexpr int SMEM_BYTES = SMEM_FLOATS * 4;
    static_assert(GDN_THREADS % DV == 0 && DK % (4 * G) == 0, "thread layout");
};

template <int DK, int DV>
__global__ void __launch_bounds__(GDN_THREADS) gdn_commit_kernel(float* __restrict__ state, int H,
                                                                 const float* __restrict__ k,
                                                                 const float* __restrict__ v,
                                                                 const float* __restrict__ alpha,
                                                                 const float* __restrict__ beta,
                                                                 const GdnPath path, int L) {
    using C = GdnCfg<DK, DV>;
    extern __shared__ float sm[];
    float* Ss = sm;                                  // [DV][SP]
    float* Ks = Ss + DV * C::SP;                     // [L][DK]
    float* Ps = Ks + GDN_MAX_L * DK;                 // [DV][L + 1]: P, then U'
    float* As = Ps + DV * (GDN_MAX_L + 1);           // [L][L + 1]
    float* gs = As + GDN_MAX_L * (GDN_MAX_L + 1);    // g_t
    float* ds = gs + GDN_MAX_L;                      // a_{t+1} ... a_L
    float* bs = ds + GDN_MAX_L;                      // beta_t
    float* as = bs + GDN_MAX_L;                      // alpha_t
    constexpr int PL = GDN_MAX_L + 1;

    const int h = blockIdx.x;
    const int tid = threadIdx.x;
    float* S = state + (size_t)h * DV * DK;

    // S_0 into shared memory (coalesced), the path's keys, gates and steps
    for (int e = tid; e < DV * DK / 4; e += GDN_THREADS) {
        const float4 q = reinterpret_cast<const float4*>(S)[e];
        const int i = (4 * e) / DK, j = (4 * e) % DK;
        float* row = Ss + i * C::SP + j;
        row[0] = q.x; row[1] = q.y; row[2] = q.z; row[3] = q.w;
    }
    for (int e = tid; e < L * DK; e += GDN_THREADS) {
        const int t = e / DK, j = e % DK;
        Ks[t * DK + j] = k[((size_t)path.idx[t] * H + h) * DK + j];
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
#pragma unroll 8
        for (int j = 0; j < DK; ++j) dot = fmaf(Ks[s * DK + j], Ks[t * DK + j], dot);
        float decay = 1.0f;
        for (int r = s + 1; r <= t; ++r) decay *= as[r];
        As[t * PL + s] = bs[t] * decay * dot;
    }
    // P = S_0 K^T: thread (row i, group gi) takes t = gi, gi + G, ...
    const int i = tid % DV, gi = tid / DV;
    {
        float acc[GDN_MAX_L / C::G];
#pragma unroll
        for (int u = 0; u < GDN_MAX_L / C::G; ++u) acc[u] = 0.0f;
        const float* srow = Ss + i * C::SP;
        for (int j = 0; j < DK; j += 4) {
            const float s0 = srow[j], s1 = srow[j + 1], s2 = srow[j + 2], s3 = srow[j + 3];
#pragma unroll
            for (int u = 0; u < GDN_MAX_L / C::G; ++u) {
                const int t = gi + C::G * u;
                if (t < L) {
                    const float4 kk = *reinterpret_cast<const float4*>(Ks + t * DK + j);
                    acc[u] = fmaf(s0, kk.x, fmaf(s1, kk.y, fmaf(s2, kk.z, fmaf(s3, kk.w, acc[u]))));
                }
            }
        }
#pragma unroll
        for (int u = 0; u < GDN_MAX_L / C::G; ++u) {
            const int t = gi + C::G * u;
            if (t < L) Ps[i * PL + t] = acc[u];
        }
    }
    __syncthreads();
    // forward substitution, one thread per row of S: u_t = r_t - sum_{s<t} A[t][s] u_s, with
    // r_t = b_t (v_t[i] - g_t P[i][t]); then U'[i][t] = (a_{t+1} ... a_L) u_t
    if (tid < DV) {
        float u[GDN_MAX_L];
#pragma unroll
        for (int t = 0; t < GDN_MAX_L; ++t) {
            if (t < L) {
                const float vt = v[((size_t)path.idx[t] * H + h) * DV + i];
                float r = bs[t] * (vt - gs[t] * Ps[i * PL + t]);
#pragma unroll
                for (int s = 0; s < t; ++s) r = fmaf(-As[t * PL + s], u[s], r);
                u[t] = r;
            }
        }
#pragma unroll
        for (int t = 0; t < GDN_MAX_L; ++t)
            if (t < L) Ps[i * PL + t] = ds[t] * u[t];
    }
    __syncthreads();
    // S_L = g_L S_0 + U' K: thread (row i, group gi) takes columns [gi * DK / G, (gi + 1) * DK / G)
    {
        constexpr int NC = DK / C::G;
        const int j0 = gi * NC;
        float acc[NC];
        const float gL = (L > 0) ? gs[L - 1] : 1.0f;
        float* srow = Ss + i * C::SP + j0;
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[c] = gL * srow[c];
        for (int t = 0; t < L; ++t) {
            const float ut = Ps[i * PL + t];
            const float* kr = Ks + t * DK + j0;
#pragma unroll
            for (int c = 0; c < NC; c += 4) {
                const float4 kk = *reinterpret_cast<const float4*>(kr + c);
                acc[c] = fmaf(ut, kk.x, acc[c]);
                acc[c + 1] = fmaf(ut, kk.y, acc[c + 1]);
                acc[c + 2] = fmaf(ut, kk.z, acc[c + 2]);
                acc[c + 3] = fmaf(ut, kk.w, acc[c + 3]);
            }
        }
        __syncthreads();   // every thread has read its S_0 elements before any is overwritten
#pragma unroll
        for (int c = 0; c < NC; ++c) srow[c] = acc[c];
    }
    __syncthreads();
    for (int e = tid; e < DV * DK / 4; e += GDN_THREADS) {
        const int r = (4 * e) / DK, j = (4 * e) % DK;
        const float* row = Ss + r * C::SP + j;
        reinterpret_cast<float4*>(S)[e] = make_float4(row[0], row[1], row[2], row[3]);
    }
}

}  // namespace tl
