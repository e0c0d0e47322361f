// xprep.cuh -- the two small kernels around the exact f16 GEMM (gemm_ex_kernel<NX>).
//
// The GEMM multiplies f16 operands: W' = e2m1 * e4m3 is exact in f16, and X (bf16) is
// exact in f16 once each row is scaled by a power of two, as long as the row's range fits:
//
//   x_prep_kernel      X row m (bf16) -> xh row m = f16(x * 2^-e_m), with e_m chosen so the
//                      row's largest |x| lands in [2^15, 2^16). A bf16 value keeps all its 8
//                      significant bits in f16 down to 2^-17 after scaling (f16 subnormals
//                      included), i.e. about 32 binades below the row's largest element. The
//                      kernel converts every element back and compares; a row where any
//                      element is not reproduced exactly (a wider range, a NaN or infinity,
//                      or a largest |x| outside 2^-45 .. 2^75, where the epilogue factor
//                      g * 2^e_m could leave the normal float range) is flagged in the
//                      matrix's row mask.
//   fallback_rows_kernel  recomputes every flagged row from the bf16 X as given, in fp64 on
//                      CUDA cores, and overwrites that row of Y. Launched after every GEMM; with
//                      no row flagged (the normal case) each CTA reads the masks and returns.
//
// So every output is the exact product rounded once through the fp32 accumulator (the f16
// products are exact), whatever the finite or non-finite X. The epilogue of the GEMM
// multiplies row m by global_scale * 2^e_m (rowfac holds 2^e_m).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "gemm_tc.cuh"
#include "nvfp4_format.cuh"

namespace tl {

constexpr int XP_THREADS = 256;
constexpr int FB_THREADS = 256;
constexpr int XP_EMIN = -60, XP_EMAX = 60;   // e_m range with a normal epilogue factor

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Grid (matrices, M): CTA (i, r) prepares row r of matrix i, its 256 threads over the row's
// 16-byte chunks. A first pass finds the row's largest |x| (and any NaN or infinity), a second
// re-reads the row (from L1) and writes it scaled; the CTA then sets or clears bit r of the
// matrix's row mask with one atomic, so concurrent rows of one matrix never race on it.
__global__ void __launch_bounds__(XP_THREADS) x_prep_kernel(const __grid_constant__ TcParams p) {
    const TcMat& m = p.mats ? p.mats[blockIdx.x] : p.one;
    constexpr int W = XP_THREADS / 32;
    __shared__ float amax_s[W];
    __shared__ int bad_s[W], inexact_s[W];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.y;
    const int K = m.K, chunks = K / 8;   // K is a multiple of 256
    const uint4* xr = reinterpret_cast<const uint4*>(m.x + (size_t)r * K);
    float amax = 0.0f;
    bool bad = false;
    for (int c = threadIdx.x; c < chunks; c += XP_THREADS) {
        const uint4 v = __ldg(xr + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float a = bf16_lo(w[j]), b = bf16_hi(w[j]);
            bad |= !isfinite(a) || !isfinite(b);
            amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    bad = __any_sync(0xFFFFFFFFu, bad);
    if (lane == 0) { amax_s[warp] = amax; bad_s[warp] = bad ? 1 : 0; }
    __syncthreads();
    amax = amax_s[0];
    int anybad = bad_s[0];
#pragma unroll
    for (int i = 1; i < W; ++i) { amax = fmaxf(amax, amax_s[i]); anybad |= bad_s[i]; }
    bad = anybad != 0;
    int e = 0;
    if (!bad && amax > 0.0f) {
        e = ilogbf(amax) - 15;   // largest |x| * 2^-e in [2^15, 2^16)
        if (e < XP_EMIN || e > XP_EMAX) bad = true;
    }
    if (bad) e = 0;
    const float down = ldexpf(1.0f, -e);
    uint4* xo = reinterpret_cast<uint4*>(m.xh + (size_t)r * K);
    bool inexact = false;
    for (int c = threadIdx.x; c < chunks; c += XP_THREADS) {
        const uint4 v = __ldg(xr + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float a = bf16_lo(w[j]) * down, b = bf16_hi(w[j]) * down;   // exact (power of two)
            const __half ha = __float2half_rn(a), hb = __float2half_rn(b);
            inexact |= (__half2float(ha) != a) || (__half2float(hb) != b);
            o[j] = (uint32_t)__half_as_ushort(ha) | ((uint32_t)__half_as_ushort(hb) << 16);
        }
        xo[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    inexact = __any_sync(0xFFFFFFFFu, inexact);
    if (lane == 0) inexact_s[warp] = inexact ? 1 : 0;
    __syncthreads();
    if (threadIdx.x == 0) {
        int flagged = bad ? 1 : 0;
#pragma unroll
        for (int i = 0; i < W; ++i) flagged |= inexact_s[i];
        m.rowfac[r] = ldexpf(1.0f, e);
        const unsigned bit = 1u << r;
        if (flagged) atomicOr(m.rowmask, bit);
        else atomicAnd(m.rowmask, ~bit);
    }
}

// Recompute the flagged rows: y[r][n] = bf16( g * sum_b e4m3(s[n][b]) * sum_{k in b} x[r][k] * e2m1(c[n][k]) )
// in fp64, lanes over 16-k blocks and a fixed butterfly across lanes (deterministic). A warp
// takes weight rows n = global warp, + all warps, ...; for each n it does every flagged row, so
// the weight row is read from memory once.
__global__ void __launch_bounds__(FB_THREADS) fallback_rows_kernel(const __grid_constant__ TcParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * (FB_THREADS / 32) + warp;
    const long long nw = (long long)gridDim.x * (FB_THREADS / 32);
    for (int i0 = 0; i0 < p.n_mats; i0 += 32) {
        const int i = i0 + lane;
        unsigned mk = 0u;
        if (i < p.n_mats) {
            const TcMat& mm = p.mats ? p.mats[i] : p.one;
            mk = __ldcg(mm.rowmask);
            // bits of rows past M can hold another call's flags
            if (p.M < 32) mk &= (1u << p.M) - 1u;
        }
        unsigned any = __ballot_sync(0xFFFFFFFFu, mk != 0u);
        while (any) {
            const int src = __ffs(any) - 1;
            any &= any - 1u;
            const unsigned rows = __shfl_sync(0xFFFFFFFFu, mk, src);
            const TcMat& m = p.mats ? p.mats[i0 + src] : p.one;
            const int K = m.K, nb = K / 16;
            for (long long n = gw; n < m.N; n += nw) {
                const uint8_t* cr = m.codes + (size_t)n * (K / 2);
                const uint8_t* sr = m.scales + (size_t)n * nb;
                unsigned todo = rows;
                while (todo) {
                    const int r = __ffs(todo) - 1;
                    todo &= todo - 1u;
                    const __nv_bfloat16* xr = m.x + (size_t)r * K;
                    double acc = 0.0;
                    for (int b = lane; b < nb; b += 32) {
                        const double s = (double)e4m3_to_float(sr[b]);
                        const uint2 cw = *reinterpret_cast<const uint2*>(cr + 8 * b);
                        const uint4 x0 = *reinterpret_cast<const uint4*>(xr + 16 * b);
                        const uint4 x1 = *reinterpret_cast<const uint4*>(xr + 16 * b + 8);
                        const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                        double blk = 0.0;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const __half2 c = e2m1x2_to_half2(((j < 4 ? cw.x : cw.y) >> (8 * (j & 3))) & 0xFFu);
                            blk += (double)bf16_lo(xw[j]) * (double)__low2float(c);
                            blk += (double)bf16_hi(xw[j]) * (double)__high2float(c);
                        }
                        acc += blk * s;
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
                    if (lane == 0) m.y[(size_t)r * m.N + n] = __double2bfloat16(acc * (double)m.g);
                }
            }
        }
    }
}

}  // namespace tl
