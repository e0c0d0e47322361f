// gemm_simt.cuh -- CUDA-core NVFP4 verify GEMM (one warp per weight row).
//
// The plain form of Y[M,N] = X[M,K] . dequant(W)[N,K]^T: each warp streams one weight
// row, lanes take 16-element K blocks in turn (lane l: blocks l, l+32, ...), every lane
// keeps an fp32 accumulator per X row, a fixed xor-butterfly adds the lanes. Per block:
// s = sum_j x[m,16b+j] * e2m1[n,16b+j], then acc += s * (e4m3[n,b] * g): the tensor scale
// goes in with the block scale, so the running sum keeps the magnitude of the result and
// cannot overflow fp32 where Y itself does not. Used for the smallest M, where the row count leaves the
// tensor core idle, and as a second GPU path for cross-checks.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "nvfp4_format.cuh"

namespace tl {

constexpr int SIMT_WARPS = 8;

template <int MAXM>
__global__ void __launch_bounds__(SIMT_WARPS * 32)
gemm_simt_kernel(const __nv_bfloat16* __restrict__ x, int M, const uint8_t* __restrict__ codes,
                 const uint8_t* __restrict__ scales, float g, __nv_bfloat16* __restrict__ y, int N, int K) {
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * SIMT_WARPS + (threadIdx.x >> 5);
    if (n >= N) return;
    const int nb = K / 16;
    const uint2* crow = reinterpret_cast<const uint2*>(codes + (int64_t)n * (K / 2));
    const uint8_t* srow = scales + (int64_t)n * nb;
    float acc[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; ++m) acc[m] = 0.0f;

    for (int b = lane; b < nb; b += 32) {
        const uint2 c = crow[b];
        const float s = e4m3_to_float(srow[b]) * g;
        float v[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t byte = ((j < 4 ? c.x : c.y) >> (8 * (j & 3))) & 0xFFu;
            const __half2 h = e2m1x2_to_half2(byte);
            v[2 * j] = __low2float(h);
            v[2 * j + 1] = __high2float(h);
        }
#pragma unroll
        for (int m = 0; m < MAXM; ++m) {
            if (m < M) {
                const uint4* xr = reinterpret_cast<const uint4*>(x + (int64_t)m * K + 16 * b);
                const uint4 x0 = __ldg(xr), x1 = __ldg(xr + 1);
                const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                float p = 0.0f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    p = fmaf(__uint_as_float(xw[j] << 16), v[2 * j], p);
                    p = fmaf(__uint_as_float(xw[j] & 0xFFFF0000u), v[2 * j + 1], p);
                }
                acc[m] = fmaf(p, s, acc[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MAXM; ++m) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xFFFFFFFFu, acc[m], o);
    }
    // lane m writes row m (each lane holds every sum after the butterfly)
#pragma unroll
    for (int m = 0; m < MAXM; ++m)
        if (m == lane && m < M) y[(int64_t)m * N + n] = __float2bfloat16_rn(acc[m]);
}

}  // namespace tl
