// kernels_aux.cuh -- quantiser and dequantiser kernels (off the hot path).
#pragma once
#include <cstdint>
#include "nvfp4_format.cuh"
#include "ptx.cuh"

namespace tl {

// Tensor absmax as fp32 bits (non-negative floats order like unsigned ints) and a
// non-finite flag. out[0] = max |w| bits, out[1] = 1 if any element is NaN or infinity.
__global__ void absmax_kernel(const float* __restrict__ w, int64_t count, uint32_t* out) {
    uint32_t m = 0, bad = 0;
    const int64_t n4 = count / 4;
    const float4* w4 = reinterpret_cast<const float4*>(w);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        float4 v = w4[i];
        uint32_t b[4] = {__float_as_uint(v.x) & 0x7FFFFFFFu, __float_as_uint(v.y) & 0x7FFFFFFFu,
                         __float_as_uint(v.z) & 0x7FFFFFFFu, __float_as_uint(v.w) & 0x7FFFFFFFu};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            bad |= (b[j] >= 0x7F800000u);
            m = max(m, b[j]);
        }
    }
    for (int o = 16; o > 0; o >>= 1) {
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        bad |= __shfl_xor_sync(0xFFFFFFFFu, bad, o);
    }
    if ((threadIdx.x & 31) == 0) {
        atomicMax(&out[0], m);
        if (bad) atomicOr(&out[1], 1u);
    }
}

// One thread per 16-element block: scale byte and eight code bytes.
__global__ void quantize_kernel(const float* __restrict__ w, int64_t n_blocks, float g,
                                uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
    int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (b >= n_blocks) return;
    const float4* src = reinterpret_cast<const float4*>(w + b * 16);
    float v[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float4 f = src[j];
        v[4 * j] = f.x; v[4 * j + 1] = f.y; v[4 * j + 2] = f.z; v[4 * j + 3] = f.w;
    }
    float bmax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) bmax = fmaxf(bmax, fabsf(v[j]));
    uint32_t s = 0;
    if (g != 0.0f) s = e4m3_encode_rne_sat((double)bmax / 6.0 / (double)g);
    const double denom = (double)e4m3_to_float(s) * (double)g;
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        uint32_t c = (denom != 0.0) ? e2m1_encode_rne((double)v[j] / denom) : 0u;
        if (j < 8) lo |= c << (4 * j);
        else hi |= c << (4 * (j - 8));
    }
    reinterpret_cast<uint2*>(codes)[b] = make_uint2(lo, hi);
    scales[b] = (uint8_t)s;
}

// One thread per 16-element block: w_out = fp32(e2m1 * e4m3 * g), one rounding.
__global__ void dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                               float g, int64_t n_blocks, float* __restrict__ w_out) {
    int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (b >= n_blocks) return;
    uint2 c = reinterpret_cast<const uint2*>(codes)[b];
    const float s = e4m3_to_float(scales[b]);
    float o[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t byte = ((j < 4 ? c.x : c.y) >> (8 * (j & 3))) & 0xFFu;
        __half2 h = e2m1x2_to_half2(byte);
        o[2 * j] = __fmul_rn(__fmul_rn(__low2float(h), s), g);       // e2m1*s exact in fp32
        o[2 * j + 1] = __fmul_rn(__fmul_rn(__high2float(h), s), g);
    }
    float4* dst = reinterpret_cast<float4*>(w_out + b * 16);
#pragma unroll
    for (int j = 0; j < 4; ++j) dst[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
}

// A bounded wait on an mbarrier that never completes: exercises the timeout path
// (status word 0x1FF) without touching any other memory.
__global__ void selftest_wait_kernel(unsigned iterations, int* err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncwarp();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, iterations)) atomicCAS(err, 0, 0x1FF);
}

}  // namespace tl
