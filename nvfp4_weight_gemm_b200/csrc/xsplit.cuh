// xsplit.cuh -- X (bf16) as a sum of FP4 pieces for the block-scaled tensor-core path.
//
// The block-scaled MMA (kind::mxf4nvf4) multiplies E2M1 by E2M1, each with one E4M3 scale per
// 16 k. W already has that form (NVFP4). X is bf16, so it is written as a sum of TC_PIECES
// such terms, per row and per 16-k block:
//
//   x[m][k] * 2^e[m]  ~=  sum_p  4^-p * e2m1(c_p[m][k]) * e4m3(s_p[m][k/16])
//
// 1. e[m] is the power of two that brings the row's largest |x| into [2^7, 2^8).
// 2. Piece p codes the block's remaining residual r, taken in units 4^-p times those of piece
//    0 (u = 4^p r): s_p is the smallest E4M3 value with 6 * s_p >= max|u| (so no code
//    saturates), c_p = RNE_e2m1(u / s_p), and u -= c_p * s_p. (The kernel keeps r in piece 0's
//    units and scales s_p instead; the powers of two make the two forms give the same bits.)
//
// Why 4^p: a piece leaves a residual of at most s_p <= 1.125 * max|u| / 6 (one E4M3 step of
// rounding up), so 4 * residual <= 0.75 * max|u|: every piece's |u| stays below 2^8 and its
// scales inside the E4M3 range, while the smallest scale (2^-9) reaches 4^-p further down
// than it would in piece 0's units. Blocks far below the row's largest value are therefore
// still coded to about 1e-3 of their own size by the later pieces.
//
// A piece leaves at most 1.125 / 6 of a block's residual, so after four pieces an element
// is off by at most about 1.2e-3 of its block's largest |x| (typically far less, and with
// random signs); on the workload's inputs the error in Y stays more than two orders of
// magnitude inside |y - y_ref| <= 1e-3 * sum|x w| + 2^-8 |y_ref|. A row whose largest |x| is
// not finite gets a NaN factor, so its outputs are NaN.
//
// Layout written per matrix, k-tile major (a k-tile is 256 k), so that one k-tile of every
// row and piece is one contiguous run that a single bulk copy brings into shared memory.
// Mp is M rounded up to a multiple of 4; rows M .. Mp-1 are written as zeros. Row m's pieces
// are adjacent: piece p of row m is "line" j = 4 m + p of the k-tile.
//   codes  [K/256][Mp][TC_PIECES][128]  bytes: the line's 256 k of the tile, k pairs packed
//                                       low nibble first like the weights; the 16-byte chunk
//                                       c of line j is stored at chunk c ^ (j & 7), the 128-byte
//                                       swizzle the tensor core's shared-memory descriptor reads
//   scales [K/256][Mp][TC_PIECES][16]   bytes: the E4M3 scales of the tile's 16 blocks
//   factor [M]                   float, 2^-e[m] (NaN for a non-finite row); piece p of row m
//                                stands for factor[m] * 4^-p * (its codes times its scales)
#pragma once
#include <cstdint>
#include <cstring>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace tl {

constexpr int TC_PIECES = 4;

struct XSplitMat {
    const __nv_bfloat16* x;   // [M][K]
    uint8_t* codes;           // [K/256][Mp][TC_PIECES][128], swizzled lines
    uint8_t* scales;          // [K/256][Mp][TC_PIECES][16]
    float* factor;            // [M]
    int K;
};

struct XSplitParams {
    const XSplitMat* mats;    // device table, or nullptr to use `one`
    int n_mats;
    int M;
    int Mp;                   // M rounded up to a multiple of 4
    XSplitMat one;
};

__host__ __device__ __forceinline__ uint32_t xs_f2u(float f) {
#ifdef __CUDA_ARCH__
    return __float_as_uint(f);
#else
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
#endif
}

__host__ __device__ __forceinline__ float xs_u2f(uint32_t u) {
#ifdef __CUDA_ARCH__
    return __uint_as_float(u);
#else
    float f;
    memcpy(&f, &u, 4);
    return f;
#endif
}

// Value of a non-negative E4M3 code (0 .. 0x7E): m * 2^-9 below exponent 1, else (1 + m/8) * 2^(e-7).
__host__ __device__ __forceinline__ float xs_e4m3_value(uint32_t code) {
    return (code >= 8u) ? xs_u2f((((code >> 3) + 120u) << 23) | ((code & 7u) << 20)) : (float)code * 0.001953125f;
}

// The smallest E4M3 code whose value v satisfies 6 v >= amax (amax > 0 finite; 0 for amax == 0),
// capped at 0x7E (448). An estimate from the bits of amax / 6, rounded up onto the E4M3 grid,
// then corrected by exact comparisons (6 v is exact in fp32).
__host__ __device__ __forceinline__ uint32_t xs_e4m3_ceil_div6(float amax) {
    if (!(amax > 0.0f)) return 0u;
    const float t = amax * (1.0f / 6.0f);
    uint32_t code;
    if (t < 0.015625f) {                                   // below 2^-6: E4M3 subnormals m * 2^-9
        float m = ceilf(t * 512.0f);
        code = (uint32_t)fminf(fmaxf(m, 1.0f), 8.0f);
    } else {
        const uint32_t b = xs_f2u(t);
        const uint32_t E = (b >> 23) - 120u;               // E4M3 biased exponent of t (>= 1)
        code = (E > 15u) ? 0x7Eu : ((E << 3) | ((b >> 20) & 7u)) + ((b & 0xFFFFFu) != 0u ? 1u : 0u);
    }
    if (code > 0x7Eu) code = 0x7Eu;
    if (code < 0x7Eu && 6.0f * xs_e4m3_value(code) < amax) ++code;
    if (code > 1u && 6.0f * xs_e4m3_value(code - 1u) >= amax) --code;
    return code;
}

// Eight floats to eight E2M1 codes (round to nearest even, saturating at +-6), packed low
// nibble first into one word, and the values of those codes as four f16 pairs (exact).
__device__ __forceinline__ uint32_t xs_e2m1x8(const float (&q)[8], uint32_t (&h)[4]) {
    uint32_t codes;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %8, %7;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %10, %9;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %12, %11;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %4, b3;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(codes), "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
    return codes;
}

constexpr int XS_THREADS = 256;
constexpr int XS_ROWS = 4;   // rows per CTA: one group of four rows of the layout

// Piece codes and scale of one 16-k block (u: the block's residual in piece-0 units, updated in
// place). inv_tab: 8 / (8 + m) for m = 0..7, then 0 and 1 / m for m = 1..7 (each correctly
// rounded), so that 1 / s is exact table value times powers of two, the same bits as a division.
__device__ __forceinline__ void xs_block_pieces(float (&u)[16], const float* inv_tab, uint8_t* cline, uint8_t* sdst,
                                                uint32_t chunk, uint32_t ph0) {
#pragma unroll
    for (int pc = 0; pc < TC_PIECES; ++pc) {
        const float unit = (float)(1 << (2 * pc));          // piece pc's units: 4^-pc of piece 0's
        float a3[6];
#pragma unroll
        for (int i = 0; i < 5; ++i) {
            float r;
            asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(fabsf(u[3 * i])), "f"(fabsf(u[3 * i + 1])), "f"(fabsf(u[3 * i + 2])));
            a3[i] = r;
        }
        a3[5] = fabsf(u[15]);
        float b0, b1, amax;
        asm("max.f32 %0, %1, %2, %3;" : "=f"(b0) : "f"(a3[0]), "f"(a3[1]), "f"(a3[2]));
        asm("max.f32 %0, %1, %2, %3;" : "=f"(b1) : "f"(a3[3]), "f"(a3[4]), "f"(a3[5]));
        amax = fmaxf(b0, b1);
        const uint32_t sc = xs_e4m3_ceil_div6(amax * unit);
        const float sv = xs_e4m3_value(sc);
        const float s = sv * (1.0f / unit);                 // the scale in piece-0 units (exact)
        // 1 / sv: normal codes (1 + m/8) 2^(E-7) -> 2^(7-E) * 8 / (8 + m); subnormal m 2^-9 -> 512 / m
        const uint32_t E = sc >> 3;
        const float pw = (E != 0u) ? __uint_as_float((134u - E) << 23) : 512.0f;
        const float inv = (inv_tab[(E != 0u) ? (sc & 7u) : (8u + sc)] * pw) * unit;   // = 1 / s (0 for sc == 0)
        uint32_t w[2];
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
            float q[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) q[i] = u[8 * hlf + i] * inv;
            uint32_t h[4];
            w[hlf] = xs_e2m1x8(q, h);
            if (pc + 1 < TC_PIECES) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 qv = __half22float2(*reinterpret_cast<const __half2*>(&h[i]));
                    u[8 * hlf + 2 * i] = fmaf(-qv.x, s, u[8 * hlf + 2 * i]);
                    u[8 * hlf + 2 * i + 1] = fmaf(-qv.y, s, u[8 * hlf + 2 * i + 1]);
                }
            }
        }
        *reinterpret_cast<uint2*>(cline + pc * 128 + ((chunk ^ ((ph0 + pc) & 7u)) << 4)) = make_uint2(w[0], w[1]);
        sdst[pc * 16] = (uint8_t)sc;
    }
}

// Grid (Mp / 4, n_mats): one CTA per group of four rows of one matrix; rows M .. Mp-1 write zero
// pieces. The four rows' 16-k blocks are shared out evenly over the CTA's threads.
__global__ void __launch_bounds__(XS_THREADS, 4) x_split_kernel(const __grid_constant__ XSplitParams p) {
    __shared__ float red[XS_THREADS / 32][XS_ROWS];
    __shared__ int bad_sh[XS_ROWS];
    __shared__ float p1_sh[XS_ROWS], p2_sh[XS_ROWS];
    __shared__ int zero_sh[XS_ROWS];
    __shared__ float inv_tab[16];
    const XSplitMat& m = p.mats ? p.mats[blockIdx.y] : p.one;
    const int row0 = blockIdx.x * XS_ROWS;
    const int K = m.K;
    const int M = p.M, Mp = p.Mp;
    const int KB = K / 16;
    const __nv_bfloat16* const x = m.x;
    uint8_t* const codes = m.codes;
    uint8_t* const scales = m.scales;
    float* const factor = m.factor;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < XS_ROWS) bad_sh[tid] = 0;
    if (tid < 16) inv_tab[tid] = (tid < 8) ? 8.0f / (float)(8 + tid) : (tid == 8) ? 0.0f : 1.0f / (float)(tid - 8);
    __syncthreads();
    // 1. each row's largest |x|, and whether any element is NaN or infinite
#pragma unroll
    for (int rr = 0; rr < XS_ROWS; ++rr) {
        float mx = 0.0f;
        bool bad = false;
        if (row0 + rr < M) {
            const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)(row0 + rr) * K);
#pragma unroll 4
            for (int k8 = tid; k8 < K / 8; k8 += XS_THREADS) {
                const uint4 v = __ldg(xr + k8);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float a = fabsf(xs_u2f(w[j] << 16)), b = fabsf(xs_u2f(w[j] & 0xFFFF0000u));
                    bad |= !(a <= 3.402823466e38f) || !(b <= 3.402823466e38f);
                    mx = fmaxf(mx, fmaxf(a, b));
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        const bool any_bad = __any_sync(0xFFFFFFFFu, bad);
        if (lane == 0) {
            red[warp][rr] = mx;
            if (any_bad) bad_sh[rr] = 1;
        }
    }
    __syncthreads();
    if (tid < XS_ROWS) {
        const int row = row0 + tid;
        float r = red[0][tid];
#pragma unroll
        for (int i = 1; i < XS_THREADS / 32; ++i) r = fmaxf(r, red[i][tid]);
        const bool pad_row = row >= M;
        const bool zero = bad_sh[tid] != 0 || pad_row;    // bad and padding rows write zero pieces
        int e = 0;                                        // r * 2^e in [2^7, 2^8)
        if (r > 0.0f && !zero) {
            int fe;
            frexpf(r, &fe);                               // r in [2^(fe-1), 2^fe)
            e = 8 - fe;
        }
        if (!pad_row) factor[row] = zero ? __int_as_float(0x7FC00000) : ldexpf(1.0f, -e);
        // exact scaling by 2^e in two steps (each factor a normal power of two)
        p1_sh[tid] = ldexpf(1.0f, e / 2);
        p2_sh[tid] = ldexpf(1.0f, e - e / 2);
        zero_sh[tid] = zero ? 1 : 0;
    }
    __syncthreads();
    // 2. four pieces per 16-k block, one thread per block; block b of row rr is item rr * KB + b
    int rr = 0, b = tid;
    while (b >= KB && rr < XS_ROWS) { b -= KB; ++rr; }
    while (rr < XS_ROWS) {
        const int row = row0 + rr;
        const int kt = b >> 4, bt = b & 15;       // k-tile, block within it
        const size_t j0 = ((size_t)kt * Mp + (size_t)row) * TC_PIECES;   // line of piece 0
        // piece p is line j0 + p; its 16-byte chunk bt/2 sits at chunk (bt/2) ^ ((j0 + p) & 7)
        uint8_t* cline = codes + j0 * 128 + 8 * (bt & 1);
        uint8_t* sdst = scales + j0 * 16 + bt;
        const uint32_t chunk = (uint32_t)(bt >> 1), ph0 = (uint32_t)(j0 & 7);
        if (zero_sh[rr]) {
#pragma unroll
            for (int pc = 0; pc < TC_PIECES; ++pc) {
                *reinterpret_cast<uint2*>(cline + pc * 128 + ((chunk ^ ((ph0 + pc) & 7u)) << 4)) = make_uint2(0u, 0u);
                sdst[pc * 16] = 0;
            }
        } else {
            // u: the block's residual, always in piece-0 units (x * 2^e)
            const float p1 = p1_sh[rr], p2 = p2_sh[rr];
            const uint4* xb = reinterpret_cast<const uint4*>(x + (size_t)row * K) + 2 * b;
            const uint4 v0 = __ldg(xb), v1 = __ldg(xb + 1);
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            float u[16];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                u[2 * j] = (xs_u2f(w[j] << 16) * p1) * p2;
                u[2 * j + 1] = (xs_u2f(w[j] & 0xFFFF0000u) * p1) * p2;
            }
            xs_block_pieces(u, inv_tab, cline, sdst, chunk, ph0);
        }
        b += XS_THREADS;
        while (b >= KB && rr < XS_ROWS) { b -= KB; ++rr; }
    }
}

}  // namespace tl
