// gemm_head.cuh -- the FP8 output head of the verify pass on sm_100a: logits and greedy top-2.
//
// The verify pass keeps the output head in FP8 while the projections are NVFP4 (TandemLLM docs
// v0.12.0, "What TandemLLM is", section 1.2: the head stays FP8 when the step's bytes are cut),
// and the agreement rule compares the best two logits, a near tie being a gap within one unit in
// the last place ("What TandemLLM is", section 1.5). For M <= 32 tree rows:
//
//   L[m, n] = (sum_k x[m, k] * e4m3(w[n, k])) * s_n        (s_n per output row, or one s)
//   token[m] = argmax_n L[m, n] (lowest n among equal maxima), top1, top2 (largest of the rest),
//   gap[m] = (top1 - top2) / ulp_bf16(top1)
//
// Operands as in gemm_ex.cuh: A = e4m3(w) in f16 (hardware convert of each pair of bytes: every
// E4M3 value is an f16 normal, so exact), written into tensor memory by CUDA cores; B = X
// prepared by xprep.cuh (row m times 2^-e_m in f16, exact); fp32 accumulation in tensor memory.
// The epilogue writes fp32 logits acc * 2^e_m * s_n; rows xprep flags are recomputed in fp64
// by head_tail_kernel, which also reduces every row of logits to its top two (partials over
// chunks of the row, merged by the row's last CTA).
//
// Tile: 128 weight rows x 256 k (32 KiB of E4M3 bytes, two 128-byte swizzled slices per row);
// roles and stream-K split as in gemm_ex.cuh (weight producer, X producer, 2 MMA issuers,
// 8 dequantisers in two tile sets of four lane quarters, 4 epilogue warps).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "gemm_tc.cuh"

namespace tl {

struct alignas(64) HeadParams {
    CUtensorMap tm_w;       // uint8 {128 B, N rows, K/128 slices}, box {128, 128, 2}, 128-byte swizzle
    CUtensorMap tm_x;       // f16 prepared X {64, M, K/64}, box {64, NX, 4}, 128-byte swizzle
    const uint8_t* w;       // E4M3 bytes [N][K] (fallback rows)
    const float* row_scale; // [N] or nullptr: then tensor_scale for every row
    float tensor_scale;
    float* logits;          // fp32 [M][N]
    const float* rowfac;    // 2^e_m of the prepared X
    const unsigned* rowmask;// rows xprep could not hold exactly in f16
    const __nv_bfloat16* x; // X as given (fallback rows)
    int M, N, K;
    int k_tiles, n_tiles;
    long long total_tiles;
    float* partials;        // [2 * gridDim.x][32][128]
    unsigned* counters;     // [4 * gridDim.x], zero between launches
    int* err;
};

template <int NX>
struct HeadCfg {
    static constexpr int NISSUE = 2;                       // k-steps 8j .. 8j + 7 for issuer j
    static constexpr int KSTEPS = 16 / NISSUE;
    static constexpr int THREADS = 32 * 16;                // 16 warps: 128 registers a thread
    static constexpr int DQ_FIRST = 4, EPI_FIRST = 12, XWARP = 3;
    static constexpr int W_STAGE_BYTES = TC_BLOCK_N * TC_BLOCK_K;          // 32768
    static constexpr int X_SUB = NX * 128;
    static constexpr int X_BYTES = 4 * X_SUB;
    static constexpr int NUM_A = 3;
    static constexpr int W_STAGES = (NX == 32) ? 5 : 6;
    static constexpr int X_RING = W_STAGES * W_STAGE_BYTES;
    static constexpr int SMEM_BYTES = X_RING + NUM_A * X_BYTES + 1024 + 512;
    static constexpr uint32_t IDESC = idesc_f16(0u, 128u, (uint32_t)NX);
    static constexpr int ACC_COL0 = 128 * NUM_A;
    static constexpr int ACC_BUF_COLS = NISSUE * NX;
    static constexpr int ACC_BUFS = (ACC_COL0 + 2 * ACC_BUF_COLS <= 512) ? 2 : 1;
    static constexpr int TMEM_COLS = 512;
    static_assert(ACC_COL0 + ACC_BUFS * ACC_BUF_COLS <= TMEM_COLS, "tensor memory budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

__host__ __device__ constexpr int head_issuer_of_warp(int w) { return (w == 1 || w == 2) ? w - 1 : -1; }

// Sixteen E4M3 bytes (k order) -> eight f16x2 words (low byte in the low half), exact.
__device__ __forceinline__ void head_decode16(uint4 q, uint32_t* out) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
            "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
            : "=r"(out[2 * j]), "=r"(out[2 * j + 1]) : "r"(w[j]));
    }
}

// One segment: the k-tiles [k0, k1) of n-tile `ntile` (the head is a single matrix).
struct HeadSeg {
    int ntile, k0, k1;
    long long t0;
};

struct HeadSegIter {
    long long t, end;
    int kt;
    __device__ HeadSegIter(int k_tiles, long long begin, long long stop) : t(begin), end(stop), kt(k_tiles) {}
    __device__ bool next(HeadSeg& s) {
        if (t >= end) return false;
        s.ntile = (int)(t / kt);
        s.k0 = (int)(t % kt);
        const long long rem = end - t;
        s.k1 = (int)((kt - s.k0) < rem ? kt : s.k0 + rem);
        s.t0 = t;
        t += s.k1 - s.k0;
        return true;
    }
};

template <int NX>
__global__ void __launch_bounds__(HeadCfg<NX>::THREADS, 1) gemm_head_kernel(const __grid_constant__ HeadParams p) {
    using C = HeadCfg<NX>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::X_RING + C::NUM_A * C::X_BYTES);
    uint64_t* wfull = bars;                         // [W_STAGES] weight bytes landed
    uint64_t* wempty = wfull + C::W_STAGES;         // [W_STAGES] read by the 4 warps of a tile set
    uint64_t* ready = wempty + C::W_STAGES;         // [NUM_A] slot filled: 4 warps + X bytes
    uint64_t* tfree = ready + C::NUM_A;             // [NUM_A] slot read by the MMAs
    uint64_t* accfull = tfree + C::NUM_A;           // [ACC_BUFS]
    uint64_t* accempty = accfull + 2;               // [ACC_BUFS]
    uint64_t* drain = accempty + 2;                 // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const long long ctas = gridDim.x;
    const long long t_begin = tc_range_start(blockIdx.x, p.total_tiles, ctas);
    const long long t_end = tc_range_start(blockIdx.x + 1, p.total_tiles, ctas);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::W_STAGES; ++i) { mbar_init(&wfull[i], 1); mbar_init(&wempty[i], 4); }
        for (int i = 0; i < C::NUM_A; ++i) { mbar_init(&ready[i], 5); mbar_init(&tfree[i], C::NISSUE); }
        for (int i = 0; i < C::ACC_BUFS; ++i) { mbar_init(&accfull[i], C::NISSUE); mbar_init(&accempty[i], 4); }
        mbar_init(drain, C::NISSUE);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ weight producer
        const uint64_t pol = policy_evict_first();
        int s = 0;
        uint32_t ph = 0, issued = 0, last_ph = 0;
        HeadSegIter it(p.k_tiles, t_begin, t_end);
        HeadSeg sg;
        bool ok = true;
        const bool leader = elect_one();
        while (ok && it.next(sg)) {
            for (int kt = sg.k0; kt < sg.k1; ++kt) {
                if (!__all_sync(0xFFFFFFFFu, tc_wait(&wempty[s], ph ^ 1u, abort_flag))) {
                    if (leader) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_PRODUCER);
                    ok = false;
                    break;
                }
                if (leader) {
                    mbar_arrive_expect_tx(&wfull[s], (uint32_t)C::W_STAGE_BYTES);
                    tma_load_3d_s(smem_u32(smem + s * C::W_STAGE_BYTES), &p.tm_w, &wfull[s], 0, sg.ntile * TC_BLOCK_N,
                                  2 * kt, pol);
                }
                __syncwarp();
                issued |= 1u << s;
                last_ph = (last_ph & ~(1u << s)) | (ph << s);
                if (++s == C::W_STAGES) { s = 0; ph ^= 1u; }
            }
        }
        if (leader) {
            for (int i = 0; i < C::W_STAGES; ++i)
                if ((issued >> i) & 1u)
                    if (!mbar_wait(&wfull[i], (last_ph >> i) & 1u, TL_WAIT_LIMIT))
                        tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DRAIN);
        }
    } else if (warp == C::XWARP) {
        // ------------------------------------------------------------ X producer
        const bool leader = elect_one();
        const uint64_t pol = policy_evict_last();
        int a = 0;
        uint32_t aph = 0, issued = 0, last_ph = 0;
        HeadSegIter it(p.k_tiles, t_begin, t_end);
        HeadSeg sg;
        bool ok = true;
        while (ok && it.next(sg)) {
            for (int kt = sg.k0; kt < sg.k1; ++kt) {
                if (!__all_sync(0xFFFFFFFFu, tc_wait(&tfree[a], aph ^ 1u, abort_flag))) {
                    if (leader) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_PRODUCER);
                    ok = false;
                    break;
                }
                if (leader) {
                    mbar_arrive_expect_tx(&ready[a], (uint32_t)C::X_BYTES);
                    tma_load_3d_s(smem_u32(smem + C::X_RING + a * C::X_BYTES), &p.tm_x, &ready[a], 0, 0, kt * 4, pol);
                }
                __syncwarp();
                issued |= 1u << a;
                last_ph = (last_ph & ~(1u << a)) | (aph << a);
                if (++a == C::NUM_A) { a = 0; aph ^= 1u; }
            }
        }
        if (leader) {
            for (int i = 0; i < C::NUM_A; ++i)
                if ((issued >> i) & 1u)
                    if (!mbar_wait(&ready[i], (last_ph >> i) & 1u, TL_WAIT_LIMIT))
                        tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DRAIN);
        }
    } else if (head_issuer_of_warp(warp) >= 0) {
        // ------------------------------------------------------------ MMA issuers (k-steps 8j .. 8j + 7)
        // warp-uniform operands (lane-0 shuffles), as in gemm_ex_kernel
        const int j = __shfl_sync(0xFFFFFFFFu, head_issuer_of_warp(warp), 0);
        const int i0 = C::KSTEPS * j;
        const bool leader = elect_one();
        int a = 0, acc = 0;
        uint32_t aph = 0, accph = 0;
        const uint32_t tmem_u = __shfl_sync(0xFFFFFFFFu, tmem, 0);
        const uint64_t bdesc_raw = smem_desc_k_sw128(smem_u32(smem + C::X_RING));
        const uint64_t bdesc_base = ((uint64_t)__shfl_sync(0xFFFFFFFFu, (uint32_t)(bdesc_raw >> 32), 0) << 32) |
                                    (uint64_t)__shfl_sync(0xFFFFFFFFu, (uint32_t)bdesc_raw, 0);
        HeadSegIter it(p.k_tiles, t_begin, t_end);
        HeadSeg sg;
        bool ok = true;
        while (ok && it.next(sg)) {
            if (!__all_sync(0xFFFFFFFFu, tc_wait(&accempty[acc], accph ^ 1u, abort_flag))) {
                if (leader) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_MMA);
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_u + (uint32_t)(C::ACC_COL0 + C::ACC_BUF_COLS * acc + NX * j);
            uint32_t first = 1;
            for (int kt = sg.k0; kt < sg.k1; ++kt) {
                if (!__all_sync(0xFFFFFFFFu, tc_wait(&ready[a], aph, abort_flag))) {
                    if (leader) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_MMA);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t bdesc0 = bdesc_base + (uint64_t)((a * C::X_BYTES) >> 4);
                const uint32_t a_tmem = tmem_u + (uint32_t)(128 * a + 8 * i0);
                if (leader) {
#pragma unroll
                    for (int u = 0; u < C::KSTEPS; ++u) {
                        const int i = i0 + u;
                        mma_ts_f16(d_tmem, a_tmem + 8u * u, bdesc0 + (uint64_t)((((i >> 2) * C::X_SUB + (i & 3) * 32)) >> 4),
                                   C::IDESC, (u == 0) ? (first ^ 1u) : 1u);
                    }
                    mma_commit(&tfree[a]);
                }
                __syncwarp();
                first = 0;
                if (++a == C::NUM_A) { a = 0; aph ^= 1u; }
            }
            if (!ok) break;
            if (leader) mma_commit(&accfull[acc]);
            __syncwarp();
            if (++acc == C::ACC_BUFS) { acc = 0; accph ^= 1u; }
        }
        if (leader) mma_commit(drain);
        __syncwarp();
        if (warp == 1 && !__all_sync(0xFFFFFFFFu, mbar_wait(drain, 0, TL_WAIT_LIMIT)) && lane == 0)
            tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DRAIN);
    } else if (warp >= C::DQ_FIRST && warp < C::DQ_FIRST + 8) {
        // ------------------------------------------------------------ dequantisers
        // warp (set, quarter q): rows 32q..32q+31, the whole 256 k, as four 64-k chunks (64 bytes
        // of the row each: piece j of slice c / 2, pieces 4 (c % 2) .. + 3 of the row's 128-byte line)
        const int set = (warp - C::DQ_FIRST) >> 2;
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
        const int row_off = r * 128, row_sw = r & 7;
        const int ntiles = (int)(t_end - t_begin);
        int s = set, a = set;
        uint32_t ph = 0, aph = 0;
        auto advance2 = [](int& idx, uint32_t& phase, int ring) {
            idx += 2;
            if (idx >= ring) { idx -= ring; phase ^= 1u; }
        };
        const uint8_t* st = smem;
        auto piece = [&](int c, int j) {
            return *reinterpret_cast<const uint4*>(st + (c >> 1) * (128 * 128) + row_off + ((((c & 1) * 4 + j) ^ row_sw) << 4));
        };
        bool ok = true;
        for (int n = set; ok && n < ntiles; n += 2) {
            if (!__all_sync(0xFFFFFFFFu, tc_wait(&wfull[s], ph, abort_flag))) { ok = false; break; }
            st = smem + s * C::W_STAGE_BYTES;
            uint4 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = piece(0, j);
            if (!__all_sync(0xFFFFFFFFu, tc_wait(&tfree[a], aph ^ 1u, abort_flag))) { ok = false; break; }
            tc_fence_after();
            const uint32_t col = t_lane + (uint32_t)(128 * a);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t out[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) head_decode16(v[j], &out[8 * j]);
                if (c < 3) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) v[j] = piece(c + 1, j);
                }
                tmem_st32(col + 32u * c, out);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&wempty[s]);   // every byte of the stage this warp reads is in registers
            advance2(s, ph, C::W_STAGES);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready[a]);
            advance2(a, aph, C::NUM_A);
        }
        if (!ok && lane == 0) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DEQUANT);
        tmem_wait_st();
    } else if (warp >= C::EPI_FIRST && warp < C::EPI_FIRST + 4) {
        // ------------------------------------------------------------ epilogue: fp32 logits
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
        const int M = p.M, N = p.N;
        int acc = 0;
        uint32_t accph = 0;
        HeadSegIter it(p.k_tiles, t_begin, t_end);
        HeadSeg sg;
        while (it.next(sg)) {
            if (!tc_wait(&accfull[acc], accph, abort_flag)) {
                tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_EPILOGUE);
                break;
            }
            tc_fence_after();
            const int n = sg.ntile * TC_BLOCK_N + r;
            const float sn = (n < N) ? (p.row_scale ? __ldg(p.row_scale + n) : p.tensor_scale) : 0.0f;
            const bool whole = (sg.k0 == 0 && sg.k1 == p.k_tiles);
            const long long ta = (long long)sg.ntile * p.k_tiles;
            const int my_slot = 2 * (int)blockIdx.x + (sg.t0 == t_begin ? 0 : 1);
            float* mine = p.partials + (size_t)my_slot * (32 * TC_BLOCK_N);
            float v[NX];
#pragma unroll
            for (int i = 0; i < NX; ++i) v[i] = 0.0f;
#pragma unroll
            for (int j = 0; j < C::NISSUE; ++j) {
#pragma unroll
                for (int c0 = 0; c0 < NX; c0 += 16) {
                    uint32_t raw[16];
                    tmem_ld16(t_lane + (uint32_t)(C::ACC_COL0 + C::ACC_BUF_COLS * acc + NX * j + c0), raw);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[c0 + i] += __uint_as_float(raw[i]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
            if (++acc == C::ACC_BUFS) { acc = 0; accph ^= 1u; }
            if (whole) {
                if (n < N) {
#pragma unroll
                    for (int i = 0; i < NX; ++i)
                        if (i < M) p.logits[(size_t)i * N + n] = (v[i] * __ldg(p.rowfac + i)) * sn;
                }
                continue;
            }
#pragma unroll
            for (int i = 0; i < NX; ++i)
                if (i < M) mine[i * TC_BLOCK_N + r] = v[i];
            const long long tb = ta + p.k_tiles;
            const int f = tc_cta_of(ta, p.total_tiles, ctas);
            const int l = tc_cta_of(tb - 1, p.total_tiles, ctas);
            __threadfence();
            __syncwarp();
            unsigned old = 0;
            if (lane == 0) old = atomicAdd(&p.counters[4 * f + q], 1u);
            old = __shfl_sync(0xFFFFFFFFu, old, 0);
            if (old == (unsigned)(l - f)) {
                __threadfence();
#pragma unroll
                for (int c0 = 0; c0 < NX; c0 += 16) {
                    float w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) w[i] = 0.0f;
                    for (int c = f; c <= l; ++c) {
                        const long long cs = tc_range_start(c, p.total_tiles, ctas);
                        const int slot = 2 * c + ((ta > cs ? ta : cs) == cs ? 0 : 1);
                        const float* part = p.partials + (size_t)slot * (32 * TC_BLOCK_N);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < M) w[i] += __ldcg(&part[(c0 + i) * TC_BLOCK_N + r]);
                    }
                    if (n < N) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < M) p.logits[(size_t)(c0 + i) * N + n] = (w[i] * __ldg(p.rowfac + c0 + i)) * sn;
                    }
                }
                if (lane == 0) p.counters[4 * f + q] = 0u;
            }
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// One logit of a row the X preparation flagged, recomputed from the bf16 X as given in fp64 by
// one warp (lanes over k, a fixed butterfly) and rounded to fp32 once.
__device__ __forceinline__ float head_logit_fp64(const HeadParams& p, int m, int n, int lane) {
    const uint8_t* wr = p.w + (size_t)n * p.K;
    const __nv_bfloat16* xr = p.x + (size_t)m * p.K;
    const double sn = p.row_scale ? (double)p.row_scale[n] : (double)p.tensor_scale;
    double acc = 0.0;
    for (int k = 2 * lane; k < p.K; k += 64) {
        const uint32_t two = (uint32_t)wr[k] | ((uint32_t)wr[k + 1] << 8);
        uint32_t h;
        asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h) : "r"(two));
        const __half2 hv = *reinterpret_cast<const __half2*>(&h);
        acc += (double)__bfloat162float(xr[k]) * (double)__low2float(hv);
        acc += (double)__bfloat162float(xr[k + 1]) * (double)__high2float(hv);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    return (float)(acc * sn);
}

// Greedy top-2 of each row of logits, one CTA per row, a fixed order of comparisons: token
// (largest logit, lowest index among equal ones; -1 if the row holds a NaN), the largest and the
// second largest values (the largest of the row without the token's entry), and their gap in
// bf16 units in the last place at the largest value.
struct HeadTop2 {
    int token;
    float top1, top2, gap_ulp;
};

constexpr int HEAD_TOP2_THREADS = 256;

struct T2 {
    float v1, v2;
    int i1;
    int nan;
};

__device__ __forceinline__ T2 t2_merge(T2 a, T2 b) {
    T2 r;
    r.nan = a.nan | b.nan;
    const bool a_first = (a.v1 > b.v1) || (a.v1 == b.v1 && a.i1 < b.i1);
    const T2& w = a_first ? a : b;
    const T2& l = a_first ? b : a;
    r.v1 = w.v1;
    r.i1 = w.i1;
    r.v2 = fmaxf(w.v2, l.v1);
    return r;
}

// bf16 spacing at |v| (finite): 2^(e - 7) for 2^e <= |v| < 2^(e + 1), e >= -126; 2^-133 below.
__device__ __forceinline__ float bf16_ulp_f(float v) {
    const float a = fabsf(v);
    if (a < 0x1p-126f) return 0x1p-133f;
    const int e = ilogbf(a);
    return ldexpf(1.0f, e - 7);
}

__device__ __forceinline__ T2 t2_warp_merge(T2 t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        T2 u;
        u.v1 = __shfl_xor_sync(0xFFFFFFFFu, t.v1, o);
        u.v2 = __shfl_xor_sync(0xFFFFFFFFu, t.v2, o);
        u.i1 = __shfl_xor_sync(0xFFFFFFFFu, t.i1, o);
        u.nan = __shfl_xor_sync(0xFFFFFFFFu, t.nan, o);
        t = t2_merge(t, u);
    }
    return t;
}

// After the GEMM, one launch: grid (chunks, M); CTA (c, m) takes logits[m][c * chunk, (c + 1) * chunk).
//   1. If the X preparation flagged row m, it first recomputes those logits in fp64 (a warp per
//      weight row) and writes them.
//   2. It reduces the chunk to one partial (best value, its lowest index, best of the rest, any
//      NaN) and stores it.
//   3. The last CTA of row m to finish (an atomic counter per row, reset by that CTA; nothing waits)
//      merges the row's partials with one warp and writes the token, the two best values and their
//      gap in bf16 units in the last place (token -1 and NaN for a row with a NaN).
// The merge keeps the largest value with the lowest index and the largest of the rest, so the answer
// does not depend on the order in which partials are merged.
__global__ void __launch_bounds__(HEAD_TOP2_THREADS) head_tail_kernel(const __grid_constant__ HeadParams p, int chunk,
                                                                      T2* part, unsigned* row_counters,
                                                                      HeadTop2* out) {
    const int c = blockIdx.x, m = blockIdx.y, chunks = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = p.N;
    float* row = p.logits + (size_t)m * N;
    const int n0 = c * chunk, n1 = min(N, n0 + chunk);
    unsigned flagged = __ldcg(p.rowmask);
    if (p.M < 32) flagged &= (1u << p.M) - 1u;
    if ((flagged >> m) & 1u) {
        for (int n = n0 + warp; n < n1; n += HEAD_TOP2_THREADS / 32) {
            const float v = head_logit_fp64(p, m, n, lane);
            if (lane == 0) row[n] = v;
        }
        __syncthreads();
    }
    T2 t = {-INFINITY, -INFINITY, 0x7FFFFFFF, 0};
    for (int n = n0 + (int)threadIdx.x; n < n1; n += HEAD_TOP2_THREADS) {
        const float v = __ldcg(row + n);
        if (isnan(v)) { t.nan = 1; continue; }
        const T2 e = {v, -INFINITY, n, 0};
        t = t2_merge(t, e);
    }
    t = t2_warp_merge(t);
    __shared__ T2 ws[HEAD_TOP2_THREADS / 32];
    __shared__ int last;
    if (lane == 0) ws[warp] = t;
    __syncthreads();
    if (threadIdx.x == 0) {
        T2 r = ws[0];
        for (int w = 1; w < HEAD_TOP2_THREADS / 32; ++w) r = t2_merge(r, ws[w]);
        part[(size_t)m * chunks + c] = r;
        __threadfence();
        last = (atomicAdd(row_counters + m, 1u) == (unsigned)(chunks - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (!last || warp != 0) return;
    __threadfence();
    T2 r = {-INFINITY, -INFINITY, 0x7FFFFFFF, 0};
    for (int q = lane; q < chunks; q += 32) {
        T2 e;
        const T2* src = part + (size_t)m * chunks + q;
        e.v1 = __ldcg(&src->v1);
        e.v2 = __ldcg(&src->v2);
        e.i1 = __ldcg(&src->i1);
        e.nan = __ldcg(&src->nan);
        r = t2_merge(r, e);
    }
    r = t2_warp_merge(r);
    if (lane == 0) {
        HeadTop2 o;
        if (r.nan) {
            o.token = -1;
            o.top1 = o.top2 = o.gap_ulp = __int_as_float(0x7FC00000);
        } else {
            o.token = r.i1;
            o.top1 = r.v1;
            o.top2 = r.v2;
            o.gap_ulp = (r.v1 - r.v2) / bf16_ulp_f(r.v1);
        }
        out[m] = o;
        row_counters[m] = 0u;   // ready for the next call
    }
}

}  // namespace tl
