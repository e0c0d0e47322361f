// gemm_tc.cuh -- tensor-core NVFP4 verify GEMM for sm_100a (tcgen05 + TMA + tensor memory).
//
// Y[M,N] = X[M,K] . dequant(W)[N,K]^T for M <= 32 draft-tree rows (TandemLLM docs v0.12.0,
// "What TandemLLM is", section 1.2: one verify pass over all tree rows streams every 4-bit
// weight once). The pass is bound by the weight bytes, so the kernel is built around the
// weight stream:
//
//   * Work. A weight tile is 128 rows x 256 k (16 KiB of codes, 2 KiB of scales). All
//     tiles of all matrices of a launch form one list (matrix, n-tile, k-tile); each
//     persistent CTA takes one contiguous, equal share of the list (stream-K). A CTA
//     whose share starts or ends inside an n-tile writes an fp32 partial; the last of an
//     n-tile's contributors (an atomic counter, no waiting) adds the partials in k order,
//     so every output has one fixed reduction order.
//   * Roles, 24 warps. Warp 0 issues TMA loads of codes, scales and the X tile into a
//     ring of shared-memory stages (three lanes, one rank-3 load each, per stage). Warps 4..19 dequantise: a thread owns one weight row and
//     a 128-k half of a tile, reads its codes/scales from shared memory, forms
//     W' = e2m1 * e4m3 in bf16 (exact) and stores it into tensor memory, the A operand. Warp 1 issues tcgen05.mma with
//     A from tensor memory, B = X tile (bf16, shared memory, 128-byte swizzle) and the
//     fp32 accumulator in tensor memory (M_mma = 128 weight rows, N_mma = 16 or 32 X rows).
//     The dequantisers form two sets of eight warps that take alternate tiles, so four
//     dequant warps share each scheduler and one set's waits overlap the other's decode. A single thread keeps
//     only about one tcgen05.mma in flight per ~90 cycles at these small N, so warps 1..3
//     each issue a third of every tile's 16 k-steps into their own accumulator.
//     Warps 20..23 read the accumulators and write Y (or a partial).
//   * Dequantisation without a table. For code c = s e1 e0 m, the bf16 bit pattern
//     (e1 e0 m) << 6 | s << 15 is exactly e2m1(c) * 2^-126 (code 1 lands on a bf16
//     subnormal). One bf16 multiply by e4m3(s) * 2^119 gives W' * 2^-7, exact (at most six
//     significant bits, no overflow, no underflow); 2^7 is folded into the epilogue scale.
//
// Every mbarrier wait is bounded; a wait that runs out records TL_ERR_TIMEOUT in the
// device status word and the CTA winds down (drains its MMAs, frees tensor memory).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "nvfp4_format.cuh"

#ifndef TL_WAIT_LIMIT
#define TL_WAIT_LIMIT (1u << 22)
#endif

namespace tl {

constexpr int TC_BLOCK_N = 128;        // weight rows per tile (MMA M)
constexpr int TC_BLOCK_K = 256;        // k per tile / pipeline stage
constexpr int TC_THREADS = 768;     // 24 warps: producer, 3 MMA issuers, 16 dequantisers, 4 epilogue
constexpr int TC_TMEM_COLS = 512;
// MMA issuers. One thread can only keep about one tcgen05.mma in flight per ~90 cycles,
// whatever N is, so three issuer warps (1..3) share each tile's 16 k-steps (6 / 5 / 5);
// issuer j accumulates into its own accumulator j and the epilogue adds them in order.
constexpr int TC_NISSUE = 3;
__host__ __device__ constexpr int tc_ks_begin(int j) { return j == 0 ? 0 : (j == 1 ? 6 : (j == 2 ? 11 : 16)); }

enum : int {
    TL_DEV_ERR_TIMEOUT_PRODUCER = 0x101,
    TL_DEV_ERR_TIMEOUT_MMA = 0x102,
    TL_DEV_ERR_TIMEOUT_DEQUANT = 0x103,
    TL_DEV_ERR_TIMEOUT_EPILOGUE = 0x104,
    TL_DEV_ERR_TIMEOUT_DRAIN = 0x105,
};

// One matrix of a launch: tensor maps of its codes, scales and X, and its work-list offset.
struct alignas(64) TcMat {
    CUtensorMap tm_codes;   // uint8 {K/2, N, 1}, box 128 B x 128 rows x 1, 128-byte swizzle
    CUtensorMap tm_scales;  // uint8 {K/16, N, 1}, box 16 B x 128 rows x 1
    CUtensorMap tm_x;       // bf16 X as 3-D {64, M, K/64}, box {64, NX, 4}: the four 64-k slices of a
                            // tile, 128-byte swizzle (rows >= M read 0)
    __nv_bfloat16* y;
    float g_out;            // epilogue multiplier: global_scale * 2^7
    int N;
    int k_tiles;            // K / 256
    int n_tiles;            // ceil(N / 128)
    long long tile_begin;   // first global tile index of this matrix
};

struct TcParams {
    const TcMat* mats;      // device table, or nullptr to use `one`
    int n_mats;
    int M;
    long long total_tiles;
    float* partials;        // [2 * gridDim.x][32][128] fp32
    unsigned* counters;     // [4 * gridDim.x], zero between launches
    int* err;               // device status word
    TcMat one;
};

template <int NX>
struct TcCfg {
    static constexpr int CODES_BYTES = TC_BLOCK_N * (TC_BLOCK_K / 2);   // 16384
    static constexpr int X_SUB = NX * 128;                              // one 64-k slice of X
    static constexpr int X_BYTES = 4 * X_SUB;
    static constexpr int SCALES_BYTES = TC_BLOCK_N * (TC_BLOCK_K / 16); // 2048
    static constexpr int STAGE_BYTES = CODES_BYTES + X_BYTES + SCALES_BYTES;
    static constexpr int STAGES = (NX == 32) ? 6 : 8;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 512 /*barriers*/;
    static constexpr uint32_t IDESC = idesc_f16(1u, 128u, (uint32_t)NX);
    // tensor memory: three A buffers (128 columns each) so a tile set never waits for the
    // MMAs of its own previous tile, then ACC_BUFS accumulator buffers of TC_NISSUE
    // accumulators of NX fp32 columns each (one buffer at NX = 32: the MMAs then wait for
    // the epilogue once per n-tile segment, which is cheaper than a third-short A ring)
    static constexpr int NUM_A = 3;
    static constexpr int ACC_BUFS = (NX == 16) ? 2 : 1;
    static constexpr int ACC_COL0 = 128 * NUM_A;
    static constexpr int ACC_BUF_COLS = TC_NISSUE * NX;
    static_assert(ACC_COL0 + ACC_BUFS * ACC_BUF_COLS <= TC_TMEM_COLS, "tensor memory budget");
};

struct TcSeg {
    int mat, ntile, k0, k1;
    long long t0;   // global index of tile k0
};

// Walks the contiguous tile range [t, end) of one CTA as segments within one n-tile.
struct TcSegIter {
    const TcMat* mats;
    int n_mats, mat;
    long long t, end;
    __device__ TcSegIter(const TcMat* m, int n, long long begin, long long stop)
        : mats(m), n_mats(n), mat(0), t(begin), end(stop) {
        int lo = 0, hi = n - 1;   // last matrix with tile_begin <= begin
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (mats[mid].tile_begin <= begin) lo = mid; else hi = mid - 1;
        }
        mat = lo;
    }
    __device__ bool next(TcSeg& s) {
        if (t >= end) return false;
        while (mat + 1 < n_mats && mats[mat + 1].tile_begin <= t) ++mat;
        const long long kt = mats[mat].k_tiles;
        const long long local = t - mats[mat].tile_begin;
        s.mat = mat;
        s.ntile = (int)(local / kt);
        s.k0 = (int)(local % kt);
        const long long rem = end - t;
        s.k1 = (int)((kt - s.k0) < rem ? kt : s.k0 + rem);
        s.t0 = t;
        t += s.k1 - s.k0;
        return true;
    }
};

__device__ __forceinline__ long long tc_range_start(long long c, long long total, long long ctas) {
    return (c * total) / ctas;
}
__device__ __forceinline__ int tc_cta_of(long long t, long long total, long long ctas) {
    return (int)(((t + 1) * ctas - 1) / total);
}

__device__ __forceinline__ void tc_fail(int* err, volatile int* abort_flag, int code) {
    atomicCAS(err, 0, code);
    *abort_flag = 1;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Eight scale bytes -> eight bf16x2 words, both halves e4m3(s) * 2^119 (exact).
// Fast path for finite, positive, normal scales (every scale the quantiser writes except
// all-zero blocks): bf16 bits of s * 2^119 are ((s & 0x7F) << 4) + (239 << 7). Anything
// else (zero or subnormal scale, sign bit, NaN) takes the exact float route.
__device__ __forceinline__ void scales8_to_bf16x2(uint2 sc, uint32_t (&S)[8]) {
    const uint32_t e0 = sc.x & 0x78787878u, e1 = sc.y & 0x78787878u;
    const uint32_t zero_exp = ((e0 - 0x01010101u) & ~e0) | ((e1 - 0x01010101u) & ~e1);   // a byte had e == 0
    const uint32_t nan_or_neg = ((sc.x | sc.y) & 0x80808080u) |
                                (((sc.x & 0x7F7F7F7Fu) + 0x01010101u) & 0x80808080u) |
                                (((sc.y & 0x7F7F7F7Fu) + 0x01010101u) & 0x80808080u);   // bit 7 set or byte 0x7F
    if (((zero_exp & 0x80808080u) | nan_or_neg) == 0u) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            // [b_lo, 0, b_hi, 0] -> bf16 of each scale * 2^119 in its own half
            const uint32_t w = prmt(p < 2 ? sc.x : sc.y, 0u, (p & 1) ? 0x4342u : 0x4140u);
            const uint32_t b = (w << 4) + 0x77807780u;
            S[2 * p] = prmt(b, 0u, 0x1010u);
            S[2 * p + 1] = prmt(b, 0u, 0x3232u);
        }
        return;
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint32_t two = ((p < 2 ? sc.x : sc.y) >> (16 * (p & 1))) & 0xFFFFu;
        const __half2 h = e4m3x2_to_half2(two);
        const float f0 = __low2float(h) * 0x1p119f;
        const float f1 = __high2float(h) * 0x1p119f;
        S[2 * p] = prmt(__float_as_uint(f0), 0u, 0x3232u);
        S[2 * p + 1] = prmt(__float_as_uint(f1), 0u, 0x3232u);
    }
}

// Four code bytes (eight weights, k order) -> four bf16x2 words W' * 2^-7 in k order.
__device__ __forceinline__ void decode8(uint32_t q, uint32_t S, uint32_t* out) {
    const uint32_t L = q & 0x0F0F0F0Fu;          // even-k nibbles, one per byte
    const uint32_t H = (q >> 4) & 0x0F0F0F0Fu;   // odd-k nibbles
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // [L.byte i, 0, H.byte i, 0]; selector 8 replicates the (zero) sign of L.byte 0
        const uint32_t t = prmt(L, H, (uint32_t)i | 0x80u | ((uint32_t)(4 + i) << 8) | 0x8000u);
        const uint32_t w = (t * 0x1040u) & 0x81C081C0u;   // e1e0m -> bits 6..8, sign -> bit 15
        out[i] = hmul2_bf16(w, S);
    }
}

// MMA issuer J (warp 1 + J, lane 0): k-steps [tc_ks_begin(J), tc_ks_begin(J + 1)) of every
// tile into accumulator J.
template <int NX, int J>
__device__ __forceinline__ void tc_mma_issuer(const TcParams& p, const TcMat* mats, long long t_begin, long long t_end,
                                              uint8_t* smem, uint32_t tmem, uint64_t* full, uint64_t* empty,
                                              uint64_t* aready, uint64_t* afree, uint64_t* accfull,
                                              uint64_t* accempty, uint64_t* drain, volatile int* abort_flag) {
    using C = TcCfg<NX>;
    constexpr int I0 = tc_ks_begin(J), I1 = tc_ks_begin(J + 1);
    int s = 0, a = 0, acc = 0;
    uint32_t ph = 0, aph = 0, accph = 0;
    TcSegIter it(mats, p.n_mats, t_begin, t_end);
    TcSeg sg;
    bool ok = true;
    while (ok && it.next(sg)) {
        if (*abort_flag || !mbar_wait(&accempty[acc], accph ^ 1u, TL_WAIT_LIMIT)) {
            tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_MMA);
            break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(C::ACC_COL0 + C::ACC_BUF_COLS * acc + NX * J);
        for (int kt = sg.k0; kt < sg.k1; ++kt) {
            if (*abort_flag || !mbar_wait(&full[s], ph, TL_WAIT_LIMIT) ||
                !mbar_wait(&aready[a], aph, TL_WAIT_LIMIT)) {
                tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_MMA);
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t xs = smem_u32(smem + s * C::STAGE_BYTES + C::CODES_BYTES);
            const uint32_t a_tmem = tmem + (uint32_t)(128 * a);
#pragma unroll
            for (int i = I0; i < I1; ++i) {
                const uint64_t bdesc = smem_desc_k_sw128(xs + (i >> 2) * C::X_SUB + (i & 3) * 32);
                mma_ts_f16(d_tmem, a_tmem + 8u * i, bdesc, C::IDESC, (kt > sg.k0 || i > I0) ? 1u : 0u);
            }
            mma_commit(&empty[s]);
            mma_commit(&afree[a]);
            if (++s == C::STAGES) { s = 0; ph ^= 1u; }
            if (++a == C::NUM_A) { a = 0; aph ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&accfull[acc]);
        if (++acc == C::ACC_BUFS) { acc = 0; accph ^= 1u; }
    }
    // no MMA of this issuer may still run when tensor memory is released
    mma_commit(drain);
}

template <int NX>
__global__ void __launch_bounds__(TC_THREADS, 1)
gemm_tc_kernel(const __grid_constant__ TcParams p) {
    using C = TcCfg<NX>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* full = bars;                          // [STAGES] TMA bytes landed
    uint64_t* empty = full + C::STAGES;             // [STAGES] stage consumed (one commit per issuer)
    uint64_t* aready = empty + C::STAGES;           // [NUM_A] A buffer written (8 warps of a tile set)
    uint64_t* afree = aready + C::NUM_A;            // [NUM_A] A buffer read (one commit per issuer)
    uint64_t* accfull = afree + C::NUM_A;           // [ACC_BUFS] accumulators complete (one commit per issuer)
    uint64_t* accempty = accfull + 2;               // [ACC_BUFS] accumulators read (4 epilogue warps)
    uint64_t* drain = accempty + 2;                 // [1] every MMA finished (one commit per issuer)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const TcMat* mats = p.mats ? p.mats : &p.one;
    const long long ctas = gridDim.x;
    const long long t_begin = tc_range_start(blockIdx.x, p.total_tiles, ctas);
    const long long t_end = tc_range_start(blockIdx.x + 1, p.total_tiles, ctas);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], TC_NISSUE); }
        for (int i = 0; i < C::NUM_A; ++i) { mbar_init(&aready[i], 8); mbar_init(&afree[i], TC_NISSUE); }
        for (int i = 0; i < C::ACC_BUFS; ++i) { mbar_init(&accfull[i], TC_NISSUE); mbar_init(&accempty[i], 4); }
        mbar_init(drain, TC_NISSUE);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TC_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp runs the loop and every lane waits for the stage itself; lane 0 posts
        // the stage's byte count, then lanes 0, 1, 2 copy codes, X and scales with one
        // converged 3-D load (all three maps are rank 3).
        const uint64_t pol = (lane == 1) ? policy_evict_last() : policy_evict_first();
        const uint32_t dst_off = (lane == 0) ? 0u : (lane == 1) ? (uint32_t)C::CODES_BYTES
                                                                : (uint32_t)(C::CODES_BYTES + C::X_BYTES);
        const uint32_t smem0 = smem_u32(smem);
        int s = 0;
        uint32_t ph = 0;
        uint32_t issued = 0;   // bit s: stage s was issued at least once
        uint32_t last_ph = 0;  // bit s: parity of its latest use
        TcSegIter it(mats, p.n_mats, t_begin, t_end);
        TcSeg sg;
        bool ok = true;
        while (ok && it.next(sg)) {
            const TcMat& m = mats[sg.mat];
            const void* tmap = (lane == 0) ? (const void*)&m.tm_codes
                             : (lane == 1) ? (const void*)&m.tm_x : (const void*)&m.tm_scales;
            const int c1 = (lane == 1) ? 0 : sg.ntile * TC_BLOCK_N;
            for (int kt = sg.k0; kt < sg.k1; ++kt) {
                const bool got = !*abort_flag && mbar_wait(&empty[s], ph ^ 1u, TL_WAIT_LIMIT);
                if (!__all_sync(0xFFFFFFFFu, got)) {
                    if (lane == 0) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_PRODUCER);
                    ok = false;
                    break;
                }
                if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)C::STAGE_BYTES);
                __syncwarp();
                const int c0 = (lane == 0) ? kt * (TC_BLOCK_K / 2) : (lane == 1) ? 0 : kt * (TC_BLOCK_K / 16);
                const int c2 = (lane == 1) ? kt * 4 : 0;
                if (lane < 3)
                    tma_load_3d_s(smem0 + (uint32_t)(s * C::STAGE_BYTES) + dst_off, tmap, &full[s], c0, c1, c2, pol);
                issued |= 1u << s;
                last_ph = (last_ph & ~(1u << s)) | (ph << s);
                if (++s == C::STAGES) { s = 0; ph ^= 1u; }
            }
        }
        // every issued copy must land before the CTA can leave
        if (lane == 0) {
            for (int i = 0; i < C::STAGES; ++i)
                if ((issued >> i) & 1u)
                    if (!mbar_wait(&full[i], (last_ph >> i) & 1u, TL_WAIT_LIMIT))
                        tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DRAIN);
        }
    } else if (warp >= 1 && warp <= TC_NISSUE) {
        // ------------------------------------------------------------ MMA issuers
        if (lane == 0) {
            if (warp == 1)
                tc_mma_issuer<NX, 0>(p, mats, t_begin, t_end, smem, tmem, full, empty, aready, afree, accfull, accempty, drain, abort_flag);
            else if (warp == 2)
                tc_mma_issuer<NX, 1>(p, mats, t_begin, t_end, smem, tmem, full, empty, aready, afree, accfull, accempty, drain, abort_flag);
            else
                tc_mma_issuer<NX, 2>(p, mats, t_begin, t_end, smem, tmem, full, empty, aready, afree, accfull, accempty, drain, abort_flag);
            if (warp == 1 && !mbar_wait(drain, 0, TL_WAIT_LIMIT)) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DRAIN);
        }
    } else if (warp >= 4 && warp < 20) {
        // ------------------------------------------------------------ dequantisers
        // 16 warps = 2 tile sets x 2 k-halves x 4 lane quarters. Set t takes the tiles with
        // parity t, so two tiles are decoded at once; within a tile, the warp of k-half h and
        // lane quarter q decodes rows 32q..32q+31, k in [128h, 128h + 128), in two chunks of
        // 64 k, and stores them into tensor-memory columns [64h, 64h + 64) of the A buffer.
        const int dq = warp - 4;
        const int set = dq >> 3;
        const int kh = (dq >> 2) & 1;
        const int q = warp & 3;                  // tensor-memory lane quarter
        const int r = 32 * q + lane;             // weight row within the tile
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
        const int row_off = r * 128, row_sw = r & 7;   // chunk j of row r sits at row_off + ((j ^ row_sw) << 4)
        int s = 0, a = 0, par = 0;
        uint32_t ph = 0, aph = 0;
        TcSegIter it(mats, p.n_mats, t_begin, t_end);
        TcSeg sg;
        bool ok = true;
        while (ok && it.next(sg)) {
            for (int kt = sg.k0; kt < sg.k1; ++kt) {
                const int ts = s, ta = a;
                const uint32_t tph = ph, taph = aph;
                const bool mine = (par == set);
                if (++s == C::STAGES) { s = 0; ph ^= 1u; }
                if (++a == C::NUM_A) { a = 0; aph ^= 1u; }
                par ^= 1;
                if (!mine) continue;
                if (*abort_flag || !mbar_wait(&full[ts], tph, TL_WAIT_LIMIT)) {
                    tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DEQUANT);
                    ok = false;
                    break;
                }
                const uint8_t* st = smem + ts * C::STAGE_BYTES;
                const uint2 sc = *reinterpret_cast<const uint2*>(st + C::CODES_BYTES + C::X_BYTES + r * 16 + 8 * kh);
                uint32_t S[8];
                scales8_to_bf16x2(sc, S);
                const uint32_t col = (uint32_t)(128 * ta + 64 * kh);
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {   // two chunks of 64 k: 32 code bytes, 4 scales
                    uint4 cw[2];
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj)
                        cw[jj] = *reinterpret_cast<const uint4*>(st + row_off + (((4 * kh + 2 * hc + jj) ^ row_sw) << 4));
                    uint32_t out[32];
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const uint4 w = cw[jj];
                        const int b = 4 * hc + 2 * jj;
                        decode8(w.x, S[b], &out[16 * jj + 0]);
                        decode8(w.y, S[b], &out[16 * jj + 4]);
                        decode8(w.z, S[b + 1], &out[16 * jj + 8]);
                        decode8(w.w, S[b + 1], &out[16 * jj + 12]);
                    }
                    if (hc == 0) {   // the A buffer must have been read by the MMAs of tile c - NUM_A
                        if (*abort_flag || !mbar_wait(&afree[ta], taph ^ 1u, TL_WAIT_LIMIT)) {
                            tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DEQUANT);
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                    }
                    tmem_st32(t_lane + col + 32 * hc, out);
                }
                if (!ok) break;
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&aready[ta]);
            }
        }
    } else if (warp >= 20) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
        const int M = p.M;
        int acc = 0;
        uint32_t accph = 0;
        TcSegIter it(mats, p.n_mats, t_begin, t_end);
        TcSeg sg;
        while (it.next(sg)) {
            if (*abort_flag || !mbar_wait(&accfull[acc], accph, TL_WAIT_LIMIT)) {
                tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_EPILOGUE);
                break;
            }
            tc_fence_after();
            const TcMat& m = mats[sg.mat];
            const int N = m.N;
            const int n = sg.ntile * TC_BLOCK_N + r;
            const bool whole = (sg.k0 == 0 && sg.k1 == m.k_tiles);
            const long long ta = m.tile_begin + (long long)sg.ntile * m.k_tiles;
            const int my_slot = 2 * (int)blockIdx.x + (sg.t0 == t_begin ? 0 : 1);
            float* mine = p.partials + (size_t)my_slot * (32 * TC_BLOCK_N);
            // 16 columns (X rows) at a time: add the issuers' accumulators in fixed order,
            // then write Y (whole n-tile) or this CTA's partial (split n-tile)
#pragma unroll
            for (int c0 = 0; c0 < NX; c0 += 16) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = 0.0f;
#pragma unroll
                for (int j = 0; j < TC_NISSUE; ++j) {
                    uint32_t raw[16];
                    tmem_ld16(t_lane + (uint32_t)(C::ACC_COL0 + C::ACC_BUF_COLS * acc + NX * j + c0), raw);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] += __uint_as_float(raw[i]);
                }
                if (whole) {
                    if (n < N) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < M) m.y[(long long)(c0 + i) * N + n] = __float2bfloat16_rn(v[i] * m.g_out);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c0 + i < M) mine[(c0 + i) * TC_BLOCK_N + r] = v[i];
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[acc]);
            if (++acc == C::ACC_BUFS) { acc = 0; accph ^= 1u; }
            if (whole) continue;

            // split n-tile: the last of the n-tile's contributors for these 32 rows adds all
            // partials in k (CTA) order
            const long long tb = ta + m.k_tiles;
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
                    float v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = 0.0f;
                    for (int c = f; c <= l; ++c) {
                        const long long cs = tc_range_start(c, p.total_tiles, ctas);
                        const int slot = 2 * c + ((ta > cs ? ta : cs) == cs ? 0 : 1);
                        const float* part = p.partials + (size_t)slot * (32 * TC_BLOCK_N);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < M) v[i] += __ldcg(&part[(c0 + i) * TC_BLOCK_N + r]);
                    }
                    if (n < N) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (c0 + i < M) m.y[(long long)(c0 + i) * N + n] = __float2bfloat16_rn(v[i] * m.g_out);
                    }
                }
                if (lane == 0) p.counters[4 * f + q] = 0u;   // ready for the next launch
            }
        }
    }
    __syncwarp();

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TC_TMEM_COLS);
    }
}

}  // namespace tl
