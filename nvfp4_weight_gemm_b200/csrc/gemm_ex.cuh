// gemm_ex.cuh -- the exact f16 tensor-core NVFP4 verify GEMM for sm_100a (the default path).
//
// Y[M,N] = X[M,K] . dequant(W)[N,K]^T for M <= 32 draft-tree rows (TandemLLM docs v0.12.0,
// "What TandemLLM is", section 1.2: one verify pass over all tree rows streams every 4-bit
// weight once, so the pass is bound by the weight bytes).
//
// Operands. A = W' = e2m1 * e4m3 in f16, written into tensor memory by CUDA cores: the hardware
// converts each code byte to two f16 E2M1 values and one f16 multiply by the block's E4M3 scale
// (also a hardware convert) gives W' exactly (at most 6 significant bits, 2^-10 <= |W'| <= 2688).
// B = the prepared X (xprep.cuh): row m of X times 2^-e_m in f16, exact. fp32 accumulator in
// tensor memory; the epilogue multiplies row m by global_scale * 2^e_m and rounds to bf16 once.
//
// Work and split-K as in gemm_tc.cuh: a weight tile is 128 rows x 256 k; all tiles of all
// matrices of a launch form one list, each persistent CTA takes one contiguous, equal share
// (stream-K), and split n-tiles are summed in k order by their last contributor.
//
// Roles (one CTA per SM):
//   * warp 0        weight producer: TMA copies of codes and scales into a ring of stages.
//   * warp 3        X producer: one TMA copy of the X tile of each k-tile into the tile's slot.
//   * warps 4..11   dequantisers, two tile sets of four lane quarters; set t takes the tiles
//                   with parity t. The warp of quarter q decodes weight rows 32q..32q+31 over the
//                   whole 256 k of a tile: it loads its row's 128 code bytes and 16 scales from
//                   shared memory at once, while the previous tile's stores complete, and hands
//                   the stage straight back (so nearly the whole ring is in flight from HBM); it
//                   decodes the first 64-k chunk before waiting for the tile's slot, then writes
//                   four chunks of 32 tensor-memory columns.
//   * issuers       warps 1 and 2: issuer j issues k-steps 8j..8j+7 of every tile into its own
//                   accumulator. Sixteen warps in all, so no SM sub-partition holds more than four
//                   and every thread may use 128 registers (eighteen warps capped them at 96, with
//                   spills at NX = 32); in paired timings this layout was 5% (M <= 16) to 8%
//                   (M >= 17) faster than four issuer warps, and eight issuers were 23% slower.
//   * warps 12..15  epilogue: add the issuers' accumulators in fixed order, write Y or a partial.
//
// Every mbarrier wait is bounded; a wait that runs out records TL_ERR_TIMEOUT in the device
// status word and the CTA winds down (drains its MMAs and copies, frees tensor memory).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "gemm_tc.cuh"

namespace tl {

template <int NX>
struct ExCfg {
    static constexpr int NISSUE = 2;
    static constexpr int KSTEPS = 16 / NISSUE;            // 16-k MMA steps per issuer per tile
    static constexpr int WARPS = 16;                       // producer, 2 issuers, X producer, 8 + 4
    static constexpr int THREADS = 32 * WARPS;
    static constexpr int DQ_FIRST = 4, DQ_WARPS = 8, EPI_FIRST = 12, XWARP = 3;
    static constexpr int CODES_BYTES = TC_BLOCK_N * (TC_BLOCK_K / 2);   // 16384
    static constexpr int SCALES_BYTES = TC_BLOCK_N * (TC_BLOCK_K / 16); // 2048
    static constexpr int W_STAGE_BYTES = CODES_BYTES + SCALES_BYTES;   // 18432
    static constexpr int X_SUB = NX * 128;                              // one 64-k slice of X (f16)
    static constexpr int X_BYTES = 4 * X_SUB;
    static constexpr int NUM_A = 3;                                    // tile slots: A buffer + X stage
    static constexpr int W_STAGES = (NX == 32) ? 9 : 11;
    static constexpr int X_RING = W_STAGES * W_STAGE_BYTES;
    static constexpr int SMEM_BYTES = X_RING + NUM_A * X_BYTES + 1024 /*align*/ + 512 /*barriers*/;
    static constexpr uint32_t IDESC = idesc_f16(0u /*f16*/, 128u, (uint32_t)NX);
    static constexpr int ACC_COL0 = 128 * NUM_A;                       // three A buffers, then the accumulators
    // accumulator buffers: two where tensor memory holds them (the next segment's MMAs then do not
    // wait for the epilogue); with two issuers that is both NX = 16 and NX = 32
    static constexpr int ACC_BUF_COLS = NISSUE * NX;
    static constexpr int ACC_BUFS = (ACC_COL0 + 2 * ACC_BUF_COLS <= 512) ? 2 : 1;
    static constexpr int TMEM_COLS = 512;
    static_assert(ACC_COL0 + ACC_BUFS * ACC_BUF_COLS <= TMEM_COLS, "tensor memory budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(WARPS * 32 <= 512, "16 warps: at most four per SM sub-partition, 128 registers a thread");
};

template <int NX>
__host__ __device__ constexpr int ex_issuer_of_warp(int w) {
    return (w >= 1 && w <= 2) ? w - 1 : -1;
}

__device__ __forceinline__ uint32_t ex_hmul2_f16(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Four scale bytes of `sc` -> four words holding e4m3(s) in both halves (exact: every E4M3 value,
// subnormals, signs and NaN included, is an f16 value; hardware convert).
__device__ __forceinline__ void ex_scales4(uint32_t sc, uint32_t (&S)[4]) {
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        uint32_t h;
        asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h) : "r"(sc >> (16 * p)));
        S[2 * p] = prmt(h, 0u, 0x1010u);
        S[2 * p + 1] = prmt(h, 0u, 0x3232u);
    }
}

// Sixteen code bytes (32 weights, k order) -> sixteen f16x2 words W' in k order (low nibble to
// the low half). Bytes 0..7 belong to the block of S0, bytes 8..15 to the block of S1. The bytes
// are unpacked with one vector move per word, which the converts read in place.
__device__ __forceinline__ void ex_decode16(uint4 q, uint32_t S0, uint32_t S1, uint32_t* out) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t c0, c1, c2, c3;
        asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
            "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
            "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
            : "=r"(c0), "=r"(c1), "=r"(c2), "=r"(c3) : "r"(w[j]));
        const uint32_t S = (j < 2) ? S0 : S1;
        out[4 * j + 0] = ex_hmul2_f16(c0, S);
        out[4 * j + 1] = ex_hmul2_f16(c1, S);
        out[4 * j + 2] = ex_hmul2_f16(c2, S);
        out[4 * j + 3] = ex_hmul2_f16(c3, S);
    }
}

template <int NX>
__global__ void __launch_bounds__(ExCfg<NX>::THREADS, 1)
gemm_ex_kernel(const __grid_constant__ TcParams p) {
    using C = ExCfg<NX>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::X_RING + C::NUM_A * C::X_BYTES);
    uint64_t* wfull = bars;                         // [W_STAGES] codes + scales landed
    uint64_t* wempty = wfull + C::W_STAGES;         // [W_STAGES] read by the 4 warps of a tile set
    uint64_t* ready = wempty + C::W_STAGES;         // [NUM_A] tile slot filled: 4 warps of a tile set + X bytes
    uint64_t* tfree = ready + C::NUM_A;             // [NUM_A] tile slot read by the MMAs (one commit per issuer)
    uint64_t* accfull = tfree + C::NUM_A;           // [ACC_BUFS] accumulators complete (one commit per issuer)
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
        // The whole warp runs the loop and every lane waits for the stage itself; lane 0 posts
        // the stage's byte count, then lanes 0 and 1 copy codes and scales with one converged
        // 3-D load.
        const uint64_t pol = policy_evict_first();
        const uint32_t dst_off = (lane == 0) ? 0u : (uint32_t)C::CODES_BYTES;
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
            const void* tmap = (lane == 0) ? (const void*)&m.tm_codes : (const void*)&m.tm_scales;
            const int c1 = sg.ntile * TC_BLOCK_N;
            for (int kt = sg.k0; kt < sg.k1; ++kt) {
                const bool got = tc_wait(&wempty[s], ph ^ 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) {
                    if (lane == 0) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_PRODUCER);
                    ok = false;
                    break;
                }
                if (lane == 0) mbar_arrive_expect_tx(&wfull[s], (uint32_t)C::W_STAGE_BYTES);
                __syncwarp();
                const int c0 = (lane == 0) ? kt * (TC_BLOCK_K / 2) : kt * (TC_BLOCK_K / 16);
                if (lane < 2)
                    tma_load_3d_s(smem0 + (uint32_t)(s * C::W_STAGE_BYTES) + dst_off, tmap, &wfull[s], c0, c1, 0, pol);
                issued |= 1u << s;
                last_ph = (last_ph & ~(1u << s)) | (ph << s);
                if (++s == C::W_STAGES) { s = 0; ph ^= 1u; }
            }
        }
        // every issued copy must land before the CTA can leave
        if (lane == 0) {
            for (int i = 0; i < C::W_STAGES; ++i)
                if ((issued >> i) & 1u)
                    if (!mbar_wait(&wfull[i], (last_ph >> i) & 1u, TL_WAIT_LIMIT))
                        tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DRAIN);
        }
    } else if (warp == C::XWARP) {
        // ------------------------------------------------------------ X producer
        // The X tile of tile n goes into the X stage of tile slot n % NUM_A; its arrival is the
        // fifth arrival (plus the bytes) on the slot's ready barrier. One elected lane issues.
        const bool leader = elect_one();
        const uint64_t pol = policy_evict_last();
        int a = 0;
        uint32_t aph = 0;
        uint32_t issued = 0, last_ph = 0;
        TcSegIter it(mats, p.n_mats, t_begin, t_end);
        TcSeg sg;
        bool ok = true;
        while (ok && it.next(sg)) {
            const TcMat& m = mats[sg.mat];
            for (int kt = sg.k0; kt < sg.k1; ++kt) {
                if (!__all_sync(0xFFFFFFFFu, tc_wait(&tfree[a], aph ^ 1u, abort_flag))) {
                    if (leader) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_PRODUCER);
                    ok = false;
                    break;
                }
                if (leader) {
                    mbar_arrive_expect_tx(&ready[a], (uint32_t)C::X_BYTES);
                    tma_load_3d_s(smem_u32(smem + C::X_RING + a * C::X_BYTES), &m.tm_x, &ready[a], 0, 0, kt * 4, pol);
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
    } else if (ex_issuer_of_warp<NX>(warp) >= 0) {
        // ------------------------------------------------------------ MMA issuers
        // The whole warp runs the loop converged; one elected lane issues every MMA and commit.
        // the issuer's index, the tensor-memory base and the X descriptor pass through a lane-0
        // shuffle, which marks them warp-uniform for the compiler: 3% off a pass at M <= 16
        const int j = __shfl_sync(0xFFFFFFFFu, ex_issuer_of_warp<NX>(warp), 0);
        const int i0 = j * C::KSTEPS;
        const uint32_t tmem_u = __shfl_sync(0xFFFFFFFFu, tmem, 0);
        const bool leader = elect_one();
        int a = 0, acc = 0;
        uint32_t aph = 0, accph = 0;
        // descriptor of slot 0's X stage; the start-address field (bits 0..13, address >> 4)
        // advances by plain addition, which never carries out of the field for shared addresses
        const uint64_t bdesc_raw = smem_desc_k_sw128(smem_u32(smem + C::X_RING));
        const uint64_t bdesc_base = ((uint64_t)__shfl_sync(0xFFFFFFFFu, (uint32_t)(bdesc_raw >> 32), 0) << 32) |
                                    (uint64_t)__shfl_sync(0xFFFFFFFFu, (uint32_t)bdesc_raw, 0);
        TcSegIter it(mats, p.n_mats, t_begin, t_end);
        TcSeg sg;
        bool ok = true;
        while (ok && it.next(sg)) {
            if (!__all_sync(0xFFFFFFFFu, tc_wait(&accempty[acc], accph ^ 1u, abort_flag))) {
                if (leader) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_MMA);
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_u + (uint32_t)(C::ACC_COL0 + C::ACC_BUF_COLS * acc + NX * j);
            uint32_t first = 1;   // the first MMA of a segment overwrites the accumulator
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
                        const int i = i0 + u;   // k-step: 64-k slice i >> 2, 16-k part i & 3
                        mma_ts_f16(d_tmem, a_tmem + 8u * u,
                                   bdesc0 + (uint64_t)((((i >> 2) * C::X_SUB + (i & 3) * 32)) >> 4), C::IDESC,
                                   (u == 0) ? (first ^ 1u) : 1u);
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
        // no MMA of this issuer may still run when tensor memory is released
        if (leader) mma_commit(drain);
        __syncwarp();
        if (warp == 1 && !__all_sync(0xFFFFFFFFu, mbar_wait(drain, 0, TL_WAIT_LIMIT)) && lane == 0)
            tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DRAIN);
    } else if (warp >= C::DQ_FIRST && warp < C::DQ_FIRST + C::DQ_WARPS) {
        // ------------------------------------------------------------ dequantisers
        const int set = (warp - C::DQ_FIRST) >> 2;
        const int q = warp & 3;                  // tensor-memory lane quarter
        const int r = 32 * q + lane;             // weight row within the tile
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
        const int row_off = r * 128, row_sw = r & 7;   // chunk j of row r sits at row_off + ((j ^ row_sw) << 4)
        const int sc_off = C::CODES_BYTES + r * 16;
        const int ntiles = (int)(t_end - t_begin);     // a CTA's share is far below 2^31 tiles
        int s = set, a = set;
        uint32_t ph = 0, aph = 0;
        auto advance2 = [](int& idx, uint32_t& phase, int ring) {
            idx += 2;
            if (idx >= ring) { idx -= ring; phase ^= 1u; }
        };
        uint4 cw[8];
        uint4 scv = make_uint4(0, 0, 0, 0);
        // wait for stage s, load this thread's 128 code bytes and 16 scales, hand the stage back
        auto load_stage = [&]() -> bool {
            if (!__all_sync(0xFFFFFFFFu, tc_wait(&wfull[s], ph, abort_flag))) return false;
            const uint8_t* st = smem + s * C::W_STAGE_BYTES;
            scv = *reinterpret_cast<const uint4*>(st + sc_off);
#pragma unroll
            for (int j = 0; j < 8; ++j) cw[j] = *reinterpret_cast<const uint4*>(st + row_off + ((j ^ row_sw) << 4));
            __syncwarp();
            if (lane == 0) mbar_arrive(&wempty[s]);   // release: the loads above are ordered before it
            advance2(s, ph, C::W_STAGES);
            return true;
        };
        bool ok = true;
        if (set < ntiles && !load_stage()) {
            if (lane == 0) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DEQUANT);
            ok = false;
        }
        for (int n = set; ok && n < ntiles; n += 2) {
            const uint32_t col = t_lane + (uint32_t)(128 * a);
            const uint32_t sw[4] = {scv.x, scv.y, scv.z, scv.w};
            uint32_t S[4];
            uint32_t out[32];
            // chunk c = 64 k = 32 tensor-memory columns
            ex_scales4(sw[0], S);
            ex_decode16(cw[0], S[0], S[1], &out[0]);
            ex_decode16(cw[1], S[2], S[3], &out[16]);
            // this tile's slot: read by the MMAs of tile n - NUM_A
            if (!__all_sync(0xFFFFFFFFu, tc_wait(&tfree[a], aph ^ 1u, abort_flag))) { ok = false; break; }
            tc_fence_after();
            tmem_st32(col, out);
#pragma unroll
            for (int c = 1; c < 4; ++c) {
                ex_scales4(sw[c], S);
                ex_decode16(cw[2 * c], S[0], S[1], &out[0]);
                ex_decode16(cw[2 * c + 1], S[2], S[3], &out[16]);
                tmem_st32(col + 32u * c, out);
            }
            // the next tile's bytes, in flight while this tile's stores complete
            if (n + 2 < ntiles && !load_stage()) { ok = false; break; }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready[a]);   // the slot goes to the MMAs
            advance2(a, aph, C::NUM_A);
        }
        if (!ok && lane == 0) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DEQUANT);
        tmem_wait_st();   // no store of this warp may be in flight when tensor memory is released
    } else if (warp >= C::EPI_FIRST && warp < C::EPI_FIRST + 4) {
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
            if (!tc_wait(&accfull[acc], accph, abort_flag)) {
                tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_EPILOGUE);
                break;
            }
            tc_fence_after();
            const TcMat& m = mats[sg.mat];
            // the matrix's fields in registers: stores to Y must not force them to be re-read
            __nv_bfloat16* const yp = m.y;
            const float g = m.g;
            const float* const rowfac = m.rowfac;
            const int N = m.N;
            const int n = sg.ntile * TC_BLOCK_N + r;
            const bool whole = (sg.k0 == 0 && sg.k1 == m.k_tiles);
            const long long ta = m.tile_begin + (long long)sg.ntile * m.k_tiles;
            const int my_slot = 2 * (int)blockIdx.x + (sg.t0 == t_begin ? 0 : 1);
            float* mine = p.partials + (size_t)my_slot * (32 * TC_BLOCK_N);
            // add the issuers' accumulators in fixed order into registers, hand the
            // accumulators back to the MMAs, then write Y (whole n-tile) or this CTA's partial
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
                        if (i < M) yp[(long long)i * N + n] = __float2bfloat16_rn(v[i] * (g * __ldg(rowfac + i)));
                }
            } else {
#pragma unroll
                for (int i = 0; i < NX; ++i)
                    if (i < M) mine[i * TC_BLOCK_N + r] = v[i];
            }
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
                            if (c0 + i < M)
                                yp[(long long)(c0 + i) * N + n] = __float2bfloat16_rn(w[i] * (g * __ldg(rowfac + c0 + i)));
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
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace tl
