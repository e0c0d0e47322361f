// gemm_bs.cuh -- block-scaled tensor-core NVFP4 verify GEMM for sm_100a (no CUDA-core dequant).
//
// Y[M,N] = X[M,K] . dequant(W)[N,K]^T for M <= 64 per launch (TandemLLM docs v0.12.0, "What
// TandemLLM is", section 1.2: the draft tree's rows, 1 to 32). W is already E2M1 with one E4M3
// scale per 16 k, which is what tcgen05.mma.kind::mxf4nvf4.block_scale consumes: the weight
// tile goes from HBM (TMA) into shared memory and from there straight into the tensor core,
// with no decode on the CUDA cores. X is brought into the same form beforehand (xsplit.cuh):
// per row a power of two and TC_PIECES FP4 pieces with E4M3 scales. The rows' pieces are
// stacked along the MMA's N dimension (row m's pieces adjacent; Mp = M rounded up to a multiple
// of 4, padding rows zero), so one MMA per 64-k chunk serves every X row and every piece:
//
//   D[n][4 m + p] = sum_k  w[n][k] * piece_p[m][k]        (fp32, in tensor memory; N = 4 Mp)
//   Y[m][n]       = bf16( (sum_p 4^-p D[n][4 m + p]) * g * factor[m] )
//
//   * Work. A tile is 128 weight rows x 256 k, or two such weight tiles (256 rows) that share
//     one copy of the X pieces (WT = 2, for 9 to 32 X rows); an n-tile is all k-tiles of its
//     weight rows. The host lays out each CTA's work as a list of segments (k-tiles [k0, k1)
//     of one n-tile), built from the matrices' shapes alone, in units of 256 weight rows:
//     - first, whole units dealt round-robin over the CTAs, so that at any moment the CTAs
//       work on neighbouring rows of one or two matrices and the X pieces they all read stay
//       in L2;
//     - then the remaining units as one list of k-tiles cut so that every CTA ends with the
//       same number of k-tiles (stream-K). A cut n-tile ("split") is reduced by its last
//       contributor, adding the parts in k order. With 128-row n-tiles a unit runs as its two
//       halves with the same cuts, so every output has one fixed reduction order that does
//       not depend on M.
//   * Roles, 12 warps.
//     - Warp 0: copies into a ring of stages, four (six with WT = 2) per tile from as many
//       lanes at once. Lanes 0 and 1 (4 and 5 for the second weight tile): a TMA tensor copy
//       each of the W codes and W scales. Lanes 2 and 3: one plain bulk copy each of the
//       tile's X piece codes (4 Mp rows of 128 B) and X piece scales (4 Mp rows of 16 B),
//       contiguous in the k-tile-major layout xsplit.cuh writes. Few, large copies: the copy
//       engine's cost per request, not the bytes, is what a per-row layout ran into.
//     - Warps 4..7: copy the tile's scales into tensor memory in the layout the MMA reads:
//       lane 32q + l, columns 4c .. 4c+3 hold the scale words (four 16-k blocks each) of rows
//       l, l + 32, l + 64, l + 96 for 64-k chunk c, for W and for the stacked X pieces.
//       A W scale byte with the sign bit set (the MMA's scales are unsigned) is handled
//       exactly: the codes of that block are negated in shared memory and the scale's sign is
//       cleared.
//     - Warp 1: one elected lane issues the MMAs of a tile (M = 128, N = 4 Mp, K = 64; four
//       per weight tile) into the segment's accumulator.
//     - Warps 8..11: the epilogue sums the pieces in fixed order and writes Y (or a partial).
//
// Every mbarrier wait is bounded; a wait that runs out records a status code and the CTA
// winds down.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "gemm_tc.cuh"
#include "xsplit.cuh"

namespace tl {

constexpr int BS_THREADS = 384;   // 12 warps
constexpr int BS_PART_ROWS = 64;  // X rows of one split-K partial slot ([64][128] fp32)

struct alignas(64) BsMat {
    CUtensorMap tm_codes;   // uint8 {K/2, N, 1}, box 128 B x 128 rows x 1, 128-byte swizzle
    CUtensorMap tm_scales;  // uint8 {K/16, N, 1}, box 16 B x 128 rows x 1
    const uint8_t* xc;      // X piece codes, [K/256][Mp][TC_PIECES][128] (swizzled lines, xsplit.cuh)
    const uint8_t* xs;      // X piece scales, [K/256][Mp][TC_PIECES][16]
    const float* xfactor;   // [M], 2^-e per X row (NaN for a non-finite row)
    __nv_bfloat16* y;
    float g;                // the weight's tensor scale
    int N;
};

// One stretch of a CTA's work: k-tiles [k0, k1) of n-tile `ntile` of matrix `mat`, in k order.
struct BsSeg {
    int mat;
    int ntile;
    uint16_t k0, k1;
    int split;              // -1: the whole n-tile; else the split's index (its four counters)
    int slot;               // split only: partial slot of this part; the split's parts use
                            // slots slot - rank .. slot - rank + parts - 1, in k order
    uint16_t rank, parts;
};

struct BsParams {
    const BsMat* mats;      // device table, or nullptr to use `one`
    int n_mats;
    int M;
    int Mp;                 // M rounded up to a multiple of 4: X rows per piece group in the layout
    const BsSeg* segs;      // every CTA's segments, CTA by CTA
    const int* seg_begin;   // [gridDim.x + 1]: CTA c runs segs[seg_begin[c] .. seg_begin[c+1])
    float* partials;        // [slots][64 x 128] fp32: [X row][128] or, with two weight tiles, [X row][256]
    unsigned* counters;     // [4 * splits] (one per 32-row quarter), zero between launches
    int* err;
    BsMat one;
};

// NX: the X rows a launch can hold (4, 8, 16, 24, 32 or 64; the smallest >= Mp is used). Fewer X
// rows leave room for more stages, and the ring's depth is what keeps enough weight bytes in
// flight. Above 32 rows the X lines are two MMA operands of up to 128 lines each (the MMA shape
// and scale layout used at every size), with one accumulator buffer.
// WT: weight tiles of 128 rows per stage (1 or 2, NX <= 32 for 2). With two, one X stage serves
// two MMAs (weight rows 0..127 and 128..255 of a 256-row n-tile), so the X pieces cost half the
// shared memory and half the L2 reads per weight byte, and more weight bytes fit in the ring.
template <int NX, int WT>
struct BsCfg {
    static constexpr int W_CODES = TC_BLOCK_N * (TC_BLOCK_K / 2);            // 16384 per weight tile
    static constexpr int W_SCALES = TC_BLOCK_N * (TC_BLOCK_K / 16);          // 2048 per weight tile
    static constexpr int CODES_BYTES = WT * W_CODES;
    static constexpr int XC_BYTES = TC_PIECES * NX * (TC_BLOCK_K / 2);       // 2048 .. 32768
    static constexpr int SCALES_BYTES = WT * W_SCALES;
    static constexpr int XS_BYTES = TC_PIECES * NX * (TC_BLOCK_K / 16);      // 256 .. 4096
    static constexpr int SC_OFF = CODES_BYTES;
    static constexpr int XC_OFF = SC_OFF + SCALES_BYTES;                     // 18432 or 36864: 1024-byte aligned
    static constexpr int XS_OFF = XC_OFF + XC_BYTES;                         // X codes and scales adjoin
    static constexpr int STAGE_BYTES = (XS_OFF + XS_BYTES + 1023) / 1024 * 1024;
    static constexpr int STAGES = (232448 - 1024 - 512) / STAGE_BYTES;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 512 /*barriers*/;
    static constexpr int N_MMA = TC_PIECES * NX;                             // X lines: 16 .. 256
    static constexpr int XH = (NX > 32) ? 2 : 1;                             // X operands per 64-k chunk (128 lines each)
    static constexpr int ACC_COLS = WT * N_MMA;                              // one accumulator: every weight tile's D
    static constexpr int SF_COLS = 16 * WT + 16 * XH;                        // scale columns per stage: W tiles, X halves
    static constexpr int ACC_BUFS = (2 * ACC_COLS + STAGES * SF_COLS <= TC_TMEM_COLS) ? 2 : 1;
    static constexpr int SF_COL0 = ACC_BUFS * ACC_COLS;                      // scale columns after the accumulators
    static constexpr int TILE_ROWS = WT * TC_BLOCK_N;                        // weight rows of an n-tile
    static constexpr int RG = (NX + 31) / 32;                                // epilogue row groups
    static constexpr int GR = (NX < 32) ? NX : 32;                           // rows per group
    // E2M1 x E2M1, UE4M3 scales, M = 128; N (bits 17..22, N / 8) is added at run time
    static constexpr uint32_t IDESC_BASE = (1u << 7) | (1u << 10) | (0u << 23) | ((uint32_t)(TC_BLOCK_N >> 4) << 24);
    static_assert(WT == 1 || (WT == 2 && NX <= 32), "two weight tiles per stage only with one X operand");
    static_assert(STAGE_BYTES % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
    static_assert(XC_OFF % 1024 == 0, "X piece codes must start on a swizzle atom");
    static_assert(SF_COL0 + STAGES * SF_COLS <= TC_TMEM_COLS, "tensor memory budget");
    static_assert(NX * WT <= BS_PART_ROWS, "a partial slot holds 64 x 128 values");
    static_assert(STAGES <= 32, "stage masks are 32 bits");
    static_assert(NX % 4 == 0 && N_MMA % 16 == 0, "MMA N must be a multiple of 16");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr),
          "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::mxf4nvf4 with one UE4M3 scale per 16 k from tensor memory.
__device__ __forceinline__ void mma_bs_f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// y[i][n] = bf16((v[i] * g) * factor[i]) for i < M (`y` already points at column n). All
// factors are read before the first store, so the loads are not serialised behind stores.
template <int NX>
__device__ __forceinline__ void bs_store_rows(float (&v)[NX], int M, float g, const float* factor,
                                              __nv_bfloat16* y, int ldy) {
#pragma unroll
    for (int i = 0; i < NX; ++i)
        if (i < M) v[i] = (v[i] * g) * __ldg(factor + i);
#pragma unroll
    for (int i = 0; i < NX; ++i)
        if (i < M) y[(long long)i * ldy] = __float2bfloat16_rn(v[i]);
}

template <int NX, int WT>
__global__ void __launch_bounds__(BS_THREADS, 1)
gemm_bs_kernel(const __grid_constant__ BsParams p) {
    using C = BsCfg<NX, WT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
    uint64_t* full = bars;                          // [STAGES] all bytes of the stage landed
    uint64_t* sfready = full + C::STAGES;           // [STAGES] scales of the stage in tensor memory (4 warps)
    uint64_t* empty = sfready + C::STAGES;          // [STAGES] stage and its scale columns read by the MMAs
    uint64_t* accfull = empty + C::STAGES;          // [2] accumulator complete
    uint64_t* accempty = accfull + 2;               // [2] accumulator read (4 epilogue warps)
    uint64_t* drain = accempty + 2;                 // [1] every MMA finished
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const BsMat* mats = p.mats ? p.mats : &p.one;
    const int s_begin = __ldg(p.seg_begin + blockIdx.x), s_end = __ldg(p.seg_begin + blockIdx.x + 1);

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&sfready[i], 4);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < C::ACC_BUFS; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], 4); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TC_TMEM_COLS);
        tmem_relinquish();
    }
    // X rows past 4 Mp stay zero: the copies only ever write rows < 4 Mp
    for (int i = threadIdx.x; i < C::STAGES * (C::XC_BYTES + C::XS_BYTES) / 16; i += BS_THREADS) {
        const int st = i / ((C::XC_BYTES + C::XS_BYTES) / 16), o = 16 * (i % ((C::XC_BYTES + C::XS_BYTES) / 16));
        *reinterpret_cast<uint4*>(smem + st * C::STAGE_BYTES + C::XC_OFF + o) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // Lanes 0, 1 (and 4, 5 for a second weight tile) copy the W codes and W scales of weight
        // tile lane / 4, lanes 2 and 3 the X piece codes and X piece scales of a stage, all at
        // once; the whole warp waits for the stage.
        const bool w_lane = (lane < 2) || (WT == 2 && (lane == 4 || lane == 5));
        const bool x_lane = (lane == 2 || lane == 3);
        const int wt = lane >> 2;                               // weight tile of a W lane
        // L2 policies: X pieces evict-last (every CTA on the matrix reads them); weights evict-first
        // with one weight tile per stage, evict-normal with two, which in paired timings keeps
        // the X pieces from being re-read from DRAM with two tiles (3-4% less time there) while
        // costing about 1% with one
        const uint64_t pol = w_lane ? ((WT == 2) ? policy_evict_normal() : policy_evict_first()) : policy_evict_last();
        // lane 2: X piece codes (4 Mp rows x 128 B), lane 3: X piece scales (4 Mp rows x 16 B)
        const uint32_t xbytes = (uint32_t)(TC_PIECES * p.Mp) * ((lane == 2) ? 128u : 16u);
        const uint32_t dst_off = x_lane ? ((lane == 2) ? (uint32_t)C::XC_OFF : (uint32_t)C::XS_OFF)
                               : ((lane & 1) ? (uint32_t)(C::SC_OFF + C::W_SCALES * wt) : (uint32_t)(C::W_CODES * wt));
        const uint32_t stage_tx = (uint32_t)(C::CODES_BYTES + C::SCALES_BYTES) + (uint32_t)p.Mp * (TC_PIECES * (128 + 16));
        const uint32_t smem0 = smem_u32(smem);
        int s = 0;
        uint32_t ph = 0, issued = 0, last_ph = 0;
        bool ok = true;
        for (int si = s_begin; ok && si < s_end; ++si) {
            const BsSeg sg = p.segs[si];
            const BsMat& m = mats[sg.mat];
            const int ntile = sg.ntile, k0 = sg.k0, k1 = sg.k1;
            const void* tmap = (lane & 1) ? (const void*)&m.tm_scales : (const void*)&m.tm_codes;
            const int c1 = ntile * C::TILE_ROWS + TC_BLOCK_N * wt;   // rows past N read as zeros
            const uint8_t* xsrc = (lane == 2) ? m.xc : m.xs;    // k-tile 0; k-tile kt is xbytes further each
            for (int kt = k0; kt < k1; ++kt) {
                const bool got = tc_wait(&empty[s], ph ^ 1u, abort_flag);
                if (!__all_sync(0xFFFFFFFFu, got)) {
                    if (lane == 0) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_PRODUCER);
                    ok = false;
                    break;
                }
                if (lane == 0) mbar_arrive_expect_tx(&full[s], stage_tx);
                __syncwarp();
                const uint32_t dst = smem0 + (uint32_t)(s * C::STAGE_BYTES) + dst_off;
                if (w_lane)
                    tma_load_3d_s(dst, tmap, &full[s], (lane & 1) ? kt * (TC_BLOCK_K / 16) : kt * (TC_BLOCK_K / 2),
                                  c1, 0, pol);
                else if (x_lane)
                    bulk_load_s(dst, xsrc + (size_t)kt * xbytes, xbytes, &full[s], pol);
                issued |= 1u << s;
                last_ph = (last_ph & ~(1u << s)) | (ph << s);
                if (++s == C::STAGES) { s = 0; ph ^= 1u; }
            }
        }
        if (lane == 0) {
            for (int i = 0; i < C::STAGES; ++i)
                if ((issued >> i) & 1u)
                    if (!mbar_wait(&full[i], (last_ph >> i) & 1u, TL_WAIT_LIMIT))
                        tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DRAIN);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (whole warp, elected lane)
        const bool leader = elect_one();
        int s = 0, acc = 0;
        uint32_t ph = 0, accph = 0;
        const uint64_t desc_w0 = smem_desc_k_sw128(smem_u32(smem));
        const uint64_t desc_x0 = smem_desc_k_sw128(smem_u32(smem + C::XC_OFF));
        // X lines 0..127 and 128..4 Mp - 1 (above 32 rows) are two MMAs into accumulator columns
        // 0..127 and 128..
        const uint32_t lines = (uint32_t)(TC_PIECES * p.Mp);
        const uint32_t idesc = C::IDESC_BASE | ((lines < 128u ? lines : 128u) >> 3) << 17;
        const uint32_t idesc_hi = C::IDESC_BASE | ((lines > 128u ? lines - 128u : 16u) >> 3) << 17;
        bool ok = true;
        for (int si = s_begin; ok && si < s_end; ++si) {
            const BsSeg sg = p.segs[si];
            const int k0 = sg.k0, k1 = sg.k1;
            if (!__all_sync(0xFFFFFFFFu, tc_wait(&accempty[acc], accph ^ 1u, abort_flag))) {
                if (leader) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_MMA);
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem + (uint32_t)(C::ACC_COLS * acc);
            uint32_t first = 1;
            for (int kt = k0; kt < k1; ++kt) {
                if (!__all_sync(0xFFFFFFFFu, tc_wait(&full[s], ph, abort_flag) &&
                                                 tc_wait(&sfready[s], ph, abort_flag))) {
                    if (leader) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_MMA);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t sdesc = (uint64_t)((s * C::STAGE_BYTES) >> 4);
                const uint32_t sf = tmem + (uint32_t)(C::SF_COL0 + C::SF_COLS * s);
                if (leader) {
                    // scale columns of the stage: 16 per weight tile, then 16 per X operand
                    const uint32_t sfx = sf + 16u * WT;
#pragma unroll
                    for (int kc = 0; kc < 4; ++kc) {
#pragma unroll
                        for (int h = 0; h < WT; ++h)
                            mma_bs_f4(d_tmem + (uint32_t)(C::N_MMA * h),
                                      desc_w0 + sdesc + (uint64_t)((C::W_CODES * h) >> 4) + (uint64_t)(2 * kc),
                                      desc_x0 + sdesc + (uint64_t)(2 * kc), idesc, sf + 16u * h + 4u * kc,
                                      sfx + 4u * kc, (kc == 0) ? (first ^ 1u) : 1u);
                        if (C::XH > 1 && lines > 128u)
                            mma_bs_f4(d_tmem + 128u, desc_w0 + sdesc + (uint64_t)(2 * kc),
                                      desc_x0 + sdesc + (uint64_t)((128 * 128) >> 4) + (uint64_t)(2 * kc), idesc_hi,
                                      sf + 4u * kc, sfx + 16u + 4u * kc, (kc == 0) ? (first ^ 1u) : 1u);
                    }
                    mma_commit(&empty[s]);
                }
                __syncwarp();
                first = 0;
                if (++s == C::STAGES) { s = 0; ph ^= 1u; }
            }
            if (!ok) break;
            if (leader) mma_commit(&accfull[acc]);
            __syncwarp();
            if (++acc == C::ACC_BUFS) { acc = 0; accph ^= 1u; }
        }
        if (leader) mma_commit(drain);
        __syncwarp();
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(drain, 0, TL_WAIT_LIMIT)) && lane == 0)
            tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DRAIN);
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ scales into tensor memory
        const int q = warp & 3;                         // this warp's tensor-memory lane quarter
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
        long long ntiles = 0;
        for (int si = s_begin; si < s_end; ++si) ntiles += p.segs[si].k1 - p.segs[si].k0;
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (long long n = 0; ok && n < ntiles; ++n) {
            if (!__all_sync(0xFFFFFFFFu, tc_wait(&full[s], ph, abort_flag))) {
                if (lane == 0) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DEQUANT);
                ok = false;
                break;
            }
            uint8_t* st = smem + s * C::STAGE_BYTES;
            const uint32_t col = t_lane + (uint32_t)(C::SF_COL0 + C::SF_COLS * s);
#pragma unroll
            for (int h = 0; h < WT; ++h) {
                uint8_t* const wc = st + C::W_CODES * h;            // this weight tile's codes
                uint4 wa[4];
#pragma unroll
                for (int gq = 0; gq < 4; ++gq)
                    wa[gq] = *reinterpret_cast<const uint4*>(st + C::SC_OFF + C::W_SCALES * h + 16 * (lane + 32 * gq));
                // a scale byte with the sign bit set: negate that block's codes, keep |scale|
                uint32_t neg = 0;
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) neg |= (wa[gq].x | wa[gq].y | wa[gq].z | wa[gq].w) & 0x80808080u;
                if (__any_sync(0xFFFFFFFFu, neg != 0u)) {
                    if (q == 0) {
#pragma unroll
                        for (int gq = 0; gq < 4; ++gq) {
                            const int r = lane + 32 * gq;
                            const uint32_t w4[4] = {wa[gq].x, wa[gq].y, wa[gq].z, wa[gq].w};
#pragma unroll
                            for (int b = 0; b < 16; ++b) {
                                if ((w4[b >> 2] >> (8 * (b & 3) + 7)) & 1u) {
                                    // block b = bytes 8b .. 8b+7 of row r: 16-byte chunk b/2, half (b&1)
                                    uint2* c = reinterpret_cast<uint2*>(wc + r * 128 + ((((b >> 1) ^ (r & 7))) << 4) + 8 * (b & 1));
                                    const uint2 v = *c;
                                    *c = make_uint2(v.x ^ 0x88888888u, v.y ^ 0x88888888u);
                                }
                            }
                        }
                        fence_proxy_async_smem();
                    }
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq) {
                        wa[gq].x &= 0x7F7F7F7Fu; wa[gq].y &= 0x7F7F7F7Fu; wa[gq].z &= 0x7F7F7F7Fu; wa[gq].w &= 0x7F7F7F7Fu;
                    }
                }
                // column 4c + gq: scale word c (four 16-k blocks of chunk c) of row lane + 32 gq
                uint32_t ca[16];
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) {
                    ca[0 + gq] = wa[gq].x; ca[4 + gq] = wa[gq].y; ca[8 + gq] = wa[gq].z; ca[12 + gq] = wa[gq].w;
                }
                tmem_st16(col + 16u * h, ca);
            }
#pragma unroll
            for (int h = 0; h < C::XH; ++h) {
                uint32_t cb[16];
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) {
                    const int rx = 128 * h + lane + 32 * gq;   // X line
                    const uint4 wb = (rx < C::N_MMA) ? *reinterpret_cast<const uint4*>(st + C::XS_OFF + 16 * rx)
                                                     : make_uint4(0, 0, 0, 0);
                    cb[0 + gq] = wb.x; cb[4 + gq] = wb.y; cb[8 + gq] = wb.z; cb[12 + gq] = wb.w;
                }
                tmem_st16(col + 16u * WT + 16u * h, cb);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfready[s]);
            if (++s == C::STAGES) { s = 0; ph ^= 1u; }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
        const int M = p.M;
        int acc = 0;
        uint32_t accph = 0;
        for (int si = s_begin; si < s_end; ++si) {
            const BsSeg sg = p.segs[si];
            const BsMat& m = mats[sg.mat];
            // the matrix's fields in registers: stores to Y must not force them to be re-read
            __nv_bfloat16* const yp = m.y;
            const float gm = m.g;
            const float* const xf = m.xfactor;
            const int N = m.N;
            if (!tc_wait(&accfull[acc], accph, abort_flag)) {
                tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_EPILOGUE);
                break;
            }
            tc_fence_after();
            const uint32_t acc_col = (uint32_t)(C::ACC_COLS * acc);
            // split only: this part's slot, [X row][TILE_ROWS] fp32
            float* part = p.partials + (size_t)sg.slot * (BS_PART_ROWS * TC_BLOCK_N);
            // Rows in groups of up to 32 (registers); per group, every weight tile h (rows 128 h + r
            // of the n-tile, accumulator columns N_MMA h ..) is read first, summing the pieces in
            // order, v[m] = sum_p 4^-p D[4 m + p] (exact scalings), 16 columns holding rows
            // 4c .. 4c+3; the accumulator is handed back after the last group's reads, before
            // its stores.
#pragma unroll 1
            for (int g = 0; g < C::RG; ++g) {
                float v[WT][C::GR];
#pragma unroll
                for (int h = 0; h < WT; ++h) {
#pragma unroll
                    for (int c = 0; c < C::GR / 4; ++c) {
                        if (32 * g + 4 * c < M) {
                            uint32_t raw[16];
                            tmem_ld16(t_lane + acc_col + (uint32_t)(C::N_MMA * h + 16 * (8 * g + c)), raw);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                float a = __uint_as_float(raw[4 * j]);
                                a = fmaf(__uint_as_float(raw[4 * j + 1]), 0.25f, a);
                                a = fmaf(__uint_as_float(raw[4 * j + 2]), 0.0625f, a);
                                v[h][4 * c + j] = fmaf(__uint_as_float(raw[4 * j + 3]), 0.015625f, a);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j) v[h][4 * c + j] = 0.0f;
                        }
                    }
                }
                if (g == C::RG - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&accempty[acc]);
                    if (++acc == C::ACC_BUFS) { acc = 0; accph ^= 1u; }
                }
                const int mg = M - 32 * g;                      // rows of this group that exist
#pragma unroll
                for (int h = 0; h < WT; ++h) {
                    const int rt = TC_BLOCK_N * h + r;          // row within the n-tile
                    const int n = sg.ntile * C::TILE_ROWS + rt;
                    if (sg.split < 0) {
                        if (n < N && mg > 0)
                            bs_store_rows<C::GR>(v[h], mg, gm, xf + 32 * g, yp + (long long)(32 * g) * N + n, N);
                    } else {
#pragma unroll
                        for (int i = 0; i < C::GR; ++i)
                            if (i < mg) part[(32 * g + i) * C::TILE_ROWS + rt] = v[h][i];
                    }
                }
            }
            if (sg.split < 0) continue;
            // a split n-tile: the last part to arrive (per 32-row quarter of each weight tile) adds
            // all parts in k order and writes Y
            __threadfence();
            __syncwarp();
            unsigned old = 0;
            if (lane == 0) old = atomicAdd(&p.counters[4 * sg.split + q], 1u);
            old = __shfl_sync(0xFFFFFFFFu, old, 0);
            if (old == (unsigned)(sg.parts - 1)) {
                __threadfence();
                const float* part0 = p.partials + (size_t)(sg.slot - sg.rank) * (BS_PART_ROWS * TC_BLOCK_N);
#pragma unroll 1
                for (int h = 0; h < WT; ++h) {
                    const int rt = TC_BLOCK_N * h + r;
                    const int n = sg.ntile * C::TILE_ROWS + rt;
#pragma unroll 1
                    for (int g = 0; g < C::RG; ++g) {
                        const int mg = M - 32 * g;
                        float v[C::GR];
#pragma unroll
                        for (int i = 0; i < C::GR; ++i) v[i] = 0.0f;
                        for (int rk = 0; rk < sg.parts; ++rk) {
                            const float* pp = part0 + (size_t)rk * (BS_PART_ROWS * TC_BLOCK_N);
#pragma unroll
                            for (int i = 0; i < C::GR; ++i)
                                if (i < mg) v[i] += __ldcg(&pp[(32 * g + i) * C::TILE_ROWS + rt]);
                        }
                        if (n < N && mg > 0)
                            bs_store_rows<C::GR>(v, mg, gm, xf + 32 * g, yp + (long long)(32 * g) * N + n, N);
                    }
                }
                if (lane == 0) p.counters[4 * sg.split + q] = 0u;   // ready for the next launch
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
