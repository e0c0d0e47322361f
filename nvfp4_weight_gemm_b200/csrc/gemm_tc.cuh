// gemm_tc.cuh -- the exact bf16 tensor-core NVFP4 verify GEMM for sm_100a (TL_PATH_BF16_EXACT and
// the no-allocation entry point), and the structures every tensor-core path shares: the matrix
// descriptor (TcMat), the launch parameters (TcParams), the stream-K work list (TcSegIter,
// tc_range_start) and the bounded mbarrier wait (tc_wait). The default exact f16 path's GEMM
// is gemm_ex.cuh.
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
//   * Roles, 26 warps. Warp 0 streams codes and scales (TMA) into a ring of weight stages;
//     a stage is handed back as soon as the dequantisers hold its bytes in registers, so
//     nearly the whole ring is in flight from HBM. Warp 24 loads the X tile of each k-tile
//     into a separate, shorter ring (an L2 hit) that the MMAs release. Warps 4..19
//     dequantise: a thread owns one weight row and a 128-k half of a tile, reads its
//     codes/scales from shared memory, forms W' = e2m1 * e4m3 in bf16 (exact) and stores it
//     into tensor memory, the A operand. Warps 1..3 issue tcgen05.mma with A from tensor
//     memory, B = X tile (bf16, shared memory, 128-byte swizzle) and the fp32 accumulator in
//     tensor memory (M_mma = 128 weight rows, N_mma = 16 or 32 X rows).
//     The dequantisers form two sets of eight warps that take alternate tiles, so four
//     dequant warps share each scheduler and one set's waits overlap the other's decode. A single thread keeps
//     only about one tcgen05.mma in flight per ~90 cycles at these small N, so warps 1..3
//     and 25 each issue a quarter of every tile's 16 k-steps into their own accumulator.
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
#include <cuda_fp16.h>
#include "ptx.cuh"
#include "nvfp4_format.cuh"

#ifndef TL_WAIT_LIMIT
#define TL_WAIT_LIMIT (1u << 22)
#endif

namespace tl {

constexpr int TC_BLOCK_N = 128;        // weight rows per tile (MMA M)
constexpr int TC_BLOCK_K = 256;        // k per tile / pipeline stage
constexpr int TC_THREADS = 832;     // 26 warps: weight producer, 4 MMA issuers, 16 dequantisers, 4 epilogue, X producer
constexpr int TC_XWARP = 24;
constexpr int TC_TMEM_COLS = 512;
// MMA issuers. One thread can only keep about one tcgen05.mma in flight per ~90 cycles,
// whatever N is, so four issuer warps (1, 2, 3 and 25) share each tile's 16 k-steps, four
// each; issuer j accumulates into its own accumulator j and the epilogue adds them in order.
constexpr int TC_NISSUE = 4;
__host__ __device__ constexpr int tc_ks_begin(int j) { return 4 * j; }
__host__ __device__ constexpr int tc_issuer_of_warp(int w) { return (w >= 1 && w <= 3) ? w - 1 : (w == 25 ? 3 : -1); }

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
    // the exact f16 path only (gemm_ex.cuh, xprep.cuh; tm_x then maps xh, the prepared copy of X)
    const __nv_bfloat16* x; // X as given, bf16 [M][K]
    __half* xh;             // X row m times 2^-e_m in f16, [M][K]
    float* rowfac;          // 2^e_m per row; that path's epilogue multiplies by global_scale * 2^e_m
    unsigned* rowmask;      // bit m set: row m is not exact in f16 (recomputed by the fallback)
    const uint8_t* codes;   // the weights as given (fallback rows)
    const uint8_t* scales;
    float g;                // global_scale
    int K;
};

struct TcParams {
    const TcMat* mats;      // device table, or nullptr to use `one`
    int n_mats;
    int M;
    long long total_tiles;
    float* partials;        // [2 * gridDim.x][32][128] fp32
    unsigned* counters;     // [4 * gridDim.x], zero between launches
    int* err;               // device status word
    uint32_t spread_mul;    // 0x1040, passed at run time so the decode multiply stays one IMAD
    uint32_t scale_mul;     // 0x00100010 (byte << 4 into both bf16 halves), likewise
    TcMat one;
};

template <int NX>
struct TcCfg {
    static constexpr int CODES_BYTES = TC_BLOCK_N * (TC_BLOCK_K / 2);   // 16384
    static constexpr int X_SUB = NX * 128;                              // one 64-k slice of X
    static constexpr int X_BYTES = 4 * X_SUB;
    static constexpr int SCALES_BYTES = TC_BLOCK_N * (TC_BLOCK_K / 16); // 2048
    // Two rings. Weight stages (codes + scales, read once from HBM) are released as soon as
    // the dequantisers have loaded them, so almost the whole weight ring is in flight; X
    // stages (an L2 hit) are released by the MMAs.
    static constexpr int W_STAGE_BYTES = CODES_BYTES + SCALES_BYTES;   // 18432
    static constexpr int W_STAGES = (NX == 32) ? 9 : 11;
    static constexpr int X_RING = W_STAGES * W_STAGE_BYTES;            // offset of the X ring
    static constexpr int NUM_A = 3;                                    // tile slots: A buffer + X stage
    static constexpr int SMEM_BYTES = X_RING + NUM_A * X_BYTES + 1024 /*align*/ + 512 /*barriers*/;
    static constexpr uint32_t IDESC = idesc_f16(1u, 128u, (uint32_t)NX);
    // tensor memory: three A buffers (128 columns each) so a tile set never waits for the
    // MMAs of its own previous tile, then ACC_BUFS accumulator buffers of TC_NISSUE
    // accumulators of NX fp32 columns each (one buffer at NX = 32: the MMAs then wait for
    // the epilogue once per n-tile segment, which is cheaper than a third-short A ring)
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

// Bounded wait that also gives up when another role has aborted the CTA.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 0; i < TL_WAIT_LIMIT; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
    }
    return false;
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

// Scale bytes -> bf16x2 words, both halves e4m3(s) * 2^119 (exact).
//
// Fast path, for finite, positive, normal scales (every scale the quantiser writes except
// all-zero blocks): the bf16 bits of s * 2^119 are (s << 4) + (239 << 7), which one IMAD forms
// in both halves at once from the byte (s << 4 | s << 20) + 0x77807780. A tile's eight bytes are
// checked once; anything else (zero or subnormal scale, sign bit, NaN) takes the exact float
// route for the whole tile.
__device__ __forceinline__ bool scales_fast_ok(uint2 sc) {
    const uint32_t e0 = sc.x & 0x78787878u, e1 = sc.y & 0x78787878u;
    const uint32_t zero_exp = ((e0 - 0x01010101u) & ~e0) | ((e1 - 0x01010101u) & ~e1);   // a byte had e == 0
    const uint32_t nan_or_neg = ((sc.x | sc.y) & 0x80808080u) |
                                (((sc.x & 0x7F7F7F7Fu) + 0x01010101u) & 0x80808080u) |
                                (((sc.y & 0x7F7F7F7Fu) + 0x01010101u) & 0x80808080u);   // bit 7 set or byte 0x7F
    return ((zero_exp & 0x80808080u) | nan_or_neg) == 0u;
}

// Four scale bytes of `sc` (fast path only; see scales_fast_ok).
__device__ __forceinline__ void scales4_fast(uint32_t sc, uint32_t mul, uint32_t (&S)[4]) {
#pragma unroll
    for (int p = 0; p < 4; ++p) S[p] = prmt(sc, 0u, 0x4440u | (uint32_t)p) * mul + 0x77807780u;
}

// Four scale bytes of `sc`, exactly, for any byte value.
__device__ __forceinline__ void scales4_exact(uint32_t sc, uint32_t (&S)[4]) {
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        const __half2 h = e4m3x2_to_half2((sc >> (16 * p)) & 0xFFFFu);
        const float f0 = __low2float(h) * 0x1p119f;
        const float f1 = __high2float(h) * 0x1p119f;
        S[2 * p] = prmt(__float_as_uint(f0), 0u, 0x3232u);
        S[2 * p + 1] = prmt(__float_as_uint(f1), 0u, 0x3232u);
    }
}

// Four code bytes (eight weights, k order) -> four bf16x2 words W' * 2^-7 in k order.
// `spread` is 0x1040 (x * 2^6 + x * 2^12); it arrives as a kernel argument so that the
// compiler keeps the multiply as one IMAD (FMA pipe) instead of shifts on the integer pipe,
// which the prmt/lop3 steps already keep busy.
__device__ __forceinline__ void decode8(uint32_t q, uint32_t S, uint32_t spread, uint32_t* out) {
    const uint32_t L = q & 0x0F0F0F0Fu;          // even-k nibbles, one per byte
    const uint32_t H = (q >> 4) & 0x0F0F0F0Fu;   // odd-k nibbles
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        // [L.byte i, 0, H.byte i, 0]; selector 8 replicates the (zero) sign of L.byte 0
        const uint32_t t = prmt(L, H, (uint32_t)i | 0x80u | ((uint32_t)(4 + i) << 8) | 0x8000u);
        const uint32_t w = (t * spread) & 0x81C081C0u;   // e1e0m -> bits 6..8, sign -> bit 15
        out[i] = hmul2_bf16(w, S);
    }
}

// MMA issuer J (a whole warp, converged; one elected lane issues): k-steps
// [tc_ks_begin(J), tc_ks_begin(J + 1)) of every tile into accumulator J. A tile slot (A buffer +
// X stage) is ready when the 8 warps of its tile set have arrived and its X bytes have landed;
// the slot is handed back by one commit per issuer.
template <int NX, int J>
__device__ __forceinline__ void tc_mma_issuer(const TcParams& p, const TcMat* mats, long long t_begin, long long t_end,
                                              uint8_t* smem, uint32_t tmem, uint64_t* ready, uint64_t* tfree,
                                              uint64_t* accfull, uint64_t* accempty, uint64_t* drain,
                                              volatile int* abort_flag) {
    using C = TcCfg<NX>;
    constexpr int I0 = tc_ks_begin(J), I1 = tc_ks_begin(J + 1);
    const bool leader = elect_one();   // issues every MMA and commit of this issuer
    int a = 0, acc = 0;
    uint32_t aph = 0, accph = 0;
    // descriptor of slot 0's X stage; the start-address field (bits 0..13, address >> 4)
    // advances by plain addition, which never carries out of the field for shared addresses
    const uint64_t bdesc_base = smem_desc_k_sw128(smem_u32(smem + C::X_RING));
    TcSegIter it(mats, p.n_mats, t_begin, t_end);
    TcSeg sg;
    bool ok = true;
    while (ok && it.next(sg)) {
        if (!__all_sync(0xFFFFFFFFu, tc_wait(&accempty[acc], accph ^ 1u, abort_flag))) {
            if (leader) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_MMA);
            break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(C::ACC_COL0 + C::ACC_BUF_COLS * acc + NX * J);
        uint32_t first = 1;   // the first MMA of a segment overwrites the accumulator
        for (int kt = sg.k0; kt < sg.k1; ++kt) {
            if (!__all_sync(0xFFFFFFFFu, tc_wait(&ready[a], aph, abort_flag))) {
                if (leader) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_MMA);
                ok = false;
                break;
            }
            tc_fence_after();
            const uint64_t bdesc0 = bdesc_base + (uint64_t)((a * C::X_BYTES) >> 4);
            const uint32_t a_tmem = tmem + (uint32_t)(128 * a + 8 * I0);
            if (leader) {
#pragma unroll
                for (int i = I0; i < I1; ++i)
                    mma_ts_f16(d_tmem, a_tmem + 8u * (i - I0),
                               bdesc0 + (uint64_t)((((i >> 2) * C::X_SUB + (i & 3) * 32)) >> 4), C::IDESC,
                               (i == I0) ? (first ^ 1u) : 1u);
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
}

template <int NX>
__global__ void __launch_bounds__(TC_THREADS, 1)
gemm_tc_kernel(const __grid_constant__ TcParams p) {
    using C = TcCfg<NX>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::X_RING + C::NUM_A * C::X_BYTES);
    uint64_t* wfull = bars;                         // [W_STAGES] codes + scales landed
    uint64_t* wempty = wfull + C::W_STAGES;         // [W_STAGES] loaded by the 8 warps of a tile set
    uint64_t* ready = wempty + C::W_STAGES;         // [NUM_A] tile slot filled: 8 warps of a tile set + X bytes
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
        for (int i = 0; i < C::W_STAGES; ++i) { mbar_init(&wfull[i], 1); mbar_init(&wempty[i], 8); }
        for (int i = 0; i < C::NUM_A; ++i) { mbar_init(&ready[i], 9); mbar_init(&tfree[i], TC_NISSUE); }
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
    } else if (warp == TC_XWARP) {
        // ------------------------------------------------------------ X producer
        // The X tile of tile n goes into the X stage of tile slot n % NUM_A; its arrival is
        // the ninth arrival (plus the bytes) on the slot's ready barrier. The warp runs the
        // loop converged; one elected lane issues.
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
        // the slot of every issued copy completes before the CTA leaves (at once on the
        // normal path, where the MMAs consumed it; bounded on an error path)
        if (leader) {
            for (int i = 0; i < C::NUM_A; ++i)
                if ((issued >> i) & 1u)
                    if (!mbar_wait(&ready[i], (last_ph >> i) & 1u, TL_WAIT_LIMIT))
                        tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DRAIN);
        }
    } else if (tc_issuer_of_warp(warp) >= 0) {
        // ------------------------------------------------------------ MMA issuers
        const int j = tc_issuer_of_warp(warp);
        if (j == 0)
            tc_mma_issuer<NX, 0>(p, mats, t_begin, t_end, smem, tmem, ready, tfree, accfull, accempty, drain, abort_flag);
        else if (j == 1)
            tc_mma_issuer<NX, 1>(p, mats, t_begin, t_end, smem, tmem, ready, tfree, accfull, accempty, drain, abort_flag);
        else if (j == 2)
            tc_mma_issuer<NX, 2>(p, mats, t_begin, t_end, smem, tmem, ready, tfree, accfull, accempty, drain, abort_flag);
        else
            tc_mma_issuer<NX, 3>(p, mats, t_begin, t_end, smem, tmem, ready, tfree, accfull, accempty, drain, abort_flag);
        if (warp == 1 && !__all_sync(0xFFFFFFFFu, mbar_wait(drain, 0, TL_WAIT_LIMIT)) && lane == 0)
            tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DRAIN);
    } else if (warp >= 4 && warp < 20) {
        // ------------------------------------------------------------ dequantisers
        // 16 warps = 2 tile sets x 2 k-halves x 4 lane quarters. Set t takes the tiles with
        // parity t, so one set's barrier and load latencies overlap the other set's decode.
        // Within a tile the warp of k-half h and lane quarter q decodes rows 32q..32q+31,
        // k in [128h, 128h + 128) (64 code bytes and 8 scales per thread) in two chunks of
        // 64 k, stored into
        // tensor-memory columns [64h, 64h + 64) of the tile's slot. Barrier tests for the next
        // tile and for this tile's slot are issued before the decode.
        // Wait outcomes are warp-uniform.
        const int dq = warp - 4;
        const int set = dq >> 3;
        const int kh = (dq >> 2) & 1;
        const int q = warp & 3;                  // tensor-memory lane quarter
        const int r = 32 * q + lane;             // weight row within the tile
        const uint32_t t_lane = tmem + ((uint32_t)(32 * q) << 16);
        const int row_off = r * 128, row_sw = r & 7;   // chunk j of row r sits at row_off + ((j ^ row_sw) << 4)
        const uint32_t sc_off = (uint32_t)(C::CODES_BYTES + r * 16 + 8 * kh);
        uint32_t cw_off[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) cw_off[j] = (uint32_t)(row_off + (((4 * kh + j) ^ row_sw) << 4));
        const int ntiles = (int)(t_end - t_begin);   // a CTA's share is far below 2^31 tiles
        const uint32_t spread = p.spread_mul;
        const uint32_t smul = p.scale_mul;
        // this set's tiles are n = set, set + 2, ...: stage n % W_STAGES, slot n % NUM_A
        int s = set, a = set;
        uint32_t ph = 0, aph = 0;
        auto advance2 = [](int& idx, uint32_t& phase, int ring) {
            idx += 2;
            if (idx >= ring) { idx -= ring; phase ^= 1u; }
        };
        // registers hold the scales and first-chunk codes of the current tile; the second
        // chunk's codes are read after the first chunk is stored, then the stage goes back
        uint2 sc = make_uint2(0, 0);
        uint4 cw0 = make_uint4(0, 0, 0, 0), cw1 = cw0;
        const uint8_t* st_cur = smem;
        bool ok = true;
        if (set < ntiles) {
            ok = __all_sync(0xFFFFFFFFu, tc_wait(&wfull[s], ph, abort_flag));
            if (ok) {
                st_cur = smem + s * C::W_STAGE_BYTES;
                sc = *reinterpret_cast<const uint2*>(st_cur + sc_off);
                cw0 = *reinterpret_cast<const uint4*>(st_cur + cw_off[0]);
                cw1 = *reinterpret_cast<const uint4*>(st_cur + cw_off[1]);
            } else if (lane == 0) {
                tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DEQUANT);
            }
        }
        int s_cur = s;
        advance2(s, ph, C::W_STAGES);
        for (int n = set; ok && n < ntiles; n += 2) {
            const bool has_next = n + 2 < ntiles;
            // the next tile's stage, and this tile's slot (read by the MMAs of tile n - NUM_A):
            // one vote when both are ready, the usual case; each is waited for on its own otherwise
            const bool both_ready = __all_sync(0xFFFFFFFFu, (!has_next || mbar_test(&wfull[s], ph)) &&
                                                             mbar_test(&tfree[a], aph ^ 1u));
            const bool fast = scales_fast_ok(sc);
            uint32_t S[4];
            if (fast) scales4_fast(sc.x, smul, S); else scales4_exact(sc.x, S);
            uint32_t out[32];
            decode8(cw0.x, S[0], spread, &out[0]);
            decode8(cw0.y, S[0], spread, &out[4]);
            decode8(cw0.z, S[1], spread, &out[8]);
            decode8(cw0.w, S[1], spread, &out[12]);
            decode8(cw1.x, S[2], spread, &out[16]);
            decode8(cw1.y, S[2], spread, &out[20]);
            decode8(cw1.z, S[3], spread, &out[24]);
            decode8(cw1.w, S[3], spread, &out[28]);
            // second chunk's codes: in flight while the first chunk is stored
            cw0 = *reinterpret_cast<const uint4*>(st_cur + cw_off[2]);
            cw1 = *reinterpret_cast<const uint4*>(st_cur + cw_off[3]);
            if (!both_ready && !__all_sync(0xFFFFFFFFu, tc_wait(&tfree[a], aph ^ 1u, abort_flag))) {
                if (lane == 0) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DEQUANT);
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t col = t_lane + (uint32_t)(128 * a + 64 * kh);
            tmem_st32(col, out);
            __syncwarp();
            if (lane == 0) mbar_arrive(&wempty[s_cur]);   // every byte of the stage this warp needs is in registers
            if (fast) scales4_fast(sc.y, smul, S); else scales4_exact(sc.y, S);
            decode8(cw0.x, S[0], spread, &out[0]);
            decode8(cw0.y, S[0], spread, &out[4]);
            decode8(cw0.z, S[1], spread, &out[8]);
            decode8(cw0.w, S[1], spread, &out[12]);
            decode8(cw1.x, S[2], spread, &out[16]);
            decode8(cw1.y, S[2], spread, &out[20]);
            decode8(cw1.z, S[3], spread, &out[24]);
            decode8(cw1.w, S[3], spread, &out[28]);
            tmem_st32(col + 32u, out);
            // the next tile's scales and first-chunk codes: in flight while the stores complete
            if (has_next) {
                if (!both_ready && !__all_sync(0xFFFFFFFFu, tc_wait(&wfull[s], ph, abort_flag))) {
                    if (lane == 0) tc_fail(p.err, abort_flag, TL_DEV_ERR_TIMEOUT_DEQUANT);
                    ok = false;
                    break;
                }
                st_cur = smem + s * C::W_STAGE_BYTES;
                s_cur = s;
                sc = *reinterpret_cast<const uint2*>(st_cur + sc_off);
                cw0 = *reinterpret_cast<const uint4*>(st_cur + cw_off[0]);
                cw1 = *reinterpret_cast<const uint4*>(st_cur + cw_off[1]);
                advance2(s, ph, C::W_STAGES);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ready[a]);   // the slot goes to the MMAs
            advance2(a, aph, C::NUM_A);
        }
        tmem_wait_st();   // no store of this warp may be in flight when tensor memory is released
    } else if (warp >= 20 && warp < 24) {
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
            const float g_out = m.g_out;
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
            for (int j = 0; j < TC_NISSUE; ++j) {
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
                        if (i < M) yp[(long long)i * N + n] = __float2bfloat16_rn(v[i] * g_out);
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
                            if (c0 + i < M) yp[(long long)(c0 + i) * N + n] = __float2bfloat16_rn(v[i] * g_out);
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
