// tl_nvfp4_api.cu -- the C ABI of libtl_nvfp4.so (declared in include/tl_nvfp4.h).
//
// Host side of the NVFP4 verify GEMM: argument validation, per-device state (split-K
// workspace, device status word), TMA descriptor construction, the stack descriptor
// cache, and the kernel launches. No allocation happens on the GEMM path after the
// per-device state and a stack's descriptor table exist.
#include "tl_nvfp4.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <queue>
#include <vector>

#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "gemm_ex.cuh"
#include "gdn_commit.cuh"
#include "gemm_head.cuh"
#include "xprep.cuh"
#include "gemm_bs.cuh"
#include "kernels_aux.cuh"

namespace {

thread_local char g_msg[512] = "no error";

tl_status fail(tl_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
tl_status fail(tl_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

#define TL_CUDA(call)                                                                       \
    do {                                                                                    \
        cudaError_t e_ = (call);                                                            \
        if (e_ != cudaSuccess)                                                              \
            return fail(TL_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));        \
    } while (0)

constexpr int kMaxDevices = 64;

// Split-K counters of one device: four per split n-tile (one per 32-row quarter), at most
// 2 * SMs splits (the block-scaled schedule's bound, checked in build_bs; the exact kernel
// uses 4 per CTA). Allocated, and cleared after a device-side timeout, in full.
constexpr int kSplitsPerSm = 2, kCountersPerSplit = 4;
size_t counter_words(int sms) { return (size_t)kCountersPerSplit * kSplitsPerSm * sms; }
constexpr int kStackCacheSlots = 8;

// One slot of the descriptor-table cache. A slot's device buffer only grows (to the largest
// table it has held); refilling it is an asynchronous copy from the slot's pinned staging
// buffer on the caller's stream, so after the slots have grown no call allocates or
// synchronises the device.
struct StackCacheEntry {
    std::vector<unsigned char> key;   // host bytes of the table the slot holds
    void* table = nullptr;            // device copy
    void* staging = nullptr;          // pinned host copy the refill reads
    size_t cap = 0;                   // bytes of `table` and `staging`
    cudaEvent_t copied = nullptr;     // recorded after the last refill copy
    unsigned long long last_use = 0;
};

struct DevState {
    bool ready = false;
    int num_sms = 0;
    int* err = nullptr;            // device status word
    float* partials = nullptr;     // [4 * num_sms][64][128]
    unsigned* counters = nullptr;  // [8 * num_sms]: four per split, up to 2 * num_sms splits
    unsigned* qscratch = nullptr;  // quantiser absmax + non-finite flag
    bool smem_attr_set = false;
    unsigned char* xs_buf = nullptr;   // X pieces of the block-scaled path (calls without a plan)
    size_t xs_cap = 0;
    unsigned char* xh_buf = nullptr;   // prepared X of the exact path (calls without a plan)
    size_t xh_cap = 0;
    StackCacheEntry cache[kStackCacheSlots];
    unsigned long long use_clock = 0;
};

std::mutex g_mu;
DevState g_dev[kMaxDevices];
int g_path = TL_PATH_EXACT;   // which tensor-core path the GEMM entry points take

// The path setting, read once per call or plan (never while g_mu is held).
int current_path() {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_path;
}
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

tl_status load_encode_fn() {
    if (g_encode) return TL_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
        return fail(TL_ERR_CUDA, "cuTensorMapEncodeTiled unavailable from the driver");
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return TL_OK;
}

// Create the state of `device` (caller holds g_mu). Switches device only temporarily.
tl_status init_locked(int device) {
    if (device < 0 || device >= kMaxDevices) return fail(TL_ERR_INVALID_VALUE, "device %d out of range", device);
    DevState& d = g_dev[device];
    if (d.ready) return TL_OK;
    int prev = 0;
    TL_CUDA(cudaGetDevice(&prev));
    if (prev != device) TL_CUDA(cudaSetDevice(device));
    tl_status st = TL_OK;
    do {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
            st = fail(TL_ERR_CUDA, "cannot query device %d", device);
            break;
        }
        if (major != 10 || minor != 0) {
            st = fail(TL_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", device,
                      major, minor);
            break;
        }
        d.num_sms = sms;
        const size_t pbytes = (size_t)4 * sms * tl::BS_PART_ROWS * tl::TC_BLOCK_N * sizeof(float);
        if (cudaMalloc(&d.err, 64) != cudaSuccess || cudaMalloc(&d.partials, pbytes) != cudaSuccess ||
            cudaMalloc(&d.counters, counter_words(sms) * sizeof(unsigned)) != cudaSuccess ||
            cudaMalloc(&d.qscratch, 64) != cudaSuccess) {
            st = fail(TL_ERR_CUDA, "cudaMalloc of the per-device state failed");
            break;
        }
        if (cudaMemset(d.err, 0, 64) != cudaSuccess ||
            cudaMemset(d.counters, 0, counter_words(sms) * sizeof(unsigned)) != cudaSuccess ||
            cudaDeviceSynchronize() != cudaSuccess) {
            st = fail(TL_ERR_CUDA, "initialising the per-device state failed");
            break;
        }
        d.ready = true;
    } while (0);
    if (prev != device) cudaSetDevice(prev);
    return st;
}

tl_status current_state(DevState** out) {
    int dev = 0;
    TL_CUDA(cudaGetDevice(&dev));
    std::lock_guard<std::mutex> lk(g_mu);
    tl_status st = init_locked(dev);
    if (st != TL_OK) return st;
    st = load_encode_fn();
    if (st != TL_OK) return st;
    *out = &g_dev[dev];
    return TL_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// Shared checks of one matrix (M already checked).
tl_status check_matrix(const void* x, int M, const void* codes, const void* scales, float g, const void* y, int N,
                       int K, bool check_xy) {
    if (N < 1) return fail(TL_ERR_INVALID_VALUE, "N = %d must be >= 1", N);
    if (K <= 0 || K % TL_NVFP4_K_ALIGN != 0)
        return fail(TL_ERR_INVALID_VALUE, "K = %d must be a positive multiple of %d", K, TL_NVFP4_K_ALIGN);
    if (!codes || !scales) return fail(TL_ERR_INVALID_VALUE, "null weight pointer");
    if (!std::isfinite(g)) return fail(TL_ERR_INVALID_VALUE, "global_scale is not finite");
    if (!aligned16(codes) || !aligned16(scales))
        return fail(TL_ERR_MISALIGNED, "weight pointers must be 16-byte aligned");
    if (check_xy) {
        if (!x || !y) return fail(TL_ERR_INVALID_VALUE, "null x or y pointer");
        if (!aligned16(x) || !aligned16(y)) return fail(TL_ERR_MISALIGNED, "x and y must be 16-byte aligned");
        const size_t ybytes = (size_t)M * N * 2;
        if (overlap(y, ybytes, x, (size_t)M * K * 2) || overlap(y, ybytes, codes, (size_t)N * K / 2) ||
            overlap(y, ybytes, scales, (size_t)N * K / 16))
            return fail(TL_ERR_INVALID_VALUE, "y overlaps x or the weights");
    }
    return TL_OK;
}

// Rank-3 tiled tensor map (dims innermost first; strides in bytes for dims 1 and 2).
tl_status encode_3d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, const cuuint64_t (&dims)[3],
                    const cuuint64_t (&strides)[2], const cuuint32_t (&box)[3], CUtensorMapSwizzle sw,
                    const char* what) {
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(tm, dt, 3, const_cast<void*>(base), const_cast<cuuint64_t*>(dims),
                          const_cast<cuuint64_t*>(strides), const_cast<cuuint32_t*>(box), estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TL_ERR_CUDA, "cuTensorMapEncodeTiled (%s) failed (%d)", what, (int)r);
    return TL_OK;
}

// Scratch of the exact path for one matrix with M rows: the prepared X (f16 [M][K]), the row
// factors (float [M]) and the row mask (one word), each part 256-byte aligned.
size_t xh_bytes_of(int M, int K) {
    return (((size_t)2 * M * K + 255) & ~size_t(255)) + (((size_t)4 * M + 255) & ~size_t(255)) + 256;
}

// xh: the matrix's exact-path scratch (xh_bytes_of bytes) for the f16 operands, or nullptr for
// the bf16 decode (X used as given).
tl_status build_mat(tl::TcMat* m, const void* x, int M, int NX, const void* codes, const void* scales, float g,
                    void* y, int N, int K, long long tile_begin, unsigned char* xh = nullptr) {
    memset(m, 0, sizeof *m);
    // All three maps are rank 3 so that one converged load instruction can issue them.
    // Codes and scales: {bytes per row, N rows, 1}; a tile box is 128 rows of one k-tile.
    const cuuint64_t n = (cuuint64_t)N, k = (cuuint64_t)K;
    tl_status st = encode_3d(&m->tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, {k / 2, n, 1}, {k / 2, n * (k / 2)},
                             {tl::TC_BLOCK_K / 2, tl::TC_BLOCK_N, 1}, CU_TENSOR_MAP_SWIZZLE_128B, "codes");
    if (st != TL_OK) return st;
    st = encode_3d(&m->tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, scales, {k / 16, n, 1}, {k / 16, n * (k / 16)},
                   {tl::TC_BLOCK_K / 16, tl::TC_BLOCK_N, 1}, CU_TENSOR_MAP_SWIZZLE_NONE, "scales");
    if (st != TL_OK) return st;
    // X viewed as {64 elements, M rows, K/64 slices}: one box {64, NX, 4} lands the four 64-k
    // slices of a tile one after another in shared memory, each NX rows x 128 B, swizzled;
    // rows >= M read zero.
    if (xh) {
        m->x = static_cast<const __nv_bfloat16*>(x);
        m->xh = reinterpret_cast<__half*>(xh);
        m->rowfac = reinterpret_cast<float*>(xh + (((size_t)2 * M * K + 255) & ~size_t(255)));
        m->rowmask = reinterpret_cast<unsigned*>(reinterpret_cast<unsigned char*>(m->rowfac) +
                                                 (((size_t)4 * M + 255) & ~size_t(255)));
        m->codes = static_cast<const uint8_t*>(codes);
        m->scales = static_cast<const uint8_t*>(scales);
        m->g = g;
        m->K = K;
    }
    st = encode_3d(&m->tm_x, xh ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   xh ? static_cast<const void*>(xh) : x, {64, (cuuint64_t)M, k / 64}, {k * 2, 128},
                   {64, (cuuint32_t)NX, 4}, CU_TENSOR_MAP_SWIZZLE_128B, "X");
    if (st != TL_OK) return st;
    m->y = static_cast<__nv_bfloat16*>(y);
    m->g_out = (float)((double)g * 128.0);   // W' reaches the accumulator scaled by 2^-7
    m->N = N;
    m->k_tiles = K / tl::TC_BLOCK_K;
    m->n_tiles = (N + tl::TC_BLOCK_N - 1) / tl::TC_BLOCK_N;
    m->tile_begin = tile_begin;
    return TL_OK;
}

template <int NX>
tl_status launch_tc(DevState& d, tl::TcParams& p, cudaStream_t stream) {
    using C = tl::TcCfg<NX>;
    // the attribute is per function; set for both variants on first use (idempotent, cheap)
    TL_CUDA(cudaFuncSetAttribute(tl::gemm_tc_kernel<NX>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
    const long long grid = p.total_tiles < d.num_sms ? p.total_tiles : d.num_sms;
    p.partials = d.partials;
    p.counters = d.counters;
    p.err = d.err;
    p.spread_mul = 0x1040u;
    p.scale_mul = 0x00100010u;
    tl::gemm_tc_kernel<NX><<<(unsigned)grid, tl::TC_THREADS, C::SMEM_BYTES, stream>>>(p);
    TL_CUDA(cudaGetLastError());
    return TL_OK;
}

template <int NX>
tl_status launch_ex(DevState& d, tl::TcParams& p, cudaStream_t stream) {
    using C = tl::ExCfg<NX>;
    TL_CUDA(cudaFuncSetAttribute(tl::gemm_ex_kernel<NX>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
    const long long grid = p.total_tiles < d.num_sms ? p.total_tiles : d.num_sms;
    p.partials = d.partials;
    p.counters = d.counters;
    p.err = d.err;
    tl::gemm_ex_kernel<NX><<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, stream>>>(p);
    TL_CUDA(cudaGetLastError());
    return TL_OK;
}

// The exact paths. bf16 decode: one GEMM launch on X as given. f16 decode: the X preparation
// (one CTA per matrix and row), the GEMM on the prepared X, then the fallback for flagged rows (it
// returns at once when no row is flagged).
tl_status launch_tc_any(DevState& d, tl::TcParams& p, bool f16, cudaStream_t stream) {
    if (!f16) return (p.M <= 16) ? launch_tc<16>(d, p, stream) : launch_tc<32>(d, p, stream);
    tl::x_prep_kernel<<<dim3((unsigned)p.n_mats, (unsigned)p.M), tl::XP_THREADS, 0, stream>>>(p);
    TL_CUDA(cudaGetLastError());
    tl_status st = (p.M <= 16) ? launch_ex<16>(d, p, stream) : launch_ex<32>(d, p, stream);
    if (st != TL_OK) return st;
    tl::fallback_rows_kernel<<<(unsigned)d.num_sms, tl::FB_THREADS, 0, stream>>>(p);
    TL_CUDA(cudaGetLastError());
    return TL_OK;
}

// Rows one launch serves: the block-scaled GEMM 64, the exact and CUDA-core kernels 32. Calls with
// more rows (up to TL_NVFP4_MAX_M) run as groups of rows, each streaming the weights again.
constexpr int kBsMaxRows = 64;
constexpr int kExactMaxRows = 32;

tl_status check_M(int M, int limit = TL_NVFP4_MAX_M) {
    if (M < 0) return fail(TL_ERR_INVALID_VALUE, "M = %d is negative", M);
    if (M > limit) return fail(TL_ERR_UNSUPPORTED, "M = %d > %d rows is not served here", M, limit);
    return TL_OK;
}

// Device copy of a stack's descriptor table (host bytes `key`): reused while the same
// matrices come back. On a miss the least recently used slot is refilled with an asynchronous
// copy on `stream` from the slot's pinned staging buffer. The slot's previous table may still be
// read by a kernel queued earlier: calls of one device are serialised on one stream (see the
// header), so that kernel runs before the copy. The staging buffer is rewritten only after its
// previous copy has executed (its event). A slot allocates (device and pinned host memory, after
// synchronising the device) only when it must grow: once the slots have held the largest table
// the caller uses, a miss neither allocates nor synchronises the device.
tl_status device_table(DevState& d, const void* key_, size_t bytes, cudaStream_t stream, const void** out) {
    const unsigned char* key = static_cast<const unsigned char*>(key_);
    std::lock_guard<std::mutex> lk(g_mu);
    ++d.use_clock;
    for (auto& e : d.cache) {
        if (e.table && e.key.size() == bytes && memcmp(e.key.data(), key, bytes) == 0) {
            e.last_use = d.use_clock;
            *out = e.table;
            return TL_OK;
        }
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    TL_CUDA(cudaStreamIsCapturing(stream, &cs));
    if (cs != cudaStreamCaptureStatusNone)
        return fail(TL_ERR_UNSUPPORTED, "a new stack must be run once before it is captured into a graph");
    StackCacheEntry* victim = &d.cache[0];
    for (auto& e : d.cache)
        if (!e.table || e.last_use < victim->last_use) victim = &e;
    if (victim->cap < bytes) {
        if (victim->table) {
            TL_CUDA(cudaDeviceSynchronize());   // the old table may be read by a kernel in flight
            TL_CUDA(cudaFree(victim->table));
            TL_CUDA(cudaFreeHost(victim->staging));
            victim->table = nullptr;
            victim->staging = nullptr;
            victim->cap = 0;
            victim->key.clear();
        }
        if (!victim->copied) TL_CUDA(cudaEventCreateWithFlags(&victim->copied, cudaEventDisableTiming));
        const size_t cap = (bytes + 4095) & ~size_t(4095);
        TL_CUDA(cudaMalloc(&victim->table, cap));
        if (cudaMallocHost(&victim->staging, cap) != cudaSuccess) {
            cudaFree(victim->table);
            victim->table = nullptr;
            return fail(TL_ERR_CUDA, "cudaMallocHost of a descriptor staging buffer failed");
        }
        victim->cap = cap;
    } else {
        TL_CUDA(cudaEventSynchronize(victim->copied));   // its last refill copy has run
    }
    victim->key.clear();   // the slot holds no valid table until the copy is queued
    memcpy(victim->staging, key, bytes);
    TL_CUDA(cudaMemcpyAsync(victim->table, victim->staging, bytes, cudaMemcpyHostToDevice, stream));
    TL_CUDA(cudaEventRecord(victim->copied, stream));
    victim->key.assign(key, key + bytes);
    victim->last_use = d.use_clock;
    *out = victim->table;
    return TL_OK;
}

tl_status stack_table(DevState& d, const std::vector<tl::TcMat>& mats, cudaStream_t stream, const tl::TcMat** out) {
    const void* t = nullptr;
    tl_status st = device_table(d, mats.data(), mats.size() * sizeof(tl::TcMat), stream, &t);
    *out = static_cast<const tl::TcMat*>(t);
    return st;
}

// Validate a stack and build its launch parameters (host side only, plus the
// state lookup). `table_out` receives the TcMat array when n_mats > 1.
// path: the GEMM path the parameters are for (the caller's copy of the setting, so that one
// call or plan never mixes two paths).
size_t xh_bytes_total(const tl_nvfp4_matrix* mats, int n_mats, int M) {
    size_t t = 0;
    for (int i = 0; i < n_mats; ++i) t += xh_bytes_of(M, mats[i].K);
    return t;
}

tl_status ensure_xh(DevState& d, size_t bytes, cudaStream_t stream);

// xh: the exact path's scratch for the whole stack (xh_bytes_total bytes); nullptr means the
// per-device buffer (grown here if needed). Unused on the other paths.
tl_status build_params(const tl_nvfp4_matrix* mats, int n_mats, int M, const unsigned char* x_dev,
                       unsigned char* y_dev, int path, DevState** dstate, tl::TcParams* p,
                       std::vector<tl::TcMat>* table_out, unsigned char* xh = nullptr,
                       cudaStream_t stream = nullptr) {
    tl_status st = check_M(M, path == TL_PATH_BLOCK_SCALED ? kBsMaxRows : kExactMaxRows);
    if (st != TL_OK) return st;
    if (!mats) return fail(TL_ERR_INVALID_VALUE, "mats is null");
    if (n_mats < 1 || n_mats > TL_NVFP4_MAX_STACK)
        return fail(TL_ERR_INVALID_VALUE, "n_mats = %d outside [1, %d]", n_mats, TL_NVFP4_MAX_STACK);
    // validate every matrix on the host before any CUDA call
    size_t xoff = 0, yoff = 0;
    for (int i = 0; i < n_mats; ++i) {
        const tl_nvfp4_matrix& m = mats[i];
        const void* x = x_dev ? static_cast<const void*>(x_dev + xoff) : m.x;
        const void* y = y_dev ? static_cast<const void*>(y_dev + yoff) : m.y;
        st = check_matrix(x, M, m.w_codes, m.w_scales, m.global_scale, y, m.N, m.K, true);
        if (st != TL_OK) {
            char why[sizeof g_msg];
            memcpy(why, g_msg, sizeof why);
            return fail(st, "matrix %d: %s", i, why);
        }
        xoff += (size_t)2 * M * m.K;
        yoff += (size_t)2 * M * m.N;
    }
    if (M == 0) return TL_OK;
    st = current_state(dstate);
    if (st != TL_OK) return st;
    if (path == TL_PATH_BLOCK_SCALED) return TL_OK;     // the block-scaled launch builds its own tables
    const bool f16 = (path == TL_PATH_EXACT);
    if (f16 && !xh) {
        st = ensure_xh(**dstate, xh_bytes_total(mats, n_mats, M), stream);
        if (st != TL_OK) return st;
        xh = (*dstate)->xh_buf;
    }
    const int NX = M <= 16 ? 16 : 32;
    size_t hoff = 0;
    std::vector<tl::TcMat>& tbl = *table_out;
    tbl.assign(n_mats, tl::TcMat());
    long long tiles = 0;
    xoff = 0;
    yoff = 0;
    for (int i = 0; i < n_mats; ++i) {
        const tl_nvfp4_matrix& m = mats[i];
        const void* x = x_dev ? static_cast<const void*>(x_dev + xoff) : m.x;
        void* y = y_dev ? static_cast<void*>(y_dev + yoff) : m.y;
        st = build_mat(&tbl[i], x, M, NX, m.w_codes, m.w_scales, m.global_scale, y, m.N, m.K, tiles,
                       f16 ? xh + hoff : nullptr);
        if (st != TL_OK) return st;
        if (f16) hoff += xh_bytes_of(M, m.K);
        tiles += (long long)tbl[i].n_tiles * tbl[i].k_tiles;
        xoff += (size_t)2 * M * m.K;
        yoff += (size_t)2 * M * m.N;
    }
    memset(p, 0, sizeof *p);
    p->n_mats = n_mats;
    p->M = M;
    p->total_tiles = tiles;
    p->mats = nullptr;
    if (n_mats == 1) p->one = tbl[0];
    return TL_OK;
}

tl_status run_stack_bs(const tl_nvfp4_matrix* mats, int n_mats, int M, const unsigned char* x_dev,
                       unsigned char* y_dev, void* stream_, DevState* d);

tl_status run_stack_rows(const tl_nvfp4_matrix* mats, int n_mats, int M, const unsigned char* x_dev,
                         unsigned char* y_dev, void* stream_);

// A stack with more rows than one launch serves: validate it whole, then run it as groups of
// rows (rows r0 .. r0 + Mg - 1 of every X_i and Y_i), each group one launch.
tl_status run_stack(const tl_nvfp4_matrix* mats, int n_mats, int M, const unsigned char* x_dev,
                    unsigned char* y_dev, void* stream_) {
    const int lim = (current_path() == TL_PATH_BLOCK_SCALED) ? kBsMaxRows : kExactMaxRows;
    if (M <= lim) return run_stack_rows(mats, n_mats, M, x_dev, y_dev, stream_);
    tl_status st = check_M(M);
    if (st != TL_OK) return st;
    if (!mats) return fail(TL_ERR_INVALID_VALUE, "mats is null");
    if (n_mats < 1 || n_mats > TL_NVFP4_MAX_STACK)
        return fail(TL_ERR_INVALID_VALUE, "n_mats = %d outside [1, %d]", n_mats, TL_NVFP4_MAX_STACK);
    std::vector<tl_nvfp4_matrix> full(mats, mats + n_mats), grp(n_mats);
    size_t xoff = 0, yoff = 0;
    for (int i = 0; i < n_mats; ++i) {
        if (x_dev) full[i].x = x_dev + xoff;
        if (y_dev) full[i].y = y_dev + yoff;
        st = check_matrix(full[i].x, M, full[i].w_codes, full[i].w_scales, full[i].global_scale, full[i].y, full[i].N,
                          full[i].K, true);
        if (st != TL_OK) {
            char why[sizeof g_msg];
            memcpy(why, g_msg, sizeof why);
            return fail(st, "matrix %d: %s", i, why);
        }
        xoff += (size_t)2 * M * mats[i].K;
        yoff += (size_t)2 * M * mats[i].N;
    }
    for (int r0 = 0; r0 < M; r0 += lim) {
        const int mg = std::min(lim, M - r0);
        for (int i = 0; i < n_mats; ++i) {
            grp[i] = full[i];
            grp[i].x = static_cast<const unsigned char*>(full[i].x) + (size_t)2 * r0 * full[i].K;
            grp[i].y = static_cast<unsigned char*>(full[i].y) + (size_t)2 * r0 * full[i].N;
        }
        st = run_stack_rows(grp.data(), n_mats, mg, nullptr, nullptr, stream_);
        if (st != TL_OK) return st;
    }
    return TL_OK;
}

tl_status run_stack_rows(const tl_nvfp4_matrix* mats, int n_mats, int M, const unsigned char* x_dev,
                         unsigned char* y_dev, void* stream_) {
    DevState* d = nullptr;
    tl::TcParams p;
    std::vector<tl::TcMat> tbl;
    const int path = current_path();
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    tl_status st = build_params(mats, n_mats, M, x_dev, y_dev, path, &d, &p, &tbl, nullptr, stream);
    if (st != TL_OK || M == 0) return st;
    if (path == TL_PATH_BLOCK_SCALED) return run_stack_bs(mats, n_mats, M, x_dev, y_dev, stream_, d);
    if (n_mats > 1) {
        st = stack_table(*d, tbl, stream, &p.mats);
        if (st != TL_OK) return st;
    }
    return launch_tc_any(*d, p, path == TL_PATH_EXACT, stream);
}


// ---------------------------------------------------------------------------
// The block-scaled path: X split into FP4 pieces, then W and the pieces straight into the
// tensor core (gemm_bs.cuh, xsplit.cuh).

size_t round256(size_t v) { return (v + 255) & ~size_t(255); }

int round4(int M) { return (M + 3) & ~3; }

// Bytes of the X pieces (codes, scales, row factors) of one matrix with M rows and K columns;
// the pieces are laid out for Mp = M rounded up to a multiple of 4 rows.
size_t xs_bytes_of(int M, int K) {
    const size_t Mp = (size_t)round4(M);
    return round256((size_t)tl::TC_PIECES * Mp * (K / 2)) + round256((size_t)tl::TC_PIECES * Mp * (K / 16)) +
           round256((size_t)4 * M);
}

size_t xs_bytes_total(const tl_nvfp4_matrix* mats, int n_mats, int M) {
    size_t t = 0;
    for (int i = 0; i < n_mats; ++i) t += xs_bytes_of(M, mats[i].K);
    return t;
}

// BsMat of one matrix whose X pieces live at `xs` (layout of xs_bytes_of).
tl_status build_bs_mat(tl::BsMat* m, tl::XSplitMat* xm, const void* x, int M, const void* codes,
                       const void* scales, float g, void* y, int N, int K, unsigned char* xs) {
    memset(m, 0, sizeof *m);
    const cuuint64_t n = (cuuint64_t)N, k = (cuuint64_t)K, P = (cuuint64_t)tl::TC_PIECES, Mp = (cuuint64_t)round4(M);
    unsigned char* xc = xs;
    unsigned char* xsc = xc + round256((size_t)P * Mp * (K / 2));
    float* xf = reinterpret_cast<float*>(xsc + round256((size_t)P * Mp * (K / 16)));
    tl_status st = encode_3d(&m->tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, {k / 2, n, 1}, {k / 2, n * (k / 2)},
                             {tl::TC_BLOCK_K / 2, tl::TC_BLOCK_N, 1}, CU_TENSOR_MAP_SWIZZLE_128B, "codes");
    if (st != TL_OK) return st;
    st = encode_3d(&m->tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, scales, {k / 16, n, 1}, {k / 16, n * (k / 16)},
                   {tl::TC_BLOCK_K / 16, tl::TC_BLOCK_N, 1}, CU_TENSOR_MAP_SWIZZLE_NONE, "scales");
    if (st != TL_OK) return st;
    // X pieces: k-tile-major runs that the kernel fetches with plain bulk copies
    m->xc = xc;
    m->xs = xsc;
    m->xfactor = xf;
    m->y = static_cast<__nv_bfloat16*>(y);
    m->g = g;
    m->N = N;
    xm->x = static_cast<const __nv_bfloat16*>(x);
    xm->codes = xc;
    xm->scales = xsc;
    xm->factor = xf;
    xm->K = K;
    return TL_OK;
}

// Each CTA's list of segments (gemm_bs.cuh), built from the shapes and the grid alone. The
// work is cut in units of 256 weight rows (all k-tiles of them):
//   - whole units dealt in order, each to the CTA with the fewest k-tiles so far (round-robin
//     when the units are alike), so that the CTAs move through the matrices side by side and
//     share the X pieces in L2;
//   - the last two to three rounds' worth of units cut into equal shares of k-tiles (stream-K),
//     so every CTA ends with the same number of k-tiles; a cut unit ("split") is summed over
//     its parts in k order.
// A launch with 128-row n-tiles runs a unit as its two halves, one after the other, with the
// same k ranges (each half its own split); a launch with 256-row n-tiles runs it as one. Either
// way every weight row gets the same cuts in k and the same order of summation, so an output
// does not depend on M (nor on the launch the size of M selects).
struct BsSchedule {
    std::vector<tl::BsSeg> segs;
    std::vector<int> begin;   // [grid + 1]
    int splits = 0;           // split n-tiles (four counters each)
    int slots = 0;            // partial slots
};

constexpr int kBsUnitRows = 256;

// Work units of a stack: 256-row units times k-tiles.
long long bs_unit_ktiles(const tl_nvfp4_matrix* mats, int n_mats) {
    long long t = 0;
    for (int i = 0; i < n_mats; ++i)
        t += (long long)((mats[i].N + kBsUnitRows - 1) / kBsUnitRows) * (mats[i].K / tl::TC_BLOCK_K);
    return t;
}

// tile_rows: weight rows of the launch's n-tiles (128, or 256 when a stage holds two weight tiles).
void build_schedule(const tl_nvfp4_matrix* mats, int n_mats, int grid, BsSchedule* out,
                    int tile_rows = tl::TC_BLOCK_N) {
    struct Unit { int mat, unit, kt; };
    std::vector<Unit> units;
    for (int i = 0; i < n_mats; ++i) {
        const int nu = (mats[i].N + kBsUnitRows - 1) / kBsUnitRows, kt = mats[i].K / tl::TC_BLOCK_K;
        for (int j = 0; j < nu; ++j) units.push_back({i, j, kt});
    }
    const int halves = kBsUnitRows / tile_rows;   // n-tiles per unit
    const long long U = (long long)units.size(), G = grid;
    // units dealt whole: all but a tail of at least two per CTA and at least two of the largest
    // units' k-tiles per CTA, enough to even out the dealt part
    int max_kt = 1;
    for (const Unit& un : units) max_kt = std::max(max_kt, un.kt);
    long long R = std::max(0LL, U - 2 * G), tail = 0;
    for (long long u = U - 1; u >= R; --u) tail += units[u].kt;
    while (R > 0 && tail < 2 * G * max_kt) tail += units[--R].kt;
    std::vector<std::vector<tl::BsSeg>> per(grid);
    std::vector<long long> load(grid, 0);
    // the n-tiles of unit u (those that hold rows < N)
    auto ntiles_of = [&](const Unit& u, int* first) {
        *first = u.unit * halves;
        const int nt_mat = (mats[u.mat].N + tile_rows - 1) / tile_rows;
        return std::min(halves, nt_mat - *first);
    };
    auto seg = [](const Unit& u, int ntile, int k0, int k1) {
        tl::BsSeg sg;
        sg.mat = u.mat;
        sg.ntile = ntile;
        sg.k0 = (uint16_t)k0;
        sg.k1 = (uint16_t)k1;
        sg.split = -1;
        sg.slot = 0;
        sg.rank = 0;
        sg.parts = 1;
        return sg;
    };
    // deal each whole unit, in order, to the CTA with the fewest k-tiles so far (the one that
    // will be free first; ties to the lowest index): round-robin when the units are alike
    std::priority_queue<std::pair<long long, int>, std::vector<std::pair<long long, int>>,
                        std::greater<std::pair<long long, int>>> freeq;
    for (int c = 0; c < grid; ++c) freeq.push({0LL, c});
    for (long long u = 0; u < R; ++u) {
        const int c = freeq.top().second;
        freeq.pop();
        int t0 = 0;
        const int nt = ntiles_of(units[u], &t0);
        for (int h = 0; h < nt; ++h) per[c].push_back(seg(units[u], t0 + h, 0, units[u].kt));
        load[c] += units[u].kt;
        freeq.push({load[c], c});
    }
    long long total = 0, rest = 0;
    for (long long c = 0; c < G; ++c) total += load[c];
    for (long long u = R; u < U; ++u) rest += units[u].kt;
    total += rest;
    const long long target = (total + G - 1) / G;
    // cut the rest: CTA c takes target - load[c] k-tiles (the last CTA whatever is left)
    struct Part { int cta; long long unit; int k0, k1; };
    std::vector<Part> parts;
    long long u = R;
    int k = 0;
    for (int c = 0; c < grid && u < U; ++c) {
        long long need = (c == grid - 1) ? (1LL << 62) : target - load[c];
        while (need > 0 && u < U) {
            const int take = (int)std::min<long long>(need, units[u].kt - k);
            parts.push_back({c, u, k, k + take});
            k += take;
            need -= take;
            if (k == units[u].kt) { ++u; k = 0; }
        }
    }
    out->splits = 0;
    out->slots = 0;
    for (size_t i = 0; i < parts.size();) {
        size_t j = i;
        while (j < parts.size() && parts[j].unit == parts[i].unit) ++j;
        const Unit& un = units[parts[i].unit];
        int t0 = 0;
        const int nt = ntiles_of(un, &t0);
        if (j - i == 1) {
            for (int h = 0; h < nt; ++h) per[parts[i].cta].push_back(seg(un, t0 + h, parts[i].k0, parts[i].k1));
        } else {
            // each n-tile of the unit is a split of its own, its parts in consecutive slots; a
            // CTA's parts of the unit's n-tiles follow one another
            int split0 = out->splits, slot0 = out->slots;
            out->splits += nt;
            out->slots += nt * (int)(j - i);
            for (size_t r = i; r < j; ++r)
                for (int h = 0; h < nt; ++h) {
                    tl::BsSeg sg = seg(un, t0 + h, parts[r].k0, parts[r].k1);
                    sg.split = split0 + h;
                    sg.rank = (uint16_t)(r - i);
                    sg.parts = (uint16_t)(j - i);
                    sg.slot = slot0 + h * (int)(j - i) + (int)(r - i);
                    per[parts[r].cta].push_back(sg);
                }
        }
        i = j;
    }
    out->segs.clear();
    out->begin.assign(grid + 1, 0);
    for (int c = 0; c < grid; ++c) {
        out->begin[c] = (int)out->segs.size();
        out->segs.insert(out->segs.end(), per[c].begin(), per[c].end());
    }
    out->begin[grid] = (int)out->segs.size();
}

// The X rows of the launch that serves Mp rows, and its weight tiles per stage: two (one X
// stage for 256 weight rows) from TL_BS_WT2_MIN_NX rows up to 32.
#ifndef TL_BS_WT2_MIN_NX
#define TL_BS_WT2_MIN_NX 16
#endif
constexpr int bs_nx(int Mp) { return Mp <= 4 ? 4 : Mp <= 8 ? 8 : Mp <= 16 ? 16 : Mp <= 24 ? 24 : Mp <= 32 ? 32 : 64; }
constexpr int bs_wt(int nx) { return (nx >= TL_BS_WT2_MIN_NX && nx <= 32) ? 2 : 1; }

struct BsLaunch {
    tl::BsParams bp;
    tl::XSplitParams xp;
    std::vector<tl::BsMat> tbl;
    std::vector<tl::XSplitMat> xtbl;
    BsSchedule sched;
    int grid = 0;
};

// Validate (as build_params) and build the block-scaled launch of a stack whose X pieces go to
// `xs` (xs_bytes_total bytes).
tl_status build_bs(const tl_nvfp4_matrix* mats, int n_mats, int M, const unsigned char* x_dev, unsigned char* y_dev,
                   unsigned char* xs, int num_sms, BsLaunch* L) {
    L->tbl.assign(n_mats, tl::BsMat());
    L->xtbl.assign(n_mats, tl::XSplitMat());
    size_t xoff = 0, yoff = 0, soff = 0;
    const int tile_rows = tl::TC_BLOCK_N * bs_wt(bs_nx(round4(M)));
    for (int i = 0; i < n_mats; ++i) {
        const tl_nvfp4_matrix& m = mats[i];
        const void* x = x_dev ? static_cast<const void*>(x_dev + xoff) : m.x;
        void* y = y_dev ? static_cast<void*>(y_dev + yoff) : m.y;
        tl_status st = build_bs_mat(&L->tbl[i], &L->xtbl[i], x, M, m.w_codes, m.w_scales, m.global_scale, y,
                                    m.N, m.K, xs + soff);
        if (st != TL_OK) return st;
        xoff += (size_t)2 * M * m.K;
        yoff += (size_t)2 * M * m.N;
        soff += xs_bytes_of(M, m.K);
    }
    // the split's CTAs in order of decreasing K, so that the longest ones start first and the
    // last wave is made of short ones (the split's outputs do not depend on the order)
    std::stable_sort(L->xtbl.begin(), L->xtbl.end(),
                     [](const tl::XSplitMat& a, const tl::XSplitMat& b) { return a.K > b.K; });
    memset(&L->bp, 0, sizeof L->bp);
    L->bp.n_mats = n_mats;
    L->bp.M = M;
    L->bp.Mp = round4(M);
    L->bp.mats = nullptr;
    L->grid = (int)std::min<long long>(bs_unit_ktiles(mats, n_mats), num_sms);
    build_schedule(mats, n_mats, L->grid, &L->sched, tile_rows);
    if (L->sched.slots > 4 * num_sms || (size_t)L->sched.splits * kCountersPerSplit > counter_words(num_sms))
        return fail(TL_ERR_DEVICE_FAULT, "internal: schedule needs %d partial slots and %d splits", L->sched.slots,
                    L->sched.splits);
    if (n_mats == 1) L->bp.one = L->tbl[0];
    memset(&L->xp, 0, sizeof L->xp);
    L->xp.n_mats = n_mats;
    L->xp.M = M;
    L->xp.Mp = round4(M);
    L->xp.mats = nullptr;
    if (n_mats == 1) L->xp.one = L->xtbl[0];
    return TL_OK;
}

template <int NX>
tl_status launch_bs_gemm(DevState& d, tl::BsParams& p, int grid, cudaStream_t stream) {
    constexpr int WT = bs_wt(NX);
    using C = tl::BsCfg<NX, WT>;
    TL_CUDA(cudaFuncSetAttribute(tl::gemm_bs_kernel<NX, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES));
    p.partials = d.partials;
    p.counters = d.counters;
    p.err = d.err;
    tl::gemm_bs_kernel<NX, WT><<<(unsigned)grid, tl::BS_THREADS, C::SMEM_BYTES, stream>>>(p);
    TL_CUDA(cudaGetLastError());
    return TL_OK;
}

// The X split, then the GEMM, on `stream` (bp.segs / bp.seg_begin already on the device).
tl_status launch_bs(DevState& d, tl::BsParams bp, const tl::XSplitParams& xp, int grid, cudaStream_t stream) {
    tl::x_split_kernel<<<dim3((unsigned)(xp.Mp / tl::XS_ROWS), (unsigned)xp.n_mats), tl::XS_THREADS, 0, stream>>>(xp);
    TL_CUDA(cudaGetLastError());
    switch (bs_nx(bp.Mp)) {
        case 4: return launch_bs_gemm<4>(d, bp, grid, stream);
        case 8: return launch_bs_gemm<8>(d, bp, grid, stream);
        case 16: return launch_bs_gemm<16>(d, bp, grid, stream);
        case 24: return launch_bs_gemm<24>(d, bp, grid, stream);
        case 32: return launch_bs_gemm<32>(d, bp, grid, stream);
        default: return launch_bs_gemm<64>(d, bp, grid, stream);
    }
}

// The schedule as one device blob: segments, then the per-CTA offsets.
std::vector<unsigned char> schedule_blob(const BsSchedule& sc, size_t* begin_off) {
    const size_t a = round256(sc.segs.size() * sizeof(tl::BsSeg));
    std::vector<unsigned char> blob(a + sc.begin.size() * sizeof(int), 0);
    memcpy(blob.data(), sc.segs.data(), sc.segs.size() * sizeof(tl::BsSeg));
    memcpy(blob.data() + a, sc.begin.data(), sc.begin.size() * sizeof(int));
    *begin_off = a;
    return blob;
}

// Grow the per-device X-piece scratch to `bytes` (never inside a graph capture).
tl_status ensure_xs(DevState& d, size_t bytes, cudaStream_t stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (d.xs_cap >= bytes) return TL_OK;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    TL_CUDA(cudaStreamIsCapturing(stream, &cs));
    if (cs != cudaStreamCaptureStatusNone)
        return fail(TL_ERR_UNSUPPORTED, "the block-scaled path must run once at this size before graph capture");
    if (d.xs_buf) {
        TL_CUDA(cudaDeviceSynchronize());   // a kernel in flight may still use the old buffer
        TL_CUDA(cudaFree(d.xs_buf));
        d.xs_buf = nullptr;
        d.xs_cap = 0;
    }
    TL_CUDA(cudaMalloc(&d.xs_buf, bytes));
    d.xs_cap = bytes;
    return TL_OK;
}

// Grow the per-device prepared-X scratch of the exact path to `bytes` (never inside a graph
// capture). It only grows: once it has the largest size the caller uses, no call allocates.
tl_status ensure_xh(DevState& d, size_t bytes, cudaStream_t stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (d.xh_cap >= bytes) return TL_OK;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    TL_CUDA(cudaStreamIsCapturing(stream, &cs));
    if (cs != cudaStreamCaptureStatusNone)
        return fail(TL_ERR_UNSUPPORTED, "the exact path must run once at this size before graph capture");
    if (d.xh_buf) {
        TL_CUDA(cudaDeviceSynchronize());   // a kernel in flight may still use the old buffer
        TL_CUDA(cudaFree(d.xh_buf));
        d.xh_buf = nullptr;
        d.xh_cap = 0;
    }
    TL_CUDA(cudaMalloc(&d.xh_buf, bytes));
    d.xh_cap = bytes;
    return TL_OK;
}

tl_status run_stack_bs(const tl_nvfp4_matrix* mats, int n_mats, int M, const unsigned char* x_dev,
                       unsigned char* y_dev, void* stream_, DevState* d) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_);
    tl_status st = ensure_xs(*d, xs_bytes_total(mats, n_mats, M), stream);
    if (st != TL_OK) return st;
    BsLaunch L;
    st = build_bs(mats, n_mats, M, x_dev, y_dev, d->xs_buf, d->num_sms, &L);
    if (st != TL_OK) return st;
    {
        size_t boff = 0;
        const std::vector<unsigned char> blob = schedule_blob(L.sched, &boff);
        const void* t = nullptr;
        st = device_table(*d, blob.data(), blob.size(), stream, &t);
        if (st != TL_OK) return st;
        L.bp.segs = static_cast<const tl::BsSeg*>(t);
        L.bp.seg_begin = reinterpret_cast<const int*>(static_cast<const unsigned char*>(t) + boff);
    }
    if (n_mats > 1) {
        const void* t = nullptr;
        st = device_table(*d, L.tbl.data(), L.tbl.size() * sizeof(tl::BsMat), stream, &t);
        if (st != TL_OK) return st;
        L.bp.mats = static_cast<const tl::BsMat*>(t);
        st = device_table(*d, L.xtbl.data(), L.xtbl.size() * sizeof(tl::XSplitMat), stream, &t);
        if (st != TL_OK) return st;
        L.xp.mats = static_cast<const tl::XSplitMat*>(t);
    }
    return launch_bs(*d, L.bp, L.xp, L.grid, stream);
}


// ---------------------------------------------------------------------------
// An entry point that allocates nothing.
//
// Some callers cannot let a library allocate device memory at call time: a serving
// engine that hands all free HBM to its KV-cache pool at start-up has nothing left
// for a first-call workspace, and some host runtimes route every device allocation
// through their own pool and forbid libraries from calling cudaMalloc. For them,
// tl_nvfp4_verify_gemm_noalloc() runs the exact bf16-decode kernel (TL_PATH_BF16_EXACT) with
// its split-K scratch in the static array below. The array is device memory of this
// library's CUDA module: with lazy module loading (the default since CUDA 12.2) the module,
// and so the array, is loaded on a device the first time the library touches it there, which
// for a caller that only uses this entry point is the set-up inside its first call. That first
// call is therefore the one that takes device memory (the array and the module's code); later
// calls take none.

// Room for the split-K partials of up to kNoAllocMaxCtas CTAs (two 32 x 128 fp32 tiles
// each, 5 MiB in all), their counters (must be zero when a launch starts) and a status word.
constexpr int kNoAllocMaxCtas = 160;
struct NoAllocScratch {
    float partials[2 * kNoAllocMaxCtas * 32 * tl::TC_BLOCK_N];
    unsigned counters[4 * kNoAllocMaxCtas];
    int err[16];
};

// Every GPU that loads this library holds this array until the process exits. In host code
// its name is only a stand-in: the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) NoAllocScratch g_noalloc_scratch;

struct NoAllocDevice {
    bool ready = false;
    int num_sms = 0;
    NoAllocScratch* scratch = nullptr;   // device address of g_noalloc_scratch on this device
};
NoAllocDevice g_noalloc[kMaxDevices];

// Once per device, with that device current: resolve the scratch address and the SM count.
tl_status noalloc_setup(int device, NoAllocDevice** out) {
    std::lock_guard<std::mutex> lk(g_mu);
    NoAllocDevice& nd = g_noalloc[device];
    if (!nd.ready) {
        int major = 0, minor = 0, sms = 0;
        TL_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device));
        TL_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device));
        TL_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device));
        if (major != 10 || minor != 0)
            return fail(TL_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", device,
                        major, minor);
        void* ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr)
            return fail(TL_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
        tl_status st = load_encode_fn();
        if (st != TL_OK) return st;
        TL_CUDA(cudaFuncSetAttribute(tl::gemm_tc_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     tl::TcCfg<16>::SMEM_BYTES));
        TL_CUDA(cudaFuncSetAttribute(tl::gemm_tc_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     tl::TcCfg<32>::SMEM_BYTES));
        nd.num_sms = sms;
        nd.scratch = static_cast<NoAllocScratch*>(ptr);
        nd.ready = true;
    }
    *out = &nd;
    return TL_OK;
}

}  // namespace

extern "C" tl_status tl_nvfp4_verify_gemm_noalloc(const void* x, int M, const void* w_codes, const void* w_scales,
                                                  float global_scale, void* y, int N, int K, void* stream) {
    tl_status st = check_M(M, kExactMaxRows);
    if (st != TL_OK) return st;
    st = check_matrix(x, M, w_codes, w_scales, global_scale, y, N, K, true);
    if (st != TL_OK) return st;
    if (M == 0) return TL_OK;
    int dev = 0;
    TL_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(TL_ERR_INVALID_VALUE, "device %d out of range", dev);
    NoAllocDevice* nd = nullptr;
    st = noalloc_setup(dev, &nd);
    if (st != TL_OK) return st;
    const int NX = M <= 16 ? 16 : 32;
    tl::TcParams p;
    memset(&p, 0, sizeof p);
    st = build_mat(&p.one, x, M, NX, w_codes, w_scales, global_scale, y, N, K, 0);
    if (st != TL_OK) return st;
    p.mats = nullptr;
    p.n_mats = 1;
    p.M = M;
    p.total_tiles = (long long)p.one.n_tiles * p.one.k_tiles;
    p.partials = nd->scratch->partials;
    p.counters = nd->scratch->counters;
    p.err = nd->scratch->err;
    p.spread_mul = 0x1040u;
    p.scale_mul = 0x00100010u;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the counters must start at zero; a launch that gave up could have left them raised. The
    // status word is not cleared here: it keeps a timeout until tl_noalloc_check_error() reads it.
    TL_CUDA(cudaMemsetAsync(p.counters, 0, sizeof(nd->scratch->counters), s));
    long long grid = p.total_tiles;
    if (grid > nd->num_sms) grid = nd->num_sms;
    if (grid > kNoAllocMaxCtas) grid = kNoAllocMaxCtas;
    if (NX == 16)
        tl::gemm_tc_kernel<16><<<(unsigned)grid, tl::TC_THREADS, tl::TcCfg<16>::SMEM_BYTES, s>>>(p);
    else
        tl::gemm_tc_kernel<32><<<(unsigned)grid, tl::TC_THREADS, tl::TcCfg<32>::SMEM_BYTES, s>>>(p);
    TL_CUDA(cudaGetLastError());
    return TL_OK;
}

struct tl_nvfp4_plan_st {
    int device = 0;
    DevState* d = nullptr;
    int path = TL_PATH_EXACT;         // fixed when the plan is made
    tl::TcParams params;
    tl::TcMat* table = nullptr;       // device copy when n_mats > 1
    tl::BsParams bparams;             // block-scaled path
    tl::XSplitParams xparams;
    int grid = 0;                     // CTAs of the block-scaled GEMM
    void* bs_tables = nullptr;        // device copies of the BsMat and XSplitMat tables (n_mats > 1) and the schedule
    unsigned char* xs = nullptr;      // the plan's own X-piece scratch
    unsigned char* xh = nullptr;      // the plan's own prepared-X scratch (exact path)
    const void* x_base = nullptr;     // packed X_i buffer (or nullptr if not packed)
    void* y_base = nullptr;           // packed Y_i buffer (or nullptr if not packed)
    size_t x_bytes = 0, y_bytes = 0;
    // Host-buffer runs, pipelined: the stack cut into chunks of consecutive matrices, each a
    // plan of its own, so that copying X of chunk c + 1 in, computing chunk c and copying Y of
    // chunk c - 1 out overlap (built at the first tl_nvfp4_plan_run_host).
    int M = 0;
    std::vector<tl_nvfp4_matrix> mats;          // copy of the descriptors (device pointers)
    bool chunks_built = false;
    std::vector<tl_nvfp4_plan_st*> chunks;
    std::vector<size_t> cx_off, cx_len, cy_off, cy_len;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    std::vector<cudaEvent_t> ev;               // start, done, then per chunk: X in, computed
};

namespace {

// The block-scaled launch of a plan: own X-piece scratch and own device tables, so that a plan
// never shares memory with another plan or with calls made without one.
tl_status plan_build_bs(tl_nvfp4_plan plan, const tl_nvfp4_matrix* mats, int n_mats, int M) {
    TL_CUDA(cudaMalloc(&plan->xs, xs_bytes_total(mats, n_mats, M)));
    BsLaunch L;
    tl_status st = build_bs(mats, n_mats, M, nullptr, nullptr, plan->xs, plan->d->num_sms, &L);
    if (st != TL_OK) return st;
    // one device allocation: descriptor tables (n_mats > 1), then the schedule
    size_t boff = 0;
    const std::vector<unsigned char> blob = schedule_blob(L.sched, &boff);
    const size_t b1 = n_mats > 1 ? round256(L.tbl.size() * sizeof(tl::BsMat)) : 0;
    const size_t b2 = n_mats > 1 ? round256(L.xtbl.size() * sizeof(tl::XSplitMat)) : 0;
    TL_CUDA(cudaMalloc(&plan->bs_tables, b1 + b2 + blob.size()));
    unsigned char* t = static_cast<unsigned char*>(plan->bs_tables);
    if (n_mats > 1) {
        TL_CUDA(cudaMemcpy(t, L.tbl.data(), L.tbl.size() * sizeof(tl::BsMat), cudaMemcpyHostToDevice));
        TL_CUDA(cudaMemcpy(t + b1, L.xtbl.data(), L.xtbl.size() * sizeof(tl::XSplitMat), cudaMemcpyHostToDevice));
        L.bp.mats = reinterpret_cast<const tl::BsMat*>(t);
        L.xp.mats = reinterpret_cast<const tl::XSplitMat*>(t + b1);
    }
    TL_CUDA(cudaMemcpy(t + b1 + b2, blob.data(), blob.size(), cudaMemcpyHostToDevice));
    L.bp.segs = reinterpret_cast<const tl::BsSeg*>(t + b1 + b2);
    L.bp.seg_begin = reinterpret_cast<const int*>(t + b1 + b2 + boff);
    plan->bparams = L.bp;
    plan->xparams = L.xp;
    plan->grid = L.grid;
    return TL_OK;
}

tl_status plan_launch(tl_nvfp4_plan plan, cudaStream_t s) {
    if (plan->path == TL_PATH_BLOCK_SCALED) {
        if (plan->grid < 1 || !plan->bparams.segs) return fail(TL_ERR_DEVICE_FAULT, "internal: plan without a schedule");
        return launch_bs(*plan->d, plan->bparams, plan->xparams, plan->grid, s);
    }
    if (plan->params.n_mats < 1 || plan->params.total_tiles < 1 || (plan->params.n_mats > 1 && !plan->params.mats))
        return fail(TL_ERR_DEVICE_FAULT, "internal: plan without descriptors");
    tl::TcParams p = plan->params;
    return launch_tc_any(*plan->d, p, plan->path == TL_PATH_EXACT, s);
}

tl_status plan_create_path(const tl_nvfp4_matrix* mats, int n_mats, int M, int path, tl_nvfp4_plan* plan_out);

// Chunks of a host-buffer run: up to kHostChunks groups of consecutive matrices with about
// equal weight bytes, each its own plan (same path), plus two copy streams and their events.
constexpr int kHostChunks = 8;

// Chunk boundaries of a host-buffer run over n matrices: 0 = cut[0] < cut[1] < ... < cut[C] = n,
// C = min(chunks, n) groups of consecutive matrices, a group ending where the running weight
// count (N x K) first reaches its share of the total.
std::vector<int> host_chunk_cuts(const tl_nvfp4_matrix* mats, int n, int chunks) {
    const int C = std::min(chunks, n);
    double total = 0.0;
    for (int i = 0; i < n; ++i) total += (double)mats[i].N * mats[i].K;
    std::vector<int> cut{0};
    double acc = 0.0;
    for (int i = 0; i + 1 < n && (int)cut.size() < C; ++i) {
        acc += (double)mats[i].N * mats[i].K;
        if (acc >= total * (double)cut.size() / C) cut.push_back(i + 1);
    }
    cut.push_back(n);
    return cut;
}

// Builds the chunks, their streams and events all at once: on any failure nothing is kept (the
// next host-buffer run tries again).
tl_status plan_build_chunks(tl_nvfp4_plan plan) {
    const int n = (int)plan->mats.size();
    if (std::min(kHostChunks, n) < 2) {
        plan->chunks_built = true;
        return TL_OK;
    }
    const std::vector<int> cut = host_chunk_cuts(plan->mats.data(), n, kHostChunks);
    std::vector<tl_nvfp4_plan> chunks;
    std::vector<size_t> cx_off, cx_len, cy_off, cy_len;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    std::vector<cudaEvent_t> ev(2 + 2 * (cut.size() - 1), nullptr);
    auto undo = [&](tl_status st) {
        for (tl_nvfp4_plan cp : chunks) tl_nvfp4_plan_destroy(cp);
        for (cudaEvent_t e : ev)
            if (e) cudaEventDestroy(e);
        if (s_in) cudaStreamDestroy(s_in);
        if (s_out) cudaStreamDestroy(s_out);
        return st;
    };
    size_t xo = 0, yo = 0;
    for (size_t c = 0; c + 1 < cut.size(); ++c) {
        const int a = cut[c], b = cut[c + 1];
        size_t xl = 0, yl = 0;
        for (int i = a; i < b; ++i) {
            xl += (size_t)2 * plan->M * plan->mats[i].K;
            yl += (size_t)2 * plan->M * plan->mats[i].N;
        }
        tl_nvfp4_plan cp = nullptr;
        tl_status st = plan_create_path(plan->mats.data() + a, b - a, plan->M, plan->path, &cp);
        if (st != TL_OK) return undo(st);
        chunks.push_back(cp);
        cx_off.push_back(xo);
        cx_len.push_back(xl);
        cy_off.push_back(yo);
        cy_len.push_back(yl);
        xo += xl;
        yo += yl;
    }
    if (cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking) != cudaSuccess)
        return undo(fail(TL_ERR_CUDA, "creating the host-buffer run's streams failed"));
    for (cudaEvent_t& e : ev)
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess)
            return undo(fail(TL_ERR_CUDA, "creating the host-buffer run's events failed"));
    plan->chunks = std::move(chunks);
    plan->cx_off = std::move(cx_off);
    plan->cx_len = std::move(cx_len);
    plan->cy_off = std::move(cy_off);
    plan->cy_len = std::move(cy_len);
    plan->s_in = s_in;
    plan->s_out = s_out;
    plan->ev = std::move(ev);
    plan->chunks_built = true;
    return TL_OK;
}

tl_status plan_create_path(const tl_nvfp4_matrix* mats, int n_mats, int M, int path, tl_nvfp4_plan* plan_out) {
    if (!plan_out) return fail(TL_ERR_INVALID_VALUE, "plan_out is null");
    *plan_out = nullptr;
    if (M == 0) return fail(TL_ERR_INVALID_VALUE, "a plan needs M >= 1");
    DevState* d = nullptr;
    tl::TcParams p;
    std::vector<tl::TcMat> tbl;
    // the exact path's scratch belongs to the plan: validate first (the bf16 decode builds no
    // scratch), then allocate it and build the descriptors over it
    tl_status st = build_params(mats, n_mats, M, nullptr, nullptr, path == TL_PATH_EXACT ? TL_PATH_BF16_EXACT : path,
                                &d, &p, &tbl);
    if (st != TL_OK) return st;
    unsigned char* xh = nullptr;
    if (path == TL_PATH_EXACT) {
        TL_CUDA(cudaMalloc(&xh, xh_bytes_total(mats, n_mats, M)));
        st = build_params(mats, n_mats, M, nullptr, nullptr, path, &d, &p, &tbl, xh);
        if (st != TL_OK) {
            cudaFree(xh);
            return st;
        }
    }
    tl_nvfp4_plan plan = new tl_nvfp4_plan_st();
    plan->xh = xh;
    TL_CUDA(cudaGetDevice(&plan->device));
    plan->d = d;
    plan->params = p;
    plan->path = path;
    plan->M = M;
    plan->mats.assign(mats, mats + n_mats);
    if (plan->path == TL_PATH_BLOCK_SCALED) {
        st = plan_build_bs(plan, mats, n_mats, M);
        if (st != TL_OK) {
            tl_nvfp4_plan_destroy(plan);
            return st;
        }
    } else if (n_mats > 1) {
        const size_t bytes = tbl.size() * sizeof(tl::TcMat);
        if (cudaMalloc(&plan->table, bytes) != cudaSuccess ||
            cudaMemcpy(plan->table, tbl.data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
            tl_nvfp4_plan_destroy(plan);
            return fail(TL_ERR_CUDA, "uploading the plan's descriptor table failed");
        }
        plan->params.mats = plan->table;
    }
    // packed X / Y buffers (needed by the host-buffer form only)
    bool xpk = true, ypk = true;
    const unsigned char* xb = static_cast<const unsigned char*>(mats[0].x);
    const unsigned char* yb = static_cast<const unsigned char*>(mats[0].y);
    size_t xo = 0, yo = 0;
    for (int i = 0; i < n_mats; ++i) {
        xpk = xpk && static_cast<const unsigned char*>(mats[i].x) == xb + xo;
        ypk = ypk && static_cast<const unsigned char*>(mats[i].y) == yb + yo;
        xo += (size_t)2 * M * mats[i].K;
        yo += (size_t)2 * M * mats[i].N;
    }
    if (xpk) { plan->x_base = xb; plan->x_bytes = xo; }
    if (ypk) { plan->y_base = (void*)yb; plan->y_bytes = yo; }
    *plan_out = plan;
    return TL_OK;
}

}  // namespace

namespace {

template <int NX>
tl_status launch_head(DevState& d, tl::HeadParams& hp, cudaStream_t stream) {
    using C = tl::HeadCfg<NX>;
    TL_CUDA(cudaFuncSetAttribute(tl::gemm_head_kernel<NX>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
    const long long grid = hp.total_tiles < d.num_sms ? hp.total_tiles : d.num_sms;
    tl::gemm_head_kernel<NX><<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, stream>>>(hp);
    TL_CUDA(cudaGetLastError());
    return TL_OK;
}

template <int DK, int DV, int LMAX>
tl_status launch_gdn_l(float* state, int H, const float* k, const float* v, const float* alpha, const float* beta,
                       const tl::GdnPath& p, int L, cudaStream_t stream) {
    using C = tl::GdnCfg<DK, DV>;
    TL_CUDA(cudaFuncSetAttribute(tl::gdn_commit_kernel<DK, DV, LMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_BYTES));
    tl::gdn_commit_kernel<DK, DV, LMAX><<<(unsigned)H, tl::GDN_THREADS, C::SMEM_BYTES, stream>>>(state, H, k, v, alpha,
                                                                                                beta, p, L);
    TL_CUDA(cudaGetLastError());
    return TL_OK;
}

template <int DK, int DV>
tl_status launch_gdn(float* state, int H, const float* k, const float* v, const float* alpha, const float* beta,
                     const tl::GdnPath& p, int L, cudaStream_t stream) {
    if (L <= 8) return launch_gdn_l<DK, DV, 8>(state, H, k, v, alpha, beta, p, L, stream);
    if (L <= 16) return launch_gdn_l<DK, DV, 16>(state, H, k, v, alpha, beta, p, L, stream);
    return launch_gdn_l<DK, DV, 32>(state, H, k, v, alpha, beta, p, L, stream);
}

}  // namespace

extern "C" {

tl_status tl_nvfp4_plan_create(const tl_nvfp4_matrix* mats, int n_mats, int M, tl_nvfp4_plan* plan_out) {
    if (!plan_out) return fail(TL_ERR_INVALID_VALUE, "plan_out is null");
    *plan_out = nullptr;
    return plan_create_path(mats, n_mats, M, current_path(), plan_out);
}

tl_status tl_nvfp4_plan_run(tl_nvfp4_plan plan, void* stream) {
    if (!plan) return fail(TL_ERR_INVALID_VALUE, "plan is null");
    return plan_launch(plan, static_cast<cudaStream_t>(stream));
}

tl_status tl_nvfp4_plan_run_host(tl_nvfp4_plan plan, const void* x_host, void* y_host, void* stream) {
    if (!plan) return fail(TL_ERR_INVALID_VALUE, "plan is null");
    if (!x_host || !y_host) return fail(TL_ERR_INVALID_VALUE, "null host buffer");
    if (!plan->x_base || !plan->y_base)
        return fail(TL_ERR_INVALID_VALUE, "the plan's X and Y buffers are not packed back to back");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!plan->chunks_built) {
        tl_status st = plan_build_chunks(plan);
        if (st != TL_OK) return st;
    }
    if (plan->chunks.empty()) {
        TL_CUDA(cudaMemcpyAsync(const_cast<void*>(plan->x_base), x_host, plan->x_bytes, cudaMemcpyHostToDevice, s));
        tl_status st = plan_launch(plan, s);
        if (st != TL_OK) return st;
        TL_CUDA(cudaMemcpyAsync(y_host, plan->y_base, plan->y_bytes, cudaMemcpyDeviceToHost, s));
        return TL_OK;
    }
    // X of every chunk in on s_in; chunk c computed on `stream` once its X is in; its Y out on
    // s_out once computed; `stream` resumes after the last Y is out.
    const unsigned char* xh = static_cast<const unsigned char*>(x_host);
    unsigned char* yh = static_cast<unsigned char*>(y_host);
    unsigned char* xd = static_cast<unsigned char*>(const_cast<void*>(plan->x_base));
    unsigned char* yd = static_cast<unsigned char*>(plan->y_base);
    const size_t C = plan->chunks.size();
    cudaEvent_t e_start = plan->ev[0], e_done = plan->ev[1];
    TL_CUDA(cudaEventRecord(e_start, s));
    TL_CUDA(cudaStreamWaitEvent(plan->s_in, e_start, 0));
    TL_CUDA(cudaStreamWaitEvent(plan->s_out, e_start, 0));
    // From here on both internal streams are forked from `s`: every return joins them back
    // (s_in into s_out, s_out into s), so that later work on `s` is ordered after everything
    // queued and a stream capture of the call stays closed.
    tl_status st = TL_OK;
    for (size_t c = 0; c < C && st == TL_OK; ++c) {
        if (cudaMemcpyAsync(xd + plan->cx_off[c], xh + plan->cx_off[c], plan->cx_len[c], cudaMemcpyHostToDevice,
                            plan->s_in) != cudaSuccess ||
            cudaEventRecord(plan->ev[2 + 2 * c], plan->s_in) != cudaSuccess)
            st = fail(TL_ERR_CUDA, "queueing the X copy of chunk %zu failed", c);
    }
    for (size_t c = 0; c < C && st == TL_OK; ++c) {
        if (cudaStreamWaitEvent(s, plan->ev[2 + 2 * c], 0) != cudaSuccess) {
            st = fail(TL_ERR_CUDA, "ordering chunk %zu after its X copy failed", c);
            break;
        }
        st = plan_launch(plan->chunks[c], s);
        if (st != TL_OK) break;
        if (cudaEventRecord(plan->ev[3 + 2 * c], s) != cudaSuccess ||
            cudaStreamWaitEvent(plan->s_out, plan->ev[3 + 2 * c], 0) != cudaSuccess ||
            cudaMemcpyAsync(yh + plan->cy_off[c], yd + plan->cy_off[c], plan->cy_len[c], cudaMemcpyDeviceToHost,
                            plan->s_out) != cudaSuccess)
            st = fail(TL_ERR_CUDA, "queueing the Y copy of chunk %zu failed", c);
    }
    // join: s_in -> s_out (e_start is free again once recorded here), s_out -> s
    const bool joined = cudaEventRecord(e_start, plan->s_in) == cudaSuccess &&
                        cudaStreamWaitEvent(plan->s_out, e_start, 0) == cudaSuccess &&
                        cudaEventRecord(e_done, plan->s_out) == cudaSuccess &&
                        cudaStreamWaitEvent(s, e_done, 0) == cudaSuccess;
    if (st != TL_OK) return st;
    if (!joined) return fail(TL_ERR_CUDA, "joining the host-buffer run's copy streams failed");
    return TL_OK;
}

tl_status tl_nvfp4_plan_destroy(tl_nvfp4_plan plan) {
    if (!plan) return TL_OK;
    for (tl_nvfp4_plan cp : plan->chunks) tl_nvfp4_plan_destroy(cp);
    if (plan->s_in || plan->s_out || !plan->ev.empty()) {
        int prev = 0;
        cudaGetDevice(&prev);
        cudaSetDevice(plan->device);
        cudaDeviceSynchronize();
        for (cudaEvent_t e : plan->ev)
            if (e) cudaEventDestroy(e);
        if (plan->s_in) cudaStreamDestroy(plan->s_in);
        if (plan->s_out) cudaStreamDestroy(plan->s_out);
        cudaSetDevice(prev);
    }
    if (plan->table || plan->bs_tables || plan->xs || plan->xh) {
        int prev = 0;
        cudaGetDevice(&prev);
        cudaSetDevice(plan->device);
        cudaDeviceSynchronize();
        if (plan->table) cudaFree(plan->table);
        if (plan->bs_tables) cudaFree(plan->bs_tables);
        if (plan->xs) cudaFree(plan->xs);
        if (plan->xh) cudaFree(plan->xh);
        cudaSetDevice(prev);
    }
    delete plan;
    return TL_OK;
}

tl_status tl_set_gemm_path(int path) {
    if (path != TL_PATH_BLOCK_SCALED && path != TL_PATH_BF16_EXACT && path != TL_PATH_EXACT)
        return fail(TL_ERR_INVALID_VALUE, "unknown GEMM path %d", path);
    std::lock_guard<std::mutex> lk(g_mu);
    g_path = path;
    return TL_OK;
}

int tl_get_gemm_path(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    return g_path;
}

tl_status tl_init(int device) {
    std::lock_guard<std::mutex> lk(g_mu);
    tl_status st = init_locked(device);
    if (st != TL_OK) return st;
    return load_encode_fn();
}

void tl_shutdown(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    int prev = 0;
    cudaGetDevice(&prev);
    for (int i = 0; i < kMaxDevices; ++i) {
        DevState& d = g_dev[i];
        if (!d.ready) continue;
        cudaSetDevice(i);
        cudaDeviceSynchronize();
        cudaFree(d.err);
        cudaFree(d.partials);
        cudaFree(d.counters);
        cudaFree(d.qscratch);
        for (auto& e : d.cache) {
            if (e.table) cudaFree(e.table);
            if (e.staging) cudaFreeHost(e.staging);
            if (e.copied) cudaEventDestroy(e.copied);
        }
        if (d.xs_buf) cudaFree(d.xs_buf);
        if (d.xh_buf) cudaFree(d.xh_buf);
        d = DevState();
    }
    cudaSetDevice(prev);
}

tl_status tl_nvfp4_verify_gemm(const void* x, int M, const void* w_codes, const void* w_scales, float global_scale,
                               void* y, int N, int K, void* stream) {
    tl_status st = check_M(M);
    if (st != TL_OK) return st;
    st = check_matrix(x, M, w_codes, w_scales, global_scale, y, N, K, true);
    if (st != TL_OK) return st;
    if (M == 0) return TL_OK;
    tl_nvfp4_matrix m{w_codes, w_scales, x, y, global_scale, N, K};
    return run_stack(&m, 1, M, nullptr, nullptr, stream);
}

tl_status tl_nvfp4_verify_gemm_simt(const void* x, int M, const void* w_codes, const void* w_scales,
                                    float global_scale, void* y, int N, int K, void* stream) {
    tl_status st = check_M(M);
    if (st != TL_OK) return st;
    st = check_matrix(x, M, w_codes, w_scales, global_scale, y, N, K, true);
    if (st != TL_OK) return st;
    if (M == 0) return TL_OK;
    DevState* d = nullptr;
    st = current_state(&d);
    if (st != TL_OK) return st;
    const unsigned grid = (unsigned)((N + tl::SIMT_WARPS - 1) / tl::SIMT_WARPS);
    auto xs = static_cast<const __nv_bfloat16*>(x);
    auto cs = static_cast<const uint8_t*>(w_codes);
    auto ss = static_cast<const uint8_t*>(w_scales);
    auto ys = static_cast<__nv_bfloat16*>(y);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int r0 = 0; r0 < M; r0 += kExactMaxRows) {   // groups of at most 32 rows
        const int mg = std::min(kExactMaxRows, M - r0);
        const __nv_bfloat16* xg = xs + (size_t)r0 * K;
        __nv_bfloat16* yg = ys + (size_t)r0 * N;
        if (mg <= 8)
            tl::gemm_simt_kernel<8><<<grid, tl::SIMT_WARPS * 32, 0, s>>>(xg, mg, cs, ss, global_scale, yg, N, K);
        else if (mg <= 16)
            tl::gemm_simt_kernel<16><<<grid, tl::SIMT_WARPS * 32, 0, s>>>(xg, mg, cs, ss, global_scale, yg, N, K);
        else
            tl::gemm_simt_kernel<32><<<grid, tl::SIMT_WARPS * 32, 0, s>>>(xg, mg, cs, ss, global_scale, yg, N, K);
        TL_CUDA(cudaGetLastError());
    }
    return TL_OK;
}

tl_status tl_nvfp4_verify_stack(const tl_nvfp4_matrix* mats, int n_mats, int M, void* stream) {
    return run_stack(mats, n_mats, M, nullptr, nullptr, stream);
}

tl_status tl_nvfp4_verify_stack_host(const tl_nvfp4_matrix* mats, int n_mats, int M, const void* x_host,
                                     void* x_dev, void* y_host, void* y_dev, void* stream) {
    tl_status st = check_M(M);
    if (st != TL_OK) return st;
    if (!mats || n_mats < 1 || n_mats > TL_NVFP4_MAX_STACK)
        return fail(TL_ERR_INVALID_VALUE, "mats is null or n_mats = %d outside [1, %d]", n_mats, TL_NVFP4_MAX_STACK);
    if (!x_host || !x_dev || !y_host || !y_dev) return fail(TL_ERR_INVALID_VALUE, "null host or device buffer");
    if (M == 0) return TL_OK;
    size_t xb = 0, yb = 0;
    for (int i = 0; i < n_mats; ++i) {
        if ((((size_t)M * mats[i].K) % 8) != 0 || (((size_t)M * mats[i].N) % 8) != 0)
            return fail(TL_ERR_MISALIGNED, "matrix %d: M*K and M*N must be multiples of 8 elements", i);
        if (mats[i].K < 0 || mats[i].N < 0) return fail(TL_ERR_INVALID_VALUE, "matrix %d: negative size", i);
        xb += (size_t)2 * M * mats[i].K;
        yb += (size_t)2 * M * mats[i].N;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TL_CUDA(cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, s));
    st = run_stack(mats, n_mats, M, static_cast<const unsigned char*>(x_dev), static_cast<unsigned char*>(y_dev),
                   stream);
    if (st != TL_OK) return st;
    TL_CUDA(cudaMemcpyAsync(y_host, y_dev, yb, cudaMemcpyDeviceToHost, s));
    return TL_OK;
}

tl_status tl_fp8_head(const void* x, int M, const void* w_fp8, int N, int K, float tensor_scale,
                      const float* row_scales, float* logits, tl_head_top2* top2, void* stream) {
    if (M < 0 || M > TL_HEAD_MAX_M) return fail(M < 0 ? TL_ERR_INVALID_VALUE : TL_ERR_UNSUPPORTED,
                                                "M = %d outside 0..%d rows", M, TL_HEAD_MAX_M);
    if (N < 2) return fail(TL_ERR_INVALID_VALUE, "N = %d: the head needs at least two rows", N);
    if (K <= 0 || K % TL_NVFP4_K_ALIGN != 0)
        return fail(TL_ERR_INVALID_VALUE, "K = %d must be a positive multiple of %d", K, TL_NVFP4_K_ALIGN);
    if (!x || !w_fp8 || !logits || !top2) return fail(TL_ERR_INVALID_VALUE, "null pointer");
    if (!aligned16(x) || !aligned16(w_fp8) || !aligned16(logits) || (row_scales && !aligned16(row_scales)))
        return fail(TL_ERR_MISALIGNED, "x, w, logits and row_scales must be 16-byte aligned");
    if (!row_scales && !std::isfinite(tensor_scale)) return fail(TL_ERR_INVALID_VALUE, "tensor_scale is not finite");
    if (overlap(logits, (size_t)4 * M * N, x, (size_t)2 * M * K) || overlap(logits, (size_t)4 * M * N, w_fp8, (size_t)N * K) ||
        overlap(top2, sizeof(tl_head_top2) * (size_t)M, logits, (size_t)4 * M * N))
        return fail(TL_ERR_INVALID_VALUE, "logits overlap x, the weights or top2");
    if (M == 0) return TL_OK;
    DevState* d = nullptr;
    tl_status st = current_state(&d);
    if (st != TL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = ensure_xh(*d, xh_bytes_of(M, K), s);
    if (st != TL_OK) return st;
    // the X preparation: a one-matrix TcParams over the per-device scratch
    const int NX = M <= 16 ? 16 : 32;
    tl::TcParams pp;
    memset(&pp, 0, sizeof pp);
    unsigned char* xh = d->xh_buf;
    pp.one.x = static_cast<const __nv_bfloat16*>(x);
    pp.one.xh = reinterpret_cast<__half*>(xh);
    pp.one.rowfac = reinterpret_cast<float*>(xh + (((size_t)2 * M * K + 255) & ~size_t(255)));
    pp.one.rowmask = reinterpret_cast<unsigned*>(reinterpret_cast<unsigned char*>(pp.one.rowfac) +
                                                 (((size_t)4 * M + 255) & ~size_t(255)));
    pp.one.K = K;
    pp.n_mats = 1;
    pp.M = M;
    tl::HeadParams hp;
    memset(&hp, 0, sizeof hp);
    const cuuint64_t n = (cuuint64_t)N, k = (cuuint64_t)K;
    st = encode_3d(&hp.tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_fp8, {128, n, k / 128}, {k, 128},
                   {128, tl::TC_BLOCK_N, 2}, CU_TENSOR_MAP_SWIZZLE_128B, "head weights");
    if (st != TL_OK) return st;
    st = encode_3d(&hp.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xh, {64, (cuuint64_t)M, k / 64}, {k * 2, 128},
                   {64, (cuuint32_t)NX, 4}, CU_TENSOR_MAP_SWIZZLE_128B, "head X");
    if (st != TL_OK) return st;
    hp.w = static_cast<const uint8_t*>(w_fp8);
    hp.row_scale = row_scales;
    hp.tensor_scale = tensor_scale;
    hp.logits = logits;
    hp.rowfac = pp.one.rowfac;
    hp.rowmask = pp.one.rowmask;
    hp.x = static_cast<const __nv_bfloat16*>(x);
    hp.M = M;
    hp.N = N;
    hp.K = K;
    hp.k_tiles = K / tl::TC_BLOCK_K;
    hp.n_tiles = (N + tl::TC_BLOCK_N - 1) / tl::TC_BLOCK_N;
    hp.total_tiles = (long long)hp.k_tiles * hp.n_tiles;
    hp.partials = d->partials;
    hp.counters = d->counters;
    hp.err = d->err;
    tl::x_prep_kernel<<<dim3(1u, (unsigned)M), tl::XP_THREADS, 0, s>>>(pp);
    TL_CUDA(cudaGetLastError());
    st = (NX == 16) ? launch_head<16>(*d, hp, s) : launch_head<32>(*d, hp, s);
    if (st != TL_OK) return st;
    // fp64 rows, partials over chunks of at most 1024 per row and the per-row merge in one launch;
    // the partials reuse the split-K scratch (free again once the GEMM has run on this stream), the
    // per-row counters sit past the GEMM's in the counter array and are left at zero
    int chunk = (N + 1023) / 1024;
    chunk = ((chunk < 4096 ? 4096 : chunk) + 255) & ~255;
    const int chunks = (N + chunk - 1) / chunk;
    tl::T2* part = reinterpret_cast<tl::T2*>(d->partials);
    unsigned* row_counters = d->counters + counter_words(d->num_sms) - TL_HEAD_MAX_M;
    tl::head_tail_kernel<<<dim3((unsigned)chunks, (unsigned)M), tl::HEAD_TOP2_THREADS, 0, s>>>(
        hp, chunk, part, row_counters, reinterpret_cast<tl::HeadTop2*>(top2));
    TL_CUDA(cudaGetLastError());
    return TL_OK;
}

tl_status tl_gdn_commit(float* state, int H, int d_k, int d_v, const float* k, const float* v, const float* alpha,
                        const float* beta, int n_nodes, const int* path, int L, void* stream) {
    if (H < 1) return fail(TL_ERR_INVALID_VALUE, "H = %d must be >= 1", H);
    if ((d_k != 64 && d_k != 128) || (d_v != 64 && d_v != 128))
        return fail(TL_ERR_UNSUPPORTED, "d_k = %d, d_v = %d: each must be 64 or 128", d_k, d_v);
    if (L < 0 || L > TL_GDN_MAX_PATH) return fail(TL_ERR_INVALID_VALUE, "L = %d outside 0..%d", L, TL_GDN_MAX_PATH);
    if (n_nodes < 1) return fail(TL_ERR_INVALID_VALUE, "n_nodes = %d must be >= 1", n_nodes);
    if (!state || !k || !v || !alpha || !beta || (L > 0 && !path)) return fail(TL_ERR_INVALID_VALUE, "null pointer");
    if (!aligned16(state) || !aligned16(k)) return fail(TL_ERR_MISALIGNED, "state and k must be 16-byte aligned");
    {
        const size_t sb = (size_t)H * d_v * d_k * 4, nh = (size_t)n_nodes * H;
        if (overlap(state, sb, k, nh * d_k * 4) || overlap(state, sb, v, nh * d_v * 4) ||
            overlap(state, sb, alpha, nh * 4) || overlap(state, sb, beta, nh * 4))
            return fail(TL_ERR_INVALID_VALUE, "state overlaps the path inputs");
    }
    tl::GdnPath p;
    memset(&p, 0, sizeof p);
    for (int t = 0; t < L; ++t) {
        if (path[t] < 0 || path[t] >= n_nodes)
            return fail(TL_ERR_INVALID_VALUE, "path[%d] = %d outside 0..%d", t, path[t], n_nodes - 1);
        p.idx[t] = path[t];
    }
    if (L == 0) return TL_OK;
    DevState* d = nullptr;
    tl_status st = current_state(&d);
    if (st != TL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d_k == 128 && d_v == 128) st = launch_gdn<128, 128>(state, H, k, v, alpha, beta, p, L, s);
    else if (d_k == 128) st = launch_gdn<128, 64>(state, H, k, v, alpha, beta, p, L, s);
    else if (d_v == 128) st = launch_gdn<64, 128>(state, H, k, v, alpha, beta, p, L, s);
    else st = launch_gdn<64, 64>(state, H, k, v, alpha, beta, p, L, s);
    (void)d;
    return st;
}

tl_status tl_nvfp4_dequant(const void* w_codes, const void* w_scales, float global_scale, float* w_out, int N, int K,
                           void* stream) {
    tl_status st = check_matrix(nullptr, 0, w_codes, w_scales, global_scale, nullptr, N, K, false);
    if (st != TL_OK) return st;
    if (!w_out) return fail(TL_ERR_INVALID_VALUE, "w_out is null");
    if (!aligned16(w_out)) return fail(TL_ERR_MISALIGNED, "w_out must be 16-byte aligned");
    DevState* d = nullptr;
    st = current_state(&d);
    if (st != TL_OK) return st;
    const long long blocks = (long long)N * (K / 16);
    tl::dequant_kernel<<<(unsigned)((blocks + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(w_codes), static_cast<const uint8_t*>(w_scales), global_scale, blocks, w_out);
    TL_CUDA(cudaGetLastError());
    return TL_OK;
}

tl_status tl_nvfp4_quantize(const float* w, int N, int K, void* w_codes, void* w_scales, float* global_scale_out,
                            void* stream) {
    if (N < 1) return fail(TL_ERR_INVALID_VALUE, "N = %d must be >= 1", N);
    if (K <= 0 || K % 16 != 0) return fail(TL_ERR_INVALID_VALUE, "K = %d must be a positive multiple of 16", K);
    if (!w || !w_codes || !w_scales || !global_scale_out) return fail(TL_ERR_INVALID_VALUE, "null pointer");
    if (!aligned16(w) || !aligned16(w_codes) || !aligned16(w_scales))
        return fail(TL_ERR_MISALIGNED, "w, codes and scales must be 16-byte aligned");
    DevState* d = nullptr;
    tl_status st = current_state(&d);
    if (st != TL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long count = (long long)N * K;
    TL_CUDA(cudaMemsetAsync(d->qscratch, 0, 8, s));
    tl::absmax_kernel<<<(unsigned)(4 * d->num_sms), 512, 0, s>>>(w, count, d->qscratch);
    TL_CUDA(cudaGetLastError());
    unsigned h[2] = {0, 0};
    TL_CUDA(cudaMemcpyAsync(h, d->qscratch, 8, cudaMemcpyDeviceToHost, s));
    TL_CUDA(cudaStreamSynchronize(s));
    if (h[1]) return fail(TL_ERR_NONFINITE, "w holds NaN or infinity");
    float amax;
    memcpy(&amax, &h[0], 4);
    const float g = (float)((double)amax / (6.0 * 448.0));
    const long long blocks = count / 16;
    tl::quantize_kernel<<<(unsigned)((blocks + 255) / 256), 256, 0, s>>>(w, blocks, g, static_cast<uint8_t*>(w_codes),
                                                                        static_cast<uint8_t*>(w_scales));
    TL_CUDA(cudaGetLastError());
    TL_CUDA(cudaStreamSynchronize(s));
    *global_scale_out = g;
    return TL_OK;
}

// The status word of the no-allocation entry point's static scratch on the current device:
// read, and cleared when set (no allocation; only the static array is touched).
static tl_status noalloc_take_error(int* code_out) {
    *code_out = 0;
    int dev = 0;
    TL_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(TL_ERR_INVALID_VALUE, "device %d out of range", dev);
    NoAllocScratch* sc = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_noalloc[dev].ready) sc = g_noalloc[dev].scratch;
    }
    if (!sc) return TL_OK;   // never used on this device
    int code = 0;
    TL_CUDA(cudaMemcpy(&code, sc->err, sizeof code, cudaMemcpyDeviceToHost));
    if (code != 0) TL_CUDA(cudaMemset(sc->err, 0, sizeof code));
    *code_out = code;
    return TL_OK;
}

static tl_status status_of_code(int code) {
    if (code == 0) return TL_OK;
    if ((code & 0xF00) == 0x100) return fail(TL_ERR_TIMEOUT, "a device-side wait ran past its limit (code 0x%x)", code);
    return fail(TL_ERR_DEVICE_FAULT, "device status word 0x%x", code);
}

tl_status tl_noalloc_check_error(void* stream) {
    TL_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    int code = 0;
    tl_status st = noalloc_take_error(&code);
    if (st != TL_OK) return st;
    return status_of_code(code);
}

tl_status tl_check_device_error(void* stream) {
    DevState* d = nullptr;
    tl_status st = current_state(&d);
    if (st != TL_OK) return st;
    TL_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    int na_code = 0;
    st = noalloc_take_error(&na_code);
    if (st != TL_OK) return st;
    int code = 0;
    TL_CUDA(cudaMemcpy(&code, d->err, sizeof code, cudaMemcpyDeviceToHost));
    if (code == 0 && na_code != 0) return status_of_code(na_code);
    if (code == 0) return TL_OK;
    // a kernel that gave up may have left split-K counters raised: clear all of them (up to
    // 2 * SMs splits of four counters each, kCounterWords) for the next launch
    TL_CUDA(cudaMemset(d->err, 0, sizeof code));
    TL_CUDA(cudaMemset(d->counters, 0, counter_words(d->num_sms) * sizeof(unsigned)));
    TL_CUDA(cudaDeviceSynchronize());
    return status_of_code(code);
}

tl_status tl_selftest_bounded_wait(unsigned iterations, void* stream) {
    DevState* d = nullptr;
    tl_status st = current_state(&d);
    if (st != TL_OK) return st;
    tl::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(iterations, d->err);
    TL_CUDA(cudaGetLastError());
    return TL_OK;
}

int tl_num_sms(int device) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (device < 0 || device >= kMaxDevices || !g_dev[device].ready) return 0;
    return g_dev[device].num_sms;
}

const char* tl_status_string(tl_status s) {
    switch (s) {
        case TL_OK: return "TL_OK";
        case TL_ERR_INVALID_VALUE: return "TL_ERR_INVALID_VALUE";
        case TL_ERR_MISALIGNED: return "TL_ERR_MISALIGNED";
        case TL_ERR_UNSUPPORTED: return "TL_ERR_UNSUPPORTED";
        case TL_ERR_CUDA: return "TL_ERR_CUDA";
        case TL_ERR_TIMEOUT: return "TL_ERR_TIMEOUT";
        case TL_ERR_NOT_INITIALIZED: return "TL_ERR_NOT_INITIALIZED";
        case TL_ERR_NONFINITE: return "TL_ERR_NONFINITE";
        case TL_ERR_DEVICE_FAULT: return "TL_ERR_DEVICE_FAULT";
    }
    return "TL_ERR_UNKNOWN";
}

const char* tl_last_error_message(void) { return g_msg; }

}  // extern "C"
