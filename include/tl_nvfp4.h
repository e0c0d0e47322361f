/*
 * tl_nvfp4.h -- C ABI of libtl_nvfp4.so, the NVFP4 verify GEMM for B200 (sm_100a).
 *
 * The operation. One verify pass of a speculative decoder checks all rows of
 * a draft tree (8/16/24/32 rows: 7/15/23/31 nodes plus the root) with one
 * forward pass of the big model, and that pass is dominated by reading every
 * weight once (TandemLLM docs v0.12.0, "What TandemLLM is", section 1.2; the
 * StairCut research page, "What it says"). Each projection of that pass is
 *
 *     Y[M,N] = X[M,K] . dequant(W)[N,K]^T,      1 <= M <= 32 (up to 128 served),
 *
 * with W stored as NVFP4: four bits a weight and one scale per 16 weights
 * (same page, section 1.2). At the bit level:
 *   codes    uint8 [N][K/2]  two E2M1 codes per byte, low nibble = even k;
 *                            E2M1 magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}, bit 3 = sign
 *   scales   uint8 [N][K/16] one E4M3 ("fn": no inf, 0x7F/0xFF NaN, max 448)
 *                            scale per 16-element K block
 *   global_scale  float      one FP32 tensor scale that multiplies:
 *                            w[n,k] = e2m1(code) * e4m3(scale) * global_scale
 *   x        bf16  [M][K]    the draft-tree rows
 *   y        bf16  [M][N]    fp32 accumulation, rounded to bf16 (nearest even) once
 * All arrays are row-major and contiguous, in device memory unless stated.
 *
 * Determinism. The reduction order of every output element is fixed: the same
 * inputs give bit-identical Y on every run (the pages' NVFP4 kernels keep a
 * fixed reduction order; "What TandemLLM is", section 1.7). No float atomics.
 *
 * Ownership and execution. The caller owns every buffer and stream. Calls are
 * asynchronous on `stream` (a cudaStream_t; NULL means the legacy default
 * stream) and do not synchronise, unless stated. The library keeps one small
 * per-device state (split-K workspace, error word, descriptor cache) created
 * by tl_init() or lazily by the first call on a device; call tl_init() before
 * capturing a stream into a CUDA graph (see "Allocation" below for when else a call
 * without a plan allocates). The host side of every entry point is
 * thread-safe. On the GPU, launches of one device share its workspace (split-K
 * partials and counters, the prepared X or X pieces of calls made without a plan): calls whose
 * kernels could overlap (different streams, or host threads without ordering)
 * must be serialised by the caller, e.g. by issuing them on one stream.
 *
 * Errors. Every entry point validates its arguments first: on a violation it
 * launches nothing and returns a status; tl_last_error_message() then holds a
 * one-line reason for the calling thread. Faults found on the device (a wait
 * that ran out, an invalid internal state) are recorded in a device status
 * word and reported by tl_check_device_error().
 */
#ifndef TL_NVFP4_H
#define TL_NVFP4_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TL_OK = 0,
    TL_ERR_INVALID_VALUE = 1,   /* a size or pointer argument is out of range */
    TL_ERR_MISALIGNED = 2,      /* a pointer is not 16-byte aligned */
    TL_ERR_UNSUPPORTED = 3,     /* valid request this library does not serve (e.g. M > 128) */
    TL_ERR_CUDA = 4,            /* a CUDA runtime/driver call failed */
    TL_ERR_TIMEOUT = 5,         /* a device-side wait ran past its iteration limit */
    TL_ERR_NOT_INITIALIZED = 6, /* no usable device / state */
    TL_ERR_NONFINITE = 7,       /* quantiser input holds NaN or infinity */
    TL_ERR_DEVICE_FAULT = 8     /* the device status word holds an internal error */
} tl_status;

/* Largest number of X rows one call serves. One launch serves up to 64 rows on the
 * block-scaled path and 32 on the exact and CUDA-core paths; a call with more rows runs as
 * groups of rows, each streaming the weights again. Plans take at most one launch's rows;
 * tl_nvfp4_verify_gemm_noalloc() takes at most 32. */
#define TL_NVFP4_MAX_M 128
/* K must be a positive multiple of this. */
#define TL_NVFP4_K_ALIGN 256
/* Largest number of matrices one tl_nvfp4_verify_stack() call takes. */
#define TL_NVFP4_MAX_STACK 1024

/* Tensor-core paths of tl_nvfp4_verify_gemm(), tl_nvfp4_verify_stack(),
 * tl_nvfp4_verify_stack_host() and of plans (a plan keeps the path that was selected
 * when it was created). tl_nvfp4_verify_gemm_noalloc() always takes TL_PATH_BF16_EXACT.
 *
 * TL_PATH_EXACT (the default). Exact operands on the f16 tensor-core MMA, fp32 accumulate:
 *   - W: CUDA cores turn each byte of codes into two f16 E2M1 values (hardware convert) and
 *     multiply by the block's E4M3 scale in f16. W' = e2m1 * e4m3 has at most 6 significant
 *     bits and lies in [2^-10, 2688], so it is exact in f16.
 *   - X: a small kernel first writes each row of X as f16(x * 2^-e_m), with e_m chosen so the
 *     row's largest |x| lands in [2^15, 2^16); every bf16 value within about 32 binades of
 *     the row's largest is then exact in f16. The epilogue multiplies row m by
 *     global_scale * 2^e_m. A row the kernel cannot reproduce exactly (a wider range, a NaN or
 *     infinity, or a largest |x| outside 2^-45 .. 2^75) is recomputed after the GEMM by an
 *     fp64 CUDA-core kernel from the bf16 X as given (slow, but such rows do not occur in
 *     activations). So every product is exact and only the fp32 sums round:
 *     |y - y_ref| <= 1e-3 * sum_k |x w| + 2^-8 |y_ref| holds for every input, and results
 *     are bit-exact wherever the exact result and its partial sums are representable.
 *   Needs scratch for the prepared X: 2*M*K bytes + 4*M + 256 bytes per matrix (each part
 *   rounded up to 256 bytes), owned by a plan, or (calls without a plan) one per-device
 *   buffer that grows to the largest size used (see "Allocation" below).
 *
 * TL_PATH_BF16_EXACT. The same exact arithmetic with the bf16 MMA: CUDA cores decode each
 * weight to bf16 with integer bit operations and X is used as given (no preparation, no
 * scratch). Slower: its decode is bound by the integer pipe.
 *
 * TL_PATH_BLOCK_SCALED (approximate; not the default). Before the GEMM, a small kernel
 * writes each row of X as a power of two times a sum of four NVFP4-shaped pieces (E2M1
 * codes with one E4M3 scale per 16 k; each piece codes what the pieces before it left
 * over), and the GEMM feeds the weights' codes and scales and those pieces straight into
 * the FP4 block-scaled MMA. It does NOT reproduce X exactly: each X element carries an
 * error of up to about 1.24e-3 of the largest |x| of its 16-element block, so the
 * per-element bound above is not guaranteed (a weight row with few nonzero weights, such as
 * an identity or one-hot matrix, can exceed it on an X element much smaller than its block's
 * largest). A row of X holding a NaN or an infinity gives NaN outputs for the whole row.
 * Scratch for the pieces: (4 * K/2 + 4 * K/16) * M + 4 * M bytes per matrix.
 *
 * All three paths have a fixed reduction order (runs are bit-identical) and compute each
 * row of Y independently of the other rows, so a row's result does not depend on M.
 * tl_set_gemm_path() returns TL_ERR_INVALID_VALUE for any other value. The setting is
 * process-wide; change it only while no call is in flight.
 *
 * Allocation. Plans allocate everything they need when they are created. Calls without a
 * plan (tl_nvfp4_verify_gemm, tl_nvfp4_verify_stack, tl_nvfp4_verify_stack_host) may allocate
 * device memory, and then synchronise the device first, only (a) at the first call on a
 * device (its per-device state), (b) when a call needs more path scratch than any earlier call
 * (the buffer grows and is kept), and (c) when a stack's descriptor table is larger than the
 * cache slot it lands in (eight slots; each grows to the largest table it has held, with a
 * pinned host staging buffer of the same size). Once those sizes have been reached, calls
 * neither allocate nor synchronise: a stack whose descriptors are not cached is uploaded with
 * an asynchronous copy on the call's stream. None of (a)-(c) may happen during stream capture
 * (the call returns TL_ERR_UNSUPPORTED): run each size once before capturing. */
#define TL_PATH_BLOCK_SCALED 0
#define TL_PATH_BF16_EXACT 1
#define TL_PATH_EXACT 2
tl_status tl_set_gemm_path(int path);
int tl_get_gemm_path(void);

/* Create the per-device state of `device` (workspace, status word). Idempotent.
 * Does not change the calling thread's current device. */
tl_status tl_init(int device);

/* Free every per-device state. No call may be in flight. */
void tl_shutdown(void);

/* Y = X . dequant(W)^T for one weight matrix (see the top of this file): one projection of the
 * verify pass, whose weights are four bits each with one scale per 16 (TandemLLM docs v0.12.0,
 * "What TandemLLM is", section 1.2).
 *   x      device bf16 [M][K], 16-byte aligned
 *   M      0..TL_NVFP4_MAX_M (0 is a no-op returning TL_OK; more returns TL_ERR_UNSUPPORTED)
 *   w_codes, w_scales  device, 16-byte aligned, layouts above
 *   global_scale       finite
 *   y      device bf16 [M][N], 16-byte aligned; must not overlap x or W
 *   N      >= 1;  K  > 0 and K % 256 == 0
 * Kernel: the selected tensor-core path (tl_set_gemm_path; tcgen05 MMAs with the
 * fp32 accumulator in tensor memory), persistent stream-K over all SMs; split-K
 * partials are combined in fixed k order. */
tl_status tl_nvfp4_verify_gemm(const void* x, int M, const void* w_codes, const void* w_scales,
                               float global_scale, void* y, int N, int K, void* stream);

/* The same operation on CUDA cores only (one warp per weight row, fp32 FMA; no tensor
 * cores, no workspace, no split-K). Same arguments, rules and determinism as
 * tl_nvfp4_verify_gemm(); an independent second GPU path for cross-checks and for the
 * smallest M, where the tensor-core tile is mostly padding. */
tl_status tl_nvfp4_verify_gemm_simt(const void* x, int M, const void* w_codes, const void* w_scales,
                                    float global_scale, void* y, int N, int K, void* stream);

/* tl_nvfp4_verify_gemm() for callers that cannot allocate device memory. The paper has
 * no counterpart to this entry point; it exists for deployment.
 *
 * Who needs it: a serving engine that gives all free HBM to its KV-cache pool at start-up
 * leaves nothing for a library's first-call workspace, and some host runtimes route all
 * device memory through their own pool and do not let a library call cudaMalloc. This
 * call allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 * Same arguments and rules as tl_nvfp4_verify_gemm(); it always runs the TL_PATH_BF16_EXACT
 * kernel (whatever tl_set_gemm_path() selected), with the same grid on GPUs of at most 160
 * SMs, so its results are bit-identical to tl_nvfp4_verify_gemm() under TL_PATH_BF16_EXACT.
 * Its split-K scratch is one static device array inside this library, 5 MiB (partials for
 * up to 160 CTAs, their counters, a status word), which every GPU that loads the library
 * holds until the process exits. Limits: M <= 32 (larger M returns TL_ERR_UNSUPPORTED with a
 * message); the grid is capped at 160 CTAs.
 *
 * When the memory is taken. The array belongs to the library's CUDA module, which the CUDA
 * runtime loads onto a device the first time the library touches that device (lazily, the
 * default since CUDA 12.2). For a caller that uses only this entry point that is the first
 * call, whose one-time set-up (with the device current: the array's device address and the
 * SM count) loads the module: the array and the module's code are allocated then, by the
 * runtime. Make that first call at start-up, before handing free memory to a pool, and
 * before capturing a stream into a graph. Later calls take no device memory.
 *
 * Every call shares the one array and each launch clears its counters first, so calls whose
 * kernels overlap on the GPU (different streams, or several host threads without ordering)
 * race and give undefined results: keep them on one stream. A device-side wait that runs out
 * is recorded in the array's status word, which tl_noalloc_check_error() (allocation-free)
 * and tl_check_device_error() read and clear. */
tl_status tl_nvfp4_verify_gemm_noalloc(const void* x, int M, const void* w_codes, const void* w_scales,
                                       float global_scale, void* y, int N, int K, void* stream);

/* One matrix of a layer stack. Every matrix has its own X and Y. */
typedef struct {
    const void* w_codes;   /* device uint8 [N][K/2] */
    const void* w_scales;  /* device uint8 [N][K/16] */
    const void* x;         /* device bf16 [M][K] */
    void* y;               /* device bf16 [M][N] */
    float global_scale;
    int N;
    int K;
} tl_nvfp4_matrix;

/* The verify GEMM of `n_mats` independent matrices (e.g. QKV, O, gate+up and
 * down of the served model's 64 layers; "What TandemLLM is", section 1.1) in one persistent launch: all matrices' k-tiles form one
 * work list that is split evenly over the SMs, so no SM idles at a matrix
 * boundary. `mats` is a HOST array read during the call; each entry obeys the
 * rules of tl_nvfp4_verify_gemm(), with the same M for all. 1 <= n_mats <=
 * TL_NVFP4_MAX_STACK. The matrices are independent: order of completion is
 * unspecified; each Y is deterministic. */
tl_status tl_nvfp4_verify_stack(const tl_nvfp4_matrix* mats, int n_mats, int M, void* stream);

/* End-to-end form of tl_nvfp4_verify_stack() for callers whose X and Y live
 * in host memory: copies X from `x_host` to `x_dev`, runs the stack, copies Y
 * from `y_dev` to `y_host`, all on `stream` (asynchronous; pinned host memory
 * makes the copies truly asynchronous). X_i (M x K_i bf16) sits at byte
 * offset sum_{j<i} 2*M*K_j of x_host and x_dev; Y_i (M x N_i bf16) at offset
 * sum_{j<i} 2*M*N_j of y_host and y_dev. The x and y fields of `mats` are
 * ignored. Offsets of each X_i/Y_i must stay 16-byte aligned (M*K_i and
 * M*N_i even multiples of 8 elements) or TL_ERR_MISALIGNED is returned. */
tl_status tl_nvfp4_verify_stack_host(const tl_nvfp4_matrix* mats, int n_mats, int M,
                                     const void* x_host, void* x_dev, void* y_host, void* y_dev,
                                     void* stream);

/* Plans: the descriptors of a stack built once, launched many times (the verify pass runs
 * every decoding round over the same weights; "What TandemLLM is", section 1.2).
 *
 * tl_nvfp4_plan_create() validates `mats` (same rules as tl_nvfp4_verify_stack),
 * encodes the TMA descriptors of every matrix and uploads them to the device once
 * (synchronous; must not run during stream capture). The plan keeps no pointer to
 * `mats`; it records the device pointers inside it, which must stay valid while the
 * plan is used. tl_nvfp4_plan_run() then only launches: a few microseconds of host
 * work, asynchronous on `stream`, and capturable into a CUDA graph.
 * tl_nvfp4_plan_run_host() is the end-to-end form: it requires that the plan's X_i
 * are packed back to back in one device buffer (X_{i+1} starts right after X_i) and
 * likewise the Y_i, then copies X from `x_host`, runs, and copies Y to `y_host`
 * (pinned host memory keeps the copies asynchronous); TL_ERR_INVALID_VALUE if the
 * plan's buffers are not packed. With two or more matrices the stack is cut into up to
 * 8 chunks of consecutive matrices (about equal weight bytes), each launched on its
 * own, so that the copy of X into chunk c + 1, the computation of chunk c and the copy
 * of Y out of chunk c - 1 overlap (two internal streams, ordered with `stream` by
 * events: the call is ordered after earlier work on `stream`, and later work on `stream`
 * sees all of Y copied out). The first such call builds the chunks (synchronous: it
 * allocates their descriptor tables and X-piece scratch, so not during stream capture).
 * Each chunk is scheduled on its own, so where the whole-stack run cuts an n-tile across
 * CTAs the chunked run may cut it elsewhere: its results are deterministic and within the
 * same tolerance, not always the same bits as tl_nvfp4_plan_run(). Destroy synchronises the
 * device before freeing.
 * One plan must not run on two streams at once (the runs share the split-K workspace
 * of the device; runs on one stream are ordered). */
typedef struct tl_nvfp4_plan_st* tl_nvfp4_plan;
tl_status tl_nvfp4_plan_create(const tl_nvfp4_matrix* mats, int n_mats, int M, tl_nvfp4_plan* plan_out);
tl_status tl_nvfp4_plan_run(tl_nvfp4_plan plan, void* stream);
tl_status tl_nvfp4_plan_run_host(tl_nvfp4_plan plan, const void* x_host, void* y_host, void* stream);
tl_status tl_nvfp4_plan_destroy(tl_nvfp4_plan plan);

/* Parity hook: w_out[n][k] = fp32(e2m1 * e4m3 * global_scale), rounded once
 * (the product e2m1 * e4m3 is exact); the weight format of "What TandemLLM is", section 1.2. w_out: device float [N][K], 16-byte
 * aligned. Same size rules as tl_nvfp4_verify_gemm(). */
tl_status tl_nvfp4_dequant(const void* w_codes, const void* w_scales, float global_scale,
                           float* w_out, int N, int K, void* stream);

/* Round-to-nearest NVFP4 quantiser (weight-pack builder). The pages build their packs with GPTQ
 * ("Installing TandemLLM", section 3.12), which needs a checkpoint and calibration data; this is
 * the plain round-to-nearest reading of the same format:
 *   g = fp32(absmax(w) / (6*448)); per 16-block s = E4M3_RNE_satfinite(absmax_block / 6 / g)
 *   in fp64; codes = E2M1_RNE(w / (e4m3(s) * g)) in fp64, ties to the even code, zero -> 0x0.
 * w: device float [N][K] (finite); codes/scales: device outputs as above.
 * Writes g to *global_scale_out (host). SYNCHRONISES `stream` (it reads g back).
 * Returns TL_ERR_NONFINITE, with outputs undefined, if w holds NaN or infinity. */
tl_status tl_nvfp4_quantize(const float* w, int N, int K, void* w_codes, void* w_scales,
                            float* global_scale_out, void* stream);

/* FP8 output head of the verify pass, with its greedy top-2 (the next row of the path).
 *
 * The pages keep the model's output head in FP8 while the projections are NVFP4 (TandemLLM docs
 * v0.12.0, "What TandemLLM is", section 1.2), and the agreement rule looks at the two best
 * logits, a near tie being a gap within one unit in the last place (same page, section 1.5). For
 * M tree rows:
 *     logits[m][n] = (sum_k x[m][k] * e4m3(w[n][k])) * s_n
 *     token = argmax_n (the lowest n among equal maxima), top1, top2 = the largest logit of the
 *     row without the token's entry, gap_ulp = (top1 - top2) / ulp_bf16(top1)
 * where ulp_bf16(v) = 2^(e - 7) for 2^e <= |v| < 2^(e + 1) (2^-133 below 2^-126).
 *   x            device bf16 [M][K], 16-byte aligned
 *   M            0..TL_HEAD_MAX_M (0 is a no-op)
 *   w_fp8        device uint8 [N][K] E4M3 ("fn") bytes, 16-byte aligned; 0x7F / 0xFF are NaN
 *   N            >= 2 (vocabulary rows);  K > 0 and K % 256 == 0
 *   tensor_scale s_n for every n when row_scales is NULL (finite)
 *   row_scales   NULL, or device float [N]: s_n per output row (the pages do not say which)
 *   logits       device float [M][N], 16-byte aligned, output (fp32, rounded once)
 *   top2         device tl_head_top2 [M], output; token -1 and NaN values for a row with a NaN
 * Arithmetic: exact f16 operands on the tensor cores (every E4M3 value is an f16 value; X rows
 * prepared as for TL_PATH_EXACT, with the same fp64 fallback for rows outside f16), fp32
 * accumulation. Three launches: X preparation, the GEMM, and one kernel that recomputes flagged
 * rows in fp64 and reduces every row to its top two (partials in the device's split-K scratch,
 * merged by the row's last CTA through a per-row counter it leaves at zero). Same scratch,
 * allocation and serialisation rules as the calls without a plan (the prepared-X buffer, the
 * split-K partials and counters of the device). Asynchronous on `stream`. */
#define TL_HEAD_MAX_M 32
typedef struct {
    int token;
    float top1;
    float top2;
    float gap_ulp;
} tl_head_top2;
tl_status tl_fp8_head(const void* x, int M, const void* w_fp8, int N, int K, float tensor_scale,
                      const float* row_scales, float* logits, tl_head_top2* top2, void* stream);

/* Closed-form commit of an accepted draft path through Gated DeltaNet states (a next row).
 *
 * 48 of the served model's 64 layers carry a recurrent state that cannot step back after a wrong
 * guess, so the engine commits the state of the accepted path in closed form (TandemLLM docs
 * v0.12.0, "What TandemLLM is", section 1.7; the author's "Research" page, StairCut abstract).
 * The pages print no equation; the rule taken is the gated delta rule, one token (key k, value v,
 * gate a, step b) mapping a head's state S (d_v x d_k) to
 *     S' = a S (I - b k k^T) + b v k^T,
 * and the call replaces every head's S by its state after the L tokens of the path, in order, in
 * one launch (a forward substitution over the path instead of L dependent updates).
 *   state     device float [H][d_v][d_k], 16-byte aligned; read and overwritten in place
 *   H         number of independent heads (layers x heads), >= 1
 *   d_k, d_v  64 or 128 each
 *   k         device float [n_nodes][H][d_k], 16-byte aligned: each draft-tree node's key per head
 *   v         device float [n_nodes][H][d_v]
 *   alpha     device float [n_nodes][H]: the gate a of each node and head
 *   beta      device float [n_nodes][H]: the step b
 *   path      HOST int [L]: the accepted nodes in path order, each in 0..n_nodes-1
 *   L         0..TL_GDN_MAX_PATH (0 is a no-op)
 * fp32 arithmetic on CUDA cores; no workspace, no allocation. Asynchronous on `stream`; the
 * host path array is copied into the launch and may be reused at once. Errors: a size out of
 * range, a node index outside 0..n_nodes-1, a null or misaligned pointer, a state buffer that
 * overlaps k, v, alpha or beta -> the status, nothing launched. */
#define TL_GDN_MAX_PATH 32
tl_status tl_gdn_commit(float* state, int H, int d_k, int d_v, const float* k, const float* v, const float* alpha,
                        const float* beta, int n_nodes, const int* path, int L, void* stream);

/* Synchronise `stream`, then report and clear the device status word:
 * TL_OK, TL_ERR_TIMEOUT (a bounded wait ran out) or TL_ERR_DEVICE_FAULT. Also reads and
 * clears the status word of tl_nvfp4_verify_gemm_noalloc()'s static scratch on the current
 * device. After a timeout it clears every split-K counter of the device. Creates the
 * per-device state if the device has none (allocates). */
tl_status tl_check_device_error(void* stream);

/* The allocation-free check for callers of tl_nvfp4_verify_gemm_noalloc(): synchronise
 * `stream`, then report and clear the status word of the static scratch on the current
 * device (TL_OK if the entry point never ran there). Touches no other state. */
tl_status tl_noalloc_check_error(void* stream);

/* Self-test of the device-side failure path: launches one thread that waits, with the
 * library's bounded wait, on an mbarrier that nothing completes, for at most
 * `iterations` polls; when the limit runs out it records a timeout in the device
 * status word and returns, leaving the context usable. The next
 * tl_check_device_error() then reports TL_ERR_TIMEOUT. Touches no caller memory. */
tl_status tl_selftest_bounded_wait(unsigned iterations, void* stream);

/* Number of SMs the persistent kernels use on `device` (after tl_init). */
int tl_num_sms(int device);

/* Static strings; never NULL. */
const char* tl_status_string(tl_status status);
const char* tl_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* TL_NVFP4_H */
