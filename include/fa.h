/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library (libfa_b200.so).
 *
 * The operation is exact scaled-dot-product attention, O = softmax(scale * Q K^T) V,
 * computed FlashAttention-style: Q, K and V are tiled into on-chip memory, the
 * score tile, the online softmax (running row maximum and sum with rescaling) and
 * the P.V product are fused in one kernel, and the N x N score matrix never
 * reaches device memory ("Flash Attention Explained", institutepm.com, section
 * "How Flash Attention Fixes It: Tiling and Recomputation"; holysheep.ai review,
 * section "What Is Flash Attention and Why Does It Matter?").  The backward pass
 * recomputes score tiles from the saved per-row log-sum-exp instead of storing
 * the matrix (same page, "Recompute during backward pass").
 *
 * Tensor layout (the flash_attn_func interface of the holysheep.ai review,
 * section "Implementing Flash Attention in Your Architecture"):
 *   q, k, v, o, dO, dq, dk, dv : bf16, [B, N, H, d] contiguous (d innermost),
 *                                element (b, n, h, x) at ((b*N + n)*H + h)*d + x.
 *   lse                        : fp32, [B, H, N] contiguous, natural-log
 *                                log-sum-exp of the scaled visible scores of each
 *                                query row: lse = ln sum_j exp(scale * q.k_j).
 * Queries and keys have the same length N.  causal = 1 lets query i see keys
 * j <= i only ("Flash Attention vs Standard Attention", avichala.com, section
 * "Engineering Perspective": autoregressive masking).  scale is the softmax
 * scale; callers normally pass 1/sqrt(d), the default of the same interface.
 *
 * Pointers: every tensor pointer is a DEVICE pointer on the current CUDA device,
 * 16-byte aligned (lse: 4-byte aligned), owned by the caller.  The library never
 * allocates or frees device memory and keeps no per-call state; it caches the
 * per-device kernel attributes and owns one small device status word.
 *
 * Execution: every call is asynchronous on `stream` (a cudaStream_t passed as
 * void*; NULL = the legacy default stream).  Arguments are validated on the host
 * BEFORE anything is enqueued; on any error nothing is launched.  Errors of the
 * asynchronous execution surface on the caller's next synchronisation, and a
 * kernel that had to give up on a bounded wait records FA_ERR_TIMEOUT in the
 * status word read by fa_get_status().  No exception crosses the ABI and there
 * is no fallback path: an unsupported case returns an error code.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* NULL pointer, B/H/N < 1, scale not finite and > 0, causal not 0/1, sizes overflow */
  FA_ERR_UNSUPPORTED = 2, /* head dimension d other than 64 or 128 */
  FA_ERR_ALIGNMENT = 3,   /* a tensor pointer not 16-byte aligned (lse: 4-byte) */
  FA_ERR_DEVICE = 4,      /* no usable CUDA device, or the current device is not sm_100 */
  FA_ERR_LAUNCH = 5,      /* kernel attribute setup or launch failed */
  FA_ERR_TIMEOUT = 6,     /* a kernel abandoned a bounded wait (reported by fa_get_status) */
  FA_ERR_WORKSPACE = 7,   /* workspace pointer NULL or smaller than the required size */
  FA_ERR_BOUNDS = 8       /* checking build only: a kernel's index left its tensor (fa_get_status) */
} fa_status;

/* Library ABI version (this header: 6; 6 added fa_get_status_site). */
int fa_abi_version(void);

/*
 * The checking build.  libfa_b200_checks.so is the same library compiled with FA_CHECKS:
 * before every TMA copy and every global load or store it computes, each kernel compares the
 * coordinates or index with the extent of the tensor addressed.  A violation records
 * FA_ERR_BOUNDS and the check's site in the device status word and skips the access (a
 * skipped copy leaves its barrier short, so the kernel unwinds through its bounded waits);
 * fa_get_status() then returns FA_ERR_BOUNDS.  It stands in for a memory checker where none
 * can run, and is slower; results are otherwise the same as the release library's.
 * fa_checks_enabled() returns 1 in the checking build and 0 in the release build.
 */
int fa_checks_enabled(void);

/*
 * Problem description for the _ex entry points.
 *   B, N, d      : batch, sequence length (queries and keys), head dimension (64 or 128)
 *   H            : query heads
 *   H_kv         : key/value heads, 1 <= H_kv <= H and H % H_kv == 0; query head h uses
 *                  key/value head h / (H / H_kv) -- grouped-query attention, and multi-query
 *                  attention for H_kv = 1 ("Flash Attention Explained", institutepm.com,
 *                  "Grouped Query Attention": orthogonal to Flash Attention).  H_kv = H is
 *                  ordinary multi-head attention.
 *   scale        : softmax scale (> 0, finite)
 *   causal       : 0 or 1
 *   window       : -1 for none; >= 0 (causal only) limits query i to keys i - window .. i,
 *                  sliding-window attention (same page, "Sliding Window Attention").
 *   dtype        : element type of every tensor except lse: FA_DTYPE_BF16 or FA_DTYPE_F16
 *                  (fp16, the type of the pages' memory example: "What Is Flash Attention?",
 *                  bestllmfor.com, the score-matrix size table).  Arithmetic is the same:
 *                  16-bit products, fp32 accumulation and softmax statistics.
 *                  FA_DTYPE_E4M3 (forward only, d = 128): q, k, v are fp8 e4m3 bytes, o is
 *                  bf16; see fa_fwd_e4m3_scaled.
 * Tensors: q, o, dO, dq are [B, N, H, d]; k, v, dk, dv are [B, N, H_kv, d]; lse is [B, H, N].
 */
typedef enum { FA_DTYPE_BF16 = 0, FA_DTYPE_F16 = 1, FA_DTYPE_E4M3 = 2 } fa_dtype;

typedef struct fa_problem {
  int B;
  int H;
  int H_kv;
  int N;
  int d;
  float scale;
  int causal;
  int window;
  int dtype;
} fa_problem;

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(int status);

/*
 * Forward pass: o = softmax(scale * q k^T [masked]) v and lse per query row.
 *   q, k, v : in,  bf16 [B, N, H, d]
 *   o       : out, bf16 [B, N, H, d]
 *   lse     : out, fp32 [B, H, N]
 *   d       : 64 or 128
 * Deterministic: the same inputs give bitwise-identical outputs.
 * Device memory used beyond the arguments: none.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, void* stream);

/* fa_fwd for a general problem (grouped-query heads, sliding window, bf16 or fp16 tensors).
 * Errors as fa_fwd, plus FA_ERR_INVALID_ARG for a NULL problem, H_kv not dividing H,
 * window < -1, or a window without causal masking, and FA_ERR_UNSUPPORTED for an unknown
 * dtype. */
fa_status fa_fwd_ex(const fa_problem* problem, const void* q, const void* k, const void* v, void* o,
                    float* lse, void* stream);

/*
 * Forward pass with fp8 e4m3 inputs (FlashAttention-3's FP8 forward: "Flash Attention
 * Explained", institutepm.com, section "Flash Attention 1, 2, and 3").  problem->dtype must
 * be FA_DTYPE_E4M3 and problem->d 128.  q, k, v hold e4m3 codes (1 byte per element, same
 * [B, N, H(_kv), d] layout); the values they stand for are code * descale, one positive
 * finite factor per tensor.  o is bf16 [B, N, H, d], lse fp32 [B, H, N] as in fa_fwd.
 * Q K^T is formed exactly from the codes on the tensor cores (fp32 accumulation) and scaled
 * by scale * q_descale * k_descale; the softmax weights are rounded to e4m3 for the P.V
 * product and normalised by the sum of the rounded weights, O is scaled by v_descale; the
 * LSE uses the unrounded fp32 sum.  fa_fwd_ex with this dtype is this call with descales 1.
 * Errors as fa_fwd_ex, plus FA_ERR_INVALID_ARG for a dtype other than FA_DTYPE_E4M3 or a
 * descale that is not positive and finite.
 */
fa_status fa_fwd_e4m3_scaled(const fa_problem* problem, const void* q, const void* k, const void* v,
                             float q_descale, float k_descale, float v_descale, void* o, float* lse, void* stream);

/*
 * Bytes of device workspace fa_bwd needs for these sizes: an fp32 dQ accumulator
 * [B, H, N, d], then the fp32 row sums D_i = sum_x dO_ix O_ix and the fp32 LSE_i * log2(e),
 * each [B*H, Npad] with Npad = N rounded up to a multiple of 128; in total
 * 4*B*H*(N*d + 2*Npad) bytes.  Returns 0 for sizes fa_bwd rejects (B, H, N < 1, d not
 * 64 / 128, or more elements than its index range allows).
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass of L = sum(o * dO): dq, dk, dv, recomputing the score tiles from
 * q, k and the saved lse (no N x N matrix is stored or read).
 *   q, k, v, o, dO : in,  bf16 [B, N, H, d]   (o and lse as returned by fa_fwd)
 *   lse            : in,  fp32 [B, H, N]
 *   dq, dk, dv     : out, bf16 [B, N, H, d]
 *   workspace      : device scratch of at least fa_bwd_workspace_size(B, H, N, d)
 *                    bytes, 16-byte aligned, caller-owned; its contents on entry do
 *                    not matter and are overwritten.
 *   scale, causal  : the values passed to fa_fwd.
 * Errors: FA_ERR_WORKSPACE if workspace is NULL or too small; otherwise as fa_fwd.
 * dk and dv are deterministic; dq is accumulated with fp32 atomics and may differ in
 * the last bits between runs.  Calls sharing one workspace must not overlap.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
                 float scale, int causal, void* stream);

/* Workspace bytes fa_bwd_ex needs for a problem (same as fa_bwd_workspace_size for its
 * B, H, N, d: the accumulator and statistics are per query head). 0 for a NULL problem. */
size_t fa_bwd_workspace_size_ex(const fa_problem* problem);

/* fa_bwd for a general problem (all 16-bit tensors in the problem's dtype; FA_DTYPE_E4M3
 * returns FA_ERR_UNSUPPORTED): k, v, dk, dv are [B, N, H_kv, d]; dK and dV of a shared
 * key/value head accumulate the contributions of all H / H_kv query heads that use it.
 * Errors as fa_bwd, plus those of fa_fwd_ex for the problem. */
fa_status fa_bwd_ex(const fa_problem* problem, const void* q, const void* k, const void* v, const void* o,
                    const void* dO, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * fa_bwd without a workspace argument, for callers that cannot allocate device memory:
 * for example code running where every byte of device memory is already handed to
 * another allocator, or where the implicit synchronisation of cudaMalloc / cudaFree is
 * not acceptable.  (The pages describe no such entry point; it has no counterpart there.)
 * It performs the same computation as fa_bwd, with the same arguments minus the
 * workspace, and calls no cudaMalloc, cudaFree or other allocating routine.  Like fa_bwd
 * it covers bf16 tensors with H_kv == H and no sliding window only; fp16, grouped-query
 * and windowed problems go through fa_bwd_ex with a caller-provided workspace.
 *
 * Scratch: a fixed 64 MiB array inside the library holding what fa_bwd's workspace would
 * (fa_bwd_workspace_size bytes).  Problems that need more return FA_ERR_WORKSPACE and launch
 * nothing; use fa_bwd with a caller-provided workspace for those.  Every GPU that loads
 * the library holds this array until the process exits, whether or not this entry point
 * is used.  All calls on a device share the one array: calls whose work can overlap on
 * the GPU (different streams without ordering between them) race and corrupt each
 * other's results; serialise them.  Whatever must start at zero is cleared by each call.
 *
 * The first call on each device looks up the array's device address (once per device,
 * with that device current); make that first call before any CUDA stream capture.
 */
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
                         int causal, void* stream);

/*
 * ---------------------------------------------------------------- decoding
 * Attention of a few NEW queries per sequence against a key/value cache: the generation
 * phase, as opposed to prompt processing ("What Is Flash Attention?", bestllmfor.com,
 * table "What you actually gain on a local machine").  The result is the same exact
 * softmax(scale * q K^T) V over each query's visible cached keys; the cache is split
 * over all SMs and the pieces are combined by their log-sum-exps.
 *
 *   B        : sequences
 *   H, H_kv  : query heads and key/value heads (H % H_kv == 0; query head h reads
 *              key/value head h / (H / H_kv))
 *   N_q      : new queries per sequence, 1 for plain decoding (more for, e.g., verifying
 *              several drafted tokens at once)
 *   N_kv     : cache capacity: positions per sequence in k_cache / v_cache
 *   d        : 64 or 128
 *   scale    : softmax scale (> 0, finite)
 *   causal   : 1: query i of sequence b stands at position len_b - N_q + i, right after
 *              the cached prefix it extends, and sees the cached keys at or before that
 *              position; 0: every query sees all len_b cached keys
 *   window   : -1, or >= 0 with causal = 1: a query at position t sees keys t - window .. t
 *   dtype    : FA_DTYPE_BF16 or FA_DTYPE_F16, the type of q, the caches and o
 * Constraint: (H / H_kv) * N_q <= 128 (the rows one key/value head contributes to a
 * 128-row tile); larger groups return FA_ERR_UNSUPPORTED.
 */
typedef struct fa_decode_problem {
  int B;
  int H;
  int H_kv;
  int N_q;
  int N_kv;
  int d;
  float scale;
  int causal;
  int window;
  int dtype;
} fa_decode_problem;

/*
 * Bytes of device workspace fa_decode needs on the CURRENT device (the split over its SMs
 * sets the number of partial results): 256-byte-aligned regions for the schedule
 * (4 * (2 + B) bytes), the partial log-sum-exps (8 * S * M) and the partial outputs
 * (4 * S * M * d), with M = (H / H_kv) * N_q and S = R * (SMs + B * H_kv - 1), where
 * R = 4 when M <= 16, 2 when M <= 32, else 1 (the copies of a head group's rows a tile holds).
 * Returns 0 for an invalid or unsupported problem or without an sm_100 device.
 */
size_t fa_decode_workspace_size(const fa_decode_problem* problem);

/*
 * Decoding forward.
 *   q        : in,  bf16 [B, N_q, H, d]
 *   k_cache  : in,  bf16 [B, N_kv, H_kv, d]; only the first len_b positions of sequence b
 *              are read as keys: the rest may hold anything (stale values, NaN)
 *   v_cache  : in,  bf16 [B, N_kv, H_kv, d], same rule
 *   seqlens  : in,  DEVICE int32 [B]: len_b, the cached length of each sequence (values
 *              are clamped to [0, N_kv]), or NULL: every sequence is N_kv long.  Read by
 *              the kernels, so a captured CUDA graph can be replayed as lengths grow.
 *   o        : out, bf16 [B, N_q, H, d]
 *   lse      : out, fp32 [B, H, N_q], natural-log log-sum-exp of each query's visible scores
 *   workspace: device scratch of at least fa_decode_workspace_size() bytes, 256-byte
 *              aligned; contents on entry do not matter
 * A query that sees no key (len_b = 0, or a position before the start of the cache) gets
 * O = 0 and LSE = -inf.  Deterministic for fixed inputs and device.  Errors: as fa_fwd,
 * FA_ERR_INVALID_ARG for a bad problem (a window without causal masking included),
 * FA_ERR_UNSUPPORTED beyond the constraint above, FA_ERR_ALIGNMENT, FA_ERR_WORKSPACE.
 */
fa_status fa_decode(const fa_decode_problem* problem, const void* q, const void* k_cache, const void* v_cache,
                    const int* seqlens, void* o, float* lse, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * Failure-detection self-test: launches one warp that waits on a barrier nothing will
 * arrive on, through the same bounded wait the attention kernels use, with a bound of
 * timeout_us microseconds (1 .. 1000000).  The wait runs out, the kernel records
 * FA_ERR_TIMEOUT in the device status word and returns; nothing faults or hangs and the
 * context stays usable.  A following fa_get_status() returns FA_ERR_TIMEOUT.
 * Returns FA_ERR_INVALID_ARG for a bound out of range, FA_ERR_DEVICE without an sm_100
 * device, FA_ERR_LAUNCH if the launch fails, else FA_OK.
 */
fa_status fa_selftest_wait_timeout(unsigned int timeout_us, void* stream);

/*
 * Checking-build self-test: launches one warp whose bounds check is given an index outside
 * its (one-element, shared-memory) target, so the check fails by construction and the access
 * is skipped; nothing outside the target is touched.  In the checking build the kernel
 * records FA_ERR_BOUNDS and a following fa_get_status() returns it; the release build has no
 * checks and returns FA_ERR_UNSUPPORTED without launching.  FA_ERR_DEVICE without an sm_100
 * device, FA_ERR_LAUNCH if the launch fails, else FA_OK.
 */
fa_status fa_selftest_bounds(void* stream);

/*
 * Synchronises `stream`, then returns and clears the device status word of the
 * current device: FA_OK, FA_ERR_TIMEOUT if a kernel gave up a bounded wait since the
 * last call, or (checking build) FA_ERR_BOUNDS if a bounds check failed.  Returns FA_ERR_DEVICE if the stream or device reports a
 * CUDA error.
 */
fa_status fa_get_status(void* stream);

/*
 * fa_get_status, and in *site (if not NULL) where the first recorded error arose: for
 * FA_ERR_TIMEOUT the wait that ran out (forward: 1 loads, 2 MMA, 3 and 4 the softmax of the
 * first and second query block; backward: 11 loads, 12 MMA, 13 key rows, 14 dQ drain;
 * decode: 21 loads, 22 MMA, 23 softmax; 98 the final wait for issued MMAs or a wait while
 * unwinding after an abort; 99 the self-test),
 * for FA_ERR_BOUNDS the check that failed (three-digit sites, 999 the self-test); 0 when
 * none was recorded.  The sources name each site beside its wait or check.
 */
fa_status fa_get_status_site(void* stream, int* site);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
