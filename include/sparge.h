/*
 * sparge.h -- C ABI of the B200 (sm_100a) SpargeAttn sparse-attention forward.
 *
 * The method is the two-stage filtered sparse FlashAttention of "SpargeAttn:
 * Accurate and Training-free Sparse Attention Accelerating Any Model
 * Inference" (paper review page, section 三 技术架构, Algorithm 1):
 *   stage 1  block-mask prediction from mean-pooled Q/K blocks (Eq. 4-9);
 *   stage 2  block-sparse online-softmax attention with the per-warp lambda
 *            skip of P~V (Eq. 1-3);
 *   plus     the Hilbert-curve token permutation for visual tokens
 *            (same page, "HilbertCurve Permutation").
 *
 * Conventions shared by every entry point
 *   Layout     Q [B, Hq, N, d], K and V [B, Hkv, N, d], O [B, Hq, N, d],
 *              row-major with d contiguous; every base pointer 16-byte aligned.
 *              Query head h reads KV head h / (Hq / Hkv).
 *   Memory     Every pointer argument is DEVICE memory unless stated, allocated
 *              and owned by the caller.  The library allocates nothing, keeps no
 *              state between calls and is re-entrant for calls with distinct
 *              workspaces.
 *   Streams    Every call is asynchronous on the given stream; no call
 *              synchronises except sparge_device_status.
 *   Devices    A call runs on the device that owns its (first) device
 *              pointer and leaves the caller's current device as it was.
 *   Errors     Arguments are validated on the host before any launch:
 *              SPARGE_EINVAL (bad pointer, size or hyper-parameter),
 *              SPARGE_EUNSUPPORTED (valid but not implemented, e.g. d = 96,
 *              b_q != 128, b_k != 64, or more than 5952 key blocks: N > 380,928),
 *              SPARGE_EWORKSPACE (workspace too small), SPARGE_ECUDA (a CUDA
 *              runtime call or launch failed).  Nothing is launched when a call
 *              returns an error.  Kernels never trap: a device-side wait that
 *              runs out of time writes SPARGE_ETIMEOUT into the workspace
 *              status word and the kernel returns; sparge_device_status reads it.
 *   Blocks     bq = 128 query rows, bk = 64 key rows (the pages' b_q, b_k);
 *              c_w = bq / 32 = 4 warps of 32 query rows each for the lambda
 *              test; T_m = ceil(N / bq), T_n = ceil(N / bk).
 */
#ifndef SPARGE_H_
#define SPARGE_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPARGE_OK = 0,
  SPARGE_EINVAL = 1,
  SPARGE_EUNSUPPORTED = 2,
  SPARGE_ECUDA = 3,
  SPARGE_ETIMEOUT = 4,
  SPARGE_EWORKSPACE = 5,
  SPARGE_ERANGE = 6 /* a bf16 V value did not fit fp16 (P~V runs in fp16); it was saturated */
} sparge_status_t;

typedef enum { SPARGE_F16 = 0, SPARGE_BF16 = 1, SPARGE_F32 = 2 } sparge_dtype_t;

/* Hyper-parameters of one attention call (Algorithm 1 "Input" line). */
typedef struct {
  int32_t B, Hq, Hkv, N, d; /* d in {64, 128}; Hq % Hkv == 0; N >= 0            */
  int32_t bq, bk;           /* must be 128 and 64                               */
  float tau;                /* TopCdf mass, Eq. 8; (0, 1], >= 1 keeps all       */
  float theta;              /* self-similarity threshold, Eq. 7 and Eq. 9       */
  float lambda;             /* P~V skip threshold of Eq. 3, natural-log units;
                               <= 0, -INFINITY disables the skip                */
  float scale;              /* score scale, normally 1/sqrt(d) (Eq. 1)          */
  int32_t causal;           /* 1: key n is visible to query m iff n <= m        */
  int32_t qk_int8;          /* 1: per-block INT8 Q K^T with K mean smoothing
                               (Algorithm 1 steps 2 and 10; d = 128 only)       */
  sparge_dtype_t io_dtype;  /* dtype of Q, K, V: SPARGE_F16 or SPARGE_BF16      */
  sparge_dtype_t o_dtype;   /* dtype of O: io_dtype or SPARGE_F32               */
} sparge_params_t;

/* Per-call work counters, accumulated with atomics into caller-zeroed device
 * memory.  A "slice" is one warp's 32 query rows of one (tile, key block). */
typedef struct {
  unsigned long long tiles;          /* query tiles processed                    */
  unsigned long long qk_blocks;      /* Q_i K_j^T block products computed         */
  unsigned long long pv_blocks;      /* P~_ij V_j products issued (any slice on) */
  unsigned long long pv_slices;      /* slices whose P~V was kept                 */
  unsigned long long skipped_slices; /* slices skipped by the lambda test (Eq. 3) */
} sparge_stats_t;

/* Bytes of workspace that sparge_predict_mask and sparge_attn_fwd need for
 * these parameters.  The SAME workspace must be passed to both calls of one
 * forward: with qk_int8 the predictor writes the INT8 codes there and the
 * attention reads them.  Returns 0 for invalid parameters. */
size_t sparge_workspace_bytes(const sparge_params_t* p);

/* Hilbert permutation table (paper review page, "HilbertCurve Permutation";
 * rebuttal page, reply to Weakness 3).  Tokens are laid out as
 * [prefix_len text tokens | T x Hg x Wg grid, (t, y, x) row-major | rest].
 * Axes of extent 1 are dropped; the remaining axes, in order (t, y, x), index
 * a Hilbert curve on the smallest 2^b cube holding them (Skilling's transpose
 * form).  Writes perm[N] (device, int32) with y[p] = x[perm[p]]: prefix and
 * trailing tokens keep their place, grid tokens follow the curve.
 * ws: device workspace of sparge_hilbert_workspace_bytes(T, Hg, Wg) bytes. */
size_t sparge_hilbert_workspace_bytes(int32_t T, int32_t Hg, int32_t Wg);
sparge_status_t sparge_hilbert_index(int32_t N, int32_t prefix_len, int32_t T, int32_t Hg,
                                     int32_t Wg, int32_t* perm, void* ws, size_t ws_bytes,
                                     cudaStream_t stream);

/* y[b, h, p, :] = x[b, h, perm[p], :] for x, y [B, H, N, d] of dtype (16-bit
 * or f32).  perm is a device array of N int32 entries, normally a
 * permutation of 0..N-1 (e.g. from sparge_hilbert_index); a row whose entry
 * lies outside [0, N) is skipped (y's row is left as it was).  x and y must
 * not overlap (SPARGE_EINVAL).  A row of d elements must be a multiple of 16
 * bytes and B * H at most 65535 (SPARGE_EUNSUPPORTED otherwise); B, H or
 * N = 0 is a no-op.  HBM-bound: each row is read once and written once. */
sparge_status_t sparge_hilbert_permute(const void* x, void* y, int32_t B, int32_t H, int32_t N,
                                       int32_t d, sparge_dtype_t dtype, const int32_t* perm,
                                       cudaStream_t stream);

/* The inverse: x[b, h, perm[p], :] = y[b, h, p, :], under the same rules (a
 * row whose entry lies outside [0, N) is not written).  perm should be a
 * permutation: if two in-range entries are equal, both source rows are
 * written to the same destination row and which one remains is unspecified. */
sparge_status_t sparge_inverse_permute(const void* y, void* x, int32_t B, int32_t H, int32_t N,
                                       int32_t d, sparge_dtype_t dtype, const int32_t* perm,
                                       cudaStream_t stream);

/* Stage 1, Algorithm 1 steps 2-5 (Eq. 4-9): block means q_i, k_j, CosSim
 * self-similarities s_q, s_k (mean of the block's token cosine matrix), the
 * compressed map S_hat = scale * q k^T with -inf columns where s_k < theta
 * (and causal-future blocks), row softmax, TopCdf(tau), the fix-block rule.
 * Outputs (device):
 *   mask   [B, Hq, T_m, T_n] uint8 M_g (1 = compute block)
 *   kv_idx [B, Hq, T_m, T_n] int32: the kept j of each tile in ascending order,
 *          first kv_cnt entries valid (the rest are left unspecified)
 *   kv_cnt [B, Hq, T_m] int32
 *   s_q    [B, Hq, T_m] float, s_k [B, Hkv, T_n] float (both nullable)
 * With qk_int8 it also quantises Q and K - mean(K) per block into ws
 * (Algorithm 1 step 2): mean(K) is the per-head mean over all N tokens, summed
 * in float64 and rounded once to float32; per block delta = absmax / 127 and
 * code = round-half-even(x / delta) of the IEEE float32 quotient. */
sparge_status_t sparge_predict_mask(const sparge_params_t* p, const void* q, const void* k,
                                    uint8_t* mask, int32_t* kv_idx, int32_t* kv_cnt, float* s_q,
                                    float* s_k, void* ws, size_t ws_bytes, cudaStream_t stream);

/* The two halves of sparge_predict_mask, for callers that time or schedule
 * them apart.  sparge_predict_pool is Algorithm 1 steps 2-3 (Eq. 4-6): block
 * means, CosSim self-similarities and, with qk_int8, the INT8 codes of Q and
 * K - mean(K) with their scales, all written into ws (the HBM-bound pass over
 * Q and K).  sparge_predict_select is steps 4-5 (Eq. 7-9): S_hat, softmax,
 * TopCdf, the fix rule, mask / kv_idx / kv_cnt (and the optional s_q, s_k
 * copies) computed from what sparge_predict_pool left in the same ws, which
 * must therefore run first on the same stream (or be ordered before it).
 * Arguments, layouts and errors as for sparge_predict_mask; pool checks q and
 * k, select checks the outputs. */
sparge_status_t sparge_predict_pool(const sparge_params_t* p, const void* q, const void* k,
                                    void* ws, size_t ws_bytes, cudaStream_t stream);
sparge_status_t sparge_predict_select(const sparge_params_t* p, uint8_t* mask, int32_t* kv_idx,
                                      int32_t* kv_cnt, float* s_q, float* s_k, void* ws,
                                      size_t ws_bytes, cudaStream_t stream);

/* sparge_predict_mask without a workspace, for callers that cannot allocate
 * device memory at call time and have no workspace to pass in (a plugin whose
 * host framework owns every device buffer, a serving loop that must not call
 * the allocator after start-up).  The paper has no counterpart: this is a
 * deployment variant of the stage-1 predictor above, with the same outputs.
 * Its scratch (pooled block means and self-similarities) lives in one static
 * 32 MiB device array compiled into the library; every GPU that loads the
 * library holds that array until the process exits.  The predictor's regions
 * must fit: 256 + align256(B*Hq*T_m*d*4) + align256(B*Hkv*T_n*d*4)
 * + align256(B*Hq*T_m*4) + align256(B*Hkv*T_n*4) <= 32 MiB, else the call
 * returns SPARGE_EWORKSPACE (align256 rounds up to a multiple of 256).
 * qk_int8 = 1 returns SPARGE_EUNSUPPORTED (the INT8 codes must outlive the
 * call); otherwise a parameter set gets the same status as from
 * sparge_predict_mask (SPARGE_EINVAL or SPARGE_EUNSUPPORTED).  The first call
 * on each device looks up the array's device address there
 * (cudaGetSymbolAddress), so make that first call before any stream capture.
 * The call allocates nothing.  All calls share the array and it keeps the
 * last call's contents; each call rewrites every region it reads, so nothing
 * has to be cleared, but calls whose kernels overlap on the GPU (unordered
 * streams) race on it.  The predictor has no device-side waits, so these
 * calls leave no device status to read (there is no workspace to hold one). */
sparge_status_t sparge_predict_mask_noalloc(const sparge_params_t* p, const void* q,
                                            const void* k, uint8_t* mask, int32_t* kv_idx,
                                            int32_t* kv_cnt, float* s_q, float* s_k,
                                            cudaStream_t stream);

/* Compacts a caller-built mask [B, Hq, T_m, T_n] (uint8, nonzero = keep) into
 * the kv_idx / kv_cnt skip list sparge_attn_fwd consumes: Algorithm 1 step 9
 * visits, for query block i, the key blocks j with M_g[i, j] = 1 in ascending
 * order, and Eq. 2 skips the others; this is that visiting order.  Causal-
 * future blocks are kept if the mask keeps them (the attention masks them
 * anyway).  Outputs as for sparge_predict_mask; errors as for every entry
 * point (SPARGE_EINVAL for null or misaligned pointers). */
sparge_status_t sparge_mask_compact(const sparge_params_t* p, const uint8_t* mask,
                                    int32_t* kv_idx, int32_t* kv_cnt, cudaStream_t stream);

/* Stage 2, Algorithm 1 steps 6-17 (Eq. 1-3): for every query tile i, the key
 * blocks kv_idx[..., :kv_cnt] in the listed order: S = scale Q_i K_j^T (INT8
 * codes times the block scales with qk_int8), online softmax of Eq. 1, then
 * P~V for every 32-row warp slice whose max(m_local - m_new) >= lambda.
 * O_i = O / l; a row with l = 0 outputs 0.  P~V runs in fp16 with fp32
 * accumulation (V is converted from bf16 into ws when io_dtype is bf16).
 * stats: nullable device pointer to caller-zeroed counters.
 * ws: the workspace passed to sparge_predict_mask (required with qk_int8). */
sparge_status_t sparge_attn_fwd(const sparge_params_t* p, const void* q, const void* k,
                                const void* v, const int32_t* kv_idx, const int32_t* kv_cnt,
                                void* o, void* ws, size_t ws_bytes, sparge_stats_t* stats,
                                cudaStream_t stream);

/* Synchronises the stream and returns the status word that kernels write to
 * the workspace (SPARGE_OK, SPARGE_ETIMEOUT or SPARGE_ERANGE), then clears it.
 * ws: the workspace of sparge_predict_mask / sparge_attn_fwd. */
sparge_status_t sparge_device_status(void* ws, cudaStream_t stream);

/* Failure-detection self-test (no counterpart in the paper): launches one
 * CTA whose time-bounded mbarrier wait -- the same wait the attention kernel
 * uses -- is on a phase that nothing ever completes.  The wait gives up after
 * its 1 s limit and writes SPARGE_ETIMEOUT into the status word of ws, which
 * sparge_device_status then returns (and clears).  Nothing faults, traps or
 * hangs; the context stays usable.  ws: any workspace of at least 256 bytes. */
sparge_status_t sparge_selftest_wait_timeout(void* ws, cudaStream_t stream);

/* Static description of a status code (never NULL). */
const char* sparge_status_string(sparge_status_t s);

#ifdef __cplusplus
}
#endif

#endif /* SPARGE_H_ */
