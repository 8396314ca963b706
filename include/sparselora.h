/*
 * sparselora.h - C ABI of libsparselora.so, a B200 (sm_100a) implementation of the
 * hot path of SparseLoRA: the contextually sparse frozen-main-branch linear layer of
 * a LoRA fine-tuning step.
 *
 * Sources (cited by page title and section):
 *   [WT] "SparseLoRA: Accelerating LLM Fine-Tuning with Contextual Sparsity",
 *        paper-graph-ui walkthrough: section 3.2 "Big-Picture Architecture" and
 *        section 3.4 parts "Oracle Sparse Neuron Selection Criteria", "SVD
 *        Sparsity Estimator" (Algorithm 1), "Token Sensitivity and
 *        Context-Output Aware Sparsity" (Figure 8), "Putting It All Together".
 *   [PN] zhaoyang97 Paper-Notes page on SparseLoRA, section 方法详解
 *        (selection criteria, SVD sparsity estimator).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are CUDA device pointers owned by the caller. The library
 *   never allocates device memory, never synchronises the stream and keeps no
 *   global state besides lazily set kernel attributes (and the fixed scratch array
 *   of sl_svd_estimate_noalloc). Scratch memory comes from the caller's sl_workspace.
 * - Matrices are row-major with an explicit leading dimension in elements.
 *   Frozen weights use nn.Linear storage order W[d_out, d_in] (the pages' math
 *   convention is y = x W_math with W_math = W^T). LoRA: A[r, d_in], B[d_out, r],
 *   y += scale * (x A^T) B^T.
 * - Token rows are in context-first order: rows [0, n_ctx) are context tokens and
 *   rows [n_ctx, n_tok) are output (loss-target) tokens. Linear layers act on rows
 *   independently, so this is the pages' in-place context/output split (Figure 8)
 *   after one permutation of the batch (sl_permute_rows).
 * - A channel set for one projection is a permutation sigma of [0, n_side):
 *   sigma[0, n_keep) are the kept channels in ascending order, sigma[n_keep,
 *   n_side) the dropped ones in ascending order (sl_select_channels writes it).
 * - "sigma layout" of an activation with n_side columns: its context rows store
 *   channel sigma[p] in column p (kept channels first); its output rows store
 *   channel c in column c. The SwiGLU path writes g, u, h (and the backward dg,
 *   du) in this layout so every GEMM operand of the sparse path is contiguous.
 * - bf16 for activations, frozen weights, estimator factors and LoRA parameters;
 *   fp32 for scores, x A^T, dy B and LoRA gradients; int32 for channel indices.
 * - Alignment: every bf16 matrix consumed by a tensor-core GEMM needs a 16-byte
 *   aligned base and a leading dimension that is a multiple of 8 elements.
 * - Errors: arguments are checked on the host before any launch and reported as a
 *   status; nothing is launched on an error. Launch failures give SL_ERR_CUDA. All
 *   device-side waits are bounded; a wait that runs out writes a non-zero code
 *   into the workspace's error word (read it with sl_read_device_flag).
 * - Environment (read once per process; each changes how a result is computed, never
 *   which result): SL_PDL=0 launches without programmatic dependent launch;
 *   SL_VERBOSE_ERRORS=1 prints the CUDA error of a failed launch to stderr;
 *   SL_GEMM_1CTA=1 runs every GEMM on the one-CTA kernel; SL_GEMM_BROWS=256
 *   forces the one-CTA kernel's widest B stage; SL_GEMM_BULK_STORE=0 stores bf16
 *   epilogues per thread instead of through bulk tensor copies.
 */
#ifndef SPARSELORA_H_
#define SPARSELORA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SL_API __attribute__((visibility("default")))
#else
#define SL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sl_stream; /* cudaStream_t; NULL = legacy default stream */

typedef enum {
  SL_OK = 0,
  SL_ERR_INVALID_ARG = 1, /* null pointer, bad enum, inconsistent counts */
  SL_ERR_SHAPE = 2,       /* sizes out of the supported range */
  SL_ERR_ALIGNMENT = 3,   /* base address or leading dimension not aligned for TMA */
  SL_ERR_WORKSPACE = 4,   /* workspace missing or too small; ws->needed holds the size */
  SL_ERR_UNSUPPORTED = 5, /* a valid request the library does not implement */
  SL_ERR_CUDA = 6,        /* a CUDA launch or driver call failed */
  SL_ERR_DEVICE_FLAG = 7  /* a kernel reported a device-side timeout */
} sl_status;

typedef enum {
  SL_CRIT_L2 = 0,        /* s_i = ||Y_hat[:, i]||_2                 ([WT] VO criterion, [PN] L2 Norm) */
  SL_CRIT_SWIGLU_L2 = 1, /* s_i = ||SiLU(G_hat) * U_hat [:, i]||_2  ([WT] FFN criterion)            */
  SL_CRIT_QK = 2         /* s = ||Q_hat||_2 * ||K_hat||_2            ([WT] QK norm, [PN] QK Norm)    */
} sl_criterion;

typedef enum { SL_DT_BF16 = 0, SL_DT_F32 = 1 } sl_dtype;
typedef enum { SL_SLICE_OUT = 0, SL_SLICE_IN = 1 } sl_slice;
typedef enum { SL_LAYOUT_NATURAL = 0, SL_LAYOUT_SIGMA = 1 } sl_layout;
typedef enum { SL_EPI_NONE = 0, SL_EPI_SWIGLU = 1 } sl_epilogue;
typedef enum { SL_LORA_FWD = 0, SL_LORA_BWD = 1 } sl_lora_mode;

/* Caller-owned scratch memory. When ptr is NULL or bytes < the size a call needs, the
 * call stores the size in `needed` and returns SL_ERR_WORKSPACE without launching.
 * The first 64 KiB are a header: the device error word (byte 0), a row of 64 bf16 zeros
 * (bytes 128..255, the zero rows past the kept count of a gathered GEMM operand; never
 * written) and the finish counters of split-K GEMM tiles (which the kernels return to
 * zero). Zero the header once with sl_workspace_init before first use. Calls that share a workspace must be ordered on
 * one stream (they reuse the same scratch and counters). */
typedef struct {
  void* ptr;
  size_t bytes;
  size_t needed;
} sl_workspace;

/* One frozen projection with its LoRA adapter. */
typedef struct {
  const void* w;      /* bf16 [d_out, d_in], frozen */
  const void* w_t;    /* bf16 [d_in, d_out] = w^T (sl_prepare_weight); required for SL_SLICE_IN */
  int64_t d_in, d_out;
  int32_t slice;      /* sl_slice: which side the channel set indexes */
  int32_t r;          /* LoRA rank, multiple of 8, <= 64 */
  const void* lora_a; /* bf16 [r, d_in] */
  const void* lora_b; /* bf16 [d_out, r] */
  float lora_scale;   /* alpha / r */
  int32_t pad_;
  /* Optional (may be NULL): the kept rows of the sliced weight for the channel set passed
   * with the call, row-major and dense: SL_SLICE_OUT: w[sigma[j], :] for j < n_keep
   * ([n_keep, d_in]); SL_SLICE_IN: w_t[sigma[j], :] ([n_keep, d_out]). With keep ratio 1
   * and the identity sigma it is w (w_t) itself. The caller keeps it consistent with sigma;
   * 16-byte aligned.
   * A compacted copy given here is the faster form on B200: the forward and the backward
   * of a step share it, and the GEMM stages it with tiled tensor copies.
   * NULL: the sliced products read the kept rows in place, each GEMM operand tile assembled
   * by row-gather tensor copies (tile::gather4, four 128-byte rows per copy) of w
   * (SL_SLICE_OUT) or w_t (SL_SLICE_IN) through sigma, with no copy of the rows, as long as
   * the gathered rows are whole 64-column boxes (d_in % 64 == 0 for SL_SLICE_OUT,
   * d_out % 64 == 0 for SL_SLICE_IN) and sigma is 16-byte aligned; otherwise each call first
   * gathers the kept rows into its workspace (sl_gather_rows_batch semantics). Every form
   * gives the same result bit for bit. */
  const void* w_kept;
} sl_linear;

/* The channel set applied to one projection's sliced side. */
typedef struct {
  const int32_t* sigma; /* [n_side] kept (ascending) then dropped (ascending) */
  int64_t n_side;       /* d_out for SL_SLICE_OUT, d_in for SL_SLICE_IN */
  int64_t n_keep;       /* 1 <= n_keep <= n_side */
} sl_channels;

SL_API const char* sl_status_string(sl_status s);
SL_API int32_t sl_version(void);

/* n_keep = ceil(ratio * n) with a 1e-9 guard against binary rounding, clamped to
 * [1, n] ([WT] Algorithm 1: the top ceil(r * D_out) channels). Host only. */
SL_API int64_t sl_keep_count(double ratio, int64_t n);

/* Zero the workspace error word (asynchronous memset on `stream`). */
SL_API sl_status sl_workspace_init(sl_workspace* ws, sl_stream stream);
/* Copy the error word to the host (synchronises `stream`). *code = 0: no error. */
SL_API sl_status sl_read_device_flag(const sl_workspace* ws, int32_t* code, sl_stream stream);

/* a1 + a2: SVD sparsity estimator and criterion ([WT] "SVD Sparsity Estimator",
 * Algorithm 1, and the criteria of "Oracle Sparse Neuron Selection Criteria";
 * [PN] SVD 稀疏估计器).
 *   x: [n_ctx, d_in] (ld ldx), the context rows of the layer input, dtype `dtype`.
 *   w_a[j]: [d_in, k], w_b[j]: [k, d_out[j]] - offline rank-k factors of projection j
 *           (same dtype as x).
 *   crit SL_CRIT_L2:        n_proj = 1; scores[d_out[0]] = ||x W_A W_B||_2 per column.
 *   crit SL_CRIT_SWIGLU_L2: n_proj = 2 (gate, up); scores[d_out[0]] from SiLU(G_hat) * U_hat.
 *   crit SL_CRIT_QK:        n_proj = 2 (q, k) or 3 (q, k, v); scores over the
 *                           n_kv_heads * head_dim KV units (g, d): ||K_hat[:, (g,d)]|| *
 *                           sum_{h in group g} ||Q_hat[:, (h,d)]|| (equal head counts give
 *                           s = q * k exactly). With n_proj = 3, scores_v[d_out[2]] receives
 *                           the L2 scores of v from the same pass over x.
 * Sums over tokens run in a fixed order (bit-identical across runs). k <= 16,
 * n_proj * k <= 64, d_in % 8 == 0. */
SL_API sl_status sl_svd_estimate(sl_criterion crit, sl_dtype dtype, const void* x, int64_t n_ctx, int64_t d_in,
                          int64_t ldx, int32_t n_proj, const void* const* w_a, const void* const* w_b,
                          const int64_t* d_out, int32_t k, int32_t n_q_heads, int32_t n_kv_heads,
                          int32_t head_dim, float* scores, float* scores_v, sl_workspace* ws,
                          sl_stream stream);

/* sl_svd_estimate without a workspace: the method itself has no counterpart of this entry;
 * it exists for callers that cannot supply device scratch (a host with no device allocator
 * of its own, or code where cudaMalloc/cudaFree must not run because cudaFree synchronises
 * the whole device). Same arguments, layouts and results as sl_svd_estimate (bit-identical
 * scores), with the scratch taken from a fixed 8 MiB array inside the library, one per
 * device; the call allocates nothing.
 *   scratch_needed: optional host int64; receives the bytes the call needs whenever the
 *     arguments are valid.
 *   device_flag: optional device int32; receives, on `stream` after the estimator's
 *     kernels, the call's device error word (0 = no device-side timeout).
 * Errors: argument errors as sl_svd_estimate; SL_ERR_WORKSPACE when the shapes need more
 * than the 8 MiB (nothing is launched); SL_ERR_CUDA when the array's address cannot be
 * looked up. The array costs 8 MiB of device memory on every device where the library is
 * loaded, whether or not this entry is called. The first call on a device (with that device
 * current) looks the address up and should precede any stream capture there; the address is
 * kept per device and CUDA context, so the first call after a device reset looks it up again
 * (and should not be captured either). All calls share the array and leave their
 * contents in it; the header is cleared at the start of each call. Calls that may execute
 * at the same time (different streams, unordered threads) race on it: serialise them. */
SL_API sl_status sl_svd_estimate_noalloc(sl_criterion crit, sl_dtype dtype, const void* x, int64_t n_ctx,
                                         int64_t d_in, int64_t ldx, int32_t n_proj, const void* const* w_a,
                                         const void* const* w_b, const int64_t* d_out, int32_t k,
                                         int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, float* scores,
                                         float* scores_v, int64_t* scratch_needed, int32_t* device_flag,
                                         sl_stream stream);

/* a1 + a2 across data-parallel ranks ([WT] "Oracle Sparse Neuron Selection Criteria": the
 * criterion is a norm over the context tokens of the batch, one index set per batch). A rank
 * holding part of the batch's context rows computes its rank-local statistics, the caller sums
 * them over the ranks (an fp64 all-reduce), and every rank turns the sum into the same scores:
 *   SL_CRIT_SWIGLU_L2: partials[d_out[0]] = sum over the rank's context rows of
 *                      (SiLU(G_hat) * U_hat)^2 per channel (fp64);
 *   SL_CRIT_L2, SL_CRIT_QK: partials[(n_proj k)^2] = the Gram matrix Z^T Z of the rank's
 *                      Z = X_ctx [W_A^(1) ...] (fp64, row-major), from which every linear
 *                      criterion follows exactly: sum_t (z_t . b)^2 = b^T (Z^T Z) b.
 * sl_svd_partials_count gives the element count (0 for invalid arguments). Arguments of
 * sl_svd_estimate_partials are those of sl_svd_estimate, with n_ctx = 0 allowed (zero
 * statistics); sl_svd_scores_from_partials takes the summed statistics and writes scores (and
 * scores_v for SL_CRIT_QK with n_proj = 3) exactly as sl_svd_estimate would for the union of the
 * ranks' context rows (up to the summation order). Sums over tokens run in a fixed order on a
 * rank; the sum over ranks is the caller's. */
SL_API int64_t sl_svd_partials_count(sl_criterion crit, int32_t n_proj, const int64_t* d_out, int32_t k);
SL_API sl_status sl_svd_estimate_partials(sl_criterion crit, sl_dtype dtype, const void* x, int64_t n_ctx,
                                          int64_t d_in, int64_t ldx, int32_t n_proj, const void* const* w_a,
                                          const void* const* w_b, const int64_t* d_out, int32_t k,
                                          int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                          double* partials, sl_workspace* ws, sl_stream stream);
SL_API sl_status sl_svd_scores_from_partials(sl_criterion crit, sl_dtype dtype, int32_t n_proj,
                                             const void* const* w_b, const int64_t* d_out, int32_t k,
                                             int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                             const double* partials, float* scores, float* scores_v,
                                             sl_stream stream);

/* a3: top-n selection ([WT] Algorithm 1; [PN] top-n). Keeps exactly n_keep of the n
 * scores: larger score first, ties to the lower index, NaN below every number.
 * Writes sigma[n] (kept ascending, then dropped ascending). When heads_per_group > 0
 * the n scores are KV units (g, d) with d < head_dim, and sigma_wide[n *
 * heads_per_group] receives the matching query-side set: channel (h, d) is kept iff
 * unit (h / heads_per_group, d) is (the kept count is n_keep * heads_per_group).
 * n <= 40960; n <= 16384 with the query-side set. */
SL_API sl_status sl_select_channels(const float* scores, int64_t n, int64_t n_keep, int32_t* sigma,
                             int32_t heads_per_group, int32_t head_dim, int32_t* sigma_wide, sl_stream stream);

/* Head-level variant of the QK selection ([WT] "Oracle Sparse Neuron Selection Criteria",
 * why not head-level pruning for QK, and the criterion ablation of Table 10: head-level pruning
 * with the same metric). scores: the n_heads * head_dim unit scores of sl_svd_estimate
 * (SL_CRIT_QK); the head score is their sum over the head's head_dim units; the n_keep_heads
 * largest heads are kept whole (ties to the lower head index, NaN below every number).
 * sigma[n_heads * head_dim] (KV channels): channels of kept heads ascending, then the others
 * ascending (kept count n_keep_heads * head_dim); sigma_wide (optional, query side,
 * [n_heads * heads_per_group * head_dim]): query channel (h, d) is kept iff KV head
 * h / heads_per_group is. n_heads <= 1024. */
SL_API sl_status sl_select_heads(const float* scores, int32_t n_heads, int32_t head_dim, int32_t n_keep_heads,
                                 int32_t heads_per_group, int32_t* sigma, int32_t* sigma_wide, sl_stream stream);

/* Wanda-style channel criterion, the FFN alternative of the criterion ablation ([WT] "Oracle
 * Sparse Neuron Selection Criteria", Table 10: Wanda against L2 norm and random pruning for the
 * FFN projections). Wanda's weight importance is |W[i, j]| ||X[:, j]||_2 with the input feature
 * norm over the context rows; the channel score sums it over the channel's row, and the n_proj
 * weights that share one index set (gate and up) add theirs:
 *   scores[i] = sum_p sum_j |w[p][i, j]| * sqrt(sum_t x[t, j]^2),  i < d_out.
 *   x: bf16 [n_ctx, d_in] (ld ldx), the context rows; w[p]: frozen bf16 [d_out, d_in] (ld ldw),
 *   16-byte aligned, d_in % 8 == 0, d_in <= 51200, n_proj <= 4. Reads every weight byte once;
 *   fp32 sums in a fixed order. Workspace: (ceil(n_ctx / 128) + 1) * d_in floats. */
SL_API sl_status sl_wanda_scores(const void* x, int64_t n_ctx, int64_t d_in, int64_t ldx, int32_t n_proj,
                                 const void* const* w, int64_t d_out, int64_t ldw, float* scores,
                                 sl_workspace* ws, sl_stream stream);

/* Decoder-layer pieces around the sparse projections ([WT] "Putting It All Together": the
 * projections sit in a LLaMA decoder layer; RMSNorm with a frozen gain). All bf16 rows
 * [n_rows, d] (ld elements, 16-byte aligned, ld % 8 == 0, d % 8 == 0), fp32 arithmetic.
 * sl_rmsnorm_fwd: s = x (+ res when res is given, written to sum_out as the new residual
 *   stream, rounded to bf16); rstd[row] = 1 / sqrt(mean_j s_j^2 + eps); y = s * rstd * gamma.
 * sl_rmsnorm_bwd: dx = rstd * gamma * dy - s * rstd^3 * (sum_j s_j gamma_j dy_j) / d
 *   (+ dres when given: the gradient arriving through the residual connection); x is the
 *   normalised input s of the forward.
 * sl_add_rows: out = a + b. */
SL_API sl_status sl_rmsnorm_fwd(const void* x, int64_t ldx, const void* res, int64_t ldr, void* sum_out,
                                int64_t lds, const void* gamma, float eps, void* y, int64_t ldy, float* rstd,
                                int64_t n_rows, int64_t d, sl_stream stream);
SL_API sl_status sl_rmsnorm_bwd(const void* dy, int64_t lddy, const void* x, int64_t ldx, const void* gamma,
                                const float* rstd, const void* dres, int64_t ldr, void* dx, int64_t lddx,
                                int64_t n_rows, int64_t d, sl_stream stream);
SL_API sl_status sl_add_rows(const void* a, int64_t lda, const void* b, int64_t ldb, void* out, int64_t ldo,
                             int64_t n_rows, int64_t d, sl_stream stream);

/* AdamW step over n fp32 parameters (the LoRA matrices of a fine-tuning step; [WT] §3.2: only
 * the adapters train): decoupled decay p -= lr * weight_decay * p; m = beta1 m + (1 - beta1) g;
 * v = beta2 v + (1 - beta2) g^2; p -= lr * m_hat / (sqrt(v_hat) + eps) with the bias corrections
 * m_hat = m / (1 - beta1^step), v_hat = v / (1 - beta2^step), step >= 1. params_bf16
 * (optional) receives the updated parameters rounded to bf16 (the working copy the kernels read). */
SL_API sl_status sl_adamw_step(float* params, const float* grads, float* m, float* v, void* params_bf16, int64_t n,
                               float lr, float beta1, float beta2, float eps, float weight_decay, int32_t step,
                               sl_stream stream);

/* a6: the dense LoRA branch ([WT] Algorithm 1 "computed densely and added"; section 3.2:
 * LoRA gradients are always dense).
 * SL_LORA_FWD: for n_ad adapters sharing the input x [n_tok, d_in] (ld ldx), with
 *   R = sum r_i and equal scales:  xa[n_tok, R] (fp32, ld ld_xa) = x A_i^T per block,
 *   xa_s[n_tok, R] (bf16, ld ld_xa) = scale * xa (the operand the sparse GEMMs fuse).
 *   in_layout SL_LAYOUT_SIGMA: x's context rows are in the sigma layout of in_ch.
 * SL_LORA_BWD: for each adapter i with output gradient dy[i] [n_tok, d_out_i] (ld ld_dy[i]):
 *   dya[i] (fp32 [n_tok, r_i], ld r_i) = scale * dy B;  dya_s[i] (bf16, same) = dya;
 *   dB[i] (fp32 [d_out_i, r_i]) = scale * dy^T xa = dy^T xa_s;
 *   dA[i] (fp32 [r_i, d_in]) = dya^T x (adapters of equal rank that share x in the natural
 *   layout, up to three, form one product over x).
 *   dya and dB come from one pass over dy whose partial sums meet in fp32 reductions, so
 *   their last bits may differ between runs; dya and dB must be 16-byte aligned.
 *   xa_s is the forward's bf16 block for adapter i (ld ld_xa, column offset = sum of
 *   earlier r). out_layout SL_LAYOUT_SIGMA: dy's context rows are in the sigma layout
 *   of out_ch[i]; in_layout SL_LAYOUT_SIGMA: x's context rows are in the sigma layout
 *   of in_ch. */
SL_API sl_status sl_lora_fwd_bwd(sl_lora_mode mode, int32_t n_ad, const sl_linear* lin, const void* x, int64_t ldx,
                          int64_t n_tok, int64_t n_ctx, int32_t in_layout, const sl_channels* in_ch, float* xa,
                          void* xa_s, int64_t ld_xa, const void* const* dy, const int64_t* ld_dy,
                          int32_t out_layout, const sl_channels* out_ch, float* const* dya, void* const* dya_s,
                          float* const* dA, float* const* dB, sl_workspace* ws, sl_stream stream);

/* a1 fused into a6's forward: the estimator's stage 1 and the adapters' x A^T from one pass over
 * x ([WT] "SVD Sparsity Estimator", Algorithm 1: Z = X_ctx W_A on the context tokens; the dense
 * LoRA branch's x A^T reads the same rows). The stacked, transposed factors of the estimated
 * projections that share x become extra rows of the skinny product's B operand, so x streams from
 * memory once for both:
 *   xa, xa_s exactly as sl_lora_fwd_bwd(SL_LORA_FWD) for the n_ad (<= 3) adapters sharing x
 *   (natural layout, equal scales);
 *   z: fp32 [n_ctx, ld_z] (ld_z >= n_proj k) = X_ctx [W_A^(1) ... W_A^(n_proj)] for the context rows
 *   [0, n_ctx) of x (rows past n_ctx are not written).
 *   w_a_t: bf16 [n_proj k, d_in] (ld ld_wat): row j k + c = column c of W_A^(j) (sl_prepare_weight
 *   of each W_A [d_in, k] gives its k rows).
 * Requires k <= 16, n_proj k <= 64 and a multiple of 4, sum of ranks + n_proj k <= 256. Sums over
 * d_in run in a fixed order (z is run-to-run identical). Errors as sl_lora_fwd_bwd. */
SL_API sl_status sl_lora_fwd_estimate(int32_t n_ad, const sl_linear* lin, const void* x, int64_t ldx, int64_t n_tok,
                                      int64_t n_ctx, float* xa, void* xa_s, int64_t ld_xa, int32_t n_proj,
                                      int32_t k, const void* w_a_t, int64_t ld_wat, float* z, int64_t ld_z,
                                      sl_workspace* ws, sl_stream stream);

/* a2 from the Z of sl_lora_fwd_estimate: the scores sl_svd_estimate gives for the same context rows
 * and factors (same criteria, arguments and results; z: fp32 [n_ctx, ld_z], n_proj k columns).
 * The linear criteria go through the fp64 Gram matrix of Z, the SwiGLU criterion through a
 * three-term bf16 expansion of Z on the tensor cores (k in {4, 8, 16}). */
SL_API sl_status sl_svd_scores_from_z(sl_criterion crit, int32_t n_proj, const void* const* w_b, const int64_t* d_out,
                                      int32_t k, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                      const float* z, int64_t ld_z, int64_t n_ctx, float* scores, float* scores_v,
                                      sl_workspace* ws, sl_stream stream);

/* a4: sparse frozen branch forward plus the fused LoRA add ([WT] Algorithm 1, Figure 8;
 * "Preliminary: what channel sparsity means structurally").
 * Context rows go through the weight sliced to the kept channels; output rows through
 * the dense weight; every row adds scale * xa B^T (xa_s from sl_lora_fwd_bwd).
 *   SL_SLICE_OUT, epi SL_EPI_NONE: n_lin projections sharing x; y[i] [n_tok, d_out_i]:
 *     kept channels = main + LoRA, dropped context channels = LoRA only. out_layout
 *     NATURAL scatters to the natural columns; SIGMA writes the sigma layout.
 *   SL_SLICE_OUT, epi SL_EPI_SWIGLU: n_lin = 2 (gate, up) with one channel set; writes
 *     y[0] = g, y[1] = u, y[2] = h = SiLU(g) * u, all [n_tok, d_out] in the sigma layout.
 *   SL_SLICE_IN: n_lin = 1 (down, o). The kept input channels of x's context rows feed
 *     w_t[kept] (w_t required); x's context rows are in the sigma layout (in_layout
 *     SIGMA, e.g. h from the SwiGLU path) or natural (gathered into the workspace).
 *     y[0] [n_tok, d_out] natural.
 * xa_s: bf16 [n_tok, sum r] (ld ld_xa), the adapters' blocks in the order of lin.
 * Never forms a frozen-weight gradient. */
SL_API sl_status sl_sparse_linear_fwd(int32_t n_lin, const sl_linear* lin, const sl_channels* ch, int32_t epi,
                               const void* x, int64_t ldx, int64_t n_tok, int64_t n_ctx, int32_t in_layout,
                               int32_t out_layout, const void* xa_s, int64_t ld_xa, void* const* y,
                               const int64_t* ldy, sl_workspace* ws, sl_stream stream);

/* a5: input-gradient backward through the same slicing, plus the fused LoRA term
 * scale * (dy B) A ([WT] section 3.2 backward pass, "Putting It All Together": no
 * frozen-weight gradient).
 *   SL_SLICE_OUT: n_lin projections whose input gradients sum into dx [n_tok, d_in]
 *     (ld lddx); dy[i] [n_tok, d_out_i] in in_layout (SIGMA: context rows in the sigma
 *     layout of ch[i]; NATURAL: kept columns gathered into the workspace).
 *   SL_SLICE_IN: n_lin = 1; dy [n_tok, d_out] natural; dx [n_tok, d_in] written in
 *     out_layout (NATURAL scatters kept channels, dropped context channels carry only
 *     the LoRA term). epi SL_EPI_SWIGLU fuses the SwiGLU backward: with g = aux[0],
 *     u = aux[1] (sigma layout, from the forward) it writes aux_out[0] = dg = dh u
 *     SiLU'(g) and aux_out[1] = du = dh SiLU(g) instead of dx (out_layout SIGMA).
 * dya_s[i]: bf16 [n_tok, r_i] (ld r_i) from sl_lora_fwd_bwd(BWD). */
SL_API sl_status sl_sparse_linear_bwd(int32_t n_lin, const sl_linear* lin, const sl_channels* ch, int32_t epi,
                               const void* const* dy, const int64_t* ld_dy, int64_t n_tok, int64_t n_ctx,
                               int32_t in_layout, int32_t out_layout, const void* const* dya_s, void* dx,
                               int64_t lddx, const void* const* aux, void* const* aux_out, sl_workspace* ws,
                               sl_stream stream);

/* Optional measurement of the library's own kernels (host-side counters, off by default).
 * While enabled, every kernel the library launches is counted, and every launch of the
 * grouped tensor-core GEMM engine is bracketed by CUDA events on its stream.
 * sl_profile_read waits for those events, returns the totals since the last read (or
 * since enabling) and resets them. Not thread-safe across concurrent callers. */
SL_API sl_status sl_profile_enable(int32_t on);
SL_API sl_status sl_profile_read(int64_t* kernel_launches, int64_t* gemm_launches, double* gemm_ms);
/* Per-launch view of the same GEMM-engine event pairs, without resetting them (call it
 * before sl_profile_read): *count = launches recorded; for the first min(count, capacity)
 * of them, in launch order, ms[i] = duration and kind[i] = 0 (one-CTA grouped launch),
 * 1 (CTA pairs, 256-row tiles), 2 (CTA pairs, 512-row tiles), 3 (fused LoRA backward
 * stream) or 4 (estimator stage 1). Waits for the events. */
SL_API sl_status sl_profile_launches(int64_t capacity, double* ms, int32_t* kind, int64_t* count);

/* The decoder layer's attention core between the sparse q/k/v and o projections ("SparseLoRA:
 * Accelerating LLM Fine-Tuning with Contextual Sparsity", walkthrough, "Putting It All Together":
 * output rows attend to the context keys and values the sparse projections computed). Causal,
 * grouped-query, no positional rotation, scores scaled by 1 / sqrt(head_dim), on the tcgen05
 * tensor cores (S = Q K^T and O = P V per 128-query tile with the softmax between them; the
 * backward recomputes P from the forward's row log-sum-exp).
 *   Rows are tokens in sequence order: n_seq sequences of seq_len tokens, T = n_seq * seq_len.
 *   q, o, d_o, dq: bf16 [T, n_q_heads * head_dim], leading dimension ldq (query head h in columns
 *     [h head_dim, (h + 1) head_dim)); k, v, dk, dv: bf16 [T, n_kv_heads * head_dim], leading
 *     dimension ldkv. Query head h attends with key/value head h / (n_q_heads / n_kv_heads).
 *   lse: fp32 [n_q_heads][T], written by the forward (natural log of sum_k exp(score)) and read by
 *     the backward.
 *   sl_attention_fwd: o[t] = sum over keys s <= t of the same sequence of softmax(q k^T) v.
 *   sl_attention_bwd: dq, dk, dv of the loss whose gradient at o is d_o. dq is summed across key
 *     tiles in fp32 reductions whose order varies between runs (last bits of dq may differ); dk and
 *     dv are run-to-run identical. Workspace: 4 n_q_heads head_dim T + 4 n_q_heads T bytes past
 *     the header (fp32 dq accumulator, per-row sum of d_o o).
 * head_dim in [8, 128], a multiple of 8; n_q_heads a multiple of n_kv_heads; every pointer 16-byte
 * aligned, ldq and ldkv multiples of 8. Errors: SL_ERR_INVALID_ARG (null pointer), SL_ERR_SHAPE,
 * SL_ERR_ALIGNMENT, SL_ERR_WORKSPACE (backward: ws->needed holds the size; the forward needs only
 * the header, whose error word receives device-side timeouts of both). */
SL_API sl_status sl_attention_fwd(const void* q, const void* k, const void* v, int64_t ldq, int64_t ldkv,
                                  int32_t n_seq, int32_t seq_len, int32_t n_q_heads, int32_t n_kv_heads,
                                  int32_t head_dim, void* o, float* lse, sl_workspace* ws, sl_stream stream);
SL_API sl_status sl_attention_bwd(const void* q, const void* k, const void* v, const void* o, const void* d_o,
                                  const float* lse, int64_t ldq, int64_t ldkv, int32_t n_seq, int32_t seq_len,
                                  int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, void* dq, void* dk,
                                  void* dv, sl_workspace* ws, sl_stream stream);

/* Tile height of the CTA-pair tensor-core GEMM that runs the sliced products (a4, a5):
 * rows = 256 (each pair of SMs computes 256 x 256 output tiles with two accumulators, so a
 * tile's epilogue overlaps the next tile's products), 512 (512 x 256 tiles: a quarter fewer
 * operand bytes per FLOP, epilogue not overlapped), 128 (no CTA pairs: every GEMM launch runs
 * on the one-CTA kernel with 128-row tiles, the slower path kept for shapes the pair kernel
 * does not take), or 0 (the default: chosen per launch by a makespan model of the persistent
 * schedule). Process-wide; applies to launches issued (or captured) after the call; changes
 * how a product is tiled, never its result beyond the fp32 summation order of the tile.
 * Errors: SL_ERR_INVALID_ARG for any other value. */
SL_API sl_status sl_set_pair_tile_rows(int32_t rows);

/* w_t[d_in, d_out] = w^T for a frozen weight (once per weight). */
SL_API sl_status sl_prepare_weight(const void* w, int64_t d_out, int64_t d_in, void* w_t, sl_stream stream);

/* dst[i, :] = src[perm[i], :] for i < n_rows, bf16 rows of n_cols columns: the context-first
 * reordering of a batch, or any row gather (an embedding lookup, kept weight rows). src has
 * src_rows rows; every perm entry must lie in [0, src_rows) (the debug build checks it).
 * Errors: SL_ERR_INVALID_ARG for a null pointer, SL_ERR_SHAPE for a non-positive size or a
 * leading dimension below n_cols. */
SL_API sl_status sl_permute_rows(const void* src, int64_t ld_src, int64_t src_rows, const int32_t* perm,
                                 int64_t n_rows, int64_t n_cols, void* dst, int64_t ld_dst, sl_stream stream);

/* Row permutation of a batch that also converts the channel order of its context rows to or
 * from the sigma layout (the layout a block's sliced products read and write; see the top of
 * this file), so that one pass does both: dst[i, :] = src[perm[i], :] for i < n_rows, n_cols
 * bf16 columns, except on context rows:
 *   to_sigma != 0: destination rows i < n_ctx store dst[i, p] = src[perm[i], sigma[p]];
 *   to_sigma == 0: source rows perm[i] < n_ctx are in the sigma layout: dst[i, sigma[p]] =
 *                  src[perm[i], p].
 * The decoder layer uses it between sequence order (the attention core) and context-first order
 * with the sigma layout (the attention block's q, k, v, x_o, dq, dk, dv): "SparseLoRA:
 * Accelerating LLM Fine-Tuning with Contextual Sparsity", walkthrough, "Putting It All Together"
 * and Figure 8 (context and output tokens of each sequence). sigma: a permutation of [0, n_cols)
 * (sl_select_channels writes it; the debug build checks its entries and perm's). n_cols <= 16384,
 * a multiple of 8, leading dimensions multiples of 8, 16-byte aligned bases; dst must not overlap
 * src. Errors: SL_ERR_INVALID_ARG for a null pointer, SL_ERR_SHAPE for a non-positive size,
 * n_cols > 16384 or a leading dimension below n_cols, SL_ERR_ALIGNMENT otherwise. */
SL_API sl_status sl_permute_rows_sigma(const void* src, int64_t ld_src, int64_t src_rows, const int32_t* perm,
                                       int64_t n_rows, int64_t n_cols, const int32_t* sigma, int64_t n_ctx,
                                       int32_t to_sigma, void* dst, int64_t ld_dst, sl_stream stream);

/* Up to 8 row gathers of bf16 rows in one launch: for each q < n, dst[q][i, :] =
 * src[q][perm[q][i], :] for i < n_rows[q], n_cols[q] columns, leading dimensions ld_src[q] and
 * ld_dst[q]; src[q] has src_rows[q] rows (every perm entry must lie in [0, src_rows[q]); the debug
 * build checks it). Used to build the kept weight rows of several projections at once (each w_kept
 * of a step: "SparseLoRA: Accelerating LLM Fine-Tuning with Contextual Sparsity",
 * walkthrough, "Putting It All Together": the weights sliced to the selected channels).
 * The arrays are host arrays of length n; every pointer in them is a device pointer. The
 * destinations must not overlap any source. Errors: SL_ERR_INVALID_ARG for n outside [1, 8]
 * or a null pointer, SL_ERR_SHAPE for a non-positive size (src_rows, n_cols) or a leading
 * dimension below n_cols. A job with zero rows is skipped (its pointers may be NULL). */
SL_API sl_status sl_gather_rows_batch(int32_t n, const void* const* src, const int64_t* ld_src,
                                      const int64_t* src_rows, const int32_t* const* perm, const int64_t* n_rows,
                                      const int64_t* n_cols, void* const* dst, const int64_t* ld_dst,
                                      sl_stream stream);

/* Debug bounds checks. A library built with them (python -m contextual_sparsity_lora_b200.build
 * --debug writes libsparselora_debug.so; the release library has none) checks, on the device,
 * every index it reads from a channel set (sigma), a row permutation or a gather list against the
 * extent it indexes, before the access that index drives: gathered weight rows against the source's
 * rows (src_rows above, d_out or d_in of a projection; also the rows a sliced product gathers
 * in place, which then read the zero row instead), gathered activation and LoRA columns
 * against their columns, scattered output columns and rows against the product's extent, dB rows
 * against the adapter's output channels. A failing check skips that access (nothing outside the
 * caller's buffers is read or written) and records a code, first writer wins: 0x101 row gather,
 * 0x102 column gather, 0x103 output column map, 0x104 output row map, 0x105 dB row. Entries with a
 * workspace record it in the workspace error word (sl_read_device_flag); sl_gather_rows_batch and
 * sl_permute_rows record it in the library's debug word, one per device.
 * sl_debug_bounds_enabled: 1 in a debug build, else 0.
 * sl_read_debug_flag: copies the debug word of the current device to *code and clears it
 * (synchronises `stream`); SL_ERR_DEVICE_FLAG when it was set. In the release build *code = 0 and
 * SL_OK. */
SL_API int32_t sl_debug_bounds_enabled(void);
SL_API sl_status sl_read_debug_flag(int32_t* code, sl_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* SPARSELORA_H_ */
