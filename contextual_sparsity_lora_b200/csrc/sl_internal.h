// Internal declarations shared by the library's translation units.
#pragma once
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <utility>
#include <cuda_runtime.h>

#include "sl_gemm.h"

namespace sl {

// ---- programmatic dependent launch
// Every library kernel is launched with programmatic stream serialisation: the launch of
// the next kernel in the stream is already in flight when the kernel before it retires, and
// its CTAs run their prologue (barrier set-up, tensor-memory allocation) before waiting in
// pdl_wait() until that kernel has completed and its memory writes are visible. pdl_wait()
// therefore comes before the first global-memory read or write of every kernel. No kernel
// signals its dependents early (that measured slower: the waiting CTAs compete with the
// running grid). SL_PDL=0 in the environment turns it off.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
bool pdl_enabled();

// True when the last launch failed; with SL_VERBOSE_ERRORS=1 in the environment the CUDA
// error and the failing launch site go to stderr.
bool launch_failed(const char* where);

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---- debug bounds checks
// A debug build (-DSL_DEBUG_BOUNDS; python -m contextual_sparsity_lora_b200.build --debug writes
// libsparselora_debug.so) checks every index read from a channel set or a row map against the
// extent it indexes, before the access that index drives: gathered rows and columns against the
// source's rows or columns, scattered output columns and rows against the problem's columns and
// rows, dB rows against the adapter's output channels. A failing check skips that access and
// records its code in the error word (first writer wins): the caller's workspace error word, or,
// for the entries that take no workspace, the library's debug word (sl_read_debug_flag). In the
// release build index_ok is `true` and compiles away.
enum : int {
  DEV_BAD_GATHER_ROW = 0x101,  // row gather: source row index out of range
  DEV_BAD_GATHER_COL = 0x102,  // column gather: source column index out of range
  DEV_BAD_COL_MAP = 0x103,     // GEMM epilogue or split-K reduce: output column map out of range
  DEV_BAD_ROW_MAP = 0x104,     // GEMM epilogue or split-K reduce: output row map out of range
  DEV_BAD_DB_ROW = 0x105,      // fused LoRA backward: dB row (sigma) out of range
};
#ifdef __CUDACC__
__device__ __forceinline__ bool index_ok(int64_t i, int64_t n, int* err, int code) {
#ifdef SL_DEBUG_BOUNDS
  if (i >= 0 && i < n) return true;
  if (err) atomicCAS(err, 0, code);
  return false;
#else
  (void)i; (void)n; (void)err; (void)code;
  return true;
#endif
}
#endif
// Device address of the library's debug word (debug builds; null in release builds), the error
// word of the checks in entries that take no workspace.
int* aux_debug_word();

// Launch accounting for the optional profiling hook (sl_profile_enable / sl_profile_read).
void note_launch(int n = 1);
bool profiling_on();
// kind: 0 one-CTA launch, 1 CTA-pair 256-row tiles, 2 CTA-pair 512-row tiles, 3 fused LoRA
// backward
void gemm_events(cudaStream_t s, bool start, int kind = 0);
#ifdef SL_PROFILE_DUMP
// Description of the next GEMM-engine launch, printed with its time by sl_profile_read.
void gemm_note(const char* desc);
#endif

// Builds the parameter block of one grouped GEMM launch on the host.
struct GemmBuilder {
  struct MapSpec {
    const void* ptr;
    int64_t rows, cols, ld;
    int box_rows;
  };
  GemmParams params;
  MapSpec specs[kMaxMaps];
  int nmaps = 0;
  int nprob = 0;
  int status = 0;  // 0 ok, 1 too many maps/problems/segments, 2 bad tensor, 3 no driver entry, 4 bad problem, 5 launch

  GemmBuilder() { memset(&params, 0, sizeof(params)); }
  // True when every problem can run as 256 x 256 tiles on CTA pairs.
  bool pair_eligible() const;
  // bf16 row-major matrix [rows, cols] with leading dimension ld (elements);
  // the TMA box is 64 columns x box_rows rows, 128-byte swizzled, zero fill.
  int map(const void* ptr, int64_t rows, int64_t cols, int64_t ld, int box_rows);
  // bf16 output block for the epilogue's 32 x 32 bulk tensor stores; -1 if not encodable
  int map_out(void* ptr, int64_t rows, int64_t cols, int64_t ld);
  void attach_output_maps();
  Prob* add(int M, int N, int tile_cols, int n_mma);
  // K is the segment's K extent; n_limit = output column limit (use N or more for "always").
  Seg* seg(Prob* pr, int a_map, int a_mn, int a_row0, int a_k0, int b_mn, int b_k0, int K, int n_limit);
  void bsrc(Seg* s, int map, int tile_off, int rows, int row0, int row_step);
  // Row-gather map of a bf16 weight [rows, cols] (box 64 columns x 1 row) for gathered B sources.
  int gmap(const void* ptr, int64_t rows, int64_t cols, int64_t ld) { return map(ptr, rows, cols, ld, 1); }
  // Make every B source of `s` (all made from gmap() maps over [g_rows, g_cols] tensors) a row
  // gather: B position q reads row idx[q] when q < n_valid, else the zero row. zero_row: 64 bf16
  // zeros in device memory (the workspace's zero row). idx 16-byte aligned; g_cols % 64 == 0.
  void gather(Seg* s, const int32_t* idx, int64_t n_valid, int64_t g_rows, int64_t g_cols, const void* zero_row);
  int zmap = -1;  // the launch's zero-row map, made by the first gather()
  // Compute a skinny problem as `ksplit` K ranges; `part` holds ksplit * M * N floats.
  void split(Prob* pr, int ksplit, float* part);
  int launch(int* err, cudaStream_t stream);
};

// Forced CTA-pair tile height of the GEMM engine: 0 = chosen per launch, 1 = 256 rows,
// 2 = 512 rows, -1 = no CTA pairs (every launch on the one-CTA kernel) (sl_set_pair_tile_rows).
void set_forced_pair_mh(int mh);
int forced_pair_mh();

// Split-K factor for a skinny problem with M rows and `kblocks` 64-wide K blocks: the
// largest split whose tiles fit one wave of `target_tiles` CTAs (default: the current
// device's SM count); 1 = no split.
int choose_ksplit(int64_t M, int64_t kblocks, int target_tiles = 0);

// ---- estimator (sl_estimator.cu)
int est_stage1(const void* x, int x_fp32, int64_t n_ctx, int64_t d_in, int64_t ldx, int n_proj,
               const void* const* wa, int wa_fp32, int k, float* zpart, int n_split, cudaStream_t s);
int est_swiglu_scores(const float* zpart, int n_split, int64_t n_ctx, int k, const void* wb_gate,
                      const void* wb_up, int wb_fp32, int64_t n_ch, float* scores, double* sumsq, int* err,
                      cudaStream_t s);
int est_gram(const float* zpart, int n_split, int64_t n_ctx, int mk, double* gram_part, int n_chunks,
             cudaStream_t s);
int est1_splits(int64_t d_in);

// ---- estimator on the tensor cores (sl_est_tc.cu)
// Stage-1 plan for bf16 inputs: K-range splits per 128-token tile and 64-wide K blocks per split.
int est_z_plan(int64_t n_ctx, int64_t d_in, int mk, int* n_split, int* kb_per);
// z[n_ctx][mk] = x[:, :d_in] [W_A^(0) .. W_A^(n_proj-1)] (W_A^(j) bf16 [d_in, k]); zpart holds
// the K-range partials (n_split * n_ctx * mk floats when n_split > 1); gram_part, when not
// null, receives each 128-token tile's fp64 Gram matrix [n_tiles][mk][mk]; zsplit, when not
// null (two projections, 3k <= 64), receives Z as bf16 terms for est_swiglu_tc. tickets: n_tiles
// finish counters that are zero between calls.
int est_z_tc(const void* x, int64_t n_ctx, int64_t d_in, int64_t ldx, int n_proj, const void* const* wa, int k,
             float* zpart, float* z, double* gram_part, void* zsplit, int* tickets, int* err, cudaStream_t s);
// SwiGLU criterion from zsplit ([n_ctx][128] bf16: Z of gate and of up as three bf16 terms,
// written by est_z_tc) and the bf16 W_B of gate and up [k, F]; scores[F].
int est_swiglu_tc(const void* zsplit, int64_t n_ctx, int k, const void* wb_g, const void* wb_u, int64_t F,
                  float* scores, double* sumsq, int* err, cudaStream_t s);
// Z (fp32 [n_ctx][ld_z], computed elsewhere) -> per-128-row-tile fp64 Gram shares
// (gram_part [tiles][mk][mk]) or the three-term bf16 split for est_swiglu_tc (zsplit
// [n_ctx][128], two projections of k columns each). One launch. gram_total (optional, with
// gram_part): the shares summed in tile order by the launch's last CTA; ticket: a counter
// that is zero between calls.
int z_finish(const float* z, int64_t ld_z, int64_t n_ctx, int mk, int k, double* gram_part, void* zsplit,
             int* ticket, double* gram_total, cudaStream_t s);
// out[mk][mk] = sum of n_parts Gram matrices in order; scores = sqrt(sumsq).
int gram_sum(const double* parts, int n_parts, int mk, double* out, cudaStream_t s);
int sqrt_scores(const double* sumsq, int64_t n, float* scores, cudaStream_t s);
// QK units and/or L2 channels from the Gram partials (sum over n_parts in order), one launch.
int est_scores(const double* gram_part, int n_parts, int mk, int k, int wb_fp32, const void* wb_q, const void* wb_k,
               int blk_q, int blk_k, int n_q_heads, int n_kv_heads, int head_dim, float* scores_qk, const void* wb_l2,
               int blk_l2, int64_t n_l2, float* scores_l2, cudaStream_t s);
// The Gram kernel runs clusters of 8 CTAs over 48 context tokens each; one fp64 partial
// Gram matrix per cluster is left for the score kernel to add.
inline int gram_groups(int64_t n_ctx) { return (int)((n_ctx + 8 * 48 - 1) / (8 * 48)); }

// ---- fused LoRA backward (sl_lora.cu)
// One adapter over one row segment of its upstream gradient: adds scale * dy B into dya and
// dy^T xa_s into dB (rows sigma[p] when sigma is set), reading dy once.
struct DualSpec {
  const void* dy;    // bf16, rows [0, row0 + rows) addressable, ld_dy elements
  int64_t ld_dy;
  const void* B;     // bf16 [cols, r]: LoRA B, or its rows permuted by sigma for sigma-layout rows
  const void* xa_s;  // bf16 [row0 + rows, r] block of this adapter (ld_xa)
  int64_t ld_xa;
  int64_t row0, rows, cols;
  int r;
  float scale;
  float* dya;        // fp32 [n_tok, ld_dya], 16-byte aligned, zeroed by the caller
  int64_t ld_dya;
  float* dB;         // fp32 [cols, r], 16-byte aligned, zeroed by the caller
  const int32_t* sigma;
};
int lora_dual_launch(const DualSpec* specs, int n, int* err, cudaStream_t s);
// dst[i][k] = bf16(src[i][k]) for k < count[i], i < n (one launch). With cat: src[i] is
// [rows, r[i]] and its values also go to columns [sum_{j<i} r[j], ... + r[i]) of cat (ld ld_cat).
int cast_f32_bf16(const float* const* src, void* const* dst, const int64_t* count, int n, cudaStream_t s,
                  void* cat = nullptr, const int* r = nullptr, int ld_cat = 0);
// Zeroes n <= 12 fp32 buffers (one launch).
int zero_f32(float* const* ptrs, const int64_t* counts, int n, cudaStream_t s);

// ---- selection (sl_select.cu)
int select_channels(const float* scores, int64_t n, int64_t n_keep, int32_t* sigma, int heads_per_group,
                    int head_dim, int64_t n_wide, int32_t* sigma_wide, int64_t* n_keep_wide_out, cudaStream_t s);
int select_heads(const float* scores, int n_heads, int head_dim, int n_keep_heads, int heads_per_group,
                 int32_t* sigma, int32_t* sigma_wide, cudaStream_t s);

// ---- decoder layer pieces (sl_layer.cu)
int rmsnorm_fwd(const void* x, int64_t ldx, const void* res, int64_t ldr, void* sum_out, int64_t lds,
                const void* gamma, float eps, void* y, int64_t ldy, float* rstd, int64_t n_rows, int64_t d,
                cudaStream_t s);
int rmsnorm_bwd(const void* dy, int64_t lddy, const void* x, int64_t ldx, const void* gamma, const float* rstd,
                const void* dres, int64_t ldr, void* dx, int64_t lddx, int64_t n_rows, int64_t d, cudaStream_t s);
int add_rows(const void* a, int64_t lda, const void* b, int64_t ldb, void* out, int64_t ldo, int64_t n_rows, int64_t d,
             cudaStream_t s);
int adamw_step(float* p, const float* g, float* m, float* v, void* p_bf16, int64_t n, float lr, float b1, float b2,
               float eps, float wd, int step, cudaStream_t s);

// ---- attention core of the decoder layer (sl_attention.cu)
// Causal GQA attention over n_seq sequences of S tokens (rows in sequence order): o [T, hq hd]
// (ld ldo), lse [hq][T] (natural log of each query row's softmax denominator, scores scaled by
// 1 / sqrt(hd)). Returns 0, 2 (tensor map), 5 (launch).
int attention_fwd(const void* q, const void* k, const void* v, int64_t ldq, int64_t ldkv, int n_seq, int S, int hq,
                  int hkv, int hd, void* o, int64_t ldo, float* lse, int* err, cudaStream_t s);
// Scratch bytes of attention_bwd: the fp32 dQ accumulator and the per-row delta = sum dO O.
size_t attention_bwd_scratch(int n_seq, int S, int hq, int hd);
// dq [T, hq hd] (ld ldq), dk, dv [T, hkv hd] (ld ldkv) from q, k, v, o, d_o and the forward's lse.
int attention_bwd(const void* q, const void* k, const void* v, const void* o, const void* d_o, const float* lse,
                  int64_t ldq, int64_t ldkv, int n_seq, int S, int hq, int hkv, int hd, void* dq, void* dk, void* dv,
                  void* scratch, int* err, cudaStream_t s);

// ---- criterion variants (sl_criteria.cu)
// Wanda-style channel scores s_i = sum_p sum_j |W_p[i, j]| ||x[:, j]||_2 over n_ctx rows of x
// (bf16 [n_ctx, d_in], ld ldx) and n_proj bf16 weights [d_out, d_in] (ld ldw); scratch holds
// wanda_scratch_floats(n_ctx, d_in) floats.
int64_t wanda_scratch_floats(int64_t n_ctx, int64_t d_in);
int wanda_scores(const void* x, int64_t n_ctx, int64_t d_in, int64_t ldx, int n_proj, const void* const* w,
                 int64_t d_out, int64_t ldw, float* scores, float* scratch, cudaStream_t s);

// ---- helpers (sl_aux.cu)
// dst[i, :] = src[idx[i], :]; src_rows: rows of src (the debug build checks idx against it);
// err: error word of the debug checks.
int gather_rows_bf16(const void* src, int64_t ld_src, int64_t src_rows, const int32_t* idx, int64_t n_rows,
                     int64_t n_cols, void* dst, int64_t ld_dst, int64_t dst_col0, int* err, cudaStream_t s);
// Row gathers batched into one launch (jobs as in gather_rows_bf16).
constexpr int kMaxGatherJobs = 8;
struct GatherJob {
  const void* src;
  const int32_t* idx;
  void* dst;
  int64_t ld_src, src_rows, n_rows, n_cols, ld_dst, col0;
  int32_t blk, blk_stride, blk_off, vec;  // destination row of row i: (i / blk) * blk_stride + blk_off + i % blk
};
struct GatherJobs {
  GatherJob j[kMaxGatherJobs];
  int32_t n;
  int* err;  // error word of the debug checks
};
struct GatherBatch {
  GatherJobs jobs{};
  // dst[drow(i), col0 + c] = src[idx[i], c] (src has src_rows rows), drow(i) = i, or with blk > 0
  // (i / blk) * blk_stride + blk_off + i % blk; returns 1 when the batch is full; empty jobs are
  // skipped
  int add(const void* src, int64_t ld_src, int64_t src_rows, const int32_t* idx, int64_t n_rows, int64_t n_cols,
          void* dst, int64_t ld_dst, int64_t dst_col0 = 0, int blk = 0, int blk_stride = 0, int blk_off = 0);
  int launch(int* err, cudaStream_t s);  // one launch for every job added, then empty
};
// dst[t, j] = src[t, idx[j]] for t < n_rows, j < n_idx; src_cols: columns of src (debug checks).
// Row permutation with the sigma-layout channel permutation of context rows (sl_permute_rows_sigma).
// Returns 2 for a shape or alignment the kernel does not take.
constexpr int64_t kPermMaxCols = 16384;
int permute_rows_sigma(const void* src, int64_t ld_src, int64_t src_rows, const int32_t* perm, int64_t n_rows,
                       int64_t n_cols, const int32_t* sigma, int64_t n_ctx, int to_sigma, void* dst, int64_t ld_dst,
                       int* err, cudaStream_t s);
int gather_cols_bf16(const void* src, int64_t ld_src, int64_t src_cols, int64_t n_rows, const int32_t* idx,
                     int64_t n_idx, void* dst, int64_t ld_dst, int* err, cudaStream_t s);
int transpose_bf16(const void* src, int64_t rows, int64_t cols, int64_t ld_src, void* dst, int64_t ld_dst,
                   cudaStream_t s);
int add_f32(float* dst, const float* src, int64_t n, cudaStream_t s);
// Tensor map of a bf16 matrix [rows, cols] (ld elements) with box_cols x box_rows boxes.
bool encode_bf16_2d(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int64_t ld, int box_cols,
                    int box_rows, bool swizzle128);

}  // namespace sl
