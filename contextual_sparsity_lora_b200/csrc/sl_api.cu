// C ABI of libsparselora.so (declared in include/sparselora.h): argument checks,
// workspace carving, and the grouped tcgen05 GEMM problem lists of each stage.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/sparselora.h"
#include "sl_internal.h"

using namespace sl;

// ------------------------------------------------------------------ profiling hook state
namespace {
std::atomic<bool> g_prof{false};
std::atomic<long long> g_launches{0};
std::mutex g_ev_mu;
std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_events;
std::vector<int32_t> g_ev_kind;  // launch kind of each event pair (sl_profile_launches)
size_t g_ev_used = 0;
#ifdef SL_PROFILE_DUMP
std::vector<std::string> g_notes;
#endif
}  // namespace

namespace sl {
void note_launch(int n) {
  if (g_prof.load(std::memory_order_relaxed)) g_launches.fetch_add(n, std::memory_order_relaxed);
}
bool profiling_on() { return g_prof.load(std::memory_order_relaxed); }
bool launch_failed(const char* where) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return false;
  static const bool verbose = [] {
    const char* v = std::getenv("SL_VERBOSE_ERRORS");
    return v && v[0] == '1';
  }();
  if (verbose) fprintf(stderr, "libsparselora: %s launch failed: %s\n", where, cudaGetErrorString(e));
  return true;
}
bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("SL_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}
#ifdef SL_PROFILE_DUMP
void gemm_note(const char* desc) {
  std::lock_guard<std::mutex> lk(g_ev_mu);
  if (g_notes.size() <= g_ev_used) g_notes.resize(g_ev_used + 1);
  g_notes[g_ev_used] = desc;
}
#endif
void gemm_events(cudaStream_t s, bool start, int kind) {
  std::lock_guard<std::mutex> lk(g_ev_mu);
  // Under stream capture the records become event nodes of the graph, re-recorded by
  // every replay (external records); otherwise they are plain stream records.
  cudaStreamCaptureStatus cst = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cst);
  const unsigned flags = cst == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
  if (start) {
    if (g_ev_used == g_events.size()) {
      cudaEvent_t a, b;
      if (cudaEventCreate(&a) != cudaSuccess) return;
      if (cudaEventCreate(&b) != cudaSuccess) return;
      g_events.emplace_back(a, b);
      g_ev_kind.push_back(0);
    }
    g_ev_kind[g_ev_used] = kind;
    cudaEventRecordWithFlags(g_events[g_ev_used].first, s, flags);
  } else {
    cudaEventRecordWithFlags(g_events[g_ev_used].second, s, flags);
    ++g_ev_used;
  }
}
}  // namespace sl

namespace {

constexpr int32_t kVersion = 1;
constexpr int kBig = 1 << 30;  // "segment always active"

inline cudaStream_t cs(sl_stream s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Two-pass carving of the caller's workspace: the first pass (base == nullptr)
// only measures. The header (error word, split-tile counters) comes first.
struct Carver {
  uint8_t* base;
  size_t off = kWorkspaceHeaderBytes;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

inline sl_status ws_check(sl_workspace* ws, size_t needed) {
  if (!ws) return SL_ERR_WORKSPACE;
  ws->needed = needed;
  if (!ws->ptr || ws->bytes < needed || !al16(ws->ptr)) return SL_ERR_WORKSPACE;
  return SL_OK;
}

inline int* err_word(sl_workspace* ws) { return static_cast<int*>(ws->ptr); }
// The workspace header's zero row (64 bf16 zeros): the rows past the kept count of a gathered operand.
inline const void* zero_row(sl_workspace* ws) { return static_cast<const char*>(ws->ptr) + kZeroRowOffsetBytes; }
// Whether the GEMM engine can read the kept rows of a weight straight from it (tile::gather4
// copies through sigma) instead of a compacted copy: the gathered rows' width (the K extent of a
// K-major operand, the N extent of an MN-major one) is whole 64-column boxes and sigma is 16-byte
// aligned.
inline bool gather_ok(const sl_channels& c, int64_t row_width) { return row_width % 64 == 0 && al16(c.sigma); }

inline sl_status from_builder(int rc) {
  switch (rc) {
    case 0: return SL_OK;
    case 2: return SL_ERR_ALIGNMENT;
    case 1: case 4: return SL_ERR_SHAPE;
    default: return SL_ERR_CUDA;
  }
}
inline sl_status from_kernel(int rc) { return rc == 0 ? SL_OK : (rc == 1 ? SL_ERR_SHAPE : SL_ERR_CUDA); }

inline int64_t rup(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

bool linear_ok(const sl_linear& L) {
  return L.w && L.d_in > 0 && L.d_out > 0 && L.lora_a && L.lora_b && L.r >= 8 && L.r <= 64 && L.r % 8 == 0 &&
         L.d_in % 8 == 0 && L.d_out % 8 == 0 && al16(L.w) && al16(L.lora_a) && al16(L.lora_b) && al16(L.w_kept) &&
         (L.slice == SL_SLICE_OUT || L.slice == SL_SLICE_IN);
}

bool channels_ok(const sl_channels& c, int64_t n_side) {
  return c.sigma && c.n_side == n_side && c.n_keep >= 1 && c.n_keep <= n_side;
}

// Split-K plan of one skinny problem: partial floats needed (0 when unsplit).
inline int64_t split_floats(int64_t M, int64_t N, int64_t K) {
  const int S = choose_ksplit(M, (K + kBK - 1) / kBK);
  return S > 1 ? (int64_t)S * M * N : 0;
}
// Marks a skinny problem for split-K, taking its partials from `region` at `*off`.
inline void maybe_split(GemmBuilder& gb, Prob* p, int64_t M, int64_t N, int64_t K, float* region, int64_t* off) {
  const int S = choose_ksplit(M, (K + kBK - 1) / kBK);
  if (!p || S <= 1 || M <= 0) return;
  gb.split(p, S, region + *off);
  *off += (int64_t)S * M * N;
}

}  // namespace

extern "C" {

const char* sl_status_string(sl_status s) {
  switch (s) {
    case SL_OK: return "ok";
    case SL_ERR_INVALID_ARG: return "invalid argument";
    case SL_ERR_SHAPE: return "unsupported or inconsistent shape";
    case SL_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case SL_ERR_WORKSPACE: return "workspace missing or too small";
    case SL_ERR_UNSUPPORTED: return "unsupported request";
    case SL_ERR_CUDA: return "CUDA error";
    case SL_ERR_DEVICE_FLAG: return "device-side timeout reported";
  }
  return "unknown status";
}

int32_t sl_version(void) { return kVersion; }

int64_t sl_keep_count(double ratio, int64_t n) {
  if (n <= 0) return 0;
  int64_t c = (int64_t)std::ceil(ratio * (double)n - 1e-9);
  if (c < 1) c = 1;
  if (c > n) c = n;
  return c;
}

sl_status sl_workspace_init(sl_workspace* ws, sl_stream stream) {
  if (!ws) return SL_ERR_WORKSPACE;
  ws->needed = kWorkspaceHeaderBytes;
  if (!ws->ptr || ws->bytes < (size_t)kWorkspaceHeaderBytes) return SL_ERR_WORKSPACE;
  return cudaMemsetAsync(ws->ptr, 0, kWorkspaceHeaderBytes, cs(stream)) == cudaSuccess ? SL_OK : SL_ERR_CUDA;
}

sl_status sl_read_device_flag(const sl_workspace* ws, int32_t* code, sl_stream stream) {
  if (!ws || !ws->ptr || !code) return SL_ERR_INVALID_ARG;
  if (cudaMemcpyAsync(code, ws->ptr, sizeof(int32_t), cudaMemcpyDeviceToHost, cs(stream)) != cudaSuccess)
    return SL_ERR_CUDA;
  if (cudaStreamSynchronize(cs(stream)) != cudaSuccess) return SL_ERR_CUDA;
  return *code ? SL_ERR_DEVICE_FLAG : SL_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ a1 + a2
namespace {

// Arguments of the criterion shared by the estimate and the scores-from-partials entries:
// the unit count, or a status.
sl_status criterion_units(sl_criterion crit, int32_t n_proj, const void* const* w_b, const int64_t* d_out, int32_t k,
                          int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, bool need_v, int64_t* units) {
  if (!w_b || !d_out) return SL_ERR_INVALID_ARG;
  if (k <= 0 || k > 16 || n_proj < 1 || n_proj * k > 64) return SL_ERR_SHAPE;
  for (int j = 0; j < n_proj; ++j)
    if (!w_b[j] || d_out[j] <= 0) return SL_ERR_INVALID_ARG;
  int64_t n_units = 0;
  switch (crit) {
    case SL_CRIT_L2:
      if (n_proj != 1) return SL_ERR_INVALID_ARG;
      n_units = d_out[0];
      break;
    case SL_CRIT_SWIGLU_L2:
      if (n_proj != 2 || d_out[0] != d_out[1]) return SL_ERR_INVALID_ARG;
      if (k != 4 && k != 8 && k != 16) return SL_ERR_UNSUPPORTED;
      n_units = d_out[0];
      break;
    case SL_CRIT_QK:
      if (n_proj != 2 && n_proj != 3) return SL_ERR_INVALID_ARG;
      if (n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0 || n_q_heads % n_kv_heads) return SL_ERR_SHAPE;
      if (d_out[0] != (int64_t)n_q_heads * head_dim || d_out[1] != (int64_t)n_kv_heads * head_dim)
        return SL_ERR_SHAPE;
      if (n_proj == 3 && need_v) return SL_ERR_INVALID_ARG;
      n_units = (int64_t)n_kv_heads * head_dim;
      break;
    default:
      return SL_ERR_INVALID_ARG;
  }
  *units = n_units;
  return SL_OK;
}

// Rank-local statistics of the criterion: per-channel sums of squares (SwiGLU) or the Gram
// matrix of Z (linear criteria).
int64_t partial_count(sl_criterion crit, int32_t n_proj, const int64_t* d_out, int32_t k) {
  return crit == SL_CRIT_SWIGLU_L2 ? d_out[0] : (int64_t)n_proj * k * n_proj * k;
}

// Estimator body: scores (and scores_v) when partials is null, else the rank-local statistics.
sl_status svd_estimate(sl_criterion crit, sl_dtype dtype, const void* x, int64_t n_ctx, int64_t d_in, int64_t ldx,
                       int32_t n_proj, const void* const* w_a, const void* const* w_b, const int64_t* d_out,
                       int32_t k, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, float* scores,
                       float* scores_v, double* partials, sl_workspace* ws, sl_stream stream) {
  if (!x || !w_a || (!scores && !partials)) return SL_ERR_INVALID_ARG;
  if (dtype != SL_DT_BF16 && dtype != SL_DT_F32) return SL_ERR_INVALID_ARG;
  int64_t n_units = 0;
  if (sl_status st = criterion_units(crit, n_proj, w_b, d_out, k, n_q_heads, n_kv_heads, head_dim,
                                     !partials && !scores_v, &n_units))
    return st;
  if (n_ctx <= 0 || d_in <= 0 || ldx < d_in) return SL_ERR_SHAPE;
  if (d_in % 8 || ldx % 8 || !al16(x)) return SL_ERR_ALIGNMENT;
  for (int j = 0; j < n_proj; ++j)
    if (!w_a[j]) return SL_ERR_INVALID_ARG;
  const int fp32 = dtype == SL_DT_F32;
  const int mk = n_proj * k;
  // bf16 inputs: stage 1 on the tensor cores (exact bf16 products, fp32 accumulation,
  // K-range partials summed in a fixed order); fp32 inputs: CUDA-core fp32 FMA kernel.
  const bool tc = !fp32 && mk % 4 == 0;
  int z_split = 1, kb_per = 0;
  if (tc && est_z_plan(n_ctx, d_in, mk, &z_split, &kb_per)) return SL_ERR_SHAPE;
  const int64_t tiles = (n_ctx + 127) / 128;
  if (tc && (tiles > kMaxSplitCounters || tiles > 65535 || n_ctx > 2147483647LL)) return SL_ERR_SHAPE;
  const int n_split = tc ? 1 : est1_splits(d_in);
  const int n_chunks = tc ? (int)tiles : gram_groups(n_ctx);
  const bool linear = crit != SL_CRIT_SWIGLU_L2;
  // SwiGLU with bf16 inputs: criterion on the tensor cores from a bf16 expansion of Z
  const bool swiglu_tc = tc && !linear;
  auto carve = [&](Carver& c, float** zp, float** zpart, double** gp, uint16_t** zs) {
    *zp = c.take<float>((size_t)n_split * n_ctx * mk);
    *zpart = tc && z_split > 1 ? c.take<float>((size_t)z_split * n_ctx * mk) : nullptr;
    *gp = linear ? c.take<double>((size_t)n_chunks * mk * mk) : nullptr;
    *zs = swiglu_tc ? c.take<uint16_t>((size_t)n_ctx * 128) : nullptr;
  };
  float* zp;
  float* zpart;
  double* gp;
  uint16_t* zs;
  {
    Carver c(nullptr);
    carve(c, &zp, &zpart, &gp, &zs);
    if (sl_status st = ws_check(ws, c.off)) return st;
  }
  Carver c(ws->ptr);
  carve(c, &zp, &zpart, &gp, &zs);
  cudaStream_t s = cs(stream);
  int rc = 0;
  if (tc) {
    int* tickets = err_word(ws) + kCounterOffsetInts;
    rc = est_z_tc(x, n_ctx, d_in, ldx, n_proj, w_a, k, zpart, zp, linear ? gp : nullptr, zs, tickets, err_word(ws),
                  s);
    if (rc) return rc == 2 ? SL_ERR_ALIGNMENT : from_kernel(rc);
  } else {
    rc = est_stage1(x, fp32, n_ctx, d_in, ldx, n_proj, w_a, fp32, k, zp, n_split, s);
    if (rc) return from_kernel(rc);
  }
  if (swiglu_tc) {
    rc = est_swiglu_tc(zs, n_ctx, k, w_b[0], w_b[1], n_units, scores, partials, err_word(ws), s);
    return rc == 2 ? SL_ERR_ALIGNMENT : from_kernel(rc);
  }
  if (crit == SL_CRIT_SWIGLU_L2) {
    rc = est_swiglu_scores(zp, 1, n_ctx, k, w_b[0], w_b[1], fp32, n_units, scores, partials, err_word(ws), s);
    return from_kernel(rc);
  }
  if (!tc && (rc = est_gram(zp, 1, n_ctx, mk, gp, n_chunks, s))) return from_kernel(rc);
  if (partials) return from_kernel(gram_sum(gp, n_chunks, mk, partials, s));
  if (crit == SL_CRIT_L2)
    rc = est_scores(gp, n_chunks, mk, k, fp32, nullptr, nullptr, 0, 0, 0, 0, 0, nullptr, w_b[0], 0, n_units, scores,
                    s);
  else
    rc = est_scores(gp, n_chunks, mk, k, fp32, w_b[0], w_b[1], 0, 1, n_q_heads, n_kv_heads, head_dim, scores,
                    n_proj == 3 ? w_b[2] : nullptr, 2, n_proj == 3 ? d_out[2] : 0, n_proj == 3 ? scores_v : nullptr,
                    s);
  return from_kernel(rc);
}

}  // namespace

extern "C" {

sl_status sl_svd_estimate(sl_criterion crit, sl_dtype dtype, const void* x, int64_t n_ctx, int64_t d_in, int64_t ldx,
                          int32_t n_proj, const void* const* w_a, const void* const* w_b, const int64_t* d_out,
                          int32_t k, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, float* scores,
                          float* scores_v, sl_workspace* ws, sl_stream stream) {
  if (!scores) return SL_ERR_INVALID_ARG;
  return svd_estimate(crit, dtype, x, n_ctx, d_in, ldx, n_proj, w_a, w_b, d_out, k, n_q_heads, n_kv_heads, head_dim,
                      scores, scores_v, nullptr, ws, stream);
}

int64_t sl_svd_partials_count(sl_criterion crit, int32_t n_proj, const int64_t* d_out, int32_t k) {
  if (!d_out || n_proj < 1 || k < 1) return 0;
  return partial_count(crit, n_proj, d_out, k);
}

sl_status sl_svd_estimate_partials(sl_criterion crit, sl_dtype dtype, const void* x, int64_t n_ctx, int64_t d_in,
                                   int64_t ldx, int32_t n_proj, const void* const* w_a, const void* const* w_b,
                                   const int64_t* d_out, int32_t k, int32_t n_q_heads, int32_t n_kv_heads,
                                   int32_t head_dim, double* partials, sl_workspace* ws, sl_stream stream) {
  if (!partials || !d_out) return SL_ERR_INVALID_ARG;
  if (n_ctx == 0) {  // no context rows on this rank: its statistics are zero
    int64_t units = 0;
    if (sl_status st = criterion_units(crit, n_proj, w_b, d_out, k, n_q_heads, n_kv_heads, head_dim, false, &units))
      return st;
    return cudaMemsetAsync(partials, 0, sizeof(double) * partial_count(crit, n_proj, d_out, k), cs(stream)) ==
                   cudaSuccess
               ? SL_OK
               : SL_ERR_CUDA;
  }
  return svd_estimate(crit, dtype, x, n_ctx, d_in, ldx, n_proj, w_a, w_b, d_out, k, n_q_heads, n_kv_heads, head_dim,
                      nullptr, nullptr, partials, ws, stream);
}

sl_status sl_svd_scores_from_partials(sl_criterion crit, sl_dtype dtype, int32_t n_proj, const void* const* w_b,
                                      const int64_t* d_out, int32_t k, int32_t n_q_heads, int32_t n_kv_heads,
                                      int32_t head_dim, const double* partials, float* scores, float* scores_v,
                                      sl_stream stream) {
  if (!partials || !scores) return SL_ERR_INVALID_ARG;
  if (dtype != SL_DT_BF16 && dtype != SL_DT_F32) return SL_ERR_INVALID_ARG;
  int64_t n_units = 0;
  if (sl_status st = criterion_units(crit, n_proj, w_b, d_out, k, n_q_heads, n_kv_heads, head_dim, !scores_v,
                                     &n_units))
    return st;
  cudaStream_t s = cs(stream);
  const int fp32 = dtype == SL_DT_F32;
  const int mk = n_proj * k;
  if (crit == SL_CRIT_SWIGLU_L2) return from_kernel(sqrt_scores(partials, n_units, scores, s));
  if (crit == SL_CRIT_L2)
    return from_kernel(est_scores(partials, 1, mk, k, fp32, nullptr, nullptr, 0, 0, 0, 0, 0, nullptr, w_b[0], 0,
                                  n_units, scores, s));
  return from_kernel(est_scores(partials, 1, mk, k, fp32, w_b[0], w_b[1], 0, 1, n_q_heads, n_kv_heads, head_dim,
                                scores, n_proj == 3 ? w_b[2] : nullptr, 2, n_proj == 3 ? d_out[2] : 0,
                                n_proj == 3 ? scores_v : nullptr, s));
}

// ------------------------------------------------------------------ a3
sl_status sl_select_channels(const float* scores, int64_t n, int64_t n_keep, int32_t* sigma, int32_t heads_per_group,
                             int32_t head_dim, int32_t* sigma_wide, sl_stream stream) {
  if (!scores || !sigma) return SL_ERR_INVALID_ARG;
  if (n <= 0 || n > 40960 || n_keep < 1 || n_keep > n) return SL_ERR_SHAPE;
  if (heads_per_group > 0 && (!sigma_wide || head_dim <= 0 || n % head_dim)) return SL_ERR_INVALID_ARG;
  const int64_t n_wide = heads_per_group > 0 ? n * heads_per_group : 0;
  return from_kernel(select_channels(scores, n, n_keep, sigma, heads_per_group, head_dim, n_wide,
                                     heads_per_group > 0 ? sigma_wide : nullptr, nullptr, cs(stream)));
}

sl_status sl_select_heads(const float* scores, int32_t n_heads, int32_t head_dim, int32_t n_keep_heads,
                          int32_t heads_per_group, int32_t* sigma, int32_t* sigma_wide, sl_stream stream) {
  if (!scores || !sigma) return SL_ERR_INVALID_ARG;
  if (n_heads < 1 || n_heads > 1024 || head_dim < 1 || n_keep_heads < 1 || n_keep_heads > n_heads)
    return SL_ERR_SHAPE;
  if (sigma_wide && heads_per_group < 1) return SL_ERR_INVALID_ARG;
  return from_kernel(select_heads(scores, n_heads, head_dim, n_keep_heads, heads_per_group, sigma, sigma_wide,
                                  cs(stream)));
}

sl_status sl_wanda_scores(const void* x, int64_t n_ctx, int64_t d_in, int64_t ldx, int32_t n_proj,
                          const void* const* w, int64_t d_out, int64_t ldw, float* scores, sl_workspace* ws,
                          sl_stream stream) {
  if (!x || !w || !scores || n_proj < 1 || n_proj > 4) return SL_ERR_INVALID_ARG;
  if (n_ctx < 1 || d_in < 8 || d_out < 1 || ldx < d_in || ldw < d_in || d_in > 51200) return SL_ERR_SHAPE;
  if (d_in % 8 || ldx % 8 || ldw % 8 || !al16(x)) return SL_ERR_ALIGNMENT;
  for (int q = 0; q < n_proj; ++q) {
    if (!w[q]) return SL_ERR_INVALID_ARG;
    if (!al16(w[q])) return SL_ERR_ALIGNMENT;
  }
  float* scratch;
  {
    Carver c(nullptr);
    scratch = c.take<float>((size_t)wanda_scratch_floats(n_ctx, d_in));
    if (sl_status st = ws_check(ws, c.off)) return st;
  }
  Carver c(ws->ptr);
  scratch = c.take<float>((size_t)wanda_scratch_floats(n_ctx, d_in));
  return from_kernel(wanda_scores(x, n_ctx, d_in, ldx, n_proj, w, d_out, ldw, scores, scratch, cs(stream)));
}

// ------------------------------------------------------------------ decoder layer pieces
namespace {
bool rows_ok(const void* p, int64_t ld, int64_t d) { return p && al16(p) && ld >= d && ld % 8 == 0; }
}  // namespace

sl_status sl_rmsnorm_fwd(const void* x, int64_t ldx, const void* res, int64_t ldr, void* sum_out, int64_t lds,
                         const void* gamma, float eps, void* y, int64_t ldy, float* rstd, int64_t n_rows, int64_t d,
                         sl_stream stream) {
  if (!x || !gamma || !y || !rstd || (res && !sum_out)) return SL_ERR_INVALID_ARG;
  if (n_rows < 1 || d < 8 || d % 8 || !(eps >= 0.f)) return SL_ERR_SHAPE;
  if (!rows_ok(x, ldx, d) || !rows_ok(y, ldy, d) || !al16(gamma) || (res && (!rows_ok(res, ldr, d) ||
                                                                             !rows_ok(sum_out, lds, d))))
    return SL_ERR_ALIGNMENT;
  return from_kernel(rmsnorm_fwd(x, ldx, res, ldr, sum_out, lds, gamma, eps, y, ldy, rstd, n_rows, d, cs(stream)));
}

sl_status sl_rmsnorm_bwd(const void* dy, int64_t lddy, const void* x, int64_t ldx, const void* gamma,
                         const float* rstd, const void* dres, int64_t ldr, void* dx, int64_t lddx, int64_t n_rows,
                         int64_t d, sl_stream stream) {
  if (!dy || !x || !gamma || !rstd || !dx) return SL_ERR_INVALID_ARG;
  if (n_rows < 1 || d < 8 || d % 8) return SL_ERR_SHAPE;
  if (!rows_ok(dy, lddy, d) || !rows_ok(x, ldx, d) || !rows_ok(dx, lddx, d) || !al16(gamma) ||
      (dres && !rows_ok(dres, ldr, d)))
    return SL_ERR_ALIGNMENT;
  return from_kernel(rmsnorm_bwd(dy, lddy, x, ldx, gamma, rstd, dres, ldr, dx, lddx, n_rows, d, cs(stream)));
}

sl_status sl_add_rows(const void* a, int64_t lda, const void* b, int64_t ldb, void* out, int64_t ldo, int64_t n_rows,
                      int64_t d, sl_stream stream) {
  if (!a || !b || !out) return SL_ERR_INVALID_ARG;
  if (n_rows < 1 || d < 8 || d % 8) return SL_ERR_SHAPE;
  if (!rows_ok(a, lda, d) || !rows_ok(b, ldb, d) || !rows_ok(out, ldo, d)) return SL_ERR_ALIGNMENT;
  return from_kernel(add_rows(a, lda, b, ldb, out, ldo, n_rows, d, cs(stream)));
}

sl_status sl_adamw_step(float* params, const float* grads, float* m, float* v, void* params_bf16, int64_t n, float lr,
                        float beta1, float beta2, float eps, float weight_decay, int32_t step, sl_stream stream) {
  if (!params || !grads || !m || !v) return SL_ERR_INVALID_ARG;
  if (n < 1 || step < 1 || !(lr >= 0.f) || !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f))
    return SL_ERR_SHAPE;
  return from_kernel(adamw_step(params, grads, m, v, params_bf16, n, lr, beta1, beta2, eps, weight_decay, step,
                                cs(stream)));
}

// ------------------------------------------------------------------ a6
sl_status sl_lora_fwd_bwd(sl_lora_mode mode, int32_t n_ad, const sl_linear* lin, const void* x, int64_t ldx,
                          int64_t n_tok, int64_t n_ctx, int32_t in_layout, const sl_channels* in_ch, float* xa,
                          void* xa_s, int64_t ld_xa, const void* const* dy, const int64_t* ld_dy, int32_t out_layout,
                          const sl_channels* out_ch, float* const* dya, void* const* dya_s, float* const* dA,
                          float* const* dB, sl_workspace* ws, sl_stream stream) {
  if (!lin || !x || n_ad < 1 || n_ad > 4) return SL_ERR_INVALID_ARG;
  if (n_tok <= 0 || n_ctx < 0 || n_ctx > n_tok) return SL_ERR_SHAPE;
  const int64_t d_in = lin[0].d_in;
  int R = 0;
  for (int i = 0; i < n_ad; ++i) {
    if (!linear_ok(lin[i]) || lin[i].d_in != d_in) return SL_ERR_INVALID_ARG;
    R += lin[i].r;
  }
  if (ldx < d_in || ldx % 8 || !al16(x)) return SL_ERR_ALIGNMENT;
  const bool in_sig = in_layout == SL_LAYOUT_SIGMA && n_ctx > 0;
  if (in_sig && (!in_ch || !channels_ok(*in_ch, d_in))) return SL_ERR_INVALID_ARG;
  if (!xa_s || ld_xa < R || ld_xa % 8 || !al16(xa_s)) return SL_ERR_ALIGNMENT;
  cudaStream_t s = cs(stream);
  const int64_t C = n_ctx, T = n_tok, O = T - C;

  if (mode == SL_LORA_FWD) {
    if (!xa) return SL_ERR_INVALID_ARG;
    if (R > 256) return SL_ERR_SHAPE;
    for (int i = 1; i < n_ad; ++i)
      if (lin[i].lora_scale != lin[0].lora_scale) return SL_ERR_UNSUPPORTED;
    const int64_t red = in_sig ? split_floats(C, R, d_in) + split_floats(O, R, d_in) : split_floats(T, R, d_in);
    auto carve = [&](Carver& c, void** asig, float** region) {
      for (int i = 0; i < n_ad; ++i) asig[i] = in_sig ? c.take<uint16_t>((size_t)lin[i].r * d_in) : nullptr;
      *region = c.take<float>((size_t)red);
    };
    void* asig[4];
    float* region;
    {
      Carver c(nullptr);
      carve(c, asig, &region);
      if (sl_status st = ws_check(ws, c.off)) return st;
    }
    Carver c(ws->ptr);
    carve(c, asig, &region);
    if (in_sig)
      for (int i = 0; i < n_ad; ++i)
        if (int rc = gather_cols_bf16(lin[i].lora_a, d_in, d_in, lin[i].r, in_ch->sigma, d_in, asig[i], d_in, err_word(ws), s))
          return from_kernel(rc);
    GemmBuilder gb;
    int64_t off = 0;
    const int mx = gb.map(x, T, d_in, ldx, kBM);
    const int n_mma = (int)rup(R, 16);
    auto add_prob = [&](int64_t M, int64_t row0, bool sig) {
      Prob* p = gb.add((int)M, R, kBN, n_mma);
      Seg* sg = gb.seg(p, mx, 0, (int)row0, 0, 0, 0, (int)d_in, kBig);
      int toff = 0;
      for (int i = 0; i < n_ad; ++i) {
        const int mb = gb.map(sig ? asig[i] : lin[i].lora_a, lin[i].r, d_in, d_in, lin[i].r);
        gb.bsrc(sg, mb, toff, lin[i].r, 0, 0);
        toff += lin[i].r;
      }
      if (!p) return;
      p->epi = EPI_XA;
      p->out_row0 = (int)row0;
      p->out0 = xa;
      p->ld0 = ld_xa;
      p->out1 = xa_s;
      p->ld1 = ld_xa;
      p->a0 = 1.f;
      p->a1 = lin[0].lora_scale;
      maybe_split(gb, p, M, R, d_in, region, &off);
    };
    if (in_sig) {
      add_prob(C, 0, true);
      add_prob(O, C, false);
    } else {
      add_prob(T, 0, false);
    }
    return from_builder(gb.launch(err_word(ws), s));
  }

  if (mode != SL_LORA_BWD) return SL_ERR_INVALID_ARG;
  if (!dy || !ld_dy || !dya || !dya_s || !dA || !dB) return SL_ERR_INVALID_ARG;
  const bool out_sig = out_layout == SL_LAYOUT_SIGMA && n_ctx > 0;
  if (out_sig && !out_ch) return SL_ERR_INVALID_ARG;
  for (int i = 0; i < n_ad; ++i) {
    if (!dy[i] || !dya[i] || !dya_s[i] || !dA[i] || !dB[i]) return SL_ERR_INVALID_ARG;
    if (ld_dy[i] < lin[i].d_out || ld_dy[i] % 8 || !al16(dy[i]) || !al16(dya_s[i]) || !al16(dya[i]) || !al16(dB[i]))
      return SL_ERR_ALIGNMENT;
    if (out_sig && !channels_ok(out_ch[i], lin[i].d_out)) return SL_ERR_INVALID_ARG;
  }
  // K extents of the dB / dA parts: pass 0 = natural part (all rows, or output rows when the
  // operand is in the sigma layout), pass 1 = context rows of a sigma-layout operand.
  auto kpart = [&](bool sig, int pass) -> int64_t { return sig ? (pass ? C : O) : (pass ? 0 : T); };
  // dA of adapters that share x and the rank (up to three, x in the natural layout) come from
  // one product x^T [dya_1 | dya_2 | ...] over an interleaved bf16 copy of their dya
  bool merge_da = n_ad >= 2 && n_ad <= 3 && !in_sig && R <= 128;
  for (int i = 1; i < n_ad; ++i) merge_da = merge_da && lin[i].r == lin[0].r;
  // split-K partials of the dA products (the two launches reuse them in stream order)
  int64_t red = 0;
  for (int pass = 0; pass < 2; ++pass) {
    const int64_t K = kpart(in_sig, pass);
    if (K <= 0) continue;
    int64_t r2 = 0;
    if (merge_da) r2 = split_floats(d_in, R, K);
    else
      for (int i = 0; i < n_ad; ++i) r2 += split_floats(d_in, lin[i].r, K);
    red = std::max(red, r2);
  }
  auto carve = [&](Carver& c, void** bsig, void** dcat, float** region) {
    for (int i = 0; i < n_ad; ++i) bsig[i] = out_sig ? c.take<uint16_t>((size_t)lin[i].d_out * lin[i].r) : nullptr;
    *dcat = merge_da ? c.take<uint16_t>((size_t)T * R) : nullptr;
    *region = c.take<float>((size_t)red);
  };
  void* bsig[4];
  void* dcat;
  float* region;
  {
    Carver c(nullptr);
    carve(c, bsig, &dcat, &region);
    if (sl_status st = ws_check(ws, c.off)) return st;
  }
  Carver c(ws->ptr);
  carve(c, bsig, &dcat, &region);
  if (out_sig) {
    GatherBatch gat;
    for (int i = 0; i < n_ad; ++i)
      gat.add(lin[i].lora_b, lin[i].r, lin[i].d_out, out_ch[i].sigma, lin[i].d_out, lin[i].r, bsig[i], lin[i].r);
    if (int rc = gat.launch(err_word(ws), s)) return from_kernel(rc);
  }
  // dya = scale * dy B and dB = dy^T xa_s from one pass over each dy (fused kernel; context rows
  // of a sigma-layout dy use the permuted B and land in dB rows sigma[p]), then dya_s = bf16(dya)
  {
    DualSpec sp[8];
    int nsp = 0;
    const float* csrc[4];
    void* cdst[4];
    int64_t ccount[4];
    int cr[4];
    int64_t koff = 0;
    // dya and dB are sums of reductions into zeroed outputs; dA accumulates its two parts
    {
      float* zp[12];
      int64_t zn[12];
      int nz = 0;
      for (int i = 0; i < n_ad; ++i) {
        zp[nz] = dya[i];
        zn[nz++] = T * lin[i].r;
        zp[nz] = dB[i];
        zn[nz++] = lin[i].d_out * lin[i].r;
        zp[nz] = dA[i];
        zn[nz++] = (int64_t)lin[i].r * d_in;
      }
      if (int rc = zero_f32(zp, zn, nz, s)) return from_kernel(rc);
    }
    for (int i = 0; i < n_ad; ++i) {
      const sl_linear& L = lin[i];
      cr[i] = L.r;
      const void* xa_blk = static_cast<const uint16_t*>(xa_s) + koff;
      koff += L.r;
      auto add = [&](int64_t row0, int64_t rows, const void* Bm, const int32_t* sig) {
        if (rows <= 0) return;
        DualSpec& d = sp[nsp++];
        d.dy = dy[i];
        d.ld_dy = ld_dy[i];
        d.B = Bm;
        d.xa_s = xa_blk;
        d.ld_xa = ld_xa;
        d.row0 = row0;
        d.rows = rows;
        d.cols = L.d_out;
        d.r = L.r;
        d.scale = L.lora_scale;
        d.dya = dya[i];
        d.ld_dya = L.r;
        d.dB = dB[i];
        d.sigma = sig;
      };
      if (out_sig) {
        add(0, C, bsig[i], out_ch[i].sigma);
        add(C, O, L.lora_b, nullptr);
      } else {
        add(0, T, L.lora_b, nullptr);
      }
      csrc[i] = dya[i];
      cdst[i] = dya_s[i];
      ccount[i] = T * L.r;
    }
    if (int rc = lora_dual_launch(sp, nsp, err_word(ws), s)) return from_builder(rc);
    if (int rc = cast_f32_bf16(csrc, cdst, ccount, n_ad, s, dcat, cr, R)) return from_kernel(rc);
  }
  // dA = (x^T dya)^T, added into the zeroed dA: launch 2 over the natural part of x (all rows,
  // or the output rows when x is in the sigma layout), launch 3 over the context rows of a
  // sigma-layout x (rows through sigma). Split-K partials are summed in a fixed order.
  for (int pass = 0; pass < 2; ++pass) {
    const int64_t K = kpart(in_sig, pass);
    if (K <= 0) continue;
    const bool ctx_part = pass == 1;
    const int64_t rows = ctx_part ? C : T;  // map extents zero-fill past the part
    const int64_t k0 = (in_sig && !ctx_part) ? C : 0;
    GemmBuilder gb;
    int64_t off = 0;
    const int ma = gb.map(x, rows, d_in, ldx, 64);
    auto add_da = [&](int n, const void* bsrc, int64_t ldb, int i0) {
      const int bcols = (int)rup(n, 64);
      const int mb = gb.map(bsrc, rows, n, ldb, 64);
      Prob* p = gb.add((int)d_in, n, kBN, (int)rup(n, 16));
      Seg* sg = gb.seg(p, ma, 1, 0, (int)k0, 1, (int)k0, (int)K, kBig);
      gb.bsrc(sg, mb, 0, bcols, 0, 0);
      if (!p) return;
      p->epi = EPI_F32_T;
      p->out0 = dA[i0];
      p->ld0 = d_in;
      p->beta = 1;
      p->row_map = ctx_part ? in_ch->sigma : nullptr;
      if (n > lin[i0].r) {
        p->col_split = lin[i0].r;
        p->out1 = dA[i0 + 1];
        p->out2 = n_ad > 2 ? dA[i0 + 2] : nullptr;
      }
      maybe_split(gb, p, d_in, n, K, region, &off);
    };
    if (merge_da) {
      add_da(R, dcat, R, 0);
    } else {
      for (int i = 0; i < n_ad; ++i) add_da(lin[i].r, dya_s[i], lin[i].r, i);
    }
    if (int rc = gb.launch(err_word(ws), s)) return from_builder(rc);
  }
  return SL_OK;
}

// a1 inside the LoRA forward: x A^T of the adapters and Z = X_ctx W_A of the estimator from one pass
// over x (the factors W_A^T as extra B rows of the same skinny product).
sl_status sl_lora_fwd_estimate(int32_t n_ad, const sl_linear* lin, const void* x, int64_t ldx, int64_t n_tok,
                               int64_t n_ctx, float* xa, void* xa_s, int64_t ld_xa, int32_t n_proj, int32_t k,
                               const void* w_a_t, int64_t ld_wat, float* z, int64_t ld_z, sl_workspace* ws,
                               sl_stream stream) {
  if (!lin || !x || !xa || !w_a_t || !z || n_ad < 1 || n_ad > kMaxBSrc - 1) return SL_ERR_INVALID_ARG;
  if (n_tok <= 0 || n_ctx < 0 || n_ctx > n_tok) return SL_ERR_SHAPE;
  if (k < 1 || k > 16 || n_proj < 1) return SL_ERR_SHAPE;
  const int mk = n_proj * k;
  const int64_t d_in = lin[0].d_in;
  int R = 0;
  for (int i = 0; i < n_ad; ++i) {
    if (!linear_ok(lin[i]) || lin[i].d_in != d_in) return SL_ERR_INVALID_ARG;
    if (lin[i].lora_scale != lin[0].lora_scale) return SL_ERR_UNSUPPORTED;
    R += lin[i].r;
  }
  if (mk > 64 || mk % 4 || R + mk > 256) return SL_ERR_SHAPE;
  if (ld_z < mk) return SL_ERR_SHAPE;
  if (ldx < d_in || ldx % 8 || !al16(x)) return SL_ERR_ALIGNMENT;
  if (ld_wat < d_in || ld_wat % 8 || !al16(w_a_t)) return SL_ERR_ALIGNMENT;
  if (!xa_s || ld_xa < R || ld_xa % 8 || !al16(xa_s)) return SL_ERR_ALIGNMENT;
  const int64_t T = n_tok;
  const int N = R + mk;
  const int64_t red = split_floats(T, N, d_in);
  {
    Carver c(nullptr);
    c.take<float>((size_t)red);
    if (sl_status st = ws_check(ws, c.off)) return st;
  }
  Carver c(ws->ptr);
  float* region = c.take<float>((size_t)red);
  GemmBuilder gb;
  int64_t off = 0;
  const int mx = gb.map(x, T, d_in, ldx, kBM);
  Prob* p = gb.add((int)T, N, kBN, (int)rup(N, 16));
  Seg* sg = gb.seg(p, mx, 0, 0, 0, 0, 0, (int)d_in, kBig);
  int toff = 0;
  for (int i = 0; i < n_ad; ++i) {
    gb.bsrc(sg, gb.map(lin[i].lora_a, lin[i].r, d_in, d_in, lin[i].r), toff, lin[i].r, 0, 0);
    toff += lin[i].r;
  }
  gb.bsrc(sg, gb.map(w_a_t, mk, d_in, ld_wat, mk), toff, mk, 0, 0);
  if (p) {
    p->epi = EPI_XA;
    p->out0 = xa;
    p->ld0 = ld_xa;
    p->out1 = xa_s;
    p->ld1 = ld_xa;
    p->a0 = 1.f;
    p->a1 = lin[0].lora_scale;
    p->z_col0 = R;
    p->z_rows = (int32_t)n_ctx;
    p->out2 = z;
    p->ld2 = ld_z;
  }
  maybe_split(gb, p, T, N, d_in, region, &off);
  return from_builder(gb.launch(err_word(ws), cs(stream)));
}

// a2 from a Z computed by sl_lora_fwd_estimate.
sl_status sl_svd_scores_from_z(sl_criterion crit, int32_t n_proj, const void* const* w_b, const int64_t* d_out,
                               int32_t k, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, const float* z,
                               int64_t ld_z, int64_t n_ctx, float* scores, float* scores_v, sl_workspace* ws,
                               sl_stream stream) {
  if (!z || !scores) return SL_ERR_INVALID_ARG;
  int64_t n_units = 0;
  if (sl_status st = criterion_units(crit, n_proj, w_b, d_out, k, n_q_heads, n_kv_heads, head_dim, !scores_v,
                                     &n_units))
    return st;
  const int mk = n_proj * k;
  if (n_ctx <= 0 || ld_z < mk || mk % 4) return SL_ERR_SHAPE;
  const int64_t tiles = (n_ctx + 127) / 128;
  const bool linear = crit != SL_CRIT_SWIGLU_L2;
  auto carve = [&](Carver& c, double** gp, uint16_t** zs) {
    *gp = linear ? c.take<double>((size_t)(tiles + 1) * mk * mk) : nullptr;  // tile shares, then their sum
    *zs = linear ? nullptr : c.take<uint16_t>((size_t)n_ctx * 128);
  };
  double* gp;
  uint16_t* zs;
  {
    Carver c(nullptr);
    carve(c, &gp, &zs);
    if (sl_status st = ws_check(ws, c.off)) return st;
  }
  Carver c(ws->ptr);
  carve(c, &gp, &zs);
  cudaStream_t s = cs(stream);
  // linear criteria: the Gram matrix of the whole context is summed inside the same launch
  double* gtot = linear ? gp + tiles * mk * mk : nullptr;
  if (int rc = z_finish(z, ld_z, n_ctx, mk, k, gp, zs, err_word(ws) + kCounterOffsetInts, gtot, s))
    return from_kernel(rc);
  int rc;
  if (!linear) {
    rc = est_swiglu_tc(zs, n_ctx, k, w_b[0], w_b[1], n_units, scores, nullptr, err_word(ws), s);
    return rc == 2 ? SL_ERR_ALIGNMENT : from_kernel(rc);
  }
  if (crit == SL_CRIT_L2)
    rc = est_scores(gtot, 1, mk, k, 0, nullptr, nullptr, 0, 0, 0, 0, 0, nullptr, w_b[0], 0, n_units, scores, s);
  else
    rc = est_scores(gtot, 1, mk, k, 0, w_b[0], w_b[1], 0, 1, n_q_heads, n_kv_heads, head_dim, scores,
                    n_proj == 3 ? w_b[2] : nullptr, 2, n_proj == 3 ? d_out[2] : 0, n_proj == 3 ? scores_v : nullptr,
                    s);
  return from_kernel(rc);
}

// ------------------------------------------------------------------ a4
sl_status sl_sparse_linear_fwd(int32_t n_lin, const sl_linear* lin, const sl_channels* ch, int32_t epi, const void* x,
                               int64_t ldx, int64_t n_tok, int64_t n_ctx, int32_t in_layout, int32_t out_layout,
                               const void* xa_s, int64_t ld_xa, void* const* y, const int64_t* ldy, sl_workspace* ws,
                               sl_stream stream) {
  if (!lin || !ch || !x || !xa_s || !y || !ldy || n_lin < 1 || n_lin > 4) return SL_ERR_INVALID_ARG;
  if (n_tok <= 0 || n_ctx < 0 || n_ctx > n_tok) return SL_ERR_SHAPE;
  const int64_t T = n_tok, C = n_ctx, O = T - C;
  const int slice = lin[0].slice;
  int R = 0;
  for (int i = 0; i < n_lin; ++i) {
    if (!linear_ok(lin[i]) || lin[i].slice != slice || lin[i].d_in != lin[0].d_in) return SL_ERR_INVALID_ARG;
    const sl_channels& c = epi == SL_EPI_SWIGLU ? ch[0] : ch[i];  // the paired SwiGLU call shares one set
    if (!channels_ok(c, slice == SL_SLICE_OUT ? lin[i].d_out : lin[i].d_in)) return SL_ERR_INVALID_ARG;
    R += lin[i].r;
  }
  const int64_t d_in = lin[0].d_in;
  if (ldx < d_in || ldx % 8 || !al16(x) || ld_xa < R || ld_xa % 8 || !al16(xa_s)) return SL_ERR_ALIGNMENT;
  cudaStream_t s = cs(stream);

  if (slice == SL_SLICE_OUT && epi == SL_EPI_NONE) {
    for (int i = 0; i < n_lin; ++i)
      if (!y[i] || ldy[i] < lin[i].d_out || ldy[i] % 8 || !al16(y[i])) return SL_ERR_ALIGNMENT;
    bool gath[4];  // kept rows read by the GEMM through sigma, no compacted copy
    for (int i = 0; i < n_lin; ++i) gath[i] = !lin[i].w_kept && gather_ok(ch[i], d_in);
    auto carve = [&](Carver& c, void** wc, void** bs) {
      for (int i = 0; i < n_lin; ++i) {
        wc[i] = lin[i].w_kept || gath[i] ? nullptr : c.take<uint16_t>((size_t)ch[i].n_keep * d_in);
        bs[i] = c.take<uint16_t>((size_t)lin[i].d_out * lin[i].r);
      }
    };
    void *wc[4], *bs[4];
    {
      Carver c(nullptr);
      carve(c, wc, bs);
      if (sl_status st = ws_check(ws, c.off)) return st;
    }
    Carver c(ws->ptr);
    carve(c, wc, bs);
    GatherBatch gat;  // sigma-ordered LoRA B (and kept weight rows that are neither given nor gathered), one launch
    for (int i = 0; i < n_lin; ++i) {
      if (lin[i].w_kept)
        wc[i] = const_cast<void*>(lin[i].w_kept);
      else if (!gath[i])
        gat.add(lin[i].w, d_in, lin[i].d_out, ch[i].sigma, ch[i].n_keep, d_in, wc[i], d_in);
      gat.add(lin[i].lora_b, lin[i].r, lin[i].d_out, ch[i].sigma, lin[i].d_out, lin[i].r, bs[i], lin[i].r);
    }
    if (int rc = gat.launch(err_word(ws), s)) return from_kernel(rc);
    GemmBuilder gb;
    const int mx = gb.map(x, T, d_in, ldx, kBM);
    int koff = 0;
    for (int i = 0; i < n_lin; ++i) {
      const sl_linear& L = lin[i];
      const int mxa = gb.map(static_cast<const uint16_t*>(xa_s) + koff, T, L.r, ld_xa, kBM);
      koff += L.r;
      if (C > 0) {
        const int mbs = gb.map(bs[i], L.d_out, L.r, L.r, kBN);
        Prob* p = gb.add((int)C, (int)L.d_out, kBN, kBN);
        Seg* sg = gb.seg(p, mx, 0, 0, 0, 0, 0, (int)d_in, (int)ch[i].n_keep);
        if (gath[i]) {
          gb.bsrc(sg, gb.gmap(L.w, L.d_out, d_in, d_in), 0, kBN, 0, kBN);
          gb.gather(sg, ch[i].sigma, ch[i].n_keep, L.d_out, d_in, zero_row(ws));
        } else {
          gb.bsrc(sg, gb.map(wc[i], ch[i].n_keep, d_in, d_in, kBN), 0, kBN, 0, kBN);
        }
        gb.bsrc(gb.seg(p, mxa, 0, 0, 0, 0, 0, L.r, kBig), mbs, 0, kBN, 0, kBN);
        if (p) {
          p->epi = EPI_BF16;
          p->out0 = y[i];
          p->ld0 = ldy[i];
          p->col_map = out_layout == SL_LAYOUT_NATURAL ? ch[i].sigma : nullptr;
        }
      }
      if (O > 0) {
        const int mw = gb.map(L.w, L.d_out, d_in, d_in, kBN);
        const int mb = gb.map(L.lora_b, L.d_out, L.r, L.r, kBN);
        Prob* p = gb.add((int)O, (int)L.d_out, kBN, kBN);
        gb.bsrc(gb.seg(p, mx, 0, (int)C, 0, 0, 0, (int)d_in, kBig), mw, 0, kBN, 0, kBN);
        gb.bsrc(gb.seg(p, mxa, 0, (int)C, 0, 0, 0, L.r, kBig), mb, 0, kBN, 0, kBN);
        if (p) {
          p->epi = EPI_BF16;
          p->out0 = y[i];
          p->ld0 = ldy[i];
          p->out_row0 = (int)C;
        }
      }
    }
    return from_builder(gb.launch(err_word(ws), s));
  }

  if (slice == SL_SLICE_OUT && epi == SL_EPI_SWIGLU) {
    if (n_lin != 2 || lin[0].d_out != lin[1].d_out || lin[0].r + lin[1].r > 64) return SL_ERR_INVALID_ARG;
    if (lin[0].lora_scale != lin[1].lora_scale) return SL_ERR_UNSUPPORTED;
    const int64_t F = lin[0].d_out;
    for (int i = 0; i < 3; ++i)
      if (!y[i] || ldy[i] < F || ldy[i] % 8 || !al16(y[i]) || ldy[i] != ldy[0]) return SL_ERR_ALIGNMENT;
    const int64_t nt = (F + 127) / 128;  // paired tiles: 128 channels each
    const bool gath = !lin[0].w_kept && !lin[1].w_kept && gather_ok(ch[0], d_in);
    auto carve = [&](Carver& c, void** wc, void** pk) {
      wc[0] = lin[0].w_kept || gath ? nullptr : c.take<uint16_t>((size_t)ch[0].n_keep * d_in);
      wc[1] = lin[1].w_kept || gath ? nullptr : c.take<uint16_t>((size_t)ch[0].n_keep * d_in);
      pk[0] = c.take<uint16_t>((size_t)nt * 256 * 64);  // sigma order
      pk[1] = c.take<uint16_t>((size_t)nt * 256 * 64);  // natural order
    };
    void *wc[2], *pk[2];
    {
      Carver c(nullptr);
      carve(c, wc, pk);
      if (sl_status st = ws_check(ws, c.off)) return st;
    }
    Carver c(ws->ptr);
    carve(c, wc, pk);
    const int32_t* sig = ch[0].sigma;
    GatherBatch gat;  // kept weight rows (when not given) and the paired LoRA B packs, one launch
    for (int i = 0; i < 2; ++i) {
      if (lin[i].w_kept)
        wc[i] = const_cast<void*>(lin[i].w_kept);
      else if (!gath)
        gat.add(lin[i].w, d_in, lin[i].d_out, sig, ch[0].n_keep, d_in, wc[i], d_in);
    }
    // LoRA B operand of a paired tile t: rows 256 t + j = [B_gate[c_j] | 0], rows 256 t + 128 + j = [0 | B_up[c_j]]
    cudaMemsetAsync(pk[0], 0, (size_t)nt * 256 * 64 * 2, s);
    cudaMemsetAsync(pk[1], 0, (size_t)nt * 256 * 64 * 2, s);
    for (int v = 0; v < 2; ++v) {
      const int32_t* idx = v == 0 ? sig : nullptr;
      gat.add(lin[0].lora_b, lin[0].r, F, idx, F, lin[0].r, pk[v], 64, 0, 128, 256, 0);
      gat.add(lin[1].lora_b, lin[1].r, F, idx, F, lin[1].r, pk[v], 64, lin[0].r, 128, 256, 128);
    }
    if (int rc = gat.launch(err_word(ws), s)) return from_kernel(rc);
    GemmBuilder gb;
    const int mx = gb.map(x, T, d_in, ldx, kBM);
    const int mxa = gb.map(xa_s, T, lin[0].r + lin[1].r, ld_xa, kBM);
    auto add_prob = [&](int64_t M, int64_t row0, int mg, int mu, int mp, int n_limit, bool gathered) {
      Prob* p = gb.add((int)M, (int)F, 128, kBN);
      Seg* sg = gb.seg(p, mx, 0, (int)row0, 0, 0, 0, (int)d_in, n_limit);
      gb.bsrc(sg, mg, 0, 128, 0, 128);
      gb.bsrc(sg, mu, 128, 128, 0, 128);
      if (gathered) gb.gather(sg, sig, ch[0].n_keep, F, d_in, zero_row(ws));
      gb.bsrc(gb.seg(p, mxa, 0, (int)row0, 0, 0, 0, 64, kBig), mp, 0, kBN, 0, kBN);
      if (!p) return;
      p->epi = EPI_SWIGLU;
      p->out0 = y[0];
      p->out1 = y[1];
      p->out2 = y[2];
      p->ld0 = ldy[0];
      p->out_row0 = (int)row0;
    };
    if (C > 0) {
      if (gath)
        add_prob(C, 0, gb.gmap(lin[0].w, F, d_in, d_in), gb.gmap(lin[1].w, F, d_in, d_in),
                 gb.map(pk[0], nt * 256, 64, 64, kBN), (int)ch[0].n_keep, true);
      else
        add_prob(C, 0, gb.map(wc[0], ch[0].n_keep, d_in, d_in, 128), gb.map(wc[1], ch[0].n_keep, d_in, d_in, 128),
                 gb.map(pk[0], nt * 256, 64, 64, kBN), (int)ch[0].n_keep, false);
    }
    if (O > 0)
      add_prob(O, C, gb.map(lin[0].w, F, d_in, d_in, 128), gb.map(lin[1].w, F, d_in, d_in, 128),
               gb.map(pk[1], nt * 256, 64, 64, kBN), kBig, false);
    return from_builder(gb.launch(err_word(ws), s));
  }

  if (slice == SL_SLICE_IN && epi == SL_EPI_NONE) {
    if (n_lin != 1) return SL_ERR_INVALID_ARG;
    const sl_linear& L = lin[0];
    if (!L.w_t || !al16(L.w_t)) return SL_ERR_INVALID_ARG;
    if (!y[0] || ldy[0] < L.d_out || ldy[0] % 8 || !al16(y[0])) return SL_ERR_ALIGNMENT;
    const int64_t nk = ch[0].n_keep;
    const bool in_sig = in_layout == SL_LAYOUT_SIGMA;
    const int64_t ldc = rup(nk, 8);
    const bool gath = !L.w_kept && gather_ok(ch[0], L.d_out);
    auto carve = [&](Carver& c, void** wtc, void** xc) {
      *wtc = L.w_kept ? const_cast<void*>(L.w_kept) : gath ? nullptr : c.take<uint16_t>((size_t)nk * L.d_out);
      *xc = (!in_sig && C > 0) ? c.take<uint16_t>((size_t)C * ldc) : nullptr;
    };
    void *wtc, *xc;
    {
      Carver c(nullptr);
      carve(c, &wtc, &xc);
      if (sl_status st = ws_check(ws, c.off)) return st;
    }
    Carver c(ws->ptr);
    carve(c, &wtc, &xc);
    if (!L.w_kept && !gath)
      if (int rc = gather_rows_bf16(L.w_t, L.d_out, L.d_in, ch[0].sigma, nk, L.d_out, wtc, L.d_out, 0, err_word(ws), s))
        return from_kernel(rc);
    if (xc)
      if (int rc = gather_cols_bf16(x, ldx, L.d_in, C, ch[0].sigma, nk, xc, ldc, err_word(ws), s)) return from_kernel(rc);
    GemmBuilder gb;
    const int mxa = gb.map(xa_s, T, L.r, ld_xa, kBM);
    const int mb = gb.map(L.lora_b, L.d_out, L.r, L.r, kBN);
    if (C > 0) {
      const int ma = in_sig ? gb.map(x, C, nk, ldx, kBM) : gb.map(xc, C, nk, ldc, kBM);
      Prob* p = gb.add((int)C, (int)L.d_out, kBN, kBN);
      Seg* sg = gb.seg(p, ma, 0, 0, 0, 1, 0, (int)nk, kBig);
      if (gath) {
        gb.bsrc(sg, gb.gmap(L.w_t, L.d_in, L.d_out, L.d_out), 0, kBN, 0, kBN);
        gb.gather(sg, ch[0].sigma, nk, L.d_in, L.d_out, zero_row(ws));
      } else {
        gb.bsrc(sg, gb.map(wtc, nk, L.d_out, L.d_out, 64), 0, kBN, 0, kBN);
      }
      gb.bsrc(gb.seg(p, mxa, 0, 0, 0, 0, 0, L.r, kBig), mb, 0, kBN, 0, kBN);
      if (p) {
        p->epi = EPI_BF16;
        p->out0 = y[0];
        p->ld0 = ldy[0];
      }
    }
    if (O > 0) {
      const int ma = gb.map(x, T, d_in, ldx, kBM);
      const int mw = gb.map(L.w, L.d_out, d_in, d_in, kBN);
      Prob* p = gb.add((int)O, (int)L.d_out, kBN, kBN);
      gb.bsrc(gb.seg(p, ma, 0, (int)C, 0, 0, 0, (int)d_in, kBig), mw, 0, kBN, 0, kBN);
      gb.bsrc(gb.seg(p, mxa, 0, (int)C, 0, 0, 0, L.r, kBig), mb, 0, kBN, 0, kBN);
      if (p) {
        p->epi = EPI_BF16;
        p->out0 = y[0];
        p->ld0 = ldy[0];
        p->out_row0 = (int)C;
      }
    }
    return from_builder(gb.launch(err_word(ws), s));
  }
  return SL_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------ a5
sl_status sl_sparse_linear_bwd(int32_t n_lin, const sl_linear* lin, const sl_channels* ch, int32_t epi,
                               const void* const* dy, const int64_t* ld_dy, int64_t n_tok, int64_t n_ctx,
                               int32_t in_layout, int32_t out_layout, const void* const* dya_s, void* dx,
                               int64_t lddx, const void* const* aux, void* const* aux_out, sl_workspace* ws,
                               sl_stream stream) {
  if (!lin || !ch || !dy || !ld_dy || !dya_s || n_lin < 1 || n_lin > 3) return SL_ERR_INVALID_ARG;
  if (n_tok <= 0 || n_ctx < 0 || n_ctx > n_tok) return SL_ERR_SHAPE;
  const int64_t T = n_tok, C = n_ctx, O = T - C;
  const int slice = lin[0].slice;
  const int64_t d_in = lin[0].d_in;
  for (int i = 0; i < n_lin; ++i) {
    if (!linear_ok(lin[i]) || lin[i].slice != slice || lin[i].d_in != d_in) return SL_ERR_INVALID_ARG;
    if (!channels_ok(ch[i], slice == SL_SLICE_OUT ? lin[i].d_out : lin[i].d_in)) return SL_ERR_INVALID_ARG;
    if (!dy[i] || !dya_s[i]) return SL_ERR_INVALID_ARG;
    if (ld_dy[i] < lin[i].d_out || ld_dy[i] % 8 || !al16(dy[i]) || !al16(dya_s[i])) return SL_ERR_ALIGNMENT;
  }
  cudaStream_t s = cs(stream);

  if (slice == SL_SLICE_OUT) {
    if (epi != SL_EPI_NONE) return SL_ERR_UNSUPPORTED;
    if (!dx || lddx < d_in || lddx % 8 || !al16(dx)) return SL_ERR_ALIGNMENT;
    const bool in_sig = in_layout == SL_LAYOUT_SIGMA;
    bool gath[3];  // kept rows read by the GEMM through sigma, no compacted copy
    for (int i = 0; i < n_lin; ++i) gath[i] = !lin[i].w_kept && gather_ok(ch[i], d_in);
    auto carve = [&](Carver& c, void** wc, void** dyc) {
      for (int i = 0; i < n_lin; ++i) {
        wc[i] = lin[i].w_kept ? const_cast<void*>(lin[i].w_kept)
                : gath[i]     ? nullptr
                              : c.take<uint16_t>((size_t)ch[i].n_keep * d_in);
        dyc[i] = (!in_sig && C > 0) ? c.take<uint16_t>((size_t)C * rup(ch[i].n_keep, 8)) : nullptr;
      }
    };
    void *wc[3], *dyc[3];
    {
      Carver c(nullptr);
      carve(c, wc, dyc);
      if (sl_status st = ws_check(ws, c.off)) return st;
    }
    Carver c(ws->ptr);
    carve(c, wc, dyc);
    GatherBatch gat;
    for (int i = 0; i < n_lin; ++i)
      if (!lin[i].w_kept && !gath[i])
        gat.add(lin[i].w, d_in, lin[i].d_out, ch[i].sigma, ch[i].n_keep, d_in, wc[i], d_in);
    if (int rc = gat.launch(err_word(ws), s)) return from_kernel(rc);
    for (int i = 0; i < n_lin; ++i) {
      if (dyc[i])
        if (int rc = gather_cols_bf16(dy[i], ld_dy[i], lin[i].d_out, C, ch[i].sigma, ch[i].n_keep, dyc[i], rup(ch[i].n_keep, 8),
                                      err_word(ws), s))
          return from_kernel(rc);
    }
    GemmBuilder gb;
    Prob* pc = C > 0 ? gb.add((int)C, (int)d_in, kBN, kBN) : nullptr;
    Prob* po = O > 0 ? gb.add((int)O, (int)d_in, kBN, kBN) : nullptr;
    for (int i = 0; i < n_lin; ++i) {
      const sl_linear& L = lin[i];
      const int mya = gb.map(dya_s[i], T, L.r, L.r, kBM);
      const int mam = gb.map(L.lora_a, L.r, d_in, d_in, 64);
      if (pc) {
        const int64_t nk = ch[i].n_keep;
        const int ma = dyc[i] ? gb.map(dyc[i], C, nk, rup(nk, 8), kBM) : gb.map(dy[i], C, nk, ld_dy[i], kBM);
        Seg* sg = gb.seg(pc, ma, 0, 0, 0, 1, 0, (int)nk, kBig);
        if (gath[i]) {
          gb.bsrc(sg, gb.gmap(L.w, L.d_out, d_in, d_in), 0, kBN, 0, kBN);
          gb.gather(sg, ch[i].sigma, nk, L.d_out, d_in, zero_row(ws));
        } else {
          gb.bsrc(sg, gb.map(wc[i], nk, d_in, d_in, 64), 0, kBN, 0, kBN);
        }
        gb.bsrc(gb.seg(pc, mya, 0, 0, 0, 1, 0, L.r, kBig), mam, 0, kBN, 0, kBN);
      }
      if (po) {
        const int ma = gb.map(dy[i], T, L.d_out, ld_dy[i], kBM);
        const int mw = gb.map(L.w, L.d_out, d_in, d_in, 64);
        gb.bsrc(gb.seg(po, ma, 0, (int)C, 0, 1, 0, (int)L.d_out, kBig), mw, 0, kBN, 0, kBN);
        gb.bsrc(gb.seg(po, mya, 0, (int)C, 0, 1, 0, L.r, kBig), mam, 0, kBN, 0, kBN);
      }
    }
    for (Prob* p : {pc, po}) {
      if (!p) continue;
      p->epi = EPI_BF16;
      p->out0 = dx;
      p->ld0 = lddx;
      p->out_row0 = p == po ? (int)C : 0;
    }
    return from_builder(gb.launch(err_word(ws), s));
  }

  // SL_SLICE_IN
  if (n_lin != 1) return SL_ERR_INVALID_ARG;
  const sl_linear& L = lin[0];
  if (!L.w_t || !al16(L.w_t)) return SL_ERR_INVALID_ARG;
  const bool swiglu = epi == SL_EPI_SWIGLU;
  if (swiglu) {
    if (!aux || !aux_out || !aux[0] || !aux[1] || !aux_out[0] || !aux_out[1]) return SL_ERR_INVALID_ARG;
    if (lddx < d_in || lddx % 8) return SL_ERR_ALIGNMENT;
    for (int i = 0; i < 2; ++i)
      if (!al16(aux[i]) || !al16(aux_out[i])) return SL_ERR_ALIGNMENT;
  } else {
    if (epi != SL_EPI_NONE) return SL_ERR_INVALID_ARG;
    if (!dx || lddx < d_in || lddx % 8 || !al16(dx)) return SL_ERR_ALIGNMENT;
  }
  const int64_t nk = ch[0].n_keep;
  const bool gath = !L.w_kept && gather_ok(ch[0], L.d_out);
  auto carve = [&](Carver& c, void** wtc, void** at, void** ats) {
    *wtc = L.w_kept ? const_cast<void*>(L.w_kept) : gath ? nullptr : c.take<uint16_t>((size_t)nk * L.d_out);
    *at = c.take<uint16_t>((size_t)d_in * L.r);
    *ats = c.take<uint16_t>((size_t)d_in * L.r);
  };
  void *wtc, *at, *ats;
  {
    Carver c(nullptr);
    carve(c, &wtc, &at, &ats);
    if (sl_status st = ws_check(ws, c.off)) return st;
  }
  Carver c(ws->ptr);
  carve(c, &wtc, &at, &ats);
  if (int rc = transpose_bf16(L.lora_a, L.r, d_in, d_in, at, L.r, s)) return from_kernel(rc);
  {
    GatherBatch gat;  // the permuted A^T (and kept rows of W^T that are neither given nor gathered), one launch
    if (!L.w_kept && !gath) gat.add(L.w_t, L.d_out, L.d_in, ch[0].sigma, nk, L.d_out, wtc, L.d_out);
    gat.add(at, L.r, d_in, ch[0].sigma, d_in, L.r, ats, L.r);
    if (int rc = gat.launch(err_word(ws), s)) return from_kernel(rc);
  }
  GemmBuilder gb;
  const int mdy = gb.map(dy[0], T, L.d_out, ld_dy[0], kBM);
  const int mya = gb.map(dya_s[0], T, L.r, L.r, kBM);
  auto set_epi = [&](Prob* p, int64_t row0, bool natural_ctx) {
    if (!p) return;
    p->out_row0 = (int)row0;
    if (swiglu) {
      p->epi = EPI_DSWIGLU;
      p->out0 = aux_out[0];
      p->out1 = aux_out[1];
      p->aux0 = aux[0];
      p->aux1 = aux[1];
      p->ld0 = lddx;
      p->ld_aux = lddx;
    } else {
      p->epi = EPI_BF16;
      p->out0 = dx;
      p->ld0 = lddx;
      p->col_map = natural_ctx ? ch[0].sigma : nullptr;
    }
  };
  if (C > 0) {
    const int mat = gb.map(ats, d_in, L.r, L.r, kBN);
    Prob* p = gb.add((int)C, (int)d_in, kBN, kBN);
    Seg* sg = gb.seg(p, mdy, 0, 0, 0, 0, 0, (int)L.d_out, (int)nk);
    if (gath) {
      gb.bsrc(sg, gb.gmap(L.w_t, L.d_in, L.d_out, L.d_out), 0, kBN, 0, kBN);
      gb.gather(sg, ch[0].sigma, nk, L.d_in, L.d_out, zero_row(ws));
    } else {
      gb.bsrc(sg, gb.map(wtc, nk, L.d_out, L.d_out, kBN), 0, kBN, 0, kBN);
    }
    gb.bsrc(gb.seg(p, mya, 0, 0, 0, 0, 0, L.r, kBig), mat, 0, kBN, 0, kBN);
    set_epi(p, 0, !swiglu && out_layout == SL_LAYOUT_NATURAL);
  }
  if (O > 0) {
    const int mw = gb.map(L.w, L.d_out, d_in, d_in, 64);
    const int mam = gb.map(L.lora_a, L.r, d_in, d_in, 64);
    Prob* p = gb.add((int)O, (int)d_in, kBN, kBN);
    gb.bsrc(gb.seg(p, mdy, 0, (int)C, 0, 1, 0, (int)L.d_out, kBig), mw, 0, kBN, 0, kBN);
    gb.bsrc(gb.seg(p, mya, 0, (int)C, 0, 1, 0, L.r, kBig), mam, 0, kBN, 0, kBN);
    set_epi(p, C, false);
  }
  return from_builder(gb.launch(err_word(ws), s));
}

sl_status sl_profile_enable(int32_t on) {
  g_prof.store(on != 0);
  return SL_OK;
}

sl_status sl_profile_read(int64_t* kernel_launches, int64_t* gemm_launches, double* gemm_ms) {
  if (!kernel_launches || !gemm_launches || !gemm_ms) return SL_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_ev_mu);
  double ms = 0.0;
  for (size_t i = 0; i < g_ev_used; ++i) {
    float t = 0.f;
    if (cudaEventSynchronize(g_events[i].second) != cudaSuccess) return SL_ERR_CUDA;
    if (cudaEventElapsedTime(&t, g_events[i].first, g_events[i].second) != cudaSuccess) return SL_ERR_CUDA;
    ms += t;
#ifdef SL_PROFILE_DUMP
    fprintf(stderr, "[sl gemm %zu] %.4f ms %s\n", i, t, i < g_notes.size() ? g_notes[i].c_str() : "");
#endif
  }
  *gemm_ms = ms;
  *gemm_launches = (int64_t)g_ev_used;
  *kernel_launches = (int64_t)g_launches.exchange(0);
  g_ev_used = 0;
  return SL_OK;
}

sl_status sl_profile_launches(int64_t capacity, double* ms, int32_t* kind, int64_t* count) {
  if (!count || capacity < 0 || (capacity > 0 && (!ms || !kind))) return SL_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_ev_mu);
  *count = (int64_t)g_ev_used;
  for (size_t i = 0; i < g_ev_used && (int64_t)i < capacity; ++i) {
    float t = 0.f;
    if (cudaEventSynchronize(g_events[i].second) != cudaSuccess) return SL_ERR_CUDA;
    if (cudaEventElapsedTime(&t, g_events[i].first, g_events[i].second) != cudaSuccess) return SL_ERR_CUDA;
    ms[i] = t;
    kind[i] = g_ev_kind[i];
  }
  return SL_OK;
}

// ------------------------------------------------------------------ attention core
namespace {
sl_status attention_args(const void* const* ptrs, int n_ptrs, int64_t ldq, int64_t ldkv, int32_t n_seq,
                         int32_t seq_len, int32_t hq, int32_t hkv, int32_t hd) {
  for (int i = 0; i < n_ptrs; ++i)
    if (!ptrs[i]) return SL_ERR_INVALID_ARG;
  if (n_seq < 1 || seq_len < 1 || hq < 1 || hkv < 1 || hq % hkv || hd < 8 || hd > 128 || hd % 8) return SL_ERR_SHAPE;
  if ((int64_t)n_seq * seq_len > (int64_t)1 << 31 || seq_len > (1 << 24) || hq > 65535 || hkv > 65535)
    return SL_ERR_SHAPE;
  if (ldq < (int64_t)hq * hd || ldkv < (int64_t)hkv * hd) return SL_ERR_SHAPE;
  if (ldq % 8 || ldkv % 8) return SL_ERR_ALIGNMENT;
  for (int i = 0; i < n_ptrs; ++i)
    if (!al16(ptrs[i])) return SL_ERR_ALIGNMENT;
  return SL_OK;
}
}  // namespace

sl_status sl_attention_fwd(const void* q, const void* k, const void* v, int64_t ldq, int64_t ldkv, int32_t n_seq,
                           int32_t seq_len, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, void* o,
                           float* lse, sl_workspace* ws, sl_stream stream) {
  const void* ptrs[5] = {q, k, v, o, lse};
  if (sl_status st = attention_args(ptrs, 5, ldq, ldkv, n_seq, seq_len, n_q_heads, n_kv_heads, head_dim)) return st;
  if (sl_status st = ws_check(ws, kWorkspaceHeaderBytes)) return st;
  const int rc = attention_fwd(q, k, v, ldq, ldkv, n_seq, seq_len, n_q_heads, n_kv_heads, head_dim, o, ldq, lse,
                               err_word(ws), cs(stream));
  return rc == 0 ? SL_OK : (rc == 2 ? SL_ERR_ALIGNMENT : SL_ERR_CUDA);
}

sl_status sl_attention_bwd(const void* q, const void* k, const void* v, const void* o, const void* d_o,
                           const float* lse, int64_t ldq, int64_t ldkv, int32_t n_seq, int32_t seq_len,
                           int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, void* dq, void* dk, void* dv,
                           sl_workspace* ws, sl_stream stream) {
  const void* ptrs[9] = {q, k, v, o, d_o, lse, dq, dk, dv};
  if (sl_status st = attention_args(ptrs, 9, ldq, ldkv, n_seq, seq_len, n_q_heads, n_kv_heads, head_dim)) return st;
  Carver c(nullptr);
  c.take<uint8_t>(attention_bwd_scratch(n_seq, seq_len, n_q_heads, head_dim));
  if (sl_status st = ws_check(ws, c.off)) return st;
  Carver c2(ws->ptr);
  void* scratch = c2.take<uint8_t>(attention_bwd_scratch(n_seq, seq_len, n_q_heads, head_dim));
  const int rc = attention_bwd(q, k, v, o, d_o, lse, ldq, ldkv, n_seq, seq_len, n_q_heads, n_kv_heads, head_dim, dq,
                               dk, dv, scratch, err_word(ws), cs(stream));
  return rc == 0 ? SL_OK : (rc == 2 ? SL_ERR_ALIGNMENT : SL_ERR_CUDA);
}

sl_status sl_set_pair_tile_rows(int32_t rows) {
  if (rows != 0 && rows != 128 && rows != 256 && rows != 512) return SL_ERR_INVALID_ARG;
  set_forced_pair_mh(rows == 128 ? -1 : rows / 256);
  return SL_OK;
}

sl_status sl_prepare_weight(const void* w, int64_t d_out, int64_t d_in, void* w_t, sl_stream stream) {
  if (!w || !w_t) return SL_ERR_INVALID_ARG;
  if (d_out <= 0 || d_in <= 0) return SL_ERR_SHAPE;
  return from_kernel(transpose_bf16(w, d_out, d_in, d_in, w_t, d_out, cs(stream)));
}

sl_status sl_permute_rows(const void* src, int64_t ld_src, int64_t src_rows, const int32_t* perm, int64_t n_rows,
                          int64_t n_cols, void* dst, int64_t ld_dst, sl_stream stream) {
  if (!src || !perm || !dst) return SL_ERR_INVALID_ARG;
  if (src_rows <= 0 || n_rows <= 0 || n_cols <= 0 || ld_src < n_cols || ld_dst < n_cols) return SL_ERR_SHAPE;
  return from_kernel(
      gather_rows_bf16(src, ld_src, src_rows, perm, n_rows, n_cols, dst, ld_dst, 0, aux_debug_word(), cs(stream)));
}

sl_status sl_permute_rows_sigma(const void* src, int64_t ld_src, int64_t src_rows, const int32_t* perm,
                                int64_t n_rows, int64_t n_cols, const int32_t* sigma, int64_t n_ctx, int32_t to_sigma,
                                void* dst, int64_t ld_dst, sl_stream stream) {
  if (!src || !perm || !sigma || !dst) return SL_ERR_INVALID_ARG;
  if (src_rows <= 0 || n_rows <= 0 || n_cols <= 0 || n_cols > kPermMaxCols || n_ctx < 0 || ld_src < n_cols ||
      ld_dst < n_cols)
    return SL_ERR_SHAPE;
  if (n_cols % 8 || ld_src % 8 || ld_dst % 8 || !al16(src) || !al16(dst)) return SL_ERR_ALIGNMENT;
  const int rc = permute_rows_sigma(src, ld_src, src_rows, perm, n_rows, n_cols, sigma, n_ctx, to_sigma ? 1 : 0, dst,
                                    ld_dst, aux_debug_word(), cs(stream));
  return rc == 2 ? SL_ERR_ALIGNMENT : from_kernel(rc);
}

sl_status sl_gather_rows_batch(int32_t n, const void* const* src, const int64_t* ld_src, const int64_t* src_rows,
                               const int32_t* const* perm, const int64_t* n_rows, const int64_t* n_cols,
                               void* const* dst, const int64_t* ld_dst, sl_stream stream) {
  if (n < 1 || n > kMaxGatherJobs || !src || !ld_src || !src_rows || !perm || !n_rows || !n_cols || !dst || !ld_dst)
    return SL_ERR_INVALID_ARG;
  GatherBatch gat;
  for (int q = 0; q < n; ++q) {
    if (n_rows[q] < 0) return SL_ERR_SHAPE;
    if (n_rows[q] == 0) continue;
    if (!src[q] || !perm[q] || !dst[q]) return SL_ERR_INVALID_ARG;
    if (n_cols[q] <= 0 || src_rows[q] <= 0 || ld_src[q] < n_cols[q] || ld_dst[q] < n_cols[q]) return SL_ERR_SHAPE;
    gat.add(src[q], ld_src[q], src_rows[q], perm[q], n_rows[q], n_cols[q], dst[q], ld_dst[q]);
  }
  return from_kernel(gat.launch(aux_debug_word(), cs(stream)));
}

int32_t sl_debug_bounds_enabled(void) {
#ifdef SL_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

sl_status sl_read_debug_flag(int32_t* code, sl_stream stream) {
  if (!code) return SL_ERR_INVALID_ARG;
  *code = 0;
  int* w = aux_debug_word();
  if (!w) return SL_OK;  // release build: no checks, nothing recorded
  if (cudaMemcpyAsync(code, w, sizeof(int32_t), cudaMemcpyDeviceToHost, cs(stream)) != cudaSuccess ||
      cudaMemsetAsync(w, 0, sizeof(int32_t), cs(stream)) != cudaSuccess ||
      cudaStreamSynchronize(cs(stream)) != cudaSuccess)
    return SL_ERR_CUDA;
  return *code ? SL_ERR_DEVICE_FLAG : SL_OK;
}

}  // extern "C"
