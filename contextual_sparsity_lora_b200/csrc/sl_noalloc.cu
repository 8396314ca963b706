// sl_svd_estimate_noalloc: the SVD estimator and criterion of sl_svd_estimate, with its
// scratch taken from a fixed array compiled into this library instead of a caller
// workspace, so a call allocates nothing.
//
// Which callers need it: a host that cannot hand the library a workspace, e.g. a plain C
// program that keeps no device allocator of its own, or code that must not call
// cudaMalloc/cudaFree at all while it runs (cudaFree synchronises the whole device and
// would stall the work queued on every other stream; an allocator can also be absent or
// capped in such a process). The estimator is the one stage whose scratch is small and
// bounded by its shapes (rank-k projections of the context rows, small Gram partials,
// the transposed rank-k factors, split-K partials), which makes a fixed array practical.
//
// The array is file-scope `static __device__` storage, one copy per device. Its device
// address is looked up once per device (cudaGetSymbolAddress, with that device current)
// on the first call made while the device is current; that first call should therefore
// precede any stream capture on that device. Every call shares the array and leaves its
// contents behind: the 64 KiB header (error word and counters) is cleared at the start
// of every call, and every other byte a call reads it has first written itself. Two calls
// whose execution overlaps (different streams, or different host threads without
// ordering) race on the array; callers serialise them.
#include <cstring>
#include <mutex>

#include "../../include/sparselora.h"
#include "sl_internal.h"

namespace {

// Fixed scratch: the 64 KiB workspace header plus up to 8 MiB - 64 KiB of estimator
// scratch. The LLaMA-7B/8B/13B projection shapes with 3072 context tokens need under
// 2.5 MiB; larger requests are rejected before any device work.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
static_assert(kNoAllocScratchBytes > (size_t)sl::kWorkspaceHeaderBytes, "scratch smaller than its header");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's copy of the array; looked up once per device.
sl_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SL_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SL_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SL_OK;
}

}  // namespace

extern "C" {

sl_status sl_svd_estimate_noalloc(sl_criterion crit, sl_dtype dtype, const void* x, int64_t n_ctx, int64_t d_in,
                                  int64_t ldx, int32_t n_proj, const void* const* w_a, const void* const* w_b,
                                  const int64_t* d_out, int32_t k, int32_t n_q_heads, int32_t n_kv_heads,
                                  int32_t head_dim, float* scores, float* scores_v, int64_t* scratch_needed,
                                  int32_t* device_flag, sl_stream stream) {
  // Size query: the workspace entry validates every argument and reports the bytes it
  // would carve, doing no device work when handed no workspace.
  sl_workspace q{nullptr, 0, 0};
  sl_status st = sl_svd_estimate(crit, dtype, x, n_ctx, d_in, ldx, n_proj, w_a, w_b, d_out, k, n_q_heads,
                                 n_kv_heads, head_dim, scores, scores_v, &q, stream);
  if (st != SL_ERR_WORKSPACE) return st;  // an argument error
  if (scratch_needed) *scratch_needed = (int64_t)q.needed;
  if (q.needed > kNoAllocScratchBytes) return SL_ERR_WORKSPACE;
  void* base = nullptr;
  if ((st = scratch_for_current_device(&base))) return st;
  sl_workspace ws{base, kNoAllocScratchBytes, 0};
  if ((st = sl_workspace_init(&ws, stream))) return st;
  st = sl_svd_estimate(crit, dtype, x, n_ctx, d_in, ldx, n_proj, w_a, w_b, d_out, k, n_q_heads, n_kv_heads,
                       head_dim, scores, scores_v, &ws, stream);
  if (st) return st;
  if (device_flag &&
      cudaMemcpyAsync(device_flag, base, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SL_ERR_CUDA;
  return SL_OK;
}

}  // extern "C"
