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
// The array is file-scope `static __device__` storage, one copy per device: every device on
// which the library's module is loaded holds these 8 MiB until the process exits (or the
// device's context is destroyed), whether or not this entry is ever called. Host code cannot
// use the array's name as an address (on the host it names a stand-in), so its device address
// is looked up with cudaGetSymbolAddress, with the device current, on the first call made while
// the device is current; that first call should therefore precede any stream capture on that
// device. The address is cached per device together with the identifier of the CUDA context it
// belongs to: after a device reset (cudaDeviceReset) the next call sees a new context and looks
// the address up again (that call, too, should not be captured). Every call shares the array
// and leaves its contents behind: the 64 KiB header (error word and counters) is cleared at the
// start of every call, and every other byte a call reads it has first written itself. Two
// calls whose execution overlaps (different streams, or different host threads without
// ordering) race on the array; callers serialise them.
#include <cstring>
#include <mutex>

#include <cuda.h>

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
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // identifier of the context g_scratch_ptr belongs to

// Identifier of the calling thread's current CUDA context (unique for the process's lifetime,
// never reused; a device reset gives the device a new one); 0 if it cannot be read.
unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of this device's copy of the array in the current context; looked up once
// per device and context.
sl_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SL_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_setup_mu);
  // no context current on this thread yet (0), a first call, or a new context after a reset:
  // look the address up (which makes the device's primary context current) and note the context
  const unsigned long long ctx = current_context_id();
  if (!g_scratch_ptr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SL_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();
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
