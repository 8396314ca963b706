// Top-n channel selection by radix select over fp32 scores (one CTA per call).
//
// Scores become order-preserving 32-bit keys (NaN lowest, -0 == +0). Four 8-bit
// passes over shared-memory histograms find the n-th largest key K*; every key
// above K* is kept, and among keys equal to K* the lowest indices are kept, so
// exactly n channels survive. The output is a permutation sigma of [0, N):
// sigma[0, n) = kept channels ascending, sigma[n, N) = dropped channels
// ascending. Optionally the selection over KV units (g, d) is expanded to the
// query side: query channel (h, d) is kept iff unit (h / heads_per_group, d) is.
#include "sl_internal.h"

namespace sl {

namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelMaxN = 40960;  // keys + flags in shared memory

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f != f) return 0u;                 // NaN ranks below every number
  if (u == 0x80000000u) u = 0u;          // -0 ranks equal to +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block scan of one int per thread (1024 threads). Returns the total.
__device__ int block_exclusive_scan(int v, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    warp_sums[lane] = wi - w;  // exclusive prefix of warp totals
    if (lane == 31) warp_sums[32] = wi;
  }
  __syncthreads();
  const int excl = warp_sums[warp] + incl - v;
  total = warp_sums[32];
  __syncthreads();
  return excl;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(const float* __restrict__ scores, int n, int n_keep,
                                                             int32_t* __restrict__ sigma, int hpg, int head_dim,
                                                             int n_wide, int32_t* __restrict__ sigma_wide) {
  pdl_wait();
  extern __shared__ uint32_t sel_smem[];
  uint32_t* keys = sel_smem;                                    // [n]
  uint8_t* keep = reinterpret_cast<uint8_t*>(keys + n);         // [n]
  __shared__ int hist[256];
  __shared__ int warp_sums[33];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_remaining;

  for (int i = threadIdx.x; i < n; i += kSelThreads) keys[i] = score_key(scores[i]);
  if (threadIdx.x == 0) {
    s_prefix = 0;
    s_mask = 0;
    s_remaining = n_keep;
  }
  __syncthreads();

  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (threadIdx.x < 256) hist[threadIdx.x] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    // Scores concentrate in few exponent bins: aggregate equal bins within a warp so each
    // bin takes one shared-memory atomic per warp instead of one per lane.
    const int n_round = (n + kSelThreads - 1) / kSelThreads * kSelThreads;
    for (int i = threadIdx.x; i < n_round; i += kSelThreads) {
      const uint32_t k = i < n ? keys[i] : 0u;
      const bool active = i < n && (k & mask) == prefix;
      const uint32_t bin = active ? ((k >> shift) & 255u) : 256u;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (active && (int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns bins [255 - 8l - 7, 255 - 8l], walked from the top
      const int lane = threadIdx.x;
      int local = 0;
      for (int j = 0; j < 8; ++j) local += hist[255 - 8 * lane - j];
      int incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int rem = s_remaining;
      const int excl = incl - local;
      const bool here = excl < rem && incl >= rem;
      const unsigned ball = __ballot_sync(0xffffffffu, here);
      if (here && lane == __ffs(ball) - 1) {
        int cum = excl;
        for (int j = 0; j < 8; ++j) {
          const int b = 255 - 8 * lane - j;
          if (cum + hist[b] >= rem) {
            s_remaining = rem - cum;
            s_prefix = prefix | ((uint32_t)b << shift);
            s_mask = mask | (255u << shift);
            break;
          }
          cum += hist[b];
        }
      }
    }
    __syncthreads();
  }
  const uint32_t thr = s_prefix;
  const int take_eq = s_remaining;

  // Each thread owns a contiguous index range, so block scans give index-order ranks.
  const int per = (n + kSelThreads - 1) / kSelThreads;
  const int i0 = min(n, (int)threadIdx.x * per), i1 = min(n, i0 + per);
  int n_eq = 0;
  for (int i = i0; i < i1; ++i) n_eq += keys[i] == thr;
  int tot;
  int eq_rank = block_exclusive_scan(n_eq, warp_sums, tot);
  int n_kept = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t k = keys[i];
    bool kp = k > thr;
    if (k == thr) {
      kp = eq_rank < take_eq;
      ++eq_rank;
    }
    keep[i] = kp;
    n_kept += kp;
  }
  int kept_before = block_exclusive_scan(n_kept, warp_sums, tot);
  int drop_before = i0 - kept_before;
  for (int i = i0; i < i1; ++i) {
    if (keep[i]) sigma[kept_before++] = i;
    else sigma[n_keep + drop_before++] = i;
  }
  if (hpg <= 0 || sigma_wide == nullptr) return;
  __syncthreads();
  // Query-side expansion: channel c = h * head_dim + d follows unit (h / hpg) * head_dim + d.
  const int n_keep_w = n_keep * hpg;
  const int perw = (n_wide + kSelThreads - 1) / kSelThreads;
  const int w0 = min(n_wide, (int)threadIdx.x * perw), w1 = min(n_wide, w0 + perw);
  auto unit_of = [&](int c) { return (c / head_dim / hpg) * head_dim + c % head_dim; };
  int nk = 0;
  for (int c = w0; c < w1; ++c) nk += keep[unit_of(c)];
  int kb = block_exclusive_scan(nk, warp_sums, tot);
  int db = w0 - kb;
  for (int c = w0; c < w1; ++c) {
    if (keep[unit_of(c)]) sigma_wide[kb++] = c;
    else sigma_wide[n_keep_w + db++] = c;
  }
}

}  // namespace

int select_channels(const float* scores, int64_t n, int64_t n_keep, int32_t* sigma, int heads_per_group, int head_dim,
                    int64_t n_wide, int32_t* sigma_wide, int64_t* n_keep_wide_out, cudaStream_t s) {
  if (n <= 0 || n > kSelMaxN || n_keep < 1 || n_keep > n) return 1;
  if (sigma_wide && (heads_per_group <= 0 || head_dim <= 0 || n % head_dim || n_wide != n * heads_per_group))
    return 1;
  const size_t smem = (size_t)n * 5;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelMaxN * 5 + 64);
    attr = true;
  }
  launch_kernel(select_kernel, 1, kSelThreads, (smem + 15) / 16 * 16, s, scores, (int)n, (int)n_keep, sigma,
                                                               sigma_wide ? heads_per_group : 0, head_dim,
                                                               (int)n_wide, sigma_wide);
  if (n_keep_wide_out) *n_keep_wide_out = sigma_wide ? n_keep * heads_per_group : 0;
  if (launch_failed("sl_select")) return 5;
  note_launch();
  return 0;
}

}  // namespace sl
