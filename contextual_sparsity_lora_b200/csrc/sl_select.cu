// Top-n channel selection over fp32 scores (one CTA per call: 256 to 1024 threads by set size).
//
// Scores become order-preserving 32-bit keys (NaN lowest, -0 == +0), held in registers:
// thread t owns the contiguous index range [t * per, (t + 1) * per). The n-th largest key
// K* is found by radix selection a byte at a time from the most significant byte in which two
// keys differ (a shared-memory histogram of 256 bins per pass, at most four passes; one warp
// picks each byte). Every key above K* is kept, and among keys equal to K* the lowest indices
// are kept, so exactly n channels survive. The output is a permutation
// sigma of [0, N): sigma[0, n) = kept channels ascending, sigma[n, N) = dropped channels
// ascending. Optionally the selection over KV units (g, d) is expanded to the query side:
// query channel (h, d) is kept iff unit (h / heads_per_group, d) is. Scores come in and
// sigma goes out through shared memory with coalesced global accesses (one CTA issues all of
// them, so per-thread strided accesses would pay a 32-byte sector per 4-byte element).
#include "sl_internal.h"

namespace sl {

namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelMaxN = 40960;
constexpr int kSelMaxNWide = 16384;  // units of a selection with the query-side expansion
constexpr int kSelStageWords = 40960;  // staging words for scores in / sigma out (160 KB)

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f != f) return 0u;                 // NaN ranks below every number
  if (u == 0x80000000u) u = 0u;          // -0 ranks equal to +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block scan of one unsigned int per thread (NT threads, arithmetic modulo 2^32)
// that also returns the block total.
template <int NT>
__device__ uint32_t block_exclusive_scan_total(uint32_t v, uint32_t* warp_sums, uint32_t* total_slot,
                                               uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < NT / 32 ? warp_sums[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < NT / 32) warp_sums[lane] = wi - w;  // exclusive prefix of warp totals
    if (lane == 31) *total_slot = wi;
  }
  __syncthreads();
  const uint32_t excl = warp_sums[warp] + incl - v;
  total = *total_slot;
  __syncthreads();
  return excl;
}

__host__ __device__ inline int stage_words(int n, int n_wide) {
  return n_wide <= kSelStageWords && n_wide > n ? n_wide : n;
}

template <int PER, int NT>
__global__ void __launch_bounds__(NT) select_kernel(const float* __restrict__ scores, int n, int n_keep,
                                                             int32_t* __restrict__ sigma, int hpg, int head_dim,
                                                             int n_wide, int32_t* __restrict__ sigma_wide) {
  pdl_wait();
  // staging words for scores in / sigma out (and sigma_wide when it fits), then, for the
  // query-side expansion, kbu[n]: the kept units before each unit
  extern __shared__ uint32_t sbuf[];
  uint16_t* kbu = reinterpret_cast<uint16_t*>(sbuf + stage_words(n, n_wide));
  __shared__ uint32_t s_or[32], s_and[32];
  __shared__ int warp_sums[32];
  __shared__ uint32_t warp_sums_u[32];
  __shared__ int hist[4][256];  // one histogram per radix pass, all zeroed before the first
  __shared__ int sel_state[2];
  __shared__ uint32_t scan_total;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per = (n + NT - 1) / NT;  // <= PER
  const int i0 = min(n, (int)threadIdx.x * per), i1 = min(n, i0 + per);
  for (int i = threadIdx.x; i < n; i += NT) sbuf[i] = __float_as_uint(scores[i]);
  for (int i = threadIdx.x; i < 4 * 256; i += NT) (&hist[0][0])[i] = 0;
  __syncthreads();

  uint32_t key[PER];
  uint32_t kor = 0u, kand = 0xffffffffu;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int i = i0 + j;
    key[j] = i < i1 ? score_key(__uint_as_float(sbuf[i])) : 0u;
    if (i < i1) {
      kor |= key[j];
      kand &= key[j];
    }
  }
  kor = __reduce_or_sync(0xffffffffu, kor);
  kand = __reduce_and_sync(0xffffffffu, kand);
  if (lane == 0) {
    s_or[warp] = kor;
    s_and[warp] = kand;
  }
  __syncthreads();
  const uint32_t bor = __reduce_or_sync(0xffffffffu, lane < NT / 32 ? s_or[lane] : 0u);
  const uint32_t band = __reduce_and_sync(0xffffffffu, lane < NT / 32 ? s_and[lane] : 0xffffffffu);
  // The n-th largest key K* by radix selection, 8 bits per pass from the byte holding the highest
  // bit in which two keys differ (every key shares the bits above it): per pass, a 256-bin
  // histogram of the next byte over the keys that match the bytes chosen so far; the chosen byte is
  // the one where the count of matching keys with a larger byte stops falling short of the places
  // still to fill. After the last pass T = K* exactly, and `need` keys equal to T are to be kept.
  const uint32_t diff = bor ^ band;
  const int top = diff ? 31 - __clz(diff) : -1;  // highest bit in which two keys differ
  uint32_t T = band;                              // every byte at or above top's is decided below
  uint32_t tmask = 0u;
  int need = n_keep;
  if (top >= 0) {
    const int first = (top / 8) * 8;
    tmask = first + 8 < 32 ? ~((1u << (first + 8)) - 1u) : 0u;  // bytes above the first pass
    T &= tmask;
    for (int shift = first, pass = 0; shift >= 0; shift -= 8, ++pass) {
#pragma unroll
      for (int j = 0; j < PER; ++j)
        if (i0 + j < i1 && (key[j] & tmask) == T) atomicAdd(&hist[pass][(key[j] >> shift) & 255u], 1);
      __syncthreads();
      if (warp == 0) {
        // lane l holds bins 255 - 8 l .. 248 - 8 l (descending), counts from the top; one warp
        // picks (all 32 warps doing it cost more issue slots than the extra barrier)
        int c[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          c[e] = hist[pass][255 - 8 * lane - e];
          tot += c[e];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int nb = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += nb;
        }
        int above = incl - tot;  // matching keys whose byte lies above this lane's bins
        int pick = -1, above_pick = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (pick < 0 && above < need && above + c[e] >= need) {
            pick = 255 - 8 * lane - e;
            above_pick = above;
          }
          above += c[e];
        }
        const unsigned who = __ballot_sync(0xffffffffu, pick >= 0);  // one lane holds the crossing
        const int src = who ? __ffs(who) - 1 : 0;
        pick = __shfl_sync(0xffffffffu, pick, src);
        above_pick = __shfl_sync(0xffffffffu, above_pick, src);
        if (lane == 0) {
          sel_state[pass & 1] = pick < 0 ? 0 : pick;  // two slots: the next pass writes the other
          warp_sums[pass & 1] = above_pick;
        }
      }
      __syncthreads();
      T |= (uint32_t)sel_state[pass & 1] << shift;
      need -= warp_sums[pass & 1];
      tmask |= 255u << shift;
    }
  }
  // Keys above T are kept; keys equal to T fill the remaining places lowest index first. One
  // exclusive scan of both per-thread counts, packed in the halves of an int (each <= 40960).
  int gt = 0, n_eq = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const bool valid = i0 + j < i1;
    gt += valid && key[j] > T ? 1 : 0;
    n_eq += valid && key[j] == T ? 1 : 0;
  }
  // (unsigned: the tied count reaches 40960 << 16, past the int range)
  uint32_t total = 0;
  const uint32_t packed = block_exclusive_scan_total<NT>((uint32_t)gt | ((uint32_t)n_eq << 16), warp_sums_u, &scan_total,
                                                     total);
  const int take_eq = n_keep - (int)(total & 0xffffu);
  int eq_rank = (int)(packed >> 16);
  int kept_before = (int)(packed & 0xffffu) + min(eq_rank, take_eq);
  uint64_t kmask = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if (i0 + j >= i1) break;
    bool kp = key[j] > T;
    if (key[j] == T) kp = eq_rank++ < take_eq;
    if (kp) kmask |= 1ull << j;
  }
  int drop_before = i0 - kept_before;
  const bool wide = hpg > 0 && sigma_wide != nullptr;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int i = i0 + j;
    if (i >= i1) break;
    const bool kp = (kmask >> j) & 1ull;
    if (wide) kbu[i] = (uint16_t)kept_before;
    // exactly n_keep keys are kept, so both ranges stay inside [0, n); the checks only
    // keep a broken invariant from writing past them
    if (kp) {
      if (kept_before < n_keep) sbuf[kept_before] = (uint32_t)i;
      ++kept_before;
    } else {
      if (n_keep + drop_before < n) sbuf[n_keep + drop_before] = (uint32_t)i;
      ++drop_before;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += NT) sigma[i] = (int32_t)sbuf[i];
  if (!wide) return;
  __syncthreads();
  // Query-side expansion: channel (h, d) = h * head_dim + d follows unit u = (h / hpg) * head_dim
  // + d. Kept query channels are ordered by head, then d; with kb(u) the kept units before u
  // (kbu) and, for the KV head g of u, kg = kb(g * head_dim) and cnt = its kept units, channel
  // (g * hpg + j, d) of a kept unit goes to hpg kg + j cnt + (kb(u) - kg), and of a dropped one to
  // n_keep hpg + hpg (g hd - kg) + j (hd - cnt) + ((u - kb(u)) - (g hd - kg)): each unit places its
  // hpg channels directly, no second scan.
  const int n_keep_w = n_keep * hpg;
  const bool staged = n_wide <= kSelStageWords;
  uint32_t* out = staged ? sbuf : reinterpret_cast<uint32_t*>(sigma_wide);
  for (int u = threadIdx.x; u < n; u += NT) {
    const int g = u / head_dim, gb = g * head_dim;
    const int kg = kbu[gb];
    const int kend = gb + head_dim < n ? (int)kbu[gb + head_dim] : n_keep;
    const int cnt = kend - kg;
    const int ku = kbu[u];
    const bool kept = (u + 1 < n ? (int)kbu[u + 1] : n_keep) > ku;
    const int c0 = g * hpg * head_dim + (u - gb);
    for (int j = 0; j < hpg; ++j) {
      const int pos = kept ? hpg * kg + j * cnt + (ku - kg)
                           : n_keep_w + hpg * (gb - kg) + j * (head_dim - cnt) + ((u - ku) - (gb - kg));
      if (pos >= 0 && pos < n_wide) out[pos] = (uint32_t)(c0 + j * head_dim);
    }
  }
  if (!staged) return;
  __syncthreads();
  for (int c = threadIdx.x; c < n_wide; c += NT) sigma_wide[c] = (int32_t)sbuf[c];
}

template <int PER, int NT>
void launch_select(const float* scores, int n, int n_keep, int32_t* sigma, int hpg, int head_dim, int n_wide,
                   int32_t* sigma_wide, cudaStream_t s) {
  if (!sigma_wide) n_wide = 0;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(select_kernel<PER, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kSelStageWords * 4 + kSelMaxNWide * 2 + 16);
    attr = true;
  }
  const size_t smem =
      (size_t)stage_words(n, sigma_wide ? n_wide : 0) * 4 + (sigma_wide ? ((size_t)n * 2 + 15) / 16 * 16 : 0);
  launch_kernel(select_kernel<PER, NT>, 1, NT, smem, s, scores, n, n_keep, sigma, hpg, head_dim, n_wide,
                sigma_wide);
}

// Head-level selection: head score H_g = sum_d s[g * head_dim + d] (fp64, d order); the
// n_keep_heads largest heads are kept (ties to the lower index, NaN below every number),
// each with all of its head_dim channels. sigma[n_kv * head_dim]: channels of kept heads
// ascending, then the others ascending; sigma_wide (query side, heads_per_group query heads
// per KV head): channel (h, d) kept iff head h / heads_per_group is.
__global__ void __launch_bounds__(kSelThreads) select_heads_kernel(const float* __restrict__ s, int n_heads,
                                                                   int head_dim, int n_keep_heads, int hpg,
                                                                   int32_t* __restrict__ sigma,
                                                                   int32_t* __restrict__ sigma_wide) {
  pdl_wait();
  __shared__ uint32_t hkey[kSelThreads];
  __shared__ uint8_t kept[kSelThreads];
  __shared__ int kept_before[kSelThreads + 1];
  const int g = threadIdx.x;
  if (g < n_heads) {
    double h = 0.0;
    for (int d = 0; d < head_dim; ++d) h += (double)s[(int64_t)g * head_dim + d];
    hkey[g] = score_key((float)h);
  }
  __syncthreads();
  if (g < n_heads) {
    // rank among the heads: larger keys first, equal keys by index
    const uint32_t k = hkey[g];
    int rank = 0;
    for (int o = 0; o < n_heads; ++o) rank += (hkey[o] > k || (hkey[o] == k && o < g)) ? 1 : 0;
    kept[g] = rank < n_keep_heads;
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // heads are few: a serial prefix count
    int c = 0;
    for (int o = 0; o < n_heads; ++o) {
      kept_before[o] = c;
      c += kept[o];
    }
    kept_before[n_heads] = c;
  }
  __syncthreads();
  // KV side: head g's channels go to its slot among kept or dropped heads
  for (int64_t c = threadIdx.x; c < (int64_t)n_heads * head_dim; c += kSelThreads) {
    const int hg = (int)(c / head_dim), d = (int)(c % head_dim);
    const int kb = kept_before[hg];
    const int64_t pos = kept[hg] ? (int64_t)kb * head_dim + d
                                 : (int64_t)n_keep_heads * head_dim + (int64_t)(hg - kb) * head_dim + d;
    sigma[pos] = (int32_t)c;
  }
  if (!sigma_wide) return;
  // query side: query head h follows KV head h / hpg; kept query heads keep index order
  const int nq = n_heads * hpg;
  for (int64_t c = threadIdx.x; c < (int64_t)nq * head_dim; c += kSelThreads) {
    const int h = (int)(c / head_dim), d = (int)(c % head_dim);
    const int hg = h / hpg, r = h % hpg;
    const int kb = kept_before[hg];
    const int64_t qkb = (int64_t)kb * hpg + r;  // kept query heads before h (kept KV heads are contiguous groups)
    const int64_t qdb = (int64_t)(hg - kb) * hpg + r;
    const int64_t pos = kept[hg] ? qkb * head_dim + d : (int64_t)n_keep_heads * hpg * head_dim + qdb * head_dim + d;
    sigma_wide[pos] = (int32_t)c;
  }
}

}  // namespace

int select_channels(const float* scores, int64_t n, int64_t n_keep, int32_t* sigma, int heads_per_group, int head_dim,
                    int64_t n_wide, int32_t* sigma_wide, int64_t* n_keep_wide_out, cudaStream_t s) {
  if (n <= 0 || n > kSelMaxN || n_keep < 1 || n_keep > n) return 1;
  if (sigma_wide && (heads_per_group <= 0 || head_dim <= 0 || n % head_dim || n_wide != n * heads_per_group ||
                     n > kSelMaxNWide))
    return 1;
  const int hpg = sigma_wide ? heads_per_group : 0;
  // Fewer, fuller threads for small sets: each block-wide phase (barrier, scan) then involves
  // fewer warps.
  if (n <= 1024)
    launch_select<4, 256>(scores, (int)n, (int)n_keep, sigma, hpg, head_dim, (int)n_wide, sigma_wide, s);
  else if (n <= 4096)
    launch_select<8, 512>(scores, (int)n, (int)n_keep, sigma, hpg, head_dim, (int)n_wide, sigma_wide, s);
  else if (n <= 16384)
    launch_select<16, 1024>(scores, (int)n, (int)n_keep, sigma, hpg, head_dim, (int)n_wide, sigma_wide, s);
  else
    launch_select<40, 1024>(scores, (int)n, (int)n_keep, sigma, hpg, head_dim, (int)n_wide, sigma_wide, s);
  if (n_keep_wide_out) *n_keep_wide_out = sigma_wide ? n_keep * heads_per_group : 0;
  if (launch_failed("sl_select")) return 5;
  note_launch();
  return 0;
}

int select_heads(const float* scores, int n_heads, int head_dim, int n_keep_heads, int heads_per_group,
                 int32_t* sigma, int32_t* sigma_wide, cudaStream_t s) {
  if (n_heads < 1 || n_heads > kSelThreads || head_dim < 1 || n_keep_heads < 1 || n_keep_heads > n_heads) return 1;
  if (sigma_wide && heads_per_group < 1) return 1;
  launch_kernel(select_heads_kernel, 1, kSelThreads, 0, s, scores, n_heads, head_dim, n_keep_heads,
                sigma_wide ? heads_per_group : 1, sigma, sigma_wide);
  if (launch_failed("sl_select")) return 5;
  note_launch();
  return 0;
}

}  // namespace sl
