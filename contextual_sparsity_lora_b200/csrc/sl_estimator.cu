// SVD sparsity estimator and criterion reductions on CUDA cores (fp32 products,
// fixed-order reductions; no floating-point atomics, so results are
// run-to-run identical).
//
// Stage 1: Z = X_ctx [W_A^(1) ... W_A^(m)]  (split over the input dimension;
//          partial sums per split, then a fixed-order sum).
// Stage 2 (SwiGLU L2): s_i = sqrt(sum_t (SiLU(g_ti) u_ti)^2) with
//          g = Z_gate W_B^gate, u = Z_up W_B^up evaluated per (token, channel).
// Stage 2 (linear criteria, V and QK): the token reduction of a linear map
//          collapses to a Gram matrix, sum_t (Z b_i)_t^2 = b_i^T (Z^T Z) b_i,
//          formed and contracted in fp64.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "sl_internal.h"
#include "sl_ptx.cuh"

namespace cg = cooperative_groups;

namespace sl {

namespace {

constexpr int kE1Rows = 128;   // tokens per CTA
constexpr int kE1Chunk = 32;   // input channels staged per step
constexpr int kE1Threads = 256;

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&f)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&f)[8]) {
  uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float2 v = __bfloat1622float2(h[j]);
    f[2 * j] = v.x;
    f[2 * j + 1] = v.y;
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&f)[8]) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

__device__ __forceinline__ float ld_any(const void* p, int64_t i, int fp32) {
  return fp32 ? reinterpret_cast<const float*>(p)[i] : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

struct WaPtrs {
  const void* p[4];
};

// grid: (ceil(n_ctx / 128), n_split). Thread = (row group of 4 tokens, column group of CPG outputs).
template <typename T, int CPG>
__global__ void __launch_bounds__(kE1Threads) est1_kernel(const T* __restrict__ x, int64_t n_ctx, int64_t d_in,
                                                          int64_t ldx, WaPtrs wa, int wa_fp32, int k, int mk,
                                                          int64_t d_per_split, float* __restrict__ zpart) {
  pdl_wait();
  constexpr int MKP = 8 * CPG;  // padded column count
  extern __shared__ float e1_smem[];
  float* xs = e1_smem;                              // [kE1Chunk][kE1Rows + 4]
  float* ws = xs + kE1Chunk * (kE1Rows + 4);        // [d_per_split][MKP]
  const int tid = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * kE1Rows;
  const int64_t d0 = (int64_t)blockIdx.y * d_per_split;
  const int64_t dn = min(d_per_split, d_in - d0);

  for (int64_t e = tid; e < dn * MKP; e += kE1Threads) {
    const int64_t d = e / MKP;
    const int j = (int)(e % MKP);
    float w = 0.f;
    if (j < mk) {
      const int pj = j / k, c = j % k;
      w = ld_any(wa.p[pj], (d0 + d) * k + c, wa_fp32);
    }
    ws[e] = w;
  }

  const int warp = tid >> 5, lane = tid & 31;
  const int rg = warp * 4 + (lane >> 3);  // 0..31
  const int cg = lane & 7;
  float acc[4][CPG];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < CPG; ++c) acc[r][c] = 0.f;

  for (int64_t dc = 0; dc < dn; dc += kE1Chunk) {
    __syncthreads();
    // stage X[t0 .. t0+128, d0+dc .. +32] transposed into xs[d][row]
    for (int e = tid; e < kE1Rows * (kE1Chunk / 8); e += kE1Threads) {
      const int row = e % kE1Rows;
      const int dq = (e / kE1Rows) * 8;
      float f[8];
      const int64_t t = t0 + row;
      const int64_t d = d0 + dc + dq;
      if (t < n_ctx && d + 8 <= d0 + dn) {
        load8<T>(x + t * ldx + d, f);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = 0.f;
        if (t < n_ctx)
          for (int i = 0; i < 8; ++i)
            if (d + i < d0 + dn) f[i] = (float)x[t * ldx + d + i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) xs[(dq + i) * (kE1Rows + 4) + row] = f[i];
    }
    __syncthreads();
    const int dlen = (int)min64(kE1Chunk, dn - dc);
    for (int dd = 0; dd < dlen; ++dd) {
      const float4 xv = *reinterpret_cast<const float4*>(&xs[dd * (kE1Rows + 4) + rg * 4]);
      const float* wrow = &ws[(dc + dd) * MKP + cg * CPG];
      float w[CPG];
#pragma unroll
      for (int c = 0; c < CPG; ++c) w[c] = wrow[c];
#pragma unroll
      for (int c = 0; c < CPG; ++c) {
        acc[0][c] = fmaf(xv.x, w[c], acc[0][c]);
        acc[1][c] = fmaf(xv.y, w[c], acc[1][c]);
        acc[2][c] = fmaf(xv.z, w[c], acc[2][c]);
        acc[3][c] = fmaf(xv.w, w[c], acc[3][c]);
      }
    }
  }
  float* zp = zpart + (int64_t)blockIdx.y * n_ctx * mk;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t t = t0 + rg * 4 + r;
    if (t >= n_ctx) continue;
#pragma unroll
    for (int c = 0; c < CPG; ++c) {
      const int j = cg * CPG + c;
      if (j < mk) zp[t * mk + j] = acc[r][c];
    }
  }
}

// Z[t][j] = sum_s zpart[s][t][j], s in increasing order. Written into split slot 0.
__global__ void est_reduce_kernel(float* zpart, int n_split, int64_t n) {
  pdl_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float acc = zpart[i];
  for (int s = 1; s < n_split; ++s) acc += zpart[(int64_t)s * n + i];
  zpart[i] = acc;
}

constexpr int kE2Threads = 256;  // 8 warps; each lane owns 2 channels of a 64-channel block
constexpr int kE2Split = 4;      // token ranges per channel block = CTAs per cluster
constexpr int kE2Buf = 4096;     // floats per staging buffer (16 KB): 4096 / (2k) tokens per chunk

// SwiGLU criterion. Grid (F / 64, kE2Split) in clusters of (1, kE2Split): the CTAs of a
// cluster share a 64-channel block and split the context tokens; their fp64 partial sums
// are combined by cluster rank 0 through distributed shared memory in rank order. The
// CTA's Z rows (2k floats per token, contiguous) arrive by bulk copies into two 16 KB
// buffers, the next chunk in flight while the current one is consumed.
template <int K>
__global__ void __cluster_dims__(1, kE2Split, 1) __launch_bounds__(kE2Threads)
    est_swiglu_kernel(const float* __restrict__ z, int64_t n_ctx, const void* wb_g, const void* wb_u, int wb_fp32,
                      int64_t n_ch, float* __restrict__ scores, double* __restrict__ sumsq, int* err) {
  constexpr int kRow = 2 * K;
  constexpr int kChunk = kE2Buf / kRow;
  __shared__ __align__(128) float zs[2][kE2Buf];
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ double part[8][64];
  __shared__ double cta_sum[64];
  pdl_wait();
  cg::cluster_group cluster = cg::this_cluster();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ch0 = (int64_t)blockIdx.x * 64 + lane;
  const int64_t ch1 = ch0 + 32;
  float wg0[K], wu0[K], wg1[K], wu1[K];
#pragma unroll
  for (int c = 0; c < K; ++c) {
    wg0[c] = ch0 < n_ch ? ld_any(wb_g, c * n_ch + ch0, wb_fp32) : 0.f;
    wu0[c] = ch0 < n_ch ? ld_any(wb_u, c * n_ch + ch0, wb_fp32) : 0.f;
    wg1[c] = ch1 < n_ch ? ld_any(wb_g, c * n_ch + ch1, wb_fp32) : 0.f;
    wu1[c] = ch1 < n_ch ? ld_any(wb_u, c * n_ch + ch1, wb_fp32) : 0.f;
  }
  const int64_t per = (n_ctx + kE2Split - 1) / kE2Split;
  const int64_t t_beg = min64(n_ctx, (int64_t)blockIdx.y * per), t_end = min64(n_ctx, t_beg + per);
  const int nchunks = (int)((t_end - t_beg + kChunk - 1) / kChunk);
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  auto issue = [&](int c) {  // thread 0: chunk c into buffer c & 1
    const int64_t t0 = t_beg + (int64_t)c * kChunk;
    const uint32_t bytes = (uint32_t)(min64(kChunk, t_end - t0) * kRow * 4);
    mbar_arrive_expect_tx(&bars[c & 1], bytes);
    bulk_load_g2s(&zs[c & 1][0], z + t0 * kRow, bytes, &bars[c & 1]);
  };
  if (threadIdx.x == 0) {
    if (nchunks > 0) issue(0);
    if (nchunks > 1) issue(1);
  }
  double acc0 = 0.0, acc1 = 0.0;
  int done = 0;  // chunks consumed
  for (int c = 0; c < nchunks; ++c) {
    const bool got = mbar_wait(&bars[c & 1], (uint32_t)((c >> 1) & 1), nullptr, err, DEV_TIMEOUT_ESTIMATOR);
    if (__syncthreads_or(!got)) break;  // uniform: every thread leaves the loop together
    const int tn = (int)min64(kChunk, t_end - (t_beg + (int64_t)c * kChunk));
    const float* zc = &zs[c & 1][0];
    float s0 = 0.f, s1 = 0.f;
    // four tokens per step (t, t + 8, t + 16, t + 24): independent FMA chains and SiLUs in flight
    constexpr int kU = 4;
    for (int tb = warp; tb < tn; tb += 8 * kU) {
      float g0[kU], u0[kU], g1[kU], u1[kU];
#pragma unroll
      for (int j = 0; j < kU; ++j) g0[j] = u0[j] = g1[j] = u1[j] = 0.f;
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        const int t = min(tb + 8 * j, tn - 1);  // clamped rows are read but not summed
        const float4* zr = reinterpret_cast<const float4*>(zc + t * kRow);
#pragma unroll
        for (int c4 = 0; c4 < K / 4; ++c4) {
          const float4 zg = zr[c4], zu = zr[K / 4 + c4];
          g0[j] = fmaf(zg.x, wg0[4 * c4], g0[j]); g0[j] = fmaf(zg.y, wg0[4 * c4 + 1], g0[j]);
          g0[j] = fmaf(zg.z, wg0[4 * c4 + 2], g0[j]); g0[j] = fmaf(zg.w, wg0[4 * c4 + 3], g0[j]);
          g1[j] = fmaf(zg.x, wg1[4 * c4], g1[j]); g1[j] = fmaf(zg.y, wg1[4 * c4 + 1], g1[j]);
          g1[j] = fmaf(zg.z, wg1[4 * c4 + 2], g1[j]); g1[j] = fmaf(zg.w, wg1[4 * c4 + 3], g1[j]);
          u0[j] = fmaf(zu.x, wu0[4 * c4], u0[j]); u0[j] = fmaf(zu.y, wu0[4 * c4 + 1], u0[j]);
          u0[j] = fmaf(zu.z, wu0[4 * c4 + 2], u0[j]); u0[j] = fmaf(zu.w, wu0[4 * c4 + 3], u0[j]);
          u1[j] = fmaf(zu.x, wu1[4 * c4], u1[j]); u1[j] = fmaf(zu.y, wu1[4 * c4 + 1], u1[j]);
          u1[j] = fmaf(zu.z, wu1[4 * c4 + 2], u1[j]); u1[j] = fmaf(zu.w, wu1[4 * c4 + 3], u1[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        if (tb + 8 * j >= tn) break;  // in order: the per-thread sum keeps a fixed token order
        const float h0 = __fdividef(g0[j], 1.0f + __expf(fminf(-g0[j], 80.f))) * u0[j];
        const float h1 = __fdividef(g1[j], 1.0f + __expf(fminf(-g1[j], 80.f))) * u1[j];
        s0 = fmaf(h0, h0, s0);
        s1 = fmaf(h1, h1, s1);
      }
    }
    acc0 += (double)s0;
    acc1 += (double)s1;
    done = c + 1;
    __syncthreads();  // buffer c & 1 is free again
    if (threadIdx.x == 0 && c + 2 < nchunks) issue(c + 2);
  }
  if (done < nchunks && threadIdx.x == 0) {
    // a copy did not land in time: wait (bounded) for the ones still in flight to finish
    // writing this CTA's shared memory before it is released
    for (int c = done; c < nchunks && c < done + 2; ++c)
      mbar_wait(&bars[c & 1], (uint32_t)((c >> 1) & 1), nullptr, nullptr, 0);
  }
  part[warp][lane] = acc0;
  part[warp][lane + 32] = acc1;
  __syncthreads();
  if (threadIdx.x < 64) {
    double s = 0.0;
    for (int w = 0; w < 8; ++w) s += part[w][threadIdx.x];
    cta_sum[threadIdx.x] = s;
  }
  cluster.sync();
  if (cluster.block_rank() == 0 && threadIdx.x < 64) {
    double s = 0.0;
    for (int rnk = 0; rnk < kE2Split; ++rnk) s += cluster.map_shared_rank(cta_sum, rnk)[threadIdx.x];
    const int64_t ch = (int64_t)blockIdx.x * 64 + threadIdx.x;
    if (ch < n_ch) {
      if (sumsq) sumsq[ch] = s;
      else scores[ch] = (float)sqrt(s);
    }
  }
  cluster.sync();  // peers keep their shared memory alive until rank 0 has read it
}

constexpr int kGramTok = 48;
constexpr int kGramCluster = 8;

// Gram matrix G[a][b] = sum_t z[t][a] z[t][b] in fp64. One cluster of kGramCluster CTAs
// splits the tokens; rank 0 adds the CTAs' partial matrices in rank order (distributed
// shared memory) and writes G.
__global__ void __cluster_dims__(kGramCluster, 1, 1) __launch_bounds__(256)
    est_gram_kernel(const float* __restrict__ z, int64_t n_ctx, int mk, double* __restrict__ gram) {
  pdl_wait();
  __shared__ float zs[kGramTok][64];
  __shared__ double gpart[64 * 64];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  // cluster c covers tokens [c * 8 * kGramTok, (c + 1) * 8 * kGramTok); its rank r the r-th kGramTok slice
  const int64_t per = kGramTok;
  const int64_t t_beg = min64(n_ctx, ((int64_t)blockIdx.x / kGramCluster * kGramCluster + rank) * per),
                t_end = min64(n_ctx, t_beg + per);
  const int ne = mk * mk;
  double acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.0;
  for (int64_t tb = t_beg; tb < t_end; tb += kGramTok) {
    __syncthreads();
    const int tn = (int)min64(kGramTok, t_end - tb);
    for (int e = threadIdx.x; e < tn * mk; e += blockDim.x) zs[e / mk][e % mk] = z[tb * mk + e];
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int e = threadIdx.x + j * 256;
      if (e < ne) {
        const int a = e / mk, b = e % mk;
        double sum = acc[j];
        for (int t = 0; t < tn; ++t) sum = fma((double)zs[t][a], (double)zs[t][b], sum);
        acc[j] = sum;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int e = threadIdx.x + j * 256;
    if (e < ne) gpart[e] = acc[j];
  }
  cluster.sync();
  if (rank == 0) {
    for (int e = threadIdx.x; e < ne; e += blockDim.x) {
      double sum = 0.0;
      for (int r = 0; r < kGramCluster; ++r) sum += cluster.map_shared_rank(gpart, r)[e];
      gram[(int64_t)(blockIdx.x / kGramCluster) * ne + e] = sum;
    }
  }
  cluster.sync();
}

}  // namespace

int est_stage1(const void* x, int x_fp32, int64_t n_ctx, int64_t d_in, int64_t ldx, int n_proj,
               const void* const* wa, int wa_fp32, int k, float* zpart, int n_split, cudaStream_t s) {
  const int mk = n_proj * k;
  if (mk > 64 || n_proj > 4 || n_ctx <= 0) return 1;
  WaPtrs w{};
  for (int i = 0; i < n_proj; ++i) w.p[i] = wa[i];
  int64_t dps = (d_in + n_split - 1) / n_split;
  dps = (dps + kE1Chunk - 1) / kE1Chunk * kE1Chunk;
  const int cpg = (mk + 7) / 8;
  const size_t smem = (size_t)kE1Chunk * (kE1Rows + 4) * 4 + (size_t)dps * 8 * cpg * 4;
  dim3 grid((unsigned)((n_ctx + kE1Rows - 1) / kE1Rows), (unsigned)((d_in + dps - 1) / dps));
  if ((int)grid.y > n_split || smem > 200 * 1024) return 1;
#define SL_E1(C)                                                                                              \
  case C: {                                                                                                   \
    if (x_fp32) {                                                                                             \
      auto kern = est1_kernel<float, C>;                                                                      \
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                     \
      launch_kernel(kern, grid, kE1Threads, smem, s, (const float*)x, n_ctx, d_in, ldx, w, wa_fp32, k, mk, dps, zpart);  \
    } else {                                                                                                  \
      auto kern = est1_kernel<__nv_bfloat16, C>;                                                              \
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                     \
      launch_kernel(kern, grid, kE1Threads, smem, s, (const __nv_bfloat16*)x, n_ctx, d_in, ldx, w, wa_fp32, k, mk, dps, \
                                          zpart);                                                             \
    }                                                                                                         \
    break;                                                                                                    \
  }
  switch (cpg) {
    SL_E1(1) SL_E1(2) SL_E1(3) SL_E1(4) SL_E1(5) SL_E1(6) SL_E1(7) SL_E1(8)
    default:
      return 1;
  }
#undef SL_E1
  const int used = (int)grid.y;
  if (used > 1) {
    const int64_t n = n_ctx * mk;
    launch_kernel(est_reduce_kernel, (unsigned)((n + 255) / 256), 256, 0, s, zpart, used, n);
  }
  if (launch_failed("sl_estimator")) return 5;
  note_launch();
  return 0;
}

int est_swiglu_scores(const float* z, int /*n_split*/, int64_t n_ctx, int k, const void* wb_gate, const void* wb_up,
                      int wb_fp32, int64_t n_ch, float* scores, double* sumsq, int* err, cudaStream_t s) {
  if (reinterpret_cast<uintptr_t>(z) & 15) return 1;  // bulk copies need 16-byte alignment
  const dim3 grid((unsigned)((n_ch + 63) / 64), kE2Split);
  switch (k) {
    case 8: launch_kernel(est_swiglu_kernel<8>, grid, kE2Threads, 0, s, z, n_ctx, wb_gate, wb_up, wb_fp32, n_ch, scores, sumsq, err); break;
    case 16: launch_kernel(est_swiglu_kernel<16>, grid, kE2Threads, 0, s, z, n_ctx, wb_gate, wb_up, wb_fp32, n_ch, scores, sumsq, err); break;
    case 4: launch_kernel(est_swiglu_kernel<4>, grid, kE2Threads, 0, s, z, n_ctx, wb_gate, wb_up, wb_fp32, n_ch, scores, sumsq, err); break;
    default: return 1;
  }
  if (launch_failed("sl_estimator")) return 5;
  note_launch();
  return 0;
}

int est_gram(const float* z, int /*n_split*/, int64_t n_ctx, int mk, double* gram, int /*n_chunks*/,
             cudaStream_t s) {
  if (mk > 64 || n_ctx <= 0) return 1;
  launch_kernel(est_gram_kernel, gram_groups(n_ctx) * kGramCluster, 256, 0, s, z, n_ctx, mk, gram);
  if (launch_failed("sl_estimator")) return 5;
  note_launch();
  return 0;
}

int est1_splits(int64_t d_in) {
  int ns = (int)((d_in + 255) / 256);
  if (ns > 64) ns = 64;
  if (ns < 1) ns = 1;
  int64_t dps = (d_in + ns - 1) / ns;
  dps = (dps + 31) / 32 * 32;
  return (int)((d_in + dps - 1) / dps);
}

}  // namespace sl
