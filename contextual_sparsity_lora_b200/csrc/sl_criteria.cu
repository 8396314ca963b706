// Wanda-style channel criterion, the FFN alternative of the criterion ablation ([WT] "Oracle
// Sparse Neuron Selection Criteria"; Table 10: Wanda against L2 norm and random pruning for the
// FFN projections). Wanda's importance of a frozen weight W[i, j] is |W[i, j]| ||X[:, j]||_2,
// the input feature norm taken over the context rows; the channel score is its sum over the
// channel's row, and channels that share one index set (gate and up) add their rows:
//   s_i = sum_p sum_j |W_p[i, j]| n_j,   n_j = sqrt(sum_t X[t, j]^2).
// Three launches: per-row-block partial sums of squares of the columns of X, their fixed-order
// sum and root, then one warp per channel streaming the weight rows (the HBM-bound part: every
// weight byte is read once).
#include <cuda_bf16.h>

#include "sl_internal.h"

namespace sl {

namespace {

constexpr int kColThreads = 256;   // two columns per thread: 512 columns per CTA
constexpr int kColRows = 128;      // context rows per CTA

// part[blockIdx.y][j] = sum over the CTA's rows of x[t][j]^2 (fp32, row order).
__global__ void __launch_bounds__(kColThreads) col_sumsq_kernel(const __nv_bfloat16* __restrict__ x, int64_t n_rows,
                                                                int64_t d, int64_t ldx, float* __restrict__ part) {
  pdl_wait();
  const int64_t j = ((int64_t)blockIdx.x * kColThreads + threadIdx.x) * 2;
  if (j >= d) return;
  const int64_t t0 = (int64_t)blockIdx.y * kColRows, t1 = min(n_rows, t0 + kColRows);
  float a = 0.f, b = 0.f;
  for (int64_t t = t0; t < t1; ++t) {
    const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(x + t * ldx + j));
    a = fmaf(v.x, v.x, a);
    b = fmaf(v.y, v.y, b);
  }
  part[(int64_t)blockIdx.y * d + j] = a;
  part[(int64_t)blockIdx.y * d + j + 1] = b;
}

// norm[j] = sqrt(sum_s part[s][j]), s in order.
__global__ void __launch_bounds__(256) col_norm_kernel(const float* __restrict__ part, int n_parts, int64_t d,
                                                       float* __restrict__ norm) {
  pdl_wait();
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  float s = 0.f;
  for (int p = 0; p < n_parts; ++p) s += part[(int64_t)p * d + j];
  norm[j] = sqrtf(s);
}

struct WandaParams {
  const __nv_bfloat16* w[4];
  int32_t n_proj, pad_;
  int64_t d_out, d_in, ldw;
  const float* norm;
  float* scores;
};

constexpr int kWandaWarps = 8;

// One warp per channel: lanes stride the row in 16-byte vectors; the lane sums meet in a fixed
// shuffle tree.
__global__ void __launch_bounds__(kWandaWarps * 32) wanda_rows_kernel(const __grid_constant__ WandaParams p) {
  extern __shared__ float sn[];  // the d_in column norms
  pdl_wait();
  for (int64_t j = threadIdx.x; j < p.d_in; j += blockDim.x) sn[j] = p.norm[j];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * kWandaWarps + (threadIdx.x >> 5);
  if (i >= p.d_out) return;
  float acc = 0.f;
  for (int q = 0; q < p.n_proj; ++q) {
    const __nv_bfloat16* row = p.w[q] + i * p.ldw;
    for (int64_t j = (int64_t)lane * 8; j < p.d_in; j += 32 * 8) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + j));
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        acc = fmaf(fabsf(f.x), sn[j + 2 * e], acc);
        acc = fmaf(fabsf(f.y), sn[j + 2 * e + 1], acc);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) p.scores[i] = acc;
}

}  // namespace

int64_t wanda_scratch_floats(int64_t n_ctx, int64_t d_in) {
  return ((n_ctx + kColRows - 1) / kColRows) * d_in + d_in;
}

int wanda_scores(const void* x, int64_t n_ctx, int64_t d_in, int64_t ldx, int n_proj, const void* const* w,
                 int64_t d_out, int64_t ldw, float* scores, float* scratch, cudaStream_t s) {
  if (n_ctx < 1 || d_in < 8 || d_in % 8 || n_proj < 1 || n_proj > 4 || d_out < 1) return 1;
  if ((size_t)d_in * sizeof(float) > 200 * 1024) return 1;
  const int n_parts = (int)((n_ctx + kColRows - 1) / kColRows);
  float* part = scratch;
  float* norm = scratch + (int64_t)n_parts * d_in;
  const dim3 g1((unsigned)((d_in / 2 + kColThreads - 1) / kColThreads), (unsigned)n_parts);
  launch_kernel(col_sumsq_kernel, g1, kColThreads, 0, s, static_cast<const __nv_bfloat16*>(x), n_ctx, d_in, ldx,
                part);
  launch_kernel(col_norm_kernel, (unsigned)((d_in + 255) / 256), 256, 0, s, (const float*)part, n_parts, d_in, norm);
  WandaParams P;
  memset(&P, 0, sizeof(P));
  for (int q = 0; q < n_proj; ++q) P.w[q] = static_cast<const __nv_bfloat16*>(w[q]);
  P.n_proj = n_proj;
  P.d_out = d_out;
  P.d_in = d_in;
  P.ldw = ldw;
  P.norm = norm;
  P.scores = scores;
  const size_t smem = (size_t)d_in * sizeof(float);
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(wanda_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    attr = true;
  }
  launch_kernel(wanda_rows_kernel, (unsigned)((d_out + kWandaWarps - 1) / kWandaWarps), kWandaWarps * 32, smem, s, P);
  if (launch_failed("sl_wanda")) return 5;
  note_launch(3);
  return 0;
}

}  // namespace sl
