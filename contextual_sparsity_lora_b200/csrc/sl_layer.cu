// The decoder layer around the sparse projections: RMSNorm forward and backward with the
// residual connections fused in ([WT] "Putting It All Together": the sparse q/k/v/o and FFN
// projections inside a LLaMA decoder layer; RMSNorm y = x / sqrt(mean(x^2) + eps) * gamma with
// a frozen gamma). One warp per row; fp32 arithmetic on bf16 rows, 16-byte vectors.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "sl_internal.h"

namespace sl {

namespace {

constexpr int kNormWarps = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 v = __bfloat1622float2(h[j]);
    f[2 * j] = v.x;
    f[2 * j + 1] = v.y;
  }
}

__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&f)[8]) {
  uint4 w;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
  for (int j = 0; j < 4; ++j) h[j] = __floats2bfloat162_rn(f[2 * j], f[2 * j + 1]);
  *reinterpret_cast<uint4*>(p) = w;
}

// y = (x [+ res]) * rstd * gamma, rstd = 1 / sqrt(mean((x [+ res])^2) + eps); with res, the
// sum x + res (the residual stream) is also written to sum_out.
__global__ void __launch_bounds__(kNormWarps * 32) rmsnorm_fwd_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t ldx, const __nv_bfloat16* __restrict__ res, int64_t ldr,
    __nv_bfloat16* __restrict__ sum_out, int64_t lds, const __nv_bfloat16* __restrict__ gamma, float eps,
    __nv_bfloat16* __restrict__ y, int64_t ldy, float* __restrict__ rstd, int64_t n_rows, int d) {
  pdl_wait();
  const int64_t row = (int64_t)blockIdx.x * kNormWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  float ss = 0.f;
  for (int j = lane * 8; j < d; j += 256) {
    float v[8];
    load8(x + row * ldx + j, v);
    if (res) {
      float r[8];
      load8(res + row * ldr + j, r);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] += r[e];
      // the residual stream is rounded to bf16 like every stored activation
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = __bfloat162float(__float2bfloat16_rn(v[e]));
      store8(sum_out + row * lds + j, v);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
  }
  ss = warp_sum(ss);
  const float rs = rsqrtf(ss / (float)d + eps);
  if (lane == 0) rstd[row] = rs;
  const __nv_bfloat16* src = res ? sum_out : x;
  const int64_t lsrc = res ? lds : ldx;
  for (int j = lane * 8; j < d; j += 256) {
    float v[8], g[8];
    load8(src + row * lsrc + j, v);
    load8(gamma + j, g);
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = v[e] * rs * g[e];
    store8(y + row * ldy + j, v);
  }
}

// dx = rstd * gamma * dy - x * rstd^3 * (sum_j x_j gamma_j dy_j) / d  [+ dres]
__global__ void __launch_bounds__(kNormWarps * 32) rmsnorm_bwd_kernel(
    const __nv_bfloat16* __restrict__ dy, int64_t lddy, const __nv_bfloat16* __restrict__ x, int64_t ldx,
    const __nv_bfloat16* __restrict__ gamma, const float* __restrict__ rstd, const __nv_bfloat16* __restrict__ dres,
    int64_t ldr, __nv_bfloat16* __restrict__ dx, int64_t lddx, int64_t n_rows, int d) {
  pdl_wait();
  const int64_t row = (int64_t)blockIdx.x * kNormWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  float dot = 0.f;
  for (int j = lane * 8; j < d; j += 256) {
    float a[8], b[8], g[8];
    load8(x + row * ldx + j, a);
    load8(dy + row * lddy + j, b);
    load8(gamma + j, g);
#pragma unroll
    for (int e = 0; e < 8; ++e) dot = fmaf(a[e], g[e] * b[e], dot);
  }
  dot = warp_sum(dot);
  const float rs = rstd[row];
  const float c = rs * rs * rs * dot / (float)d;
  for (int j = lane * 8; j < d; j += 256) {
    float a[8], b[8], g[8], o[8];
    load8(x + row * ldx + j, a);
    load8(dy + row * lddy + j, b);
    load8(gamma + j, g);
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = rs * g[e] * b[e] - a[e] * c;
    if (dres) {
      float r[8];
      load8(dres + row * ldr + j, r);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] += r[e];
    }
    store8(dx + row * lddx + j, o);
  }
}

// out = a + b (bf16 rows)
__global__ void __launch_bounds__(kNormWarps * 32) add_rows_kernel(const __nv_bfloat16* __restrict__ a, int64_t lda,
                                                                   const __nv_bfloat16* __restrict__ b, int64_t ldb,
                                                                   __nv_bfloat16* __restrict__ out, int64_t ldo,
                                                                   int64_t n_rows, int d) {
  pdl_wait();
  const int64_t row = (int64_t)blockIdx.x * kNormWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  for (int j = lane * 8; j < d; j += 256) {
    float u[8], v[8];
    load8(a + row * lda + j, u);
    load8(b + row * ldb + j, v);
#pragma unroll
    for (int e = 0; e < 8; ++e) u[e] += v[e];
    store8(out + row * ldo + j, u);
  }
}

}  // namespace

int rmsnorm_fwd(const void* x, int64_t ldx, const void* res, int64_t ldr, void* sum_out, int64_t lds,
                const void* gamma, float eps, void* y, int64_t ldy, float* rstd, int64_t n_rows, int64_t d,
                cudaStream_t s) {
  const unsigned grid = (unsigned)((n_rows + kNormWarps - 1) / kNormWarps);
  launch_kernel(rmsnorm_fwd_kernel, grid, kNormWarps * 32, 0, s, static_cast<const __nv_bfloat16*>(x), ldx,
                static_cast<const __nv_bfloat16*>(res), ldr, static_cast<__nv_bfloat16*>(sum_out), lds,
                static_cast<const __nv_bfloat16*>(gamma), eps, static_cast<__nv_bfloat16*>(y), ldy, rstd, n_rows,
                (int)d);
  if (launch_failed("sl_rmsnorm")) return 5;
  note_launch();
  return 0;
}

int rmsnorm_bwd(const void* dy, int64_t lddy, const void* x, int64_t ldx, const void* gamma, const float* rstd,
                const void* dres, int64_t ldr, void* dx, int64_t lddx, int64_t n_rows, int64_t d, cudaStream_t s) {
  const unsigned grid = (unsigned)((n_rows + kNormWarps - 1) / kNormWarps);
  launch_kernel(rmsnorm_bwd_kernel, grid, kNormWarps * 32, 0, s, static_cast<const __nv_bfloat16*>(dy), lddy,
                static_cast<const __nv_bfloat16*>(x), ldx, static_cast<const __nv_bfloat16*>(gamma), rstd,
                static_cast<const __nv_bfloat16*>(dres), ldr, static_cast<__nv_bfloat16*>(dx), lddx, n_rows, (int)d);
  if (launch_failed("sl_rmsnorm")) return 5;
  note_launch();
  return 0;
}

int add_rows(const void* a, int64_t lda, const void* b, int64_t ldb, void* out, int64_t ldo, int64_t n_rows, int64_t d,
             cudaStream_t s) {
  const unsigned grid = (unsigned)((n_rows + kNormWarps - 1) / kNormWarps);
  launch_kernel(add_rows_kernel, grid, kNormWarps * 32, 0, s, static_cast<const __nv_bfloat16*>(a), lda,
                static_cast<const __nv_bfloat16*>(b), ldb, static_cast<__nv_bfloat16*>(out), ldo, n_rows, (int)d);
  if (launch_failed("sl_add")) return 5;
  note_launch();
  return 0;
}

}  // namespace sl

// ---- AdamW on the LoRA parameters (the optimiser of a fine-tuning step)

namespace sl {

namespace {

// Decoupled weight decay (AdamW): p -= lr * wd * p; m = b1 m + (1 - b1) g; v = b2 v + (1 - b2) g^2;
// p -= lr * (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps); the bf16 working copy gets p.
__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ p, const float* __restrict__ g,
                                                    float* __restrict__ m, float* __restrict__ v,
                                                    __nv_bfloat16* __restrict__ p_bf16, int64_t n, float lr, float b1,
                                                    float b2, float eps, float wd, float c1, float c2) {
  pdl_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    float pi = p[i];
    const float gi = g[i];
    pi -= lr * wd * pi;
    const float mi = b1 * m[i] + (1.f - b1) * gi;
    const float vi = b2 * v[i] + (1.f - b2) * gi * gi;
    m[i] = mi;
    v[i] = vi;
    pi -= lr * (mi / c1) / (sqrtf(vi / c2) + eps);
    p[i] = pi;
    if (p_bf16) p_bf16[i] = __float2bfloat16_rn(pi);
  }
}

}  // namespace

int adamw_step(float* p, const float* g, float* m, float* v, void* p_bf16, int64_t n, float lr, float b1, float b2,
               float eps, float wd, int step, cudaStream_t s) {
  if (n < 1 || step < 1) return 1;
  const float c1 = 1.f - powf(b1, (float)step), c2 = 1.f - powf(b2, (float)step);
  const unsigned grid = (unsigned)std::min<int64_t>((n + 255) / 256, 1184);
  launch_kernel(adamw_kernel, grid, 256, 0, s, p, g, m, v, static_cast<__nv_bfloat16*>(p_bf16), n, lr, b1, b2, eps, wd,
                c1, c2);
  if (launch_failed("sl_adamw")) return 5;
  note_launch();
  return 0;
}

}  // namespace sl
