// Estimator stage 1 on the tensor cores, and the linear criteria from the token Gram
// matrix ([WT] "SVD Sparsity Estimator": the rank-k factors W_A, W_B of each projection
// give Y_hat = (X W_A) W_B; the criteria of "Oracle Sparse Neuron Selection Criteria").
//
// Stage 1, Z = X_ctx [W_A^(1) ... W_A^(m)] (bf16 operands, fp32 accumulation in TMEM):
// one CTA per (128-token tile, K range). The context rows stream through a 6-stage TMA ring
// (128 x 64 bf16 boxes, 128-byte swizzle); the CTA's slice of the factors, W_A^T rows
// j * k + c, is written once into shared memory in the same swizzled K-major layout, so the
// factors are read in their stored [d_in, k] layout with no transposition pass. The K-range
// partials of a tile are summed by the tile's last CTA to finish (a finish counter per tile)
// in K-range order, so Z is run-to-run identical. That CTA also forms the tile's share of
// the Gram matrix sum_t z_t z_t^T in fp64 when a linear criterion follows.
//
// Linear criteria (V: ||Y_hat[:, i]||, QK: products of such norms): for a linear map the
// token sum collapses, sum_t (z_t . b_i)^2 = b_i^T (Z^T Z) b_i with b_i = W_B[:, i]; one
// launch sums the per-tile Gram matrices in tile order and evaluates the QK units and the
// V channels.
#include <cuda_bf16.h>

#include <algorithm>

#include "sl_internal.h"
#include "sl_ptx.cuh"

namespace sl {

struct EstZParams {
  CUtensorMap xmap;                 // X_ctx [n_ctx, d_in] bf16, 64 x 128 boxes, 128-byte swizzle
  const __nv_bfloat16* wa[4];       // W_A^(j) [d_in, k] bf16
  int32_t n_proj, k, mk, n_pad;     // n_pad = mk rounded up to 16 (MMA N)
  int32_t n_ctx, d_in;
  int32_t kb_total, kb_per, n_split, wa_bulk;
  int32_t stages, ring_bytes;       // ring depth; ring span (>= stages boxes and the tail's row staging)
  int32_t b_bytes, raw_bytes;       // W_A^T image and raw slice sizes (per CTA)
  float* zpart;                     // [n_split][n_ctx][mk] when n_split > 1
  float* z;                         // [n_ctx][mk]
  double* gram_part;                // [n_tiles][mk][mk] or null
  __nv_bfloat16* zsplit;            // [n_ctx][128] or null: Z of the two projections as bf16 parts
  int* tickets;                     // [n_tiles] finish counters (zero between calls)
  int* err;
};

namespace {

constexpr int kZThreads = 192;      // warp 0 TMA, warp 1 MMA + TMEM, warps 2..5 epilogue
constexpr int kZMaxStages = 12;
constexpr int kZTile = 128 * 64 * 2;
constexpr int kZSmem = 232448;      // the whole opt-in shared memory of an SM
constexpr int kZBarBytes = 512;
constexpr int kZAvail = kZSmem - 1024 - kZBarBytes;  // ring + W_A^T image + raw slice
// Row groups of the tile's Gram: four for up to 6 x 6 blocks of 4 x 4, two up to 9 x 9, else one.
__host__ __device__ inline int gram_row_groups(int mk) {
  const int blocks = (mk / 4) * (mk / 4);
  return blocks <= 48 ? 4 : (blocks <= 96 ? 2 : 1);
}
// The tail's staging in the ring: Z rows as fp64 [128][mk] plus the Gram row-group partials
// [RG][mk][mk] (at most 64 KB + 32 KB), or Z rows as fp32 with row stride mk + 1.
constexpr int kZRowStage = 128 * 64 * 8 + 64 * 64 * 8;

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void stage_bar() { asm volatile("bar.sync 2, 160;" ::: "memory"); }


// Z rows staged in shared memory (fp32, row stride mk + 1) -> the bf16 expansion rows of
// the tile in global memory, one work item per (row, projection): the three terms of its k
// values, then zeros up to 64 elements (eight 16-byte stores). K = k at compile time.
// Expansion z = z1 + z2 + z3 with z1 = bf16(z), z2 = bf16(z - z1), z3 = bf16(z - z1 - z2):
// each difference is exact in fp32 and the residual stays below 2^-24 |z| (8 significant
// bits per term).
template <int K>
__device__ void write_zsplit_rows(const float* zr, int mk, int64_t row0, int64_t n_ctx, __nv_bfloat16* zsplit,
                                  int nthreads) {
  static_assert(3 * K <= 64 && K % 2 == 0, "three terms of k values fill at most 64 elements");
  for (int it = threadIdx.x; it < 256; it += nthreads) {
    const int rr = it >> 1, pj = it & 1;
    const int64_t row = row0 + rr;
    if (row >= n_ctx) continue;
    const float* z = zr + rr * (mk + 1) + pj * K;
    uint32_t w[32];  // 64 bf16, element part * K + c
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i] = 0u;
#pragma unroll
    for (int c = 0; c < K; c += 2) {
      const float2 v = make_float2(z[c], z[c + 1]);
      const __nv_bfloat162 t1 = __float22bfloat162_rn(v);
      const float2 f1 = __bfloat1622float2(t1);
      const float2 r1 = make_float2(v.x - f1.x, v.y - f1.y);
      const __nv_bfloat162 t2 = __float22bfloat162_rn(r1);
      const float2 f2 = __bfloat1622float2(t2);
      const __nv_bfloat162 t3 = __float22bfloat162_rn(make_float2(r1.x - f2.x, r1.y - f2.y));
      w[c / 2] = *reinterpret_cast<const uint32_t*>(&t1);
      w[(K + c) / 2] = *reinterpret_cast<const uint32_t*>(&t2);
      w[(2 * K + c) / 2] = *reinterpret_cast<const uint32_t*>(&t3);
    }
    uint4* dst = reinterpret_cast<uint4*>(zsplit + row * 128 + pj * 64);
#pragma unroll
    for (int q = 0; q < 8; ++q) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

__device__ void write_zsplit_k(int k, const float* zr, int mk, int64_t row0, int64_t n_ctx, __nv_bfloat16* zsplit,
                               int nthreads) {
  switch (k) {
    case 4: write_zsplit_rows<4>(zr, mk, row0, n_ctx, zsplit, nthreads); break;
    case 8: write_zsplit_rows<8>(zr, mk, row0, n_ctx, zsplit, nthreads); break;
    case 16: write_zsplit_rows<16>(zr, mk, row0, n_ctx, zsplit, nthreads); break;
  }
}

// The Gram share of one 128-row tile, G[a][b] = sum over its rows of z[a] z[b] in fp64 (products
// of fp32 values are exact), from the tile's rows staged as fp64 [128][mk] in shared memory (rows
// past the context hold zeros). Work items (row group, 4 x 4 block of G): each sums its rows in
// order into 16 registers; the row-group partials (gp, shared memory [RG][mk][mk]) are then added
// in row-group order into out [mk][mk]. Block-wide (every thread calls it).
__device__ void gram_tile(const double* zs, int mk, double* gp, double* out, int nthreads) {
  const int nb4 = mk / 4, blocks = nb4 * nb4;
  const int RG = gram_row_groups(mk), rows_per = 128 / RG;
  for (int it = threadIdx.x; it < blocks * RG; it += nthreads) {
    const int rg = it / blocks, blk = it - rg * blocks;
    const int ba = blk / nb4, bb = blk - ba * nb4;
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int t = rg * rows_per; t < (rg + 1) * rows_per; ++t) {
      const double2* ra = reinterpret_cast<const double2*>(zs + t * mk + ba * 4);
      const double2* rb = reinterpret_cast<const double2*>(zs + t * mk + bb * 4);
      const double2 a01 = ra[0], a23 = ra[1], b01 = rb[0], b23 = rb[1];
      const double va[4] = {a01.x, a01.y, a23.x, a23.y}, vb[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(va[i], vb[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) gp[((int64_t)rg * mk + ba * 4 + i) * mk + bb * 4 + j] = acc[i][j];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < mk * mk; e += nthreads) {
    double sum = gp[e];
    for (int rg = 1; rg < RG; ++rg) sum += gp[(int64_t)rg * mk * mk + e];
    out[e] = sum;
  }
}

__global__ void __launch_bounds__(kZThreads, 1) est_z_kernel(const __grid_constant__ EstZParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  uint8_t* sa = smem;                          // S x 16 KB context-row boxes (ring_bytes span)
  uint8_t* sb = sa + p.ring_bytes;             // W_A^T image, one 64-wide K block per n_pad x 128 B
  uint8_t* sraw = sb + p.b_bytes;              // raw W_A slices as stored ([d][k] per projection)
  uint64_t* full = reinterpret_cast<uint64_t*>(sraw + p.raw_bytes);
  uint64_t* empty = full + kZMaxStages;
  uint64_t* done = empty + kZMaxStages;
  uint64_t* wbar = done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wbar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, tile = blockIdx.y;
  const int kb0 = split * p.kb_per;
  const int nkb = min(p.kb_per, p.kb_total - kb0);  // >= 1 by construction of the plan
  const int64_t d_beg = (int64_t)kb0 * 64;
  const int d_cnt = (int)min((int64_t)nkb * 64, (int64_t)p.d_in - d_beg);
  const int raw_stride = p.kb_per * 64 * p.k * 2;   // bytes per projection in the raw region
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    mbar_init(wbar, 1);
    *abort_flag = 0;
    *s_last = p.n_split == 1;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  // The factor slices are requested first (ahead of the row stream in the memory queues),
  // then as many context-row boxes as the ring holds.
  int issued = 0;
  uint32_t fmask = 0, fpar = 0;  // producer: stages with a copy in flight, and its phase
  if (warp == 0 && lane == 0) {
    if (p.wa_bulk) {
      mbar_arrive_expect_tx(wbar, (uint32_t)(p.n_proj * d_cnt * p.k * 2));
      for (int j = 0; j < p.n_proj; ++j)
        bulk_load_g2s(sraw + j * raw_stride, p.wa[j] + d_beg * p.k, (uint32_t)(d_cnt * p.k * 2), wbar);
    }
    for (; issued < nkb && issued < S; ++issued) {
      mbar_arrive_expect_tx(&full[issued], (uint32_t)kZTile);
      fmask |= 1u << issued;
      tma_load_2d(sa + issued * kZTile, &p.xmap, &full[issued], (kb0 + issued) * 64, tile * 128);
    }
  }

  // W_A^T image: row n = j * k + c holds W_A^(j)[d][c] at K position d; rows past mk and K
  // positions past d_in stay zero. Element (n, kk) of K block b sits at byte
  // b * n_pad * 128 + n * 128 + ((kk / 8) ^ (n % 8)) * 16 + (kk % 8) * 2 (128-byte swizzle).
  // Warps 1..5 build it from the raw slices while warp 0 keeps the rows streaming; the MMA
  // warp is one of the builders, so it starts only once the image is complete.
  if (warp > 0) {
    constexpr int kStagers = kZThreads - 32;
    const int ts = threadIdx.x - 32;
    const int nb = nkb * p.n_pad * 128;
    for (int i = ts; i < nb / 16; i += kStagers) reinterpret_cast<uint4*>(sb)[i] = make_uint4(0, 0, 0, 0);
    auto put = [&](int n, int d, __nv_bfloat16 v) {
      const int kk = d & 63;
      *reinterpret_cast<__nv_bfloat16*>(sb + (d >> 6) * p.n_pad * 128 + n * 128 + ((((kk >> 3) ^ (n & 7))) << 4) +
                                        (kk & 7) * 2) = v;
    };
    if (p.wa_bulk) {
      const bool got = mbar_wait(wbar, 0, abort_flag, p.err, DEV_TIMEOUT_PRODUCER);
      stage_bar();  // zero fill complete everywhere
      if (got) {
        const int kc = p.k;
        for (int e = ts; e < p.n_proj * d_cnt; e += kStagers) {
          const int j = e / d_cnt, d = e - j * d_cnt;
          const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(sraw + j * raw_stride) + d * kc;
          for (int c = 0; c < kc; ++c) put(j * kc + c, d, src[c]);
        }
      }
    } else {
      stage_bar();
      for (int e = ts; e < p.n_proj * d_cnt * p.k; e += kStagers) {
        const int c = e % p.k;
        const int d = (e / p.k) % d_cnt;
        const int j = e / (p.k * d_cnt);
        put(j * p.k + c, d, p.wa[j][(d_beg + d) * p.k + c]);
      }
    }
    fence_proxy_async_smem();  // generic-proxy writes before the tensor cores read them
    stage_bar();
  }

  if (warp == 0) {
    if (lane == 0) {
      for (int i = issued; i < nkb && !*abort_flag; ++i) {
        const int st = i % S;
        const uint32_t ph = (uint32_t)(i / S) & 1u;
        if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.err, DEV_TIMEOUT_PRODUCER)) break;
        mbar_arrive_expect_tx(&full[st], (uint32_t)kZTile);
        fmask |= 1u << st;
        fpar = (fpar & ~(1u << st)) | (ph << st);
        tma_load_2d(sa + st * kZTile, &p.xmap, &full[st], (kb0 + i) * 64, tile * 128);
      }
      // every copy in flight lands before the CTA's shared memory can be released
      for (int s = 0; s < S; ++s)
        if (fmask & (1u << s)) mbar_wait(&full[s], (fpar >> s) & 1u, nullptr, p.err, DEV_TIMEOUT_DRAIN);
      if (p.wa_bulk) mbar_wait(wbar, 0, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, p.n_pad, 0, 0);
      for (int i = 0; i < nkb && !*abort_flag; ++i) {
        const int st = i % S;
        if (!mbar_wait(&full[st], (uint32_t)(i / S) & 1u, abort_flag, p.err, DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sa + st * kZTile);
        const uint32_t b_addr = smem_u32(sb + i * p.n_pad * 128);
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16)
          umma_bf16(tmem_base, smem_desc_sw128(a_addr + k16 * 32, 16, 1024), smem_desc_sw128(b_addr + k16 * 32, 16, 1024),
                    idesc, (i > 0 || k16 > 0) ? 1u : 0u);
        umma_commit(&empty[st]);
      }
      umma_commit(done);  // also after an abort: the epilogue leaves once the issued MMAs are done
    }
  } else {
    // epilogue: TMEM lane quarter q = warp % 4, one context row per thread
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int64_t row = (int64_t)tile * 128 + r;
    const bool in = row < p.n_ctx;
    bool ok = mbar_wait(done, 0, abort_flag, p.err, DEV_TIMEOUT_EPILOGUE);
    ok = __all_sync(0xffffffffu, ok && !*abort_flag);
    tc_fence_after();
    uint32_t a0[32], a1[32];
    if (ok) {
      tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16), a0);
      if (p.n_pad > 32) tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + 32u, a1);
      tmem_ld_wait_regs(a0);
      regs_after_wait(a1);
    }
    const int nq = p.mk / 4;
    if (ok && in) {
      float* dst = p.n_split > 1 ? p.zpart + ((int64_t)split * p.n_ctx + row) * p.mk : p.z + row * p.mk;
#pragma unroll
      for (int c4 = 0; c4 < 16; ++c4) {
        if (c4 >= nq) break;
        const uint32_t* a = c4 < 8 ? a0 : a1;
        const int o = (c4 & 7) * 4;
        reinterpret_cast<float4*>(dst)[c4] = make_float4(__uint_as_float(a[o]), __uint_as_float(a[o + 1]),
                                                         __uint_as_float(a[o + 2]), __uint_as_float(a[o + 3]));
      }
    }
    if (p.n_split == 1) {
      // this CTA holds the whole K range: its rows go straight to the tail's staging
      float* zr = reinterpret_cast<float*>(sa) + r * (p.mk + 1);
      double* zd = reinterpret_cast<double*>(sa) + r * p.mk;
#pragma unroll
      for (int c4 = 0; c4 < 16; ++c4) {
        if (c4 >= nq) break;
        const uint32_t* a = c4 < 8 ? a0 : a1;
        const int o = (c4 & 7) * 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float v = (ok && in) ? __uint_as_float(a[o + i]) : 0.f;
          if (p.gram_part) zd[c4 * 4 + i] = (double)v;
          else zr[c4 * 4 + i] = v;
        }
      }
    } else {
      // every CTA of the tile counts in, also after an abort, so the counter returns to zero;
      // the fences around the count release this CTA's partials and acquire the others'
      epi_bar();
      if (threadIdx.x == 64) {
        __threadfence();
        const int t = atomicAdd(&p.tickets[blockIdx.y], 1);
        const int l = t == p.n_split - 1;
        if (l) {
          p.tickets[blockIdx.y] = 0;  // all CTAs of the tile have counted
          __threadfence();
        }
        *s_last = l;
      }
    }
  }
  __syncthreads();
  const bool last = *s_last != 0;
  const int nq = p.mk / 4;
  const int64_t row0 = (int64_t)tile * 128;
  if (last && p.n_split > 1) {
    // Z = sum of the K-range partials in K-range order. Work items (row, 4 columns) over all
    // threads; the partials of four items are in flight together.
    const int64_t sstride = (int64_t)p.n_ctx * p.mk / 4;  // float4s per partial
    const int n_items = 128 * nq;
    for (int base = threadIdx.x; base < n_items; base += 4 * kZThreads) {
      float4 acc[4];
      for (int s0 = 0; s0 < p.n_split; s0 += 8) {
        float4 v[4][8];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int it = base + g * kZThreads;
          const int rr = it / nq, c4 = it - rr * nq;
          const bool live = it < n_items && row0 + rr < p.n_ctx;
          const float4* zp = reinterpret_cast<const float4*>(p.zpart + (row0 + rr) * p.mk) + c4;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            v[g][u] = live && s0 + u < p.n_split ? __ldcg(zp + (s0 + u) * sstride) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (s0 + u >= p.n_split) break;
            if (s0 + u == 0) {
              acc[g] = v[g][u];
            } else {
              acc[g].x += v[g][u].x;
              acc[g].y += v[g][u].y;
              acc[g].z += v[g][u].z;
              acc[g].w += v[g][u].w;
            }
          }
      }
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int it = base + g * kZThreads;
        if (it >= n_items) break;
        const int rr = it / nq, c4 = it - rr * nq;
        if (row0 + rr < p.n_ctx) reinterpret_cast<float4*>(p.z + (row0 + rr) * p.mk)[c4] = acc[g];
        else acc[g] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p.gram_part) {
          double* zd = reinterpret_cast<double*>(sa) + rr * p.mk + c4 * 4;
          zd[0] = acc[g].x;
          zd[1] = acc[g].y;
          zd[2] = acc[g].z;
          zd[3] = acc[g].w;
        } else {
          float* zr = reinterpret_cast<float*>(sa) + rr * (p.mk + 1) + c4 * 4;
          zr[0] = acc[g].x;
          zr[1] = acc[g].y;
          zr[2] = acc[g].z;
          zr[3] = acc[g].w;
        }
      }
    }
    __syncthreads();
  }
  if (last && p.zsplit != nullptr) {
    // Z rows of the two projections (gate, up) as three bf16 terms each, for the SwiGLU
    // criterion's tensor-core products: row t holds 128 bf16, [proj * 64 + part * k + c] =
    // part `part` of Z[t][proj * k + c], zero past 3k. Work items (row, 8 outputs).
    write_zsplit_k(p.k, reinterpret_cast<const float*>(sa), p.mk, row0, p.n_ctx, p.zsplit, kZThreads);
  }
  if (last && p.gram_part != nullptr) {
    const double* zs = reinterpret_cast<const double*>(sa);  // [128][mk]
    gram_tile(zs, p.mk, reinterpret_cast<double*>(sa) + 128 * p.mk, p.gram_part + (int64_t)blockIdx.y * p.mk * p.mk,
              kZThreads);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem_base, 64);
}

// Z computed outside this file (the estimator's stage 1 as extra columns of the LoRA x A^T
// launch: fp32 [n_ctx][ld_z]) -> the per-tile Gram shares of the linear criteria or the
// three-term bf16 split of the SwiGLU criterion, exactly as est_z_kernel's tail forms them from its
// own Z. One CTA per 128-row tile; rows past n_ctx count as zeros. With gram_total set, the last
// CTA to finish (a ticket that it returns to zero) also adds the tile shares in tile order into
// gram_total, the Gram matrix of the whole context.
__global__ void __launch_bounds__(kZThreads) z_finish_kernel(const float* __restrict__ z, int64_t ld_z, int64_t n_ctx,
                                                             int mk, int k, double* __restrict__ gram_part,
                                                             __nv_bfloat16* __restrict__ zsplit, int* ticket,
                                                             double* __restrict__ gram_total) {
  extern __shared__ __align__(16) uint8_t zsm[];
  __shared__ int s_last;
  pdl_wait();
  const int64_t row0 = (int64_t)blockIdx.x * 128;
  if (gram_part) {
    double* zs = reinterpret_cast<double*>(zsm);  // [128][mk], then the row-group partials
    for (int e = threadIdx.x; e < 128 * mk; e += kZThreads) {
      const int rr = e / mk, c = e - rr * mk;
      const int64_t row = row0 + rr;
      zs[e] = row < n_ctx ? (double)z[row * ld_z + c] : 0.0;
    }
    __syncthreads();
    gram_tile(zs, mk, zs + 128 * mk, gram_part + (int64_t)blockIdx.x * mk * mk, kZThreads);
    if (!gram_total) return;
    __threadfence();  // this CTA's share is visible before its ticket
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1) == (int)gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int ne = mk * mk, n_parts = (int)gridDim.x;
    for (int e = threadIdx.x; e < ne; e += kZThreads) {
      double sum = 0.0;
      for (int c0 = 0; c0 < n_parts; c0 += 8) {
        double v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = c0 + u < n_parts ? __ldcg(gram_part + (int64_t)(c0 + u) * ne + e) : 0.0;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (c0 + u < n_parts) sum += v[u];
      }
      gram_total[e] = sum;
    }
    if (threadIdx.x == 0) *ticket = 0;
  } else {
    float* zr = reinterpret_cast<float*>(zsm);  // [128][mk + 1]
    for (int e = threadIdx.x; e < 128 * mk; e += kZThreads) {
      const int rr = e / mk, c = e - rr * mk;
      const int64_t row = row0 + rr;
      zr[rr * (mk + 1) + c] = row < n_ctx ? z[row * ld_z + c] : 0.f;
    }
    __syncthreads();
    write_zsplit_k(k, zr, mk, row0, n_ctx, zsplit, kZThreads);
  }
}

// ---- linear criteria from the Gram matrix

struct ScoreParams {
  const double* gram_part;  // [n_parts][mk][mk]
  int32_t n_parts, mk, k, wb_fp32;
  // QK units (g, d): ||K_hat[:, (g,d)]|| * sum_{h in g} ||Q_hat[:, (h,d)]||
  const void* wb_q;         // [k, n_q_heads * head_dim]
  const void* wb_k;         // [k, n_kv_heads * head_dim]
  int32_t blk_q, blk_k, hpg, head_dim;
  int64_t n_q, n_kv, n_qk;  // q channels, kv channels, QK units (0: none)
  float* scores_qk;
  // L2 channels: ||Y_hat[:, i]||
  const void* wb_l2;        // [k, n_l2]
  int32_t blk_l2, pad_;
  int64_t n_l2;             // 0: none
  float* scores_l2;
};

template <int KMAX>
__device__ __forceinline__ void load_b(const void* wb, int wb_fp32, int k, int64_t n, int64_t col, float (&b)[KMAX]) {
#pragma unroll
  for (int c = 0; c < KMAX; ++c)
    b[c] = c < k ? (wb_fp32 ? reinterpret_cast<const float*>(wb)[c * n + col]
                            : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(wb)[c * n + col]))
                 : 0.f;
}

// b^T G b over the k x k block of G at (off, off) (row stride mk), in fp64; negative
// rounding residue clamps to 0.
template <int KMAX>
__device__ __forceinline__ double quad_form(const double* G, int mk, int k, const float (&b)[KMAX]) {
  double s = 0.0;
#pragma unroll
  for (int a = 0; a < KMAX; ++a) {
    if (a >= k) break;
    double row = 0.0;
#pragma unroll
    for (int c = 0; c < KMAX; ++c)
      if (c < k) row = fma(G[a * mk + c], (double)b[c], row);
    s = fma((double)b[a], row, s);
  }
  return s > 0.0 ? s : 0.0;
}

constexpr int kScoreThreads = 128;

template <int KMAX>
__global__ void __launch_bounds__(kScoreThreads) est_scores_kernel(const __grid_constant__ ScoreParams p) {
  pdl_wait();
  extern __shared__ double gs[];  // [mk][mk], the Gram matrix of the whole context
  const int ne = p.mk * p.mk;
  // The unit's W_B columns (the K column and the first four query heads' columns of a QK unit,
  // or the channel's column) are requested first, so their latency overlaps the Gram sum's.
  const int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const bool is_qk = u < p.n_qk, is_l2 = !is_qk && u < p.n_qk + p.n_l2;
  float bk[KMAX], bq[4][KMAX];
  int g = 0, d = 0;
  if (is_qk) {
    g = (int)(u / p.head_dim);
    d = (int)(u % p.head_dim);
    load_b<KMAX>(p.wb_k, p.wb_fp32, p.k, p.n_kv, u, bk);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (j < p.hpg) load_b<KMAX>(p.wb_q, p.wb_fp32, p.k, p.n_q, (int64_t)(g * p.hpg + j) * p.head_dim + d, bq[j]);
  } else if (is_l2) {
    load_b<KMAX>(p.wb_l2, p.wb_fp32, p.k, p.n_l2, u - p.n_qk, bk);
  }
  // Sum of the per-tile matrices in tile order, eight loads in flight per step.
  for (int e = threadIdx.x; e < ne; e += blockDim.x) {
    double s = 0.0;
    for (int c0 = 0; c0 < p.n_parts; c0 += 8) {
      double v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = c0 + u < p.n_parts ? p.gram_part[(int64_t)(c0 + u) * ne + e] : 0.0;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (c0 + u < p.n_parts) s += v[u];
    }
    gs[e] = s;
  }
  __syncthreads();
  if (is_qk) {
    const double* Gq = gs + p.blk_q * p.k * p.mk + p.blk_q * p.k;
    const double* Gk = gs + p.blk_k * p.k * p.mk + p.blk_k * p.k;
    double qs = 0.0;  // the group's query heads in ascending order
    for (int h0 = 0; h0 < p.hpg; h0 += 4) {
      if (h0 > 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (h0 + j < p.hpg)
            load_b<KMAX>(p.wb_q, p.wb_fp32, p.k, p.n_q, (int64_t)(g * p.hpg + h0 + j) * p.head_dim + d, bq[j]);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (h0 + j < p.hpg) qs += sqrt(quad_form<KMAX>(Gq, p.mk, p.k, bq[j]));
    }
    p.scores_qk[u] = (float)(qs * sqrt(quad_form<KMAX>(Gk, p.mk, p.k, bk)));
  } else if (is_l2) {
    p.scores_l2[u - p.n_qk] = (float)sqrt(quad_form<KMAX>(gs + p.blk_l2 * p.k * p.mk + p.blk_l2 * p.k, p.mk, p.k, bk));
  }
}

// ---- SwiGLU criterion on the tensor cores

struct SwigluParams {
  CUtensorMap zmap;           // zsplit [n_ctx, 128] bf16, 64 x 128 boxes, 128-byte swizzle
  const __nv_bfloat16* wb_g;  // W_B of gate [k, F]
  const __nv_bfloat16* wb_u;  // W_B of up [k, F]
  int32_t k, n_k16, n_ctx, F, n_blocks, pad_;
  float* scores;
  double* sumsq;              // when not null: the sums of squares instead of the scores
  int* err;
};

constexpr int kSwThreads = 320;            // warp 0 TMA, warp 1 MMA + TMEM, warps 2..9 epilogue
constexpr int kSwStages = 4;
constexpr int kSwA = 128 * 128;            // 128 channels x 64 K bf16 (16 KB), one per projection
constexpr int kSwB = 2 * 128 * 128;        // 128 tokens x (gate 64 K | up 64 K), 32 KB per stage
constexpr int kSwSmem = 2 * kSwA + kSwStages * kSwB + 1024 + 256 + 2 * 128 * 8;

__device__ __forceinline__ void sw_epi_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ void sw_build_bar() { asm volatile("bar.sync 2, 288;" ::: "memory"); }

__device__ __forceinline__ float swiglu_sq_acc(uint32_t gbits, uint32_t ubits, float s) {
  const float g = __uint_as_float(gbits), u = __uint_as_float(ubits);
  const float h = __fdividef(g, 1.0f + __expf(fminf(-g, 80.f))) * u;  // SiLU(g) u
  return fmaf(h, h, s);
}

// One CTA per 128 output channels. A = W_B^T of gate and of up in three stacked copies
// (rows = channels, K = part * k + c), built once in shared memory; B = 128-token blocks
// of the Z expansion, streamed by TMA. Per block two MMAs give G_hat and U_hat for the
// CTA's channels x 128 tokens in TMEM (double-buffered); the epilogue threads own one
// channel and half the block's tokens each and accumulate (SiLU(g) u)^2 in a fixed order.
__global__ void __launch_bounds__(kSwThreads, 1) est_swiglu_tc_kernel(const __grid_constant__ SwigluParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sa = smem;                         // [2] x 16 KB (gate, up)
  uint8_t* sbuf = sa + 2 * kSwA;              // kSwStages x 32 KB token blocks
  uint64_t* full = reinterpret_cast<uint64_t*>(sbuf + kSwStages * kSwB);
  uint64_t* empty = full + kSwStages;
  uint64_t* tfull = empty + kSwStages;        // [2]
  uint64_t* tempty = tfull + 2;               // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  double* part = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(full) + 256);  // [2][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSwStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  const int64_t ch0 = (int64_t)blockIdx.x * 128;

  if (warp > 0) {
    // A tiles: row = channel, element (chl, part * k + c) = W_B[c][ch0 + chl], zero elsewhere
    const int tb = threadIdx.x - 32;
    for (int i = tb; i < 2 * kSwA / 16; i += kSwThreads - 32) reinterpret_cast<uint4*>(sa)[i] = make_uint4(0, 0, 0, 0);
    sw_build_bar();
    for (int e = tb; e < 2 * p.k * 128; e += kSwThreads - 32) {
      const int pj = e / (p.k * 128), rem = e % (p.k * 128);
      const int c = rem / 128, chl = rem % 128;
      const int64_t ch = ch0 + chl;
      const __nv_bfloat16* wb = pj ? p.wb_u : p.wb_g;
      const __nv_bfloat16 v = ch < p.F ? wb[(int64_t)c * p.F + ch] : __float2bfloat16_rn(0.f);
      uint8_t* at = sa + pj * kSwA + chl * 128;
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        const int kk = part * p.k + c;
        *reinterpret_cast<__nv_bfloat16*>(at + (((kk >> 3) ^ (chl & 7)) << 4) + (kk & 7) * 2) = v;
      }
    }
    fence_proxy_async_smem();
    sw_build_bar();
  }

  if (warp == 0) {
    if (lane == 0) {
      uint32_t fmask = 0, fpar = 0;
      for (int j = 0; j < p.n_blocks && !*abort_flag; ++j) {
        const int st = j % kSwStages;
        const uint32_t ph = (uint32_t)(j / kSwStages) & 1u;
        if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.err, DEV_TIMEOUT_PRODUCER)) break;
        mbar_arrive_expect_tx(&full[st], (uint32_t)kSwB);
        fmask |= 1u << st;
        fpar = (fpar & ~(1u << st)) | (ph << st);
        tma_load_2d(sbuf + st * kSwB, &p.zmap, &full[st], 0, j * 128);
        tma_load_2d(sbuf + st * kSwB + kSwA, &p.zmap, &full[st], 64, j * 128);
      }
      for (int s = 0; s < kSwStages; ++s)
        if (fmask & (1u << s)) mbar_wait(&full[s], (fpar >> s) & 1u, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, 128, 0, 0);
      const uint32_t ag = smem_u32(sa), au = smem_u32(sa + kSwA);
      for (int j = 0; j < p.n_blocks && !*abort_flag; ++j) {
        const int st = j % kSwStages, ab = j & 1;
        if (!mbar_wait(&full[st], (uint32_t)(j / kSwStages) & 1u, abort_flag, p.err, DEV_TIMEOUT_MMA)) break;
        if (!mbar_wait(&tempty[ab], ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag, p.err, DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t bg = smem_u32(sbuf + st * kSwB), bu = bg + kSwA;
        const uint32_t d = tmem_base + (uint32_t)(ab * 256);
        for (int k16 = 0; k16 < p.n_k16; ++k16) {
          umma_bf16(d, smem_desc_sw128(ag + k16 * 32, 16, 1024), smem_desc_sw128(bg + k16 * 32, 16, 1024), idesc,
                    k16 > 0 ? 1u : 0u);
          umma_bf16(d + 128u, smem_desc_sw128(au + k16 * 32, 16, 1024), smem_desc_sw128(bu + k16 * 32, 16, 1024),
                    idesc, k16 > 0 ? 1u : 0u);
        }
        umma_commit(&empty[st]);
        umma_commit(&tfull[ab]);
      }
    }
  } else {
    // warps 2..9: TMEM lane quarter q = warp % 4 (channel), token half hc of each block
    const int q = warp & 3, hc = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    double acc = 0.0;
    for (int j = 0; j < p.n_blocks; ++j) {
      const int ab = j & 1;
      bool ok = mbar_wait(&tfull[ab], (uint32_t)(j >> 1) & 1u, abort_flag, p.err, DEV_TIMEOUT_EPILOGUE);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t g0[32], u0[32], g1[32], u1[32];
      const uint32_t base = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * 256 + hc * 64);
      tmem_ld32(base, g0);
      tmem_ld32(base + 128u, u0);
      tmem_ld32(base + 32u, g1);
      tmem_ld32(base + 160u, u1);
      tmem_ld_wait_regs(g0);
      regs_after_wait(u0);
      regs_after_wait(g1);
      regs_after_wait(u1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ab]);  // the buffer may be refilled while the sums run
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) s = swiglu_sq_acc(g0[i], u0[i], s);
#pragma unroll
      for (int i = 0; i < 32; ++i) s = swiglu_sq_acc(g1[i], u1[i], s);
      acc += (double)s;
    }
    part[hc * 128 + row] = acc;
    sw_epi_bar();
    if (hc == 0) {
      const int64_t ch = ch0 + row;
      if (ch < p.F) {
        const double tot = part[row] + part[128 + row];
        if (p.sumsq) p.sumsq[ch] = tot;
        else p.scores[ch] = (float)sqrt(tot);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// out[e] = sum of n_parts matrices in part order (the rank-local Gram matrix).
__global__ void __launch_bounds__(256) gram_sum_kernel(const double* __restrict__ parts, int n_parts, int ne,
                                                       double* __restrict__ out) {
  pdl_wait();
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < ne; e += gridDim.x * blockDim.x) {
    double s = 0.0;
    for (int c = 0; c < n_parts; ++c) s += parts[(int64_t)c * ne + e];
    out[e] = s;
  }
}

// scores[i] = sqrt(sumsq[i]) (the SwiGLU criterion from summed squares).
__global__ void __launch_bounds__(256) sqrt_scores_kernel(const double* __restrict__ sumsq, int64_t n,
                                                          float* __restrict__ scores) {
  pdl_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    scores[i] = (float)sqrt(sumsq[i] > 0.0 ? sumsq[i] : 0.0);
}

}  // namespace

int est_z_plan(int64_t n_ctx, int64_t d_in, int mk, int* n_split, int* kb_per) {
  if (n_ctx <= 0 || d_in <= 0 || mk <= 0 || mk > 64 || mk % 4) return 1;
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (n_ctx + 127) / 128;
  const int kb_total = (int)((d_in + 63) / 64);
  const int n_pad = (mk + 15) / 16 * 16;
  // per K block: the W_A^T image (n_pad rows) and the raw slice (mk columns), both 128 B per
  // row; the ring keeps at least the tail's row staging (four or more stages)
  const int kb_cap = (kZAvail - kZRowStage) / (n_pad * 128 + mk * 128);
  const int64_t target = tiles >= sms ? 1 : sms / tiles;  // one wave of CTAs
  int per = (int)((kb_total + target - 1) / target);
  per = per < 1 ? 1 : (per > kb_cap ? kb_cap : per);
  *kb_per = per;
  *n_split = (kb_total + per - 1) / per;
  return 0;
}

int est_z_tc(const void* x, int64_t n_ctx, int64_t d_in, int64_t ldx, int n_proj, const void* const* wa, int k,
             float* zpart, float* z, double* gram_part, void* zsplit, int* tickets, int* err, cudaStream_t s) {
  if (zsplit && (n_proj != 2 || 3 * k > 64)) return 1;
  const int mk = n_proj * k;
  if (n_proj < 1 || n_proj > 4 || n_ctx > 2147483647LL || d_in > 2147483647LL) return 1;
  int n_split = 0, kb_per = 0;
  if (est_z_plan(n_ctx, d_in, mk, &n_split, &kb_per)) return 1;
  const int64_t tiles = (n_ctx + 127) / 128;
  if (tiles > kMaxSplitCounters || tiles > 65535) return 1;
  EstZParams P;
  memset(&P, 0, sizeof(P));
  if (!encode_bf16_2d(&P.xmap, x, n_ctx, d_in, ldx, 64, 128, true)) return 2;
  bool bulk = true;  // raw slices by bulk copy: 16-byte aligned factors
  for (int j = 0; j < n_proj; ++j) {
    P.wa[j] = static_cast<const __nv_bfloat16*>(wa[j]);
    bulk = bulk && (reinterpret_cast<uintptr_t>(wa[j]) & 15) == 0;
  }
  P.n_proj = n_proj;
  P.k = k;
  P.mk = mk;
  P.n_pad = (mk + 15) / 16 * 16;
  P.n_ctx = (int32_t)n_ctx;
  P.d_in = (int32_t)d_in;
  P.kb_total = (int32_t)((d_in + 63) / 64);
  P.kb_per = kb_per;
  P.n_split = n_split;
  P.wa_bulk = bulk ? 1 : 0;
  P.b_bytes = kb_per * P.n_pad * 128;
  P.raw_bytes = bulk ? n_proj * kb_per * 64 * k * 2 : 0;
  int stages = (kZAvail - P.b_bytes - P.raw_bytes) / kZTile;
  stages = std::min(std::min(stages, kZMaxStages), kb_per);
  if (stages < 1) return 1;
  P.stages = stages;
  const int row_stage = gram_part ? 128 * mk * 8 + gram_row_groups(mk) * mk * mk * 8
                                  : (zsplit ? 128 * (mk + 1) * 4 : 0);
  P.ring_bytes = std::max(stages * kZTile, (row_stage + 1023) / 1024 * 1024);
  if (P.ring_bytes + P.b_bytes + P.raw_bytes > kZAvail) return 1;
  P.zpart = zpart;
  P.z = z;
  P.gram_part = gram_part;
  P.zsplit = static_cast<__nv_bfloat16*>(zsplit);
  P.tickets = tickets;
  P.err = err;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(est_z_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kZSmem);
    attr = true;
  }
  const bool prof = profiling_on();
  if (prof) gemm_events(s, true, 4);
  launch_kernel(est_z_kernel, dim3((unsigned)n_split, (unsigned)tiles), kZThreads, kZSmem, s, P);
  if (prof) gemm_events(s, false, 4);
  if (launch_failed("sl_estimator")) return 5;
  note_launch();
  return 0;
}

int est_swiglu_tc(const void* zsplit, int64_t n_ctx, int k, const void* wb_g, const void* wb_u, int64_t F,
                  float* scores, double* sumsq, int* err, cudaStream_t s) {
  if (k < 1 || 3 * k > 64 || F <= 0 || n_ctx <= 0 || n_ctx > 2147483647LL || F > 2147483647LL) return 1;
  SwigluParams P;
  memset(&P, 0, sizeof(P));
  if (!encode_bf16_2d(&P.zmap, zsplit, n_ctx, 128, 128, 64, 128, true)) return 2;
  P.wb_g = static_cast<const __nv_bfloat16*>(wb_g);
  P.wb_u = static_cast<const __nv_bfloat16*>(wb_u);
  P.k = k;
  P.n_k16 = (3 * k + 15) / 16;
  P.n_ctx = (int32_t)n_ctx;
  P.F = (int32_t)F;
  P.n_blocks = (int32_t)((n_ctx + 127) / 128);
  P.scores = scores;
  P.sumsq = sumsq;
  P.err = err;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(est_swiglu_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSwSmem);
    attr = true;
  }
  launch_kernel(est_swiglu_tc_kernel, (unsigned)((F + 127) / 128), kSwThreads, kSwSmem, s, P);
  if (launch_failed("sl_estimator")) return 5;
  note_launch();
  return 0;
}

int gram_sum(const double* parts, int n_parts, int mk, double* out, cudaStream_t s) {
  if (n_parts < 1 || mk < 1 || mk > 64) return 1;
  const int ne = mk * mk;
  launch_kernel(gram_sum_kernel, (unsigned)((ne + 255) / 256), 256, 0, s, parts, n_parts, ne, out);
  if (launch_failed("sl_estimator")) return 5;
  note_launch();
  return 0;
}

int sqrt_scores(const double* sumsq, int64_t n, float* scores, cudaStream_t s) {
  if (n < 1) return 1;
  const unsigned grid = (unsigned)std::min<int64_t>((n + 255) / 256, 1184);
  launch_kernel(sqrt_scores_kernel, grid, 256, 0, s, sumsq, n, scores);
  if (launch_failed("sl_estimator")) return 5;
  note_launch();
  return 0;
}

int est_scores(const double* gram_part, int n_parts, int mk, int k, int wb_fp32, const void* wb_q, const void* wb_k,
               int blk_q, int blk_k, int n_q_heads, int n_kv_heads, int head_dim, float* scores_qk, const void* wb_l2,
               int blk_l2, int64_t n_l2, float* scores_l2, cudaStream_t s) {
  if (k < 1 || k > 16 || mk > 64 || n_parts < 1) return 1;
  ScoreParams P;
  memset(&P, 0, sizeof(P));
  P.gram_part = gram_part;
  P.n_parts = n_parts;
  P.mk = mk;
  P.k = k;
  P.wb_fp32 = wb_fp32;
  if (scores_qk) {
    P.wb_q = wb_q;
    P.wb_k = wb_k;
    P.blk_q = blk_q;
    P.blk_k = blk_k;
    P.hpg = n_q_heads / n_kv_heads;
    P.head_dim = head_dim;
    P.n_q = (int64_t)n_q_heads * head_dim;
    P.n_kv = (int64_t)n_kv_heads * head_dim;
    P.n_qk = P.n_kv;
    P.scores_qk = scores_qk;
  }
  if (scores_l2) {
    P.wb_l2 = wb_l2;
    P.blk_l2 = blk_l2;
    P.n_l2 = n_l2;
    P.scores_l2 = scores_l2;
  }
  const int64_t units = P.n_qk + P.n_l2;
  if (units <= 0) return 1;
  const unsigned grid = (unsigned)((units + kScoreThreads - 1) / kScoreThreads);
  const size_t smem = (size_t)mk * mk * sizeof(double);
  if (k <= 8)
    launch_kernel(est_scores_kernel<8>, grid, kScoreThreads, smem, s, P);
  else
    launch_kernel(est_scores_kernel<16>, grid, kScoreThreads, smem, s, P);
  if (launch_failed("sl_estimator")) return 5;
  note_launch();
  return 0;
}

int z_finish(const float* z, int64_t ld_z, int64_t n_ctx, int mk, int k, double* gram_part, void* zsplit,
             int* ticket, double* gram_total, cudaStream_t s) {
  if (n_ctx <= 0 || mk <= 0 || mk > 64 || mk % 4 || ld_z < mk || (!gram_part && !zsplit)) return 1;
  if (gram_total && (!gram_part || !ticket)) return 1;
  if (!gram_part && (k != 4 && k != 8 && k != 16)) return 1;
  const int64_t tiles = (n_ctx + 127) / 128;
  if (tiles > 2147483647LL) return 1;
  const size_t smem = gram_part ? (size_t)128 * mk * 8 + (size_t)gram_row_groups(mk) * mk * mk * 8
                                : (size_t)128 * (mk + 1) * 4;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(z_finish_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 64 * 8 + 64 * 64 * 8) !=
        cudaSuccess)
      return 5;
    attr = true;
  }
  launch_kernel(z_finish_kernel, (unsigned)tiles, kZThreads, smem, s, z, ld_z, n_ctx, mk, k, gram_part,
                static_cast<__nv_bfloat16*>(zsplit), ticket, gram_total);
  if (launch_failed("sl_est_tc")) return 5;
  note_launch();
  return 0;
}

}  // namespace sl
