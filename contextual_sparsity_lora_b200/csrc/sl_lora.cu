// Fused LoRA backward stream: for each adapter, the two products that read the upstream
// gradient dy, dya = scale * dy B (reduced over output channels) and dB = dy^T xa_s (reduced
// over tokens), from one pass over dy ([WT] section 3.2: LoRA gradients are dense).
//
// dy is cut into items of G x H tiles of 128 tokens x 128 channels, ordered row group fastest
// inside a channel group; each persistent CTA takes a contiguous range of items. Over a run
// of items of one channel group it keeps the H chunks of B resident in shared memory and its
// column accumulators in TMEM, stages xa_s rows once per row block, and streams the dy tiles
// through a 3-stage ring. Every dy tile feeds two tcgen05 MMAs from the same shared memory:
//   row product    acc_row[128 tokens x 64] += dy_tile (K-major, K = 128 channels) * B_chunk
//   column product acc_col[128 channels x 64] += dy_tile^T (the same tile read MN-major,
//                                                 K = 128 tokens) * xa_s_chunk
// (rank r <= 64; the B and xa_s boxes are 64 wide, zero-filled past r). acc_row is complete
// for the item's channel range after each row block and acc_col for the run's tokens at the
// end of the run; both are added into fp32 dya / dB with vector reductions in L2, so the
// summation order over CTAs is not fixed (results agree to fp32 rounding).
// Context rows of an operand in the sigma layout use the permuted B (rows B[sigma[p]]) and
// add their dB rows at sigma[p].
//
// Roles: warp 0 issues TMA loads, warp 1 owns TMEM and issues the MMAs, warps 2..5 read
// the accumulators (one TMEM lane quarter each). Every wait is bounded.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdio>
#include <cstring>

#include "sl_internal.h"
#include "sl_ptx.cuh"

namespace sl {

namespace {

constexpr int kDualThreads = 192;
constexpr int kDualStages = 3;
constexpr int kDualMaxH = 6;                    // channel blocks per item (TMEM: 2 x 64 + 6 x 64 columns)
constexpr int kXTile = 2 * 128 * 64 * 2;        // 128 tokens x 128 channels bf16 = 32 KB (two 64-col boxes)
constexpr int kChunk = 2 * 64 * 64 * 2;         // 128 K-rows x 64 columns bf16 = 16 KB (two 64-row boxes)
constexpr int kDualSmem = kDualStages * kXTile + kDualMaxH * kChunk + 2 * kChunk + 1024 + 256;

}  // namespace

constexpr int kMaxDualJobs = 8;

struct DualJob {
  int16_t x_map, w_map, v_map, pad_;
  int32_t row0;       // first token row of the segment (coordinate in the dy and xa_s maps)
  int32_t rows;       // tokens in the segment
  int32_t cols;       // output channels
  int32_t G, H;       // 128-row and 128-channel blocks per item
  int32_t n_rg, n_cg; // items = n_rg * n_cg
  int32_t item_begin;
  float scale;        // dya = scale * dy B
  float* dya;         // [n_tok, ld_dya] fp32 (token rows relative to row 0 of the batch)
  int32_t ld_dya, r;
  float* dB;          // [cols, r] fp32
  const int32_t* sigma;  // dB row of channel position p: sigma[p] (context rows in the sigma layout), or null
};

struct DualParams {
  CUtensorMap maps[3 * kMaxDualJobs];
  DualJob jobs[kMaxDualJobs];
  int32_t njobs, total_items;
  int* err;
};

namespace {

struct ItemInfo {
  int job, rg, cg;
};

__device__ __forceinline__ ItemInfo decode_item(const DualParams& p, int it) {
  int j = 0;
  for (int i = 0; i < p.njobs; ++i)
    if (it >= p.jobs[i].item_begin) j = i;
  const DualJob& jb = p.jobs[j];
  const int local = it - jb.item_begin;
  return ItemInfo{j, local % jb.n_rg, local / jb.n_rg};
}

// Items of a CTA: a contiguous range of the item list (items run row group fastest inside a
// channel group), so consecutive items mostly share their channel group: the B chunks stay
// resident and the column accumulators keep adding over the whole run of a channel group.
__device__ __forceinline__ void cta_items(const DualParams& p, int& it0, int& it1) {
  it0 = (int)((int64_t)blockIdx.x * p.total_items / gridDim.x);
  it1 = (int)((int64_t)(blockIdx.x + 1) * p.total_items / gridDim.x);
}
__device__ __forceinline__ bool same_run(const ItemInfo& a, const ItemInfo& b) {
  return a.job == b.job && a.cg == b.cg;
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__global__ void __launch_bounds__(kDualThreads, 1) lora_dual_kernel(const __grid_constant__ DualParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sx = smem;                                   // kDualStages x 32 KB dy tiles
  uint8_t* sw = sx + kDualStages * kXTile;              // kDualMaxH x 16 KB B chunks (resident per item)
  uint8_t* sv = sw + kDualMaxH * kChunk;                // 2 x 16 KB xa_s chunks (one per row block)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sv + 2 * kChunk);
  uint64_t* xfull = bars;                               // [kDualStages]
  uint64_t* xempty = xfull + kDualStages;               // [kDualStages]
  uint64_t* wfull = xempty + kDualStages;               // B chunks landed
  uint64_t* wempty = wfull + 1;                         // MMAs of the item done with the B chunks
  uint64_t* vfull = wempty + 1;                         // [2]
  uint64_t* vempty = vfull + 2;                         // [2]
  uint64_t* rfull = vempty + 2;                         // [2] acc_row slot ready for the epilogue
  uint64_t* rempty = rfull + 2;                         // [2] acc_row slot drained
  uint64_t* cfull = rempty + 2;                         // acc_col ready
  uint64_t* cempty = cfull + 1;                         // acc_col drained
  uint64_t* drain = cempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDualStages; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], 1);
    }
    mbar_init(wfull, 1);
    mbar_init(wempty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&vfull[b], 1);
      mbar_init(&vempty[b], 1);
      mbar_init(&rfull[b], 1);
      mbar_init(&rempty[b], 128);
    }
    mbar_init(cfull, 1);
    mbar_init(cempty, 128);
    mbar_init(drain, 1);
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

  if (warp == 0) {
    if (lane == 0) {
      int xs = 0;
      uint32_t xph = 0, wph = 0;
      int vb = 0;
      uint32_t vph = 0;
      uint32_t xmask = 0, xpar = 0;  // stages with copies issued, and their phase
      uint32_t vmask = 0, vpar = 0;
      bool w_issued = false;
      uint32_t w_par = 0;
      int it0, it1;
      cta_items(p, it0, it1);
      for (int it = it0; it < it1 && !*abort_flag; ++it) {
        const ItemInfo ii = decode_item(p, it);
        const DualJob& jb = p.jobs[ii.job];
        const int cb0 = ii.cg * jb.H, ncb = min(jb.H, (jb.cols + 127) / 128 - cb0);
        const int rb0 = ii.rg * jb.G, nrb = min(jb.G, (jb.rows + 127) / 128 - rb0);
        if (it == it0 || !same_run(decode_item(p, it - 1), ii)) {
          // resident B chunks of the run's channel blocks
          if (!mbar_wait(wempty, wph ^ 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER)) break;
          mbar_arrive_expect_tx(wfull, (uint32_t)(ncb * kChunk));
          w_issued = true;
          w_par = wph;
          for (int c = 0; c < ncb; ++c)
            for (int h = 0; h < 2; ++h)
              tma_load_2d(sw + c * kChunk + h * 8192, &p.maps[jb.w_map], wfull, 0, (cb0 + c) * 128 + 64 * h);
          wph ^= 1;
        }
        for (int rb = 0; rb < nrb; ++rb) {
          const int row = jb.row0 + (rb0 + rb) * 128;
          if (!mbar_wait(&vempty[vb], vph ^ 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER)) goto producer_done;
          mbar_arrive_expect_tx(&vfull[vb], (uint32_t)kChunk);
          vmask |= 1u << vb;
          vpar = (vpar & ~(1u << vb)) | (vph << vb);
          for (int h = 0; h < 2; ++h)
            tma_load_2d(sv + vb * kChunk + h * 8192, &p.maps[jb.v_map], &vfull[vb], 0, row + 64 * h);
          if (++vb == 2) {
            vb = 0;
            vph ^= 1;
          }
          for (int c = 0; c < ncb; ++c) {
            if (!mbar_wait(&xempty[xs], xph ^ 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER)) goto producer_done;
            mbar_arrive_expect_tx(&xfull[xs], (uint32_t)kXTile);
            xmask |= 1u << xs;
            xpar = (xpar & ~(1u << xs)) | (xph << xs);
            for (int h = 0; h < 2; ++h)
              tma_load_2d(sx + xs * kXTile + h * 16384, &p.maps[jb.x_map], &xfull[xs], (cb0 + c) * 128 + 64 * h,
                          row);
            if (++xs == kDualStages) {
              xs = 0;
              xph ^= 1;
            }
          }
        }
      }
    producer_done:
      // every copy in flight has landed before the CTA's shared memory is released
      for (int s = 0; s < kDualStages; ++s)
        if (xmask & (1u << s)) mbar_wait(&xfull[s], (xpar >> s) & 1u, nullptr, p.err, DEV_TIMEOUT_DRAIN);
      for (int b = 0; b < 2; ++b)
        if (vmask & (1u << b)) mbar_wait(&vfull[b], (vpar >> b) & 1u, nullptr, p.err, DEV_TIMEOUT_DRAIN);
      if (w_issued) mbar_wait(wfull, w_par, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_row = idesc_bf16(128, 64, 0, 1);  // A = dy (K-major), B = B chunk (MN-major)
      const uint32_t id_col = idesc_bf16(128, 64, 1, 1);  // A = dy^T (MN-major view), B = xa_s (MN-major)
      int xs = 0;
      uint32_t xph = 0, wph = 0, cph = 0;
      int vb = 0, rs = 0;
      uint32_t vph = 0, rph = 0;
      int it0, it1;
      cta_items(p, it0, it1);
      for (int it = it0; it < it1 && !*abort_flag; ++it) {
        const ItemInfo ii = decode_item(p, it);
        const DualJob& jb = p.jobs[ii.job];
        const int cb0 = ii.cg * jb.H, ncb = min(jb.H, (jb.cols + 127) / 128 - cb0);
        const int rb0 = ii.rg * jb.G, nrb = min(jb.G, (jb.rows + 127) / 128 - rb0);
        const bool run_start = it == it0 || !same_run(decode_item(p, it - 1), ii);
        const bool run_end = it + 1 == it1 || !same_run(ii, decode_item(p, it + 1));
        if (run_start) {
          if (!mbar_wait(wfull, wph, abort_flag, p.err, DEV_TIMEOUT_MMA)) break;
          wph ^= 1;
          if (!mbar_wait(cempty, cph ^ 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) break;
          tc_fence_after();
        }
        for (int rb = 0; rb < nrb; ++rb) {
          if (!mbar_wait(&vfull[vb], vph, abort_flag, p.err, DEV_TIMEOUT_MMA)) goto mma_done;
          if (!mbar_wait(&rempty[rs], rph ^ 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) goto mma_done;
          tc_fence_after();
          const uint32_t d_row = tmem_base + (uint32_t)(rs * 64);
          const uint32_t v_addr = smem_u32(sv + vb * kChunk);
          for (int c = 0; c < ncb; ++c) {
            if (!mbar_wait(&xfull[xs], xph, abort_flag, p.err, DEV_TIMEOUT_MMA)) goto mma_done;
            tc_fence_after();
            const uint32_t x_addr = smem_u32(sx + xs * kXTile);
            const uint32_t w_addr = smem_u32(sw + c * kChunk);
            const uint32_t d_col = tmem_base + (uint32_t)(128 + c * 64);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              // row product: K step over 16 channels (box k / 4, 32 B per step inside a 128 B row)
              const uint64_t a_r = smem_desc_sw128(x_addr + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
              const uint64_t b_r = smem_desc_sw128(w_addr + (k >> 2) * 8192 + (k & 3) * 2048, 8192, 1024);
              umma_bf16(d_row, a_r, b_r, id_row, (c > 0 || k > 0) ? 1u : 0u);
              // column product: K step over 16 tokens (16 rows of 128 B), M = 128 channels in two
              // 64-channel chunks 16 KB apart
              const uint64_t a_c = smem_desc_sw128(x_addr + k * 2048, 16384, 1024);
              const uint64_t b_c = smem_desc_sw128(v_addr + (k >> 2) * 8192 + (k & 3) * 2048, 8192, 1024);
              umma_bf16(d_col, a_c, b_c, id_col, (!run_start || rb > 0 || k > 0) ? 1u : 0u);
            }
            umma_commit(&xempty[xs]);
            if (++xs == kDualStages) {
              xs = 0;
              xph ^= 1;
            }
          }
          umma_commit(&rfull[rs]);
          umma_commit(&vempty[vb]);
          if (++vb == 2) {
            vb = 0;
            vph ^= 1;
          }
          if (++rs == 2) {
            rs = 0;
            rph ^= 1;
          }
        }
        if (run_end) {
          umma_commit(wempty);
          umma_commit(cfull);
          cph ^= 1;
        }
      }
    mma_done:
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else {
    // epilogue warps 2..5: TMEM lane quarter q = warp % 4, lane = token row / channel
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t tq = (uint32_t)(q * 32) << 16;
    int rs = 0;
    uint32_t rph = 0, cph = 0;
    int it0, it1;
    cta_items(p, it0, it1);
    for (int it = it0; it < it1; ++it) {
      const ItemInfo ii = decode_item(p, it);
      const DualJob& jb = p.jobs[ii.job];
      const int cb0 = ii.cg * jb.H, ncb = min(jb.H, (jb.cols + 127) / 128 - cb0);
      const int rb0 = ii.rg * jb.G, nrb = min(jb.G, (jb.rows + 127) / 128 - rb0);
      const bool run_end = it + 1 == it1 || !same_run(ii, decode_item(p, it + 1));
      const int nr = jb.r;  // valid accumulator columns
      bool stop = false;
      for (int rb = 0; rb < nrb; ++rb) {
        if (!mbar_wait(&rfull[rs], rph, abort_flag, p.err, DEV_TIMEOUT_EPILOGUE)) {
          stop = true;
          break;
        }
        tc_fence_after();
        uint32_t a[32], b[32];
        tmem_ld32(tmem_base + tq + (uint32_t)(rs * 64), a);
        tmem_ld32(tmem_base + tq + (uint32_t)(rs * 64 + 32), b);
        tmem_ld_wait_regs(a);
        regs_after_wait(b);
        tc_fence_before();
        mbar_arrive(&rempty[rs]);  // the slot may be refilled while the sums leave
        const int row = (rb0 + rb) * 128 + r;
        if (row < jb.rows) {
          float* d = jb.dya + (int64_t)(jb.row0 + row) * jb.ld_dya;
          const float s = jb.scale;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            if (i < nr)
              red_add_v4(d + i, s * __uint_as_float(a[i]), s * __uint_as_float(a[i + 1]),
                         s * __uint_as_float(a[i + 2]), s * __uint_as_float(a[i + 3]));
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            if (i + 32 < nr)
              red_add_v4(d + 32 + i, s * __uint_as_float(b[i]), s * __uint_as_float(b[i + 1]),
                         s * __uint_as_float(b[i + 2]), s * __uint_as_float(b[i + 3]));
        }
        if (++rs == 2) {
          rs = 0;
          rph ^= 1;
        }
      }
      if (stop) break;
      if (!run_end) continue;  // the column sums keep accumulating over the run
      if (!mbar_wait(cfull, cph, abort_flag, p.err, DEV_TIMEOUT_EPILOGUE)) break;
      cph ^= 1;
      tc_fence_after();
      for (int c = 0; c < ncb; ++c) {
        uint32_t a[32], b[32];
        tmem_ld32(tmem_base + tq + (uint32_t)(128 + c * 64), a);
        tmem_ld32(tmem_base + tq + (uint32_t)(128 + c * 64 + 32), b);
        tmem_ld_wait_regs(a);
        regs_after_wait(b);
        const int col = (cb0 + c) * 128 + r;
        if (col < jb.cols) {
          const int dst = jb.sigma ? jb.sigma[col] : col;
          if (jb.sigma && !index_ok(dst, jb.cols, p.err, DEV_BAD_DB_ROW)) continue;
          float* d = jb.dB + (int64_t)dst * nr;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            if (i < nr)
              red_add_v4(d + i, __uint_as_float(a[i]), __uint_as_float(a[i + 1]), __uint_as_float(a[i + 2]),
                         __uint_as_float(a[i + 3]));
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            if (i + 32 < nr)
              red_add_v4(d + 32 + i, __uint_as_float(b[i]), __uint_as_float(b[i + 1]), __uint_as_float(b[i + 2]),
                         __uint_as_float(b[i + 3]));
        }
      }
      tc_fence_before();
      mbar_arrive(cempty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, 512);
  }
}

// dya_s = bf16(dya) for every adapter of the call (dya already holds the scale); with `cat`,
// the same values also go to column block [coff, coff + r) of cat [rows, ld_cat].
struct CastJob {
  const float* src;
  __nv_bfloat16* dst;
  int64_t n;
  __nv_bfloat16* cat;
  int32_t r, coff, ld_cat, pad_;
};
struct CastParams {
  CastJob j[kMaxDualJobs];
  int n;
};

__global__ void __launch_bounds__(256) cast_bf16_kernel(const __grid_constant__ CastParams p) {
  pdl_wait();
  const CastJob& c = p.j[blockIdx.y];
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < c.n; i += (int64_t)gridDim.x * blockDim.x) {
    const __nv_bfloat16 v = __float2bfloat16_rn(c.src[i]);
    c.dst[i] = v;
    if (c.cat) c.cat[(i / c.r) * c.ld_cat + c.coff + i % c.r] = v;
  }
}

// Zeroes up to kMaxZero fp32 buffers in one launch (blockIdx.y = buffer).
constexpr int kMaxZero = 12;
struct ZeroParams {
  float* p[kMaxZero];
  int64_t n[kMaxZero];
};

__global__ void __launch_bounds__(256) zero_f32_kernel(const __grid_constant__ ZeroParams z) {
  pdl_wait();
  float* p = z.p[blockIdx.y];
  const int64_t n = z.n[blockIdx.y];
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if ((reinterpret_cast<uintptr_t>(p) & 15) == 0) {
    float4* q = reinterpret_cast<float4*>(p);
    for (int64_t i = i0; i < n / 4; i += stride) q[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t i = n / 4 * 4 + i0; i < n; i += stride) p[i] = 0.f;
  } else {
    for (int64_t i = i0; i < n; i += stride) p[i] = 0.f;
  }
}

bool encode(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int64_t ld, int box_cols, int box_rows) {
  return encode_bf16_2d(m, ptr, rows, cols, ld, box_cols, box_rows, true);
}

}  // namespace

int lora_dual_launch(const DualSpec* specs, int n, int* err, cudaStream_t s) {
  if (n <= 0) return 0;
  if (n > kMaxDualJobs) return 1;
  DualParams P;
  memset(&P, 0, sizeof(P));
  int sms = 148, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // tiles over all jobs; items of G x H tiles with H = 6 channel blocks and G chosen so that
  // the item count is about four per CTA
  int64_t tiles = 0;
  for (int i = 0; i < n; ++i) tiles += (int64_t)((specs[i].rows + 127) / 128) * ((specs[i].cols + 127) / 128);
  int total = 0;
  for (int i = 0; i < n; ++i) {
    const DualSpec& sp = specs[i];
    DualJob& jb = P.jobs[i];
    if (sp.r < 1 || sp.r > 64 || sp.r % 4 || sp.rows <= 0 || sp.cols <= 0) return 1;
    jb.x_map = (int16_t)(3 * i);
    jb.w_map = (int16_t)(3 * i + 1);
    jb.v_map = (int16_t)(3 * i + 2);
    if (!encode(&P.maps[3 * i], sp.dy, sp.row0 + sp.rows, sp.cols, sp.ld_dy, 64, 128) ||
        !encode(&P.maps[3 * i + 1], sp.B, sp.cols, sp.r, sp.r, 64, 64) ||
        !encode(&P.maps[3 * i + 2], sp.xa_s, sp.row0 + sp.rows, sp.r, sp.ld_xa, 64, 64))
      return 2;
    jb.row0 = (int32_t)sp.row0;
    jb.rows = (int32_t)sp.rows;
    jb.cols = (int32_t)sp.cols;
    const int nrb = (int)((sp.rows + 127) / 128), ncb = (int)((sp.cols + 127) / 128);
    jb.H = std::min(kDualMaxH, ncb);
    const int64_t target_items = 4LL * sms;  // short items: the CTA's contiguous range shares channel groups
    const int64_t per_item = std::max<int64_t>(1, tiles / target_items);
    jb.G = (int)std::max<int64_t>(1, std::min<int64_t>(nrb, per_item / jb.H));
    jb.n_rg = (nrb + jb.G - 1) / jb.G;
    jb.n_cg = (ncb + jb.H - 1) / jb.H;
    jb.item_begin = total;
    total += jb.n_rg * jb.n_cg;
    jb.scale = sp.scale;
    jb.dya = sp.dya;
    jb.ld_dya = (int32_t)sp.ld_dya;
    jb.r = sp.r;
    jb.dB = sp.dB;
    jb.sigma = sp.sigma;
  }
  P.njobs = n;
  P.total_items = total;
  P.err = err;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(lora_dual_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDualSmem) != cudaSuccess)
      return 5;
    attr = true;
  }
  const int grid = std::min(total, sms);
  const bool prof = profiling_on();
  if (prof) gemm_events(s, true, 3);
  launch_kernel(lora_dual_kernel, grid, kDualThreads, kDualSmem, s, P);
  if (launch_failed("sl_lora")) return 5;
  if (prof) gemm_events(s, false, 3);
  note_launch();
  return 0;
}

int cast_f32_bf16(const float* const* src, void* const* dst, const int64_t* count, int n, cudaStream_t s,
                  void* cat, const int* r, int ld_cat) {
  if (n <= 0) return 0;
  if (n > kMaxDualJobs) return 1;
  CastParams P;
  memset(&P, 0, sizeof(P));
  int64_t mx = 0;
  int coff = 0;
  for (int i = 0; i < n; ++i) {
    P.j[i] = CastJob{src[i], static_cast<__nv_bfloat16*>(dst[i]), count[i], nullptr, 1, 0, 0, 0};
    if (cat) {
      P.j[i].cat = static_cast<__nv_bfloat16*>(cat);
      P.j[i].r = r[i];
      P.j[i].coff = coff;
      P.j[i].ld_cat = ld_cat;
      coff += r[i];
    }
    mx = std::max(mx, count[i]);
  }
  P.n = n;
  const unsigned gx = (unsigned)std::min<int64_t>((mx + 255) / 256, 1184);
  launch_kernel(cast_bf16_kernel, dim3(gx, n), 256, 0, s, P);
  if (launch_failed("sl_lora")) return 5;
  note_launch();
  return 0;
}

int zero_f32(float* const* ptrs, const int64_t* counts, int n, cudaStream_t s) {
  if (n <= 0) return 0;
  if (n > kMaxZero) return 1;
  ZeroParams Z;
  memset(&Z, 0, sizeof(Z));
  int64_t mx = 0;
  for (int i = 0; i < n; ++i) {
    Z.p[i] = ptrs[i];
    Z.n[i] = counts[i];
    mx = std::max(mx, counts[i]);
  }
  const unsigned gx = (unsigned)std::max<int64_t>(1, std::min<int64_t>((mx / 4 + 255) / 256, 592));
  launch_kernel(zero_f32_kernel, dim3(gx, n), 256, 0, s, Z);
  if (launch_failed("sl_lora")) return 5;
  note_launch();
  return 0;
}

}  // namespace sl
