// Persistent, warp-specialised tcgen05 GEMM engine for sm_100a (see sl_gemm.h).
//
// Roles per CTA (192 threads, one CTA per SM):
//   warp 0      one thread issues TMA tile loads into a kStages-deep ring
//   warp 1      allocates 512 TMEM columns (two 256-column fp32 accumulators);
//               one thread issues tcgen05.mma (M = 128, N = n_mma, K = 16 each)
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (one TMEM lane = one
//               output row per thread), fused elementwise work, global stores
// Tiles are handed out round-robin over the problem list; the two accumulators
// let the epilogue of tile i overlap the main loop of tile i+1.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <functional>
#include <queue>
#include <vector>

#include "sl_gemm.h"
#include "sl_internal.h"
#include "sl_ptx.cuh"

namespace sl {

struct TileInfo {
  int prob, tm, tn, ks, kb0, kb1;  // ks: split-K index; [kb0, kb1): k-block range (over all segments)
};

// Row `col` of the transposed fp32 output of an EPI_F32_T problem (col_split: columns in
// blocks of col_split go to out0, out1, out2).
__device__ __forceinline__ float* f32t_dst(const Prob& pr, int64_t col) {
  if (pr.col_split) {
    const int j = (int)(col / pr.col_split);
    void* o = j == 0 ? pr.out0 : (j == 1 ? pr.out1 : pr.out2);
    return reinterpret_cast<float*>(o) + (col - (int64_t)j * pr.col_split) * pr.ld0;
  }
  return reinterpret_cast<float*>(pr.out0) + col * pr.ld0;
}

// Slots of the CTA-pair schedule: pair c runs slots c, c + pairs, ... in order; slot s holds
// tile order[s] (-1: nothing) when the launch carries a tile order, else tile s.
__device__ __forceinline__ int slot_count(const GemmParams& p) { return p.n_slots ? p.n_slots : p.total_tiles; }
__device__ __forceinline__ int slot_tile(const GemmParams& p, int s) { return p.n_slots ? (int)p.order[s] : s; }

__device__ __forceinline__ TileInfo decode_tile(const GemmParams& p, int t) {
  int pi = 0;
  for (int i = 0; i < p.nprob; ++i)
    if (t >= p.probs[i].tile_begin) pi = i;
  const Prob& pr = p.probs[pi];
  const int local = t - pr.tile_begin;
  const int per = pr.tiles_m * pr.tiles_n;
  const int ks = local / per, rem = local % per;
  TileInfo ti{pi, rem % pr.tiles_m, rem / pr.tiles_m, ks, 0, 1 << 30};
  if (pr.ksplit > 1) {
    ti.kb0 = (int)((long long)ks * pr.kblocks / pr.ksplit);
    ti.kb1 = (int)((long long)(ks + 1) * pr.kblocks / pr.ksplit);
  }
  return ti;
}

__device__ __forceinline__ uint32_t seg_tx_bytes(const Seg& sg) {
  uint32_t bytes = kStageABytes;
  for (int i = 0; i < sg.nb; ++i) bytes += sg.b_mn ? (uint32_t)(sg.b[i].rows / 64) * 8192u : (uint32_t)sg.b[i].rows * 128u;
  return bytes;
}

// The logistic function from one exponential of -|g| (it never overflows) and one division
// by 1 + e in (1, 2]: sigma(g) = 1 / (1 + e) for g >= 0 and e / (1 + e) for g < 0, with
// e = exp(-|g|). Neither branch subtracts nearly equal numbers, so the relative error of
// sigma(g), and of SiLU(g) = g sigma(g), stays at a few ulp of the two approximate operations
// over the whole range, the far negative tail included (where a form built on 1 + tanh(g/2)
// cancels: its absolute error, about 2^-12, exceeds sigma(g) itself below g = -8).
__device__ __forceinline__ float sigmoid_f(float g) {
  const float e = __expf(-fabsf(g));
  const float q = __fdividef(1.0f, 1.0f + e);
  return g >= 0.0f ? q : e * q;
}
__device__ __forceinline__ float silu_f(float g) { return g * sigmoid_f(g); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void store_bf16_row(__nv_bfloat16* dst, const float* v, int n, bool vec_ok) {
  if (vec_ok && n == 32) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      d4[i] = make_uint4(pack_bf16x2(v[8 * i + 0], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                         pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < n) dst[i] = __float2bfloat16_rn(v[i]);
  }
}

__device__ __forceinline__ void load_bf16_row(const __nv_bfloat16* src, float* v, int n, bool vec_ok) {
  if (vec_ok && n == 32) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint4 w = s4[i];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 f = __bfloat1622float2(h[j]);
        v[8 * i + 2 * j] = f.x;
        v[8 * i + 2 * j + 1] = f.y;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = i < n ? __bfloat162float(src[i]) : 0.f;
  }
}

// 32 bf16 of row `lane` of a 64-byte-swizzled 32 x 32 box (as loaded by a bulk tensor copy).
__device__ __forceinline__ void load_box_row(const uint8_t* box, int lane, float* v) {
  const uint4* s4 = reinterpret_cast<const uint4*>(box + lane * 64);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 w = s4[i ^ ((lane >> 1) & 3)];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 f = __bfloat1622float2(h[j]);
      v[8 * i + 2 * j] = f.x;
      v[8 * i + 2 * j + 1] = f.y;
    }
  }
}

// Bulk-store path of the bf16 epilogues: the warp's 32 rows x 32 columns of one output go
// through one of the warp's two 2 KB shared-memory boxes (lane = row of 64 bytes) and leave
// with one bulk tensor store issued by lane 0, so the warp moves on while the copy drains and
// every write is a whole line. The boxes use the tensor map's 64-byte swizzle: 16-byte chunk i of
// row r sits at chunk position i ^ ((r / 2) % 4) (the boxes are 512-byte aligned), so one 16-byte
// store of the warp touches every bank at most four times (four wavefronts for 512 bytes) instead
// of sixteen with rows of 64 bytes side by side. Rows and columns outside the problem are
// clipped by the tensor map (it covers exactly the problem's M x N block). Lane 0 waits, before
// a box is rewritten, until at most one of its bulk groups (the other box) is still reading.
// Warp-collective; the caller skips warps whose rows all lie outside the problem.
__device__ __forceinline__ int swz64(int lane, int i) { return i ^ ((lane >> 1) & 3); }

__device__ __forceinline__ void bulk_store_chunk(const CUtensorMap* map, uint8_t* bufs, int& sb, const float* v,
                                                 int col, int row0) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) bulk_wait_read<1>();
  __syncwarp();
  uint8_t* buf = bufs + sb * 2048;
  uint4* d = reinterpret_cast<uint4*>(buf + lane * 64);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    d[swz64(lane, i)] =
        make_uint4(pack_bf16x2(v[8 * i + 0], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                   pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, buf, col, row0);
    bulk_commit();
  }
  sb ^= 1;
}

// Epilogue of one tile for one thread (one output row). All tcgen05.ld are
// executed by every lane of the warp (they are warp-collective).
// `half` selects the 32-column chunks this warp handles (even or odd); the other epilogue
// warp on the same TMEM lane quarter takes the rest.
// Aux loads of the SwiGLU backward: per epilogue warp one mbarrier (abar), its phase (aph)
// and whether a load is still outstanding (apend, drained at the end of the kernel).
struct AuxWait {
  uint64_t* bar;
  uint32_t phase;
  bool pending;
  volatile int* abort;
  int* err;
};

__device__ void epilogue_tile(const Prob& pr, const CUtensorMap* maps, int m0, int n0, int r, uint32_t tb,
                              float* stage, int half, int& sb, AuxWait& aw) {
  const int row = m0 + r;
  bool rv = row < pr.M;
  const int64_t orow = pr.row_map ? (rv ? (int64_t)pr.row_map[row] : 0) : (int64_t)pr.out_row0 + row;
  if (pr.row_map && rv) rv = index_ok(orow, pr.M, aw.err, DEV_BAD_ROW_MAP);
  float v[32];
  uint32_t raw[32];
  // bulk tensor stores: warp-uniform; rows of this warp start at wrow0 (problem-local)
  const bool bulk = pr.omap[0] >= 0;
  const int wrow0 = m0 + (r & ~31);
  const bool wlive = wrow0 < pr.M;
  uint8_t* bufs = reinterpret_cast<uint8_t*>(stage);

  if (pr.epi == EPI_SWIGLU) {
    const int ncols = min(128, pr.N - n0);
    for (int c0 = 32 * half; c0 < 128; c0 += 64) {
      if (c0 >= ncols) break;
      float g[32];
      uint32_t rawu[32];
      __syncwarp();
      tmem_ld32(tb + c0, raw);  // g and u in flight together, one wait
      tmem_ld32(tb + 128 + c0, rawu);
      tmem_ld_wait_regs(raw);
      regs_after_wait(rawu);
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = __uint_as_float(raw[i]);
#pragma unroll
      for (int i = 0; i < 32; ++i) raw[i] = rawu[i];
      const int n = min(32, ncols - c0);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);  // u
      if (bulk) {
        if (!wlive) continue;
        bulk_store_chunk(&maps[pr.omap[0]], bufs, sb, g, n0 + c0, wrow0);
        bulk_store_chunk(&maps[pr.omap[1]], bufs, sb, v, n0 + c0, wrow0);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = silu_f(g[i]) * v[i];
        bulk_store_chunk(&maps[pr.omap[2]], bufs, sb, v, n0 + c0, wrow0);
        continue;
      }
      if (!rv) continue;
      const int64_t off = orow * pr.ld0 + n0 + c0;
      const bool vec = ((off & 7) == 0);
      store_bf16_row(reinterpret_cast<__nv_bfloat16*>(pr.out0) + off, g, n, vec);
      store_bf16_row(reinterpret_cast<__nv_bfloat16*>(pr.out1) + off, v, n, vec);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = silu_f(g[i]) * v[i];
      store_bf16_row(reinterpret_cast<__nv_bfloat16*>(pr.out2) + off, v, n, vec);
    }
    return;
  }

  const int ncols = min(pr.tile_cols, pr.N - n0);
  const int cend = min(pr.n_mma, ncols);
  // One 32-column chunk: TMEM values in `raw` (already waited for), columns c0 .. c0 + 31.
  auto chunk = [&](uint32_t (&raw)[32], int c0) {
    const int n = min(32, ncols - c0);
    if (pr.epi == EPI_BF16 && pr.col_map) {
      // Scatter through a 32 x 32 shared-memory transpose (element (r, c) at r * 32 + (c ^ r): the
      // row writes and the column reads both hit 32 different banks): each store instruction then
      // writes 32 columns of one row (a few sectors) instead of one column of 32 rows.
      // (The transpose buffer is also the bulk-store boxes: let pending bulk reads finish.)
      const int lane = r & 31;
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 32; ++i) stage[lane * 32 + (i ^ lane)] = __uint_as_float(raw[i]) * pr.a0;
      __syncwarp();
      bool cv = lane < n;
      const int64_t ocol = cv ? (int64_t)pr.col_map[n0 + c0 + lane] : 0;
      if (cv) cv = index_ok(ocol, pr.N, aw.err, DEV_BAD_COL_MAP);
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(pr.out0);
      const int wrow0 = m0 + r - lane;
      for (int rr = 0; rr < 32; ++rr) {
        const int row2 = wrow0 + rr;
        if (cv && row2 < pr.M) {
          const int64_t o2 = pr.row_map ? (int64_t)pr.row_map[row2] : (int64_t)pr.out_row0 + row2;
          if (!pr.row_map || index_ok(o2, pr.M, aw.err, DEV_BAD_ROW_MAP))
            out[o2 * pr.ld0 + ocol] = __float2bfloat16_rn(stage[rr * 32 + (lane ^ rr)]);
        }
      }
      __syncwarp();
      return;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(raw[i]);
    if (bulk && pr.epi == EPI_BF16) {
      if (!wlive) return;
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= pr.a0;
      bulk_store_chunk(&maps[pr.omap[0]], bufs, sb, v, n0 + c0, wrow0);
      return;
    }
    if (bulk && pr.epi == EPI_DSWIGLU) {
      if (!wlive) return;
      float g[32], u[32];
      const int lane = r & 31;
      // g and u of the warp's 32 rows x 32 columns arrive by two bulk tensor loads into the
      // warp's two boxes, once its earlier bulk stores have read them; one lane = one row
      if (lane == 0) {
        bulk_wait_read<0>();
        mbar_arrive_expect_tx(aw.bar, 4096);
        tma_load_2d(bufs, &maps[pr.omap[2]], aw.bar, n0 + c0, wrow0);
        tma_load_2d(bufs + 2048, &maps[pr.omap[3]], aw.bar, n0 + c0, wrow0);
      }
      aw.pending = true;
      if (!mbar_wait(aw.bar, aw.phase, aw.abort, aw.err, DEV_TIMEOUT_EPILOGUE)) return;
      aw.pending = false;
      aw.phase ^= 1;
      load_box_row(bufs, lane, g);
      load_box_row(bufs + 2048, lane, u);
      __syncwarp();
      float dg[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float sg = sigmoid_f(g[i]);
        const float dh = v[i];
        dg[i] = dh * u[i] * (sg * (1.0f + g[i] * (1.0f - sg)));
        v[i] = dh * g[i] * sg;  // du = dh * SiLU(g)
      }
      bulk_store_chunk(&maps[pr.omap[0]], bufs, sb, dg, n0 + c0, wrow0);
      bulk_store_chunk(&maps[pr.omap[1]], bufs, sb, v, n0 + c0, wrow0);
      return;
    }
    if (!rv) return;
    switch (pr.epi) {
      case EPI_BF16: {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= pr.a0;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(pr.out0);
        if (pr.col_map) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < n) {
              const int64_t oc = pr.col_map[n0 + c0 + i];
              if (index_ok(oc, pr.N, aw.err, DEV_BAD_COL_MAP)) out[orow * pr.ld0 + oc] = __float2bfloat16_rn(v[i]);
            }
        } else {
          const int64_t off = orow * pr.ld0 + n0 + c0;
          store_bf16_row(out + off, v, n, (off & 7) == 0);
        }
        break;
      }
      case EPI_F32:
      case EPI_F32_T: {
        // out += a0 v goes out as a reduction in L2 (no load round trip; each element receives
        // one addition per launch, so the result does not depend on timing). Without a column
        // map or split, column i of the chunk is base + i * step: a short instruction stream,
        // which matters when each CTA runs this code once (its first fetch is the cost).
        if (!pr.col_map && !pr.col_split) {
          const bool tr = pr.epi == EPI_F32_T;
          const int64_t step = tr ? pr.ld0 : 1;
          float* base = reinterpret_cast<float*>(pr.out0) + (tr ? (int64_t)(n0 + c0) * pr.ld0 + orow
                                                                 : orow * pr.ld0 + n0 + c0);
          if (pr.beta) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < n) atomicAdd(base + i * step, pr.a0 * v[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < n) base[i * step] = pr.a0 * v[i];
          }
          break;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (i >= n) break;
          const int64_t col = pr.col_map ? pr.col_map[n0 + c0 + i] : n0 + c0 + i;
          if (pr.col_map && !index_ok(col, pr.N, aw.err, DEV_BAD_COL_MAP)) continue;
          float* d = pr.epi == EPI_F32 ? reinterpret_cast<float*>(pr.out0) + orow * pr.ld0 + col : f32t_dst(pr, col) + orow;
          if (pr.beta)
            atomicAdd(d, pr.a0 * v[i]);
          else
            *d = pr.a0 * v[i];
        }
        break;
      }
      case EPI_XA: {
        float* o0 = reinterpret_cast<float*>(pr.out0) + orow * pr.ld0 + n0 + c0;
        __nv_bfloat16* o1 = reinterpret_cast<__nv_bfloat16*>(pr.out1) + orow * pr.ld1 + n0 + c0;
        const int zc = pr.z_col0 > 0 ? pr.z_col0 - (n0 + c0) : 1 << 30;  // first Z column of the chunk
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (i >= n) break;
          if (i >= zc) {
            if (orow < pr.z_rows) reinterpret_cast<float*>(pr.out2)[orow * pr.ld2 + (i - zc)] = pr.a0 * v[i];
          } else {
            o0[i] = pr.a0 * v[i];
            o1[i] = __float2bfloat16_rn(pr.a1 * v[i]);
          }
        }
        break;
      }
      case EPI_DSWIGLU: {
        float g[32], u[32];
        const int64_t aoff = orow * pr.ld_aux + n0 + c0;
        const bool vec = (aoff & 7) == 0;
        load_bf16_row(reinterpret_cast<const __nv_bfloat16*>(pr.aux0) + aoff, g, n, vec);
        load_bf16_row(reinterpret_cast<const __nv_bfloat16*>(pr.aux1) + aoff, u, n, vec);
        float dg[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float s = sigmoid_f(g[i]);
          const float dh = v[i];
          dg[i] = dh * u[i] * (s * (1.0f + g[i] * (1.0f - s)));
          v[i] = dh * g[i] * s;  // du = dh * SiLU(g)
        }
        const int64_t off = orow * pr.ld0 + n0 + c0;
        store_bf16_row(reinterpret_cast<__nv_bfloat16*>(pr.out0) + off, dg, n, (off & 7) == 0);
        store_bf16_row(reinterpret_cast<__nv_bfloat16*>(pr.out1) + off, v, n, (off & 7) == 0);
        break;
      }
      default:
        break;
    }
    };
  // Two chunks in flight per TMEM wait (columns c0 and c0 + 64 of this warp's half).
  uint32_t raw2[32];
  for (int c0 = 32 * half; c0 < cend; c0 += 128) {
    const bool two = c0 + 64 < cend;
    __syncwarp();
    tmem_ld32(tb + c0, raw);
    if (two) tmem_ld32(tb + c0 + 64, raw2);
    tmem_ld_wait_regs(raw);
    regs_after_wait(raw2);
    chunk(raw, c0);
    if (two) chunk(raw2, c0 + 64);
  }
}

// Split-K tile: the raw fp32 accumulator goes to part[ks][col][row] (column-major, so the
// threads of a warp, one row each, store 128 contiguous bytes per column); the reduce kernel
// sums the splits in a fixed order and applies the problem's epilogue.
__device__ void epilogue_partial(const Prob& pr, int m0, int ks, int r, uint32_t tb, int half) {
  const int row = m0 + r;
  const bool rv = row < pr.M;
  uint32_t raw[32];
  float* dst = pr.part + (int64_t)ks * pr.N * pr.M + row;
  for (int c0 = 32 * half; c0 < pr.n_mma; c0 += 64) {
    if (c0 >= pr.N) break;
    __syncwarp();
    tmem_ld32(tb + c0, raw);
    tmem_ld_wait();
    if (!rv) continue;
    const int n = min(32, pr.N - c0);
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < n) dst[(int64_t)(c0 + i) * pr.M] = __uint_as_float(raw[i]);
  }
}

struct RedProb {
  int32_t M, N, ksplit, epi, beta, out_row0, col_split, z_col0, z_rows, pad_;
  int* err;
  int64_t ld0, ld1, ld2;
  void* out0;
  void* out1;
  void* out2;
  const int32_t* row_map;
  const int32_t* col_map;
  const float* part;
  float a0, a1;
};
struct RedParams {
  RedProb p[kMaxProbs];
};

__device__ __forceinline__ float* f32t_out(const RedProb& pr, int64_t col) {
  if (pr.col_split) {
    const int j = (int)(col / pr.col_split);
    void* o = j == 0 ? pr.out0 : (j == 1 ? pr.out1 : pr.out2);
    return reinterpret_cast<float*>(o) + (col - (int64_t)j * pr.col_split) * pr.ld0;
  }
  return reinterpret_cast<float*>(pr.out0) + col * pr.ld0;
}

// Fixed-order sum of split-K partials (column-major [ksplit][N][M]) + the problem's epilogue
// (EPI_XA, EPI_F32, EPI_F32_T). Consecutive threads take consecutive rows of a column, so the
// partial loads and the transposed stores are contiguous.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const __grid_constant__ RedParams rp) {
  pdl_wait();
  const RedProb& pr = rp.p[blockIdx.y];
  const int64_t total = (int64_t)pr.M * pr.N;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
    const int64_t row = e % pr.M, col = e / pr.M;
    float acc = 0.f;
    for (int s = 0; s < pr.ksplit; ++s) acc += __ldg(pr.part + (int64_t)s * total + e);
    const int64_t orow = pr.row_map ? (int64_t)pr.row_map[row] : pr.out_row0 + row;
    const int64_t ocol = pr.col_map ? (int64_t)pr.col_map[col] : col;
    if (pr.row_map && !index_ok(orow, pr.M, pr.err, DEV_BAD_ROW_MAP)) continue;
    if (pr.col_map && !index_ok(ocol, pr.N, pr.err, DEV_BAD_COL_MAP)) continue;
    if (pr.epi == EPI_XA) {
      if (pr.z_col0 > 0 && ocol >= pr.z_col0) {
        if (orow < pr.z_rows) reinterpret_cast<float*>(pr.out2)[orow * pr.ld2 + (ocol - pr.z_col0)] = pr.a0 * acc;
      } else {
        reinterpret_cast<float*>(pr.out0)[orow * pr.ld0 + ocol] = pr.a0 * acc;
        reinterpret_cast<__nv_bfloat16*>(pr.out1)[orow * pr.ld1 + ocol] = __float2bfloat16_rn(pr.a1 * acc);
      }
    } else {
      float* d = pr.epi == EPI_F32_T ? f32t_out(pr, ocol) + orow : reinterpret_cast<float*>(pr.out0) + orow * pr.ld0 + ocol;
      *d = pr.a0 * acc + (pr.beta ? *d : 0.f);
    }
  }
}

// ---- row-gathered B operands (Seg::gidx)
//
// A gathered segment reads its B rows straight from the full weight: B row q of the stage is
// weight row gidx[q] (q < g_valid), fetched by tile::gather4 copies of four 128-byte rows
// each, and a zero row from the zero map past the kept count. The producer warp's lanes
// issue the copies of one group of four rows each.
struct Rows4 {
  int32_t r[4];
  uint32_t m;  // bit i set: row i comes from the weight; clear: from the zero row
};

// Weight rows of B positions q .. q + 3 (q a multiple of 4, gidx 16-byte aligned).
__device__ __forceinline__ Rows4 gather_rows4(const Seg& sg, int q, int* err) {
  Rows4 o;
  if (q + 3 < sg.g_valid) {
    const int4 v = __ldg(reinterpret_cast<const int4*>(sg.gidx + q));
    o.r[0] = v.x;
    o.r[1] = v.y;
    o.r[2] = v.z;
    o.r[3] = v.w;
    o.m = 15u;
  } else {
    o.m = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool v = q + i < sg.g_valid;
      o.r[i] = v ? __ldg(sg.gidx + q + i) : 0;
      o.m |= (uint32_t)v << i;
    }
  }
#ifdef SL_DEBUG_BOUNDS
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (((o.m >> i) & 1u) && !index_ok(o.r[i], sg.g_rows, err, DEV_BAD_GATHER_ROW)) o.m &= ~(1u << i);
#else
  (void)err;
#endif
  return o;
}

// Four B rows at dst (512 bytes, 128-byte rows): one gather4 copy when all four come from the
// weight or all from the zero row, else one single-row copy each. Every copy lands 512 bytes
// on the stage barrier in total, whatever the mix.
template <bool PAIR>
__device__ __forceinline__ void gather_issue4(uint8_t* dst, const CUtensorMap* mw, const CUtensorMap* mz,
                                              uint64_t* bar, int x, const Rows4& g) {
  if (g.m == 15u) {
    if (PAIR)
      tma_gather4_pair(dst, mw, bar, x, g.r[0], g.r[1], g.r[2], g.r[3]);
    else
      tma_gather4(dst, mw, bar, x, g.r[0], g.r[1], g.r[2], g.r[3]);
  } else if (g.m == 0u) {
    if (PAIR)
      tma_gather4_pair(dst, mz, bar, 0, 0, 0, 0, 0);
    else
      tma_gather4(dst, mz, bar, 0, 0, 0, 0, 0);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool w = (g.m >> i) & 1u;
      if (PAIR)
        tma_load_2d_pair(dst + 128 * i, w ? mw : mz, bar, w ? x : 0, w ? g.r[i] : 0);
      else
        tma_load_2d(dst + 128 * i, w ? mw : mz, bar, w ? x : 0, w ? g.r[i] : 0);
    }
  }
}

// The one-CTA kernel's stage ring holds B tiles of BROWS rows (or N columns): skinny
// launches (the rank-r LoRA products, estimator stage 1) stage only the B rows they use
// and keep 6 or 8 stages of A in flight instead of 4 in the same shared memory.
template <int BROWS>
struct OneCfg {
  static constexpr int kStageB = BROWS * kBK * 2;
  static constexpr int kStages = (sl::kStages * (kStageABytes + kStageBBytes)) / (kStageABytes + kStageB);
};
static_assert(OneCfg<64>::kStages == 8 && OneCfg<128>::kStages == 6 && OneCfg<256>::kStages == 4, "stage ring");

template <int BROWS>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  using C = OneCfg<BROWS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smem_a = smem;
  uint8_t* smem_b = smem + C::kStages * kStageABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_b + C::kStages * C::kStageB);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* tfull = bars + 2 * C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_stage = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + kBarBlockBytes);  // kEpiWarps x 4 KB
  uint64_t* aux_bars = bars + 24;  // one per epilogue warp (bytes 192..255 of the barrier block)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 32 * kEpiWarps);
    }
    mbar_init(drain, 1);
    for (int w = 0; w < kEpiWarps; ++w) mbar_init(&aux_bars[w], 1);
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
  pdl_wait();  // the prologue above overlaps the previous kernel's tail

  if (warp == 0 && !p.any_gather) {
    // No gathered B rows in this launch: lane 0 alone runs the producer loop.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      for (int t = blockIdx.x; t < p.total_tiles && !*abort_flag; t += gridDim.x) {
        const TileInfo ti = decode_tile(p, t);
        const Prob& pr = p.probs[ti.prob];
        const int n0 = ti.tn * pr.tile_cols;
        int g = 0;  // k-blocks of earlier active segments
        for (int s = 0; s < pr.nseg; ++s) {
          const Seg& sg = pr.seg[s];
          if (n0 >= sg.n_limit) continue;
          const uint32_t bytes = seg_tx_bytes(sg);
          const int kb_lo = max(0, ti.kb0 - g), kb_hi = min(sg.nk, ti.kb1 - g);
          g += sg.nk;
          for (int kb = kb_lo; kb < kb_hi; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER)) goto plain_done;
            mbar_arrive_expect_tx(&full[stage], bytes);
            issued_mask |= 1u << stage;
            issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
            uint8_t* sa = smem_a + stage * kStageABytes;
            uint8_t* sb = smem_b + stage * C::kStageB;
            const int kc = kb * kBK;
            if (!sg.a_mn) {
              tma_load_2d(sa, &p.maps[sg.a_map], &full[stage], sg.a_k0 + kc, sg.a_row0 + ti.tm * kBM);
            } else {
              tma_load_2d(sa, &p.maps[sg.a_map], &full[stage], sg.a_row0 + ti.tm * kBM, sg.a_k0 + kc);
              tma_load_2d(sa + 8192, &p.maps[sg.a_map], &full[stage], sg.a_row0 + ti.tm * kBM + 64, sg.a_k0 + kc);
            }
            for (int i = 0; i < sg.nb; ++i) {
              const BSrc& b = sg.b[i];
              const int coord = b.row0 + b.row_step * ti.tn;
              if (!sg.b_mn) {
                tma_load_2d(sb + b.tile_off * 128, &p.maps[b.map], &full[stage], sg.b_k0 + kc, coord);
              } else {
                for (int c = 0; c < b.rows / 64; ++c)
                  tma_load_2d(sb + (b.tile_off / 64 + c) * 8192, &p.maps[b.map], &full[stage], coord + 64 * c,
                              sg.b_k0 + kc);
              }
            }
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
      }
    plain_done:
      // Every issued copy must land before the CTA may exit.
      for (int s = 0; s < C::kStages; ++s)
        if (issued_mask & (1u << s)) mbar_wait(&full[s], (issued_par >> s) & 1u, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else if (warp == 0) {
    // The whole warp runs the loop (lanes issue the copies of gathered B rows); lane 0 waits
    // on the ring, arms the stage and issues every other copy.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_par = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
      if (__shfl_sync(0xffffffffu, lane == 0 ? *abort_flag : 0, 0)) break;
      const TileInfo ti = decode_tile(p, t);
      const Prob& pr = p.probs[ti.prob];
      const int n0 = ti.tn * pr.tile_cols;
      int g = 0;  // k-blocks of earlier active segments
      for (int s = 0; s < pr.nseg; ++s) {
        const Seg& sg = pr.seg[s];
        if (n0 >= sg.n_limit) continue;
        const uint32_t bytes = seg_tx_bytes(sg);
        const int kb_lo = max(0, ti.kb0 - g), kb_hi = min(sg.nk, ti.kb1 - g);
        g += sg.nk;
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          int ok = 1;
          if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER);
          if (!__shfl_sync(0xffffffffu, ok, 0)) goto producer_done;
          uint8_t* sa = smem_a + stage * kStageABytes;
          uint8_t* sb = smem_b + stage * C::kStageB;
          const int kc = kb * kBK;
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[stage], bytes);
            issued_mask |= 1u << stage;
            issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
            if (!sg.a_mn) {
              tma_load_2d(sa, &p.maps[sg.a_map], &full[stage], sg.a_k0 + kc, sg.a_row0 + ti.tm * kBM);
            } else {
              tma_load_2d(sa, &p.maps[sg.a_map], &full[stage], sg.a_row0 + ti.tm * kBM, sg.a_k0 + kc);
              tma_load_2d(sa + 8192, &p.maps[sg.a_map], &full[stage], sg.a_row0 + ti.tm * kBM + 64, sg.a_k0 + kc);
            }
          }
          for (int i = 0; i < sg.nb; ++i) {
            const BSrc& b = sg.b[i];
            const int coord = b.row0 + b.row_step * ti.tn;
            if (b.gather) {
              const int ng = sg.b_mn ? 16 * (b.rows / 64) : b.rows / 4;  // groups of four rows
              for (int q4 = lane; q4 < ng; q4 += 32) {
                if (!sg.b_mn) {
                  const Rows4 r = gather_rows4(sg, coord + 4 * q4, p.err);
                  gather_issue4<false>(sb + b.tile_off * 128 + q4 * 512, &p.maps[b.map], &p.maps[sg.zmap], &full[stage],
                                       sg.b_k0 + kc, r);
                } else {
                  const int c = q4 >> 4, x = coord + 64 * c;
                  Rows4 r = gather_rows4(sg, sg.b_k0 + kc + 4 * (q4 & 15), p.err);
                  if (x >= sg.g_cols) r.m = 0u;
                  gather_issue4<false>(sb + (b.tile_off / 64 + c) * 8192 + (q4 & 15) * 512, &p.maps[b.map],
                                       &p.maps[sg.zmap], &full[stage], x, r);
                }
              }
            } else if (lane == 0) {
              if (!sg.b_mn) {
                tma_load_2d(sb + b.tile_off * 128, &p.maps[b.map], &full[stage], sg.b_k0 + kc, coord);
              } else {
                for (int c = 0; c < b.rows / 64; ++c)
                  tma_load_2d(sb + (b.tile_off / 64 + c) * 8192, &p.maps[b.map], &full[stage], coord + 64 * c,
                              sg.b_k0 + kc);
              }
            }
          }
          __syncwarp();
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  producer_done:
    // Every issued copy must land before the CTA may exit.
    if (lane == 0)
      for (int s = 0; s < C::kStages; ++s)
        if (issued_mask & (1u << s)) mbar_wait(&full[s], (issued_par >> s) & 1u, nullptr, p.err, DEV_TIMEOUT_DRAIN);
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = blockIdx.x; t < p.total_tiles && !*abort_flag; t += gridDim.x) {
        const TileInfo ti = decode_tile(p, t);
        const Prob& pr = p.probs[ti.prob];
        const int n0 = ti.tn * pr.tile_cols;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kBN);
        uint32_t accumulate = 0;
        int g = 0;
        for (int s = 0; s < pr.nseg; ++s) {
          const Seg& sg = pr.seg[s];
          if (n0 >= sg.n_limit) continue;
          const uint32_t idesc = idesc_bf16(kBM, pr.n_mma, sg.a_mn, sg.b_mn);
          const int kb_lo = max(0, ti.kb0 - g), kb_hi = min(sg.nk, ti.kb1 - g);
          g += sg.nk;
          for (int kb = kb_lo; kb < kb_hi; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag, p.err, DEV_TIMEOUT_MMA)) goto mma_done;
            tc_fence_after();
            const uint32_t sa = smem_u32(smem_a + stage * kStageABytes);
            const uint32_t sb = smem_u32(smem_b + stage * C::kStageB);
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              const uint64_t ad = sg.a_mn ? smem_desc_sw128(sa + k * 2048, 8192, 1024)
                                          : smem_desc_sw128(sa + k * 32, 16, 1024);
              const uint64_t bd = sg.b_mn ? smem_desc_sw128(sb + k * 2048, 8192, 1024)
                                          : smem_desc_sw128(sb + k * 32, 16, 1024);
              umma_bf16(d_tmem, ad, bd, idesc, accumulate);
              accumulate = 1;
            }
            umma_commit(&empty[stage]);
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
    mma_done:
      // Wait for every issued MMA before TMEM is released.
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else {
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;   // which 32-column chunks of the tile
    const int r = q * 32 + lane;
    int acc = 0, sbuf = 0;
    AuxWait aw{aux_bars + (warp - 2), 0u, false, abort_flag, p.err};
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
      const TileInfo ti = decode_tile(p, t);
      const Prob& pr = p.probs[ti.prob];
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, DEV_TIMEOUT_EPILOGUE)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kBN);
      if (pr.ksplit > 1)
        epilogue_partial(pr, ti.tm * kBM, ti.ks, r, tb, half);
      else
        epilogue_tile(pr, p.maps, ti.tm * kBM, ti.tn * pr.tile_cols, r, tb, epi_stage + (warp - 2) * (kEpiWarpBytes / 4), half,
                      sbuf, aw);
      __syncwarp();
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    if (aw.pending) mbar_wait(aw.bar, aw.phase, nullptr, nullptr, 0);  // an aux load in flight lands first
    if (lane == 0) bulk_wait_all();  // bulk stores complete before the CTA's shared memory goes away
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------ CTA-pair variant
//
// Same roles and problem list, but a cluster of two CTAs (two SMs) computes one tile of
// 256 * MH rows x 256 columns with cta_group::2 MMAs: each CTA stages its own 128 * MH
// rows of A and its half (128 rows) of the B tile, the even CTA issues the MMAs for both,
// and each CTA's TMEM holds the accumulators of its rows. Only full-width tiles
// (n_mma = 256) use it.
//   MH = 1: 256 x 256 tiles, two accumulator buffers (the epilogue of one tile overlaps
//           the main loop of the next), six 32 KB stages.
//   MH = 2: 512 x 256 tiles: per K step two M = 256 MMAs share the B tile, so operand
//           bytes per FLOP drop by a quarter; one accumulator fills all 512 TMEM columns
//           (the epilogue is not overlapped), four 48 KB stages.
constexpr int kStageB2Bytes = 128 * kBK * 2;
template <int MH>
struct PairCfg {
  static constexpr int kStages = MH == 1 ? 6 : 4;
  static constexpr int kStageA = MH * kStageABytes;
  static constexpr int kAccBufs = MH == 1 ? 2 : 1;
  static constexpr int kTileM = 256 * MH;
};
static_assert(PairCfg<1>::kStages * (PairCfg<1>::kStageA + kStageB2Bytes) <= kStages * (kStageABytes + kStageBBytes),
              "pair stages exceed the shared-memory budget");
static_assert(PairCfg<2>::kStages * (PairCfg<2>::kStageA + kStageB2Bytes) <= kStages * (kStageABytes + kStageBBytes),
              "pair stages exceed the shared-memory budget");

__device__ __forceinline__ void pair_b_loads(const GemmParams& p, const Seg& sg, int tn, uint32_t rank, uint8_t* sb,
                                             uint64_t* full, int kc) {
  for (int i = 0; i < sg.nb; ++i) {
    const BSrc& b = sg.b[i];
    const int coord = b.row0 + b.row_step * tn;
    if (!sg.b_mn) {
      if (b.rows == 256)
        tma_load_2d_pair(sb, &p.maps[b.map], full, sg.b_k0 + kc, coord + 128 * (int)rank);
      else if (b.tile_off / 128 == (int)rank)
        tma_load_2d_pair(sb, &p.maps[b.map], full, sg.b_k0 + kc, coord);
    } else {
      for (int c = 0; c < 2; ++c)
        tma_load_2d_pair(sb + c * 8192, &p.maps[b.map], full, coord + 128 * (int)rank + 64 * c, sg.b_k0 + kc);
    }
  }
}

template <int MH>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_pair_kernel(const __grid_constant__ GemmParams p) {
  using C = PairCfg<MH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smem_a = smem;
  uint8_t* smem_b = smem + C::kStages * C::kStageA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_b + C::kStages * kStageB2Bytes);
  uint64_t* full = bars;              // used in the even CTA: both CTAs' copies count here
  uint64_t* empty = bars + C::kStages;  // both CTAs: armed by the even CTA's MMA commits
  uint64_t* tfull = bars + 2 * C::kStages;
  uint64_t* tempty = tfull + 2;       // used in the even CTA: both CTAs' epilogue threads arrive
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_stage = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + kBarBlockBytes);
  uint64_t* aux_bars = bars + 24;  // one per epilogue warp (bytes 192..255 of the barrier block)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cl = blockIdx.x >> 1, n_cl = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * 32 * kEpiWarps);
    }
    mbar_init(drain, 1);
    for (int w = 0; w < kEpiWarps; ++w) mbar_init(&aux_bars[w], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before any copy or arrive targets them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // the prologue above overlaps the previous kernel's tail

  if (warp == 0 && !p.any_gather) {
    // No gathered B rows in this launch: lane 0 alone runs the producer loop.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      for (int slot = cl; slot < slot_count(p) && !*abort_flag; slot += n_cl) {
        const int t = slot_tile(p, slot);
        if (t < 0) continue;
        const TileInfo ti = decode_tile(p, t);
        const Prob& pr = p.probs[ti.prob];
        const int n0 = ti.tn * pr.tile_cols;
        for (int s = 0; s < pr.nseg; ++s) {
          const Seg& sg = pr.seg[s];
          if (n0 >= sg.n_limit) continue;
          for (int kb = 0; kb < sg.nk; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER)) goto plain_done;
            if (leader) {
              mbar_arrive_expect_tx(&full[stage], 2u * (C::kStageA + kStageB2Bytes));
              issued_mask |= 1u << stage;
              issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
            }
            uint8_t* sa = smem_a + stage * C::kStageA;
            uint8_t* sb = smem_b + stage * kStageB2Bytes;
            const int kc = kb * kBK;
            const int arow = sg.a_row0 + ti.tm * C::kTileM + 128 * MH * (int)rank;
#pragma unroll
            for (int h = 0; h < MH; ++h) {
              uint8_t* sah = sa + h * kStageABytes;
              if (!sg.a_mn) {
                tma_load_2d_pair(sah, &p.maps[sg.a_map], &full[stage], sg.a_k0 + kc, arow + 128 * h);
              } else {
                tma_load_2d_pair(sah, &p.maps[sg.a_map], &full[stage], arow + 128 * h, sg.a_k0 + kc);
                tma_load_2d_pair(sah + 8192, &p.maps[sg.a_map], &full[stage], arow + 128 * h + 64, sg.a_k0 + kc);
              }
            }
            pair_b_loads(p, sg, ti.tn, rank, sb, &full[stage], kc);
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
      }
    plain_done:
      // The even CTA's barriers count both CTAs' copies: wait for every stage it armed.
      for (int s = 0; s < C::kStages; ++s)
        if (issued_mask & (1u << s)) mbar_wait(&full[s], (issued_par >> s) & 1u, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else if (warp == 0) {
    // The whole warp runs the loop (lanes issue the copies of gathered B rows, one group of
    // four rows each); lane 0 waits on the ring, arms the stage (even CTA) and issues the
    // copies of A and of plain B sources.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_par = 0;
    for (int slot = cl; slot < slot_count(p); slot += n_cl) {
      if (__shfl_sync(0xffffffffu, lane == 0 ? *abort_flag : 0, 0)) break;
      const int t = slot_tile(p, slot);
      if (t < 0) continue;
      const TileInfo ti = decode_tile(p, t);
      const Prob& pr = p.probs[ti.prob];
      const int n0 = ti.tn * pr.tile_cols;
      for (int s = 0; s < pr.nseg; ++s) {
        const Seg& sg = pr.seg[s];
        if (n0 >= sg.n_limit) continue;
        // Gathered segment: this CTA stages 128 B rows (K-major: positions qb + j of the one
        // source it loads) or two 64-column blocks of 64 K rows (MN-major).
        const bool gat = sg.gidx != nullptr;
        const BSrc& gb = sg.b[sg.nb == 1 ? 0 : (int)rank];
        const int gcoord = gb.row0 + gb.row_step * ti.tn;
        int gx = 0, gq = 0;
        int gdst = 0;  // byte offset of this lane's four rows within the stage's B tile
        Rows4 gr;
        gr.m = 0u;
        if (gat) {
          if (!sg.b_mn) {
            gq = gcoord + (gb.rows == 256 ? 128 * (int)rank : 0) + 4 * lane;
            gdst = lane * 512;
            gr = gather_rows4(sg, gq, p.err);  // the same rows for every k-block of the tile
          } else {
            gx = gcoord + 128 * (int)rank + 64 * (lane >> 4);
            gq = sg.b_k0 + 4 * (lane & 15);
            gdst = (lane >> 4) * 8192 + (lane & 15) * 512;
            gr = gather_rows4(sg, gq, p.err);  // k-block 0; each later block's rows are loaded one ahead
            if (gx >= sg.g_cols) gr.m = 0u;
          }
        }
        for (int kb = 0; kb < sg.nk; ++kb) {
          int ok = 1;
          if (lane == 0) ok = mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER);
          if (!__shfl_sync(0xffffffffu, ok, 0)) goto producer_done;
          uint8_t* sa = smem_a + stage * C::kStageA;
          uint8_t* sb = smem_b + stage * kStageB2Bytes;
          const int kc = kb * kBK;
          if (lane == 0) {
            if (leader) {
              mbar_arrive_expect_tx(&full[stage], 2u * (C::kStageA + kStageB2Bytes));
              issued_mask |= 1u << stage;
              issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
            }
            const int arow = sg.a_row0 + ti.tm * C::kTileM + 128 * MH * (int)rank;
#pragma unroll
            for (int h = 0; h < MH; ++h) {
              uint8_t* sah = sa + h * kStageABytes;
              if (!sg.a_mn) {
                tma_load_2d_pair(sah, &p.maps[sg.a_map], &full[stage], sg.a_k0 + kc, arow + 128 * h);
              } else {
                tma_load_2d_pair(sah, &p.maps[sg.a_map], &full[stage], arow + 128 * h, sg.a_k0 + kc);
                tma_load_2d_pair(sah + 8192, &p.maps[sg.a_map], &full[stage], arow + 128 * h + 64, sg.a_k0 + kc);
              }
            }
            if (!gat) pair_b_loads(p, sg, ti.tn, rank, sb, &full[stage], kc);
          }
          if (gat) {
            gather_issue4<true>(sb + gdst, &p.maps[gb.map], &p.maps[sg.zmap],
                                &full[stage], sg.b_mn ? gx : sg.b_k0 + kc, gr);
            if (sg.b_mn && kb + 1 < sg.nk) {
              gr = gather_rows4(sg, gq + (kb + 1) * kBK, p.err);
              if (gx >= sg.g_cols) gr.m = 0u;
            }
          }
          __syncwarp();
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  producer_done:
    // The even CTA's barriers count both CTAs' copies: wait for every stage it armed.
    if (lane == 0)
      for (int s = 0; s < C::kStages; ++s)
        if (issued_mask & (1u << s)) mbar_wait(&full[s], (issued_par >> s) & 1u, nullptr, p.err, DEV_TIMEOUT_DRAIN);
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int slot = cl; slot < slot_count(p) && !*abort_flag; slot += n_cl) {
        const int t = slot_tile(p, slot);
        if (t < 0) continue;
        const TileInfo ti = decode_tile(p, t);
        const Prob& pr = p.probs[ti.prob];
        const int n0 = ti.tn * pr.tile_cols;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kBN * MH);
        uint32_t accumulate = 0;
        for (int s = 0; s < pr.nseg; ++s) {
          const Seg& sg = pr.seg[s];
          if (n0 >= sg.n_limit) continue;
          const uint32_t idesc = idesc_bf16(256, pr.n_mma, sg.a_mn, sg.b_mn);
          for (int kb = 0; kb < sg.nk; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag, p.err, DEV_TIMEOUT_MMA)) goto mma_done;
            tc_fence_after();
            const uint32_t sa = smem_u32(smem_a + stage * C::kStageA);
            const uint32_t sb = smem_u32(smem_b + stage * kStageB2Bytes);
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              const uint64_t bd = sg.b_mn ? smem_desc_sw128(sb + k * 2048, 8192, 1024)
                                          : smem_desc_sw128(sb + k * 32, 16, 1024);
#pragma unroll
              for (int h = 0; h < MH; ++h) {
                const uint32_t sah = sa + h * kStageABytes;
                const uint64_t ad = sg.a_mn ? smem_desc_sw128(sah + k * 2048, 8192, 1024)
                                            : smem_desc_sw128(sah + k * 32, 16, 1024);
                umma_bf16_pair(d_tmem + h * kBN, ad, bd, idesc, accumulate);
              }
              accumulate = 1;
            }
            umma_commit_pair_mc(&empty[stage], 0x3);
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
        umma_commit_pair_mc(&tfull[acc], 0x3);
        if (++acc == C::kAccBufs) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
    mma_done:
      umma_commit_pair(drain);
      mbar_wait(drain, 0, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else {
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = q * 32 + lane;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int acc = 0, sbuf = 0;
    AuxWait aw{aux_bars + (warp - 2), 0u, false, abort_flag, p.err};
    uint32_t acc_phase = 0;
    for (int slot = cl; slot < slot_count(p); slot += n_cl) {
      const int t = slot_tile(p, slot);
      if (t < 0) continue;
      const TileInfo ti = decode_tile(p, t);
      const Prob& pr = p.probs[ti.prob];
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, DEV_TIMEOUT_EPILOGUE)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kBN * MH);
#pragma unroll 1
      for (int h = 0; h < MH; ++h)
        epilogue_tile(pr, p.maps, ti.tm * C::kTileM + 128 * MH * (int)rank + 128 * h, ti.tn * pr.tile_cols, r,
                      tb + (uint32_t)(h * kBN), epi_stage + (warp - 2) * (kEpiWarpBytes / 4), half, sbuf, aw);
      __syncwarp();
      tc_fence_before();
      mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
      if (++acc == C::kAccBufs) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (aw.pending) mbar_wait(aw.bar, aw.phase, nullptr, nullptr, 0);  // an aux load in flight lands first
    if (lane == 0) bulk_wait_all();  // bulk stores complete before the CTA's shared memory goes away
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && !leader) {
    // copies of this CTA signal the even CTA's barriers: give any in flight time to land
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 2000000ull) {
    }
  }
  cluster_sync_all();  // no CTA leaves while its peer may still read its shared memory or TMEM
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

int GemmBuilder::map(const void* ptr, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  if (status != 0) return 0;
  if (nmaps >= kMaxMaps) {
    status = 1;
    return 0;
  }
  if (!ptr || rows <= 0 || cols <= 0 || ld < cols || (reinterpret_cast<uintptr_t>(ptr) & 15) || (ld % 8) ||
      box_rows <= 0 || box_rows > 256) {
    status = 2;
    return 0;
  }
  auto enc = get_encode();
  if (!enc) {
    status = 3;
    return 0;
  }
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&params.maps[nmaps], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    status = 2;
    return 0;
  }
  specs[nmaps] = MapSpec{ptr, rows, cols, ld, box_rows};
  return nmaps++;
}

// Tensor map of a bf16 output block [rows, cols] (ld elements) for 32 x 32 bulk stores (64-byte
// swizzle, matching the epilogue's box layout); -1 when it cannot be encoded (the epilogue then
// stores per thread).
int GemmBuilder::map_out(void* ptr, int64_t rows, int64_t cols, int64_t ld) {
  if (nmaps >= kMaxMaps || !ptr || rows <= 0 || cols <= 0 || ld < cols || (reinterpret_cast<uintptr_t>(ptr) & 15) ||
      (ld % 8))
    return -1;
  auto enc = get_encode();
  if (!enc) return -1;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  if (enc(&params.maps[nmaps], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, gdim, gstride, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return -1;
  specs[nmaps] = MapSpec{ptr, rows, cols, ld, 32};
  return nmaps++;
}

// bf16 epilogues without row or column maps store through bulk tensor copies unless
// SL_GEMM_BULK_STORE=0.
void GemmBuilder::attach_output_maps() {
  static const bool disabled = [] {
    const char* e = getenv("SL_GEMM_BULK_STORE");
    return e && e[0] == '0';
  }();
  for (int i = 0; i < nprob; ++i) {
    Prob& pr = params.probs[i];
    for (int k = 0; k < 4; ++k) pr.omap[k] = -1;
    const bool eligible = pr.ksplit <= 1 && !pr.row_map && pr.M > 0 && pr.N > 0 &&
                          ((pr.epi == EPI_BF16 && !pr.col_map) || pr.epi == EPI_SWIGLU || pr.epi == EPI_DSWIGLU);
    if (disabled || !eligible) continue;
    // SwiGLU backward: two outputs (dg, du) and two inputs (g, u) read through the same boxes
    const int nout = pr.epi == EPI_SWIGLU ? 3 : (pr.epi == EPI_DSWIGLU ? 4 : 1);
    void* outs[4] = {pr.out0, pr.out1, pr.epi == EPI_DSWIGLU ? const_cast<void*>(pr.aux0) : pr.out2,
                     const_cast<void*>(pr.aux1)};
    int idx[4] = {-1, -1, -1, -1};
    const int saved = nmaps;
    bool ok = true;
    for (int k = 0; k < nout && ok; ++k) {
      const int64_t ld = (pr.epi == EPI_DSWIGLU && k >= 2) ? pr.ld_aux : pr.ld0;
      idx[k] = map_out(static_cast<uint16_t*>(outs[k]) + (int64_t)pr.out_row0 * ld, pr.M, pr.N, ld);
      ok = idx[k] >= 0;
    }
    if (!ok) {
      nmaps = saved;
      continue;
    }
    for (int k = 0; k < nout; ++k) pr.omap[k] = (int8_t)idx[k];
  }
}

bool GemmBuilder::pair_eligible() const {
  static const bool disabled = [] {
    const char* e = getenv("SL_GEMM_1CTA");
    return e && e[0] == '1';
  }();
  if (disabled || nprob == 0 || forced_pair_mh() < 0) return false;
  for (int i = 0; i < nprob; ++i) {
    const Prob& pr = params.probs[i];
    if (pr.ksplit > 1 || pr.n_mma != kBN) return false;
    for (int s = 0; s < pr.nseg; ++s) {
      const Seg& sg = pr.seg[s];
      // each CTA must stage exactly 128 rows (or 128 N columns) of every B tile
      const bool full_one = sg.nb == 1 && sg.b[0].tile_off == 0 && sg.b[0].rows == 256;
      const bool split_two = !sg.b_mn && sg.nb == 2 && sg.b[0].tile_off == 0 && sg.b[0].rows == 128 &&
                             sg.b[1].tile_off == 128 && sg.b[1].rows == 128;
      if (!full_one && !split_two) return false;
    }
  }
  return true;
}

Prob* GemmBuilder::add(int M, int N, int tile_cols, int n_mma) {
  if (status != 0) return nullptr;
  if (nprob >= kMaxProbs) {
    status = 1;
    return nullptr;
  }
  Prob* pr = &params.probs[nprob++];
  memset(pr, 0, sizeof(Prob));
  pr->M = M;
  pr->N = N;
  pr->tile_cols = tile_cols;
  pr->n_mma = n_mma;
  pr->a0 = 1.f;
  pr->a1 = 1.f;
  return pr;
}

Seg* GemmBuilder::seg(Prob* pr, int a_map, int a_mn, int a_row0, int a_k0, int b_mn, int b_k0, int K, int n_limit) {
  if (!pr || status != 0) return nullptr;
  if (pr->nseg >= kMaxSegs) {
    status = 1;
    return nullptr;
  }
  Seg* s = &pr->seg[pr->nseg++];
  memset(s, 0, sizeof(Seg));
  s->a_map = (int16_t)a_map;
  s->a_mn = (int16_t)a_mn;
  s->a_row0 = a_row0;
  s->a_k0 = a_k0;
  s->b_mn = (int16_t)b_mn;
  s->b_k0 = b_k0;
  s->nk = (K + kBK - 1) / kBK;
  s->n_limit = n_limit;
  return s;
}

int choose_ksplit(int64_t M, int64_t kblocks, int target_tiles) {
  if (M <= 0 || kblocks <= 1) return 1;
  if (target_tiles <= 0) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sms = 148;
    target_tiles = sms;
  }
  const int64_t tm = (M + kBM - 1) / kBM;
  // the largest split that still fits one wave of `target_tiles` tiles
  int64_t s = target_tiles / tm;
  const int64_t smax = kblocks / 2;
  if (s > smax) s = smax;
  if (s > 32) s = 32;
  return s < 1 ? 1 : (int)s;
}

void GemmBuilder::split(Prob* pr, int ksplit, float* part) {
  if (!pr || status != 0) return;
  pr->ksplit = ksplit;
  pr->part = part;
}

void GemmBuilder::bsrc(Seg* s, int map, int tile_off, int rows, int row0, int row_step) {
  if (!s || status != 0) return;
  if (s->nb >= kMaxBSrc) {
    status = 1;
    return;
  }
  BSrc& b = s->b[s->nb++];
  b.map = (int16_t)map;
  b.tile_off = (int16_t)tile_off;
  b.rows = (int16_t)rows;
  b.row0 = row0;
  b.row_step = row_step;
}

void GemmBuilder::gather(Seg* s, const int32_t* idx, int64_t n_valid, int64_t g_rows, int64_t g_cols,
                         const void* zero_row) {
  if (!s || status != 0) return;
  if (!idx || (reinterpret_cast<uintptr_t>(idx) & 15) || n_valid < 0 || n_valid > g_rows || g_rows <= 0 ||
      g_rows > INT32_MAX || g_cols <= 0 || g_cols % 64 || g_cols > INT32_MAX || !zero_row || s->nb == 0) {
    status = 2;
    return;
  }
  if (zmap < 0) {
    zmap = map(zero_row, 1, 64, 64, 1);
    if (status != 0) return;
  }
  s->gidx = idx;
  s->g_valid = (int32_t)n_valid;
  s->g_rows = (int32_t)g_rows;
  s->g_cols = (int32_t)g_cols;
  s->zmap = (int16_t)zmap;
  for (int i = 0; i < s->nb; ++i) s->b[i].gather = 1;
}

// Rows per CTA pair (256 or 512) for a pair-eligible launch: the one with the smaller
// estimated makespan of the longest-first schedule over `pairs` CTA pairs (the schedule the
// launch then runs, pair_tile_order). Cost
// of a tile in 64-wide k-block units of a 256 x 256 tile: a 512-row tile moves 1.5x the
// operand bytes of a 256-row tile for twice the FLOPs, and its epilogue is not
// overlapped; a 256-row tile's epilogue overlaps the next tile's main loop and only shows
// when that main loop is shorter. Epilogue weights (same units, measured on B200): plain
// stores 4 per 256 rows; column scatter 8; the SwiGLU backward, which reads g and u from
// global memory row by row, 20. sl_set_pair_tile_rows(256 | 512) forces the choice.
static std::atomic<int> g_forced_mh{0};
void set_forced_pair_mh(int mh) { g_forced_mh.store(mh, std::memory_order_relaxed); }
int forced_pair_mh() { return g_forced_mh.load(std::memory_order_relaxed); }

// Estimated work of every tile of a CTA-pair launch at tile height MH, in the natural tile order
// (problem by problem, M fastest): cost units as above.
static void pair_tile_costs(const GemmParams& P, int nprob, int mh, std::vector<double>& cost) {
  cost.clear();
  for (int i = 0; i < nprob; ++i) {
    const Prob& pr = P.probs[i];
    if (pr.M <= 0 || pr.N <= 0) continue;
    const int tm = (pr.M + 256 * mh - 1) / (256 * mh);
    const int tn = (pr.N + pr.tile_cols - 1) / pr.tile_cols;
    const double epi = pr.epi == EPI_DSWIGLU ? 20.0 : (pr.col_map ? 8.0 : (pr.epi == EPI_SWIGLU ? 6.0 : 4.0));
    for (int n = 0; n < tn; ++n) {
      int kb = 0;
      for (int sg = 0; sg < pr.nseg; ++sg)
        if (n * pr.tile_cols < pr.seg[sg].n_limit) kb += pr.seg[sg].nk;
      // plus about 1.5 units per tile to refill the operand pipeline
      const double c = (mh == 1 ? std::max<double>(kb, epi) : 1.5 * kb + 2.0 * epi) + 1.5;
      for (int m = 0; m < tm; ++m) cost.push_back(c);
    }
  }
}

// Longest-first assignment of the tiles to `pairs` CTA pairs: tiles by decreasing cost (ties
// in tile order, so the first tiles of every pair are neighbours in the problem and share
// operands in L2), each to the pair with the least work so far (ties to the lower pair).
// Fills each pair's tile list in running order when `lists` is given; returns the makespan.
static double lpt_assign(const std::vector<double>& cost, int pairs, std::vector<std::vector<int>>* lists) {
  std::vector<int> idx(cost.size());
  for (size_t i = 0; i < idx.size(); ++i) idx[i] = (int)i;
  std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  typedef std::pair<double, int> Load;
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int c = 0; c < pairs; ++c) heap.push(Load(0.0, c));
  if (lists) lists->assign((size_t)pairs, std::vector<int>());
  double span = 0.0;
  for (int t : idx) {
    Load l = heap.top();
    heap.pop();
    l.first += cost[t];
    span = std::max(span, l.first);
    if (lists) (*lists)[(size_t)l.second].push_back(t);
    heap.push(l);
  }
  return span;
}

// Makespan of the natural order: tile t runs on pair t % pairs.
static double rr_span(const std::vector<double>& cost, int pairs) {
  std::vector<double> load((size_t)pairs, 0.0);
  for (size_t t = 0; t < cost.size(); ++t) load[t % (size_t)pairs] += cost[t];
  return load.empty() ? 0.0 : *std::max_element(load.begin(), load.end());
}

// The longest-first order replaces the natural one only where the model expects a clear gain:
// it runs the problems' tiles in another order, which costs L2 reuse where the tiles of a
// launch are all alike (measured: the FFN gate/up input gradient 3% slower).
constexpr double kOrderGain = 0.97;
static double schedule_span(const std::vector<double>& cost, int pairs, bool* use_order) {
  const double rr = rr_span(cost, pairs), lpt = lpt_assign(cost, pairs, nullptr);
  const bool order = lpt < kOrderGain * rr;
  if (use_order) *use_order = order;
  return order ? lpt : rr;
}

static int choose_pair_mh(const GemmParams& P, int nprob, int pairs) {
  const int forced = forced_pair_mh();
  if (forced == 1 || forced == 2) return forced;
  double best = 0.0;
  int best_mh = 1;
  std::vector<double> cost;
  for (int mh = 1; mh <= 2; ++mh) {
    pair_tile_costs(P, nprob, mh, cost);
    const double span = schedule_span(cost, pairs, nullptr);
    if (mh == 1 || span < best) {
      best = span;
      best_mh = mh;
    }
  }
  return best_mh;
}

// The slot order of a CTA-pair launch over `pairs` pairs (0 slots, the natural order, when the
// longest-first order gains too little or its table would not fit).
static void pair_tile_order(GemmParams& P, int nprob, int mh, int pairs) {
  P.n_slots = 0;
  std::vector<double> cost;
  pair_tile_costs(P, nprob, mh, cost);
  if ((int)cost.size() != P.total_tiles || P.total_tiles <= pairs) return;
  bool use = false;
  schedule_span(cost, pairs, &use);
  if (!use) return;
  std::vector<std::vector<int>> lists;
  lpt_assign(cost, pairs, &lists);
  size_t longest = 0;
  for (const auto& l : lists) longest = std::max(longest, l.size());
  const size_t n = longest * (size_t)pairs;
  if (n > (size_t)kMaxSlots) return;
  for (size_t k = 0; k < longest; ++k)
    for (int c = 0; c < pairs; ++c)
      P.order[k * pairs + c] = (int16_t)(k < lists[(size_t)c].size() ? lists[(size_t)c][k] : -1);
  P.n_slots = (int32_t)n;
}

// B-tile height of a one-CTA launch: the smallest stage layout (64, 128 or 256 rows) that
// holds every problem's B sources and MMA width. SL_GEMM_BROWS=256 forces the widest.
static int one_cta_brows(const GemmParams& P, int nprob) {
  static const bool wide = [] {
    const char* e = getenv("SL_GEMM_BROWS");
    return e && atoi(e) == 256;
  }();
  if (wide) return 256;
  int need = 0;
  for (int i = 0; i < nprob; ++i) {
    const Prob& pr = P.probs[i];
    need = std::max(need, pr.n_mma);
    for (int sgi = 0; sgi < pr.nseg; ++sgi)
      for (int b = 0; b < pr.seg[sgi].nb; ++b)
        need = std::max(need, (int)pr.seg[sgi].b[b].tile_off + (int)pr.seg[sgi].b[b].rows);
  }
  return need <= 64 ? 64 : (need <= 128 ? 128 : 256);
}

int GemmBuilder::launch(int* err, cudaStream_t stream) {
  if (status != 0) return status;
  const bool pair = pair_eligible();
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int mh = pair ? choose_pair_mh(params, nprob, std::max(1, sms / 2)) : 1;
  const int tile_m = pair ? 256 * mh : kBM;
  if (pair) {
    // each CTA of a pair stages 128 rows of a 256-row K-major B source: re-encode those
    // maps with a 128-row box (shared by every source that uses the same map)
    int remap[kMaxMaps];
    for (int m = 0; m < kMaxMaps; ++m) remap[m] = -1;
    for (int i = 0; i < nprob; ++i)
      for (int s = 0; s < params.probs[i].nseg; ++s) {
        Seg& sg = params.probs[i].seg[s];
        if (sg.b_mn) continue;
        for (int b = 0; b < sg.nb; ++b) {
          BSrc& bs = sg.b[b];
          if (bs.rows != 256 || bs.gather) continue;
          if (remap[bs.map] < 0) {
            const MapSpec sp = specs[bs.map];
            remap[bs.map] = map(sp.ptr, sp.rows, sp.cols, sp.ld, 128);
            if (status != 0) return status;
          }
          bs.map = (int16_t)remap[bs.map];
        }
      }
  }
  int total = 0;
  for (int i = 0; i < nprob; ++i) {
    Prob& pr = params.probs[i];
    // Every problem needs at least one segment active on every tile, a valid MMA
    // shape, and segment sources inside the B tile.
    if (pr.n_mma < 16 || pr.n_mma > kBN || pr.n_mma % 16 || pr.nseg == 0) return 4;
    if (pr.epi == EPI_SWIGLU && (pr.tile_cols != 128 || pr.n_mma != 256)) return 4;
    bool always = false;
    for (int s = 0; s < pr.nseg; ++s) {
      const Seg& sg = pr.seg[s];
      if (sg.n_limit >= pr.N) always = true;
      for (int b = 0; b < sg.nb; ++b) {
        const BSrc& bs = sg.b[b];
        if (bs.tile_off + bs.rows > kBN || bs.tile_off % 8) return 4;
        if (sg.b_mn && (bs.rows % 64 || bs.tile_off % 64)) return 4;
        if (bs.gather) {
          // a row-gather map over the segment's gathered tensor; group positions 16-byte aligned
          const MapSpec& sp = specs[bs.map];
          if (!sg.gidx || sp.box_rows != 1 || sp.cols != sg.g_cols || sp.rows != sg.g_rows || bs.rows % 4 ||
              bs.row0 % 4 || bs.row_step % 4 || sg.b_k0 % 4)
            return 4;
          if (!sg.b_mn && sg.b_k0 + sg.nk * kBK > sg.g_cols) return 4;  // every K box inside the rows
        }
      }
      if (sg.gidx && pr.ksplit > 1) return 4;
    }
    if (!always) return 4;
    pr.tiles_m = pr.M > 0 ? (pr.M + tile_m - 1) / tile_m : 0;
    pr.tiles_n = pr.N > 0 ? (pr.N + pr.tile_cols - 1) / pr.tile_cols : 0;
    pr.kblocks = 0;
    for (int s = 0; s < pr.nseg; ++s) pr.kblocks += pr.seg[s].nk;
    if (pr.ksplit > 1) {
      // split-K: skinny problems only; every segment active on every tile; partial buffer set
      if (pr.tiles_n != 1 || !pr.part || pr.ksplit > pr.kblocks ||
          (pr.epi != EPI_XA && pr.epi != EPI_F32 && pr.epi != EPI_F32_T))
        return 4;
      for (int s = 0; s < pr.nseg; ++s)
        if (pr.seg[s].n_limit < pr.N) return 4;
    } else {
      pr.ksplit = 1;
    }
    pr.tile_begin = total;
    total += pr.tiles_m * pr.tiles_n * pr.ksplit;
  }
  params.nprob = nprob;
  params.total_tiles = total;
  params.err = err;
  params.any_gather = 0;
  for (int i = 0; i < nprob; ++i)
    for (int s = 0; s < params.probs[i].nseg; ++s)
      if (params.probs[i].seg[s].gidx) params.any_gather = 1;
  if (total == 0) return 0;
  attach_output_maps();
  static int smem_set = 0;
  if (!smem_set) {
    if (cudaFuncSetAttribute(gemm_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(gemm_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(gemm_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) !=
            cudaSuccess)
      return 5;
    if (cudaFuncSetAttribute(gemm_pair_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) !=
        cudaSuccess)
      return 5;
    if (cudaFuncSetAttribute(gemm_pair_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes) !=
        cudaSuccess)
      return 5;
    smem_set = 1;
  }
  const bool prof = profiling_on();
#ifdef SL_PROFILE_DUMP
  if (prof) {
    // per-launch description for the profiling dump: problem shapes and MMA work issued
    char buf[1024];
    int o = snprintf(buf, sizeof(buf), "%s%d tiles=%d", pair ? "pair" : "1cta", mh, total);
    double issued = 0.0;
    for (int i = 0; i < nprob && o < (int)sizeof(buf) - 96; ++i) {
      const Prob& pr = params.probs[i];
      o += snprintf(buf + o, sizeof(buf) - o, " | M=%d N=%d nmma=%d tc=%d kb=%d ks=%d epi=%d segs=%d", pr.M, pr.N,
                    pr.n_mma, pr.tile_cols, pr.kblocks, pr.ksplit, pr.epi, pr.nseg);
      issued += 2.0 * pr.tiles_m * tile_m * pr.tiles_n * pr.n_mma * (double)pr.kblocks * kBK;
    }
    snprintf(buf + o, sizeof(buf) - o, " | issued_gflop=%.2f", issued / 1e9);
    gemm_note(buf);
  }
#endif
  if (prof) gemm_events(stream, true, pair ? mh : 0);
  if (pair) {
    const int clusters = std::min(total, sms / 2);
    pair_tile_order(params, nprob, mh, clusters);
    if (mh == 2)
      launch_kernel(gemm_pair_kernel<2>, 2 * clusters, kGemmThreads, kGemmSmemBytes, stream, params);
    else
      launch_kernel(gemm_pair_kernel<1>, 2 * clusters, kGemmThreads, kGemmSmemBytes, stream, params);
  } else {
    const int grid = total < sms ? total : sms;
    const int brows = one_cta_brows(params, nprob);
    if (brows == 64)
      launch_kernel(gemm_kernel<64>, grid, kGemmThreads, kGemmSmemBytes, stream, params);
    else if (brows == 128)
      launch_kernel(gemm_kernel<128>, grid, kGemmThreads, kGemmSmemBytes, stream, params);
    else
      launch_kernel(gemm_kernel<256>, grid, kGemmThreads, kGemmSmemBytes, stream, params);
  }
  if (launch_failed("sl_gemm")) return 5;
  if (prof) gemm_events(stream, false, pair ? mh : 0);
  note_launch();
  // reduce the split-K problems (one launch for all of them)
  RedParams rp;
  memset(&rp, 0, sizeof(rp));
  int nred = 0;
  int64_t maxmn = 0;
  for (int i = 0; i < nprob; ++i) {
    const Prob& pr = params.probs[i];
    if (pr.ksplit <= 1 || pr.M <= 0 || pr.N <= 0) continue;
    RedProb& q = rp.p[nred++];
    q.M = pr.M; q.N = pr.N; q.ksplit = pr.ksplit; q.epi = pr.epi; q.beta = pr.beta; q.out_row0 = pr.out_row0;
    q.col_split = pr.col_split; q.out2 = pr.out2;
    q.ld0 = pr.ld0; q.ld1 = pr.ld1; q.out0 = pr.out0; q.out1 = pr.out1; q.row_map = pr.row_map;
    q.col_map = pr.col_map; q.part = pr.part; q.a0 = pr.a0; q.a1 = pr.a1; q.err = err;
    q.z_col0 = pr.z_col0; q.z_rows = pr.z_rows; q.ld2 = pr.ld2;
    maxmn = std::max<int64_t>(maxmn, (int64_t)pr.M * pr.N);
  }
  if (nred) {
    const unsigned gx = (unsigned)std::min<int64_t>((maxmn + 255) / 256, 1184);
    launch_kernel(splitk_reduce_kernel, dim3(gx, nred), 256, 0, stream, rp);
    if (launch_failed("sl_gemm")) return 5;
    note_launch();
  }
  return 0;
}

}  // namespace sl
