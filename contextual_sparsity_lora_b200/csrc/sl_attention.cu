// Causal grouped-query attention core of the decoder layer, forward and backward, on the
// tcgen05 tensor cores ("SparseLoRA: Accelerating LLM Fine-Tuning with Contextual Sparsity",
// walkthrough, "Putting It All Together": the sparse q/k/v and o projections sit around the
// layer's attention; output rows attend to the context keys and values the sparse projections
// computed).
//
//   S = Q K^T / sqrt(d) per query head h (key/value head h / (Hq / Hkv)), keys k <= query q of the
//   same sequence; P = softmax_row(S); O = P V; LSE_q = log sum_k exp(S_qk).
//   Backward with D_q = sum_d dO_qd O_qd: dV = P^T dO, dP = dO V^T, dS = P (dP - D), dQ = dS K / sqrt(d),
//   dK = dS^T Q / sqrt(d).
//
// Rows are tokens in sequence order: n_seq sequences of seq_len tokens. Operand tiles (128 tokens
// x 64 head-dimension elements, 128-byte swizzle) come from 4-D tensor maps [head_dim, heads,
// seq_len, n_seq]: positions past a sequence's end and head-dimension elements past head_dim read
// as zeros, so ragged sequence lengths and head_dim < 64 need no padding copies. One tile in shared
// memory serves both operand majors: loaded with tokens as rows, it is K-major when the head
// dimension is the contraction (Q K^T, dO V^T) and MN-major when the tokens are (P V, P^T dO,
// dS^T Q, dS K).
//
// Forward: persistent CTAs (one per SM) over the units (128-query tile, query head, sequence), the
// units with the most key tiles first. Warp 0 loads each unit's Q and the K/V tiles through a
// two-stage ring (K and V of a stage on their own barriers; the ring runs on over unit
// boundaries); warp 1 issues the MMAs (S into two alternating TMEM buffers, so S of the next key
// tile, also the next unit's first, is computed while the softmax or the epilogue runs, then
// O += P V into one of two accumulators by unit); warps 2-9 run the online softmax, one query row
// (its TMEM lane) and half of the key columns per thread: row maximum, exponentials, rescaling of
// O in TMEM when the maximum grows, P (bf16) into shared memory for the P V MMA; at a unit's end
// O / l goes through a staging tile to bulk tensor stores.
// Backward: one CTA per (128-key tile, key/value head, sequence), the first key tiles (the most
// query tiles) started first, looping over the query heads of the group and the query tiles at or
// after the key tile: S^T and dP^T by MMA, P^T and dS^T by
// eight compute warps (one key row per thread, half of the query columns per warp), then
// dV += P^T dO, dK += dS^T Q and dQ = dS K by MMA. dO and Q have separate barriers, so the next
// dO loads once dV has read this one and dP^T of the next iteration starts while dQ is drained.
// dK and dV stay in TMEM for the whole loop and are stored once; dQ leaves TMEM every iteration
// into shared-memory boxes (over P^T and dS^T, free by then) and reaches the workspace accumulator
// through bulk tensor reductions (fp32 adds in L2; several key tiles add to the same query rows).
#include <cuda_bf16.h>
#include <type_traits>

#include <algorithm>
#include <cmath>

#include "sl_internal.h"
#include "sl_ptx.cuh"

namespace sl {

namespace {

constexpr int kSoftThreads = 256;                   // forward: warps 2..9 softmax / epilogue
constexpr int kAttnThreads = 64 + kSoftThreads;     // warp 0 TMA, warp 1 MMA + TMEM
constexpr int kBwdComputeThreads = 256;                   // backward: warps 2..9
constexpr int kAttnBwdThreads = 64 + kBwdComputeThreads;  // warp 0 TMA, warp 1 MMA + TMEM
constexpr int kTile = 128;           // tokens per tile (TMEM lanes)
constexpr int kChunk = 128 * 64 * 2;  // one 128-token x 64-element bf16 tile chunk (16 KB)

struct AttnFwdParams {
  CUtensorMap qmap, kmap, vmap;  // [head_dim, heads, seq_len, n_seq], boxes 64 x 1 x 128 x 1
  CUtensorMap omap;              // the same view of o (bulk stores of the output tile)
  __nv_bfloat16* o;
  int64_t ldo;
  float* lse;                    // [n_q_heads][n_seq * seq_len]
  int32_t n_seq, S, hq, hkv, hd, nd;
  float scale, scale_log2;       // 1 / sqrt(hd); log2(e) / sqrt(hd)
  int* err;
};

struct AttnBwdParams {
  CUtensorMap qmap, kmap, vmap, domap;
  CUtensorMap dqmap;             // dq_acc as [head_dim, hq, seq_len, n_seq] fp32, boxes 32 x 1 x 128 x 1
  const float* lse;              // [hq][T]
  const float* delta;            // [hq][T]: sum_d dO O per query row
  float* dq_acc;                 // [T][hq * hd] fp32, zero on entry
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int64_t ldkv;
  int32_t n_seq, S, hq, hkv, hd, nd;
  float scale, scale_log2;
  int* err;
};

__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* m, uint64_t* bar, int32_t c0,
                                            int32_t c1, int32_t c2, int32_t c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Each thread of the warp writes 32 consecutive fp32 columns of its TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Shared-memory descriptors of a tile stored as nc chunks (16 KB apart) of 128 token rows x 128 B.
// K-major use (contraction over the head dimension, or over the 128 columns of a P-like tile):
// 16-element step t lies in chunk t / 4 at byte 32 (t % 4) of each row.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int t) {
  return smem_desc_sw128(base + (uint32_t)(t >> 2) * kChunk + (uint32_t)(t & 3) * 32, 16, 1024);
}
// MN-major use (contraction over the 128 token rows): step t covers rows 16 t .. 16 t + 15; the
// 64-wide chunks of the other dimension are 16 KB apart.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, int t) {
  return smem_desc_sw128(base + (uint32_t)t * 2048, kChunk, 1024);
}

// Writes 32 bf16 values (v[0..31] as 16 packed pairs) of row r into a 128-byte-swizzled K-major
// tile (the layout the tensor maps produce): element c of the row sits in chunk c / 64, 16-byte
// unit ((c % 64) / 8) ^ (r % 8).
__device__ __forceinline__ void st_swizzled_row32(uint8_t* tile, int r, int c0, const uint32_t (&w)[16]) {
  uint8_t* row = tile + (c0 >> 6) * kChunk + r * 128;
  const int u0 = (c0 & 63) >> 3;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int u = (u0 + q) ^ (r & 7);
    *reinterpret_cast<uint4*>(row + u * 16) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

// Barrier of the forward's softmax warps that also returns whether `ok` holds in all of them.
__device__ __forceinline__ bool bar_and_soft(bool ok) {
  uint32_t all;
  asm volatile(
      "{\n\t.reg .pred q, a;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred a, 1, 256, q;\n\t"
      "selp.u32 %0, 1, 0, a;\n\t}"
      : "=r"(all)
      : "r"((uint32_t)ok)
      : "memory");
  return all != 0;
}
// Barrier of the backward's compute warps that also returns whether `ok` holds in all of them.
__device__ __forceinline__ bool bar_and_bwd(bool ok) {
  uint32_t all;
  asm volatile(
      "{\n\t.reg .pred q, a;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred a, 1, 256, q;\n\t"
      "selp.u32 %0, 1, 0, a;\n\t}"
      : "=r"(all)
      : "r"((uint32_t)ok)
      : "memory");
  return all != 0;
}

// Writes row r of a box of 32-element fp32 rows (128-byte swizzle: 16-byte unit u of row r sits at
// unit u ^ (r % 8); the box starts on a 1024-byte boundary) from 32 raw fp32 values, each
// multiplied by `mul`.
__device__ __forceinline__ void st_dq_box_row(uint8_t* box, int r, const uint32_t (&v)[32], float mul) {
  uint8_t* row = box + r * 128;
#pragma unroll
  for (int u = 0; u < 8; ++u)
    *reinterpret_cast<float4*>(row + ((u ^ (r & 7)) * 16)) =
        make_float4(__uint_as_float(v[4 * u]) * mul, __uint_as_float(v[4 * u + 1]) * mul,
                    __uint_as_float(v[4 * u + 2]) * mul, __uint_as_float(v[4 * u + 3]) * mul);
}

// Bulk tensor store of a shared-memory box through a 4-D tensor map (elements outside the tensor
// are not written), tracked in the issuing thread's bulk async-groups.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* m, const void* smem_src, int32_t c0, int32_t c1,
                                             int32_t c2, int32_t c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// Adds a shared-memory box to global memory through a 4-D tensor map (fp32 add in L2; elements
// outside the tensor are skipped), tracked in the issuing thread's bulk async-groups.
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap* m, const void* smem_src, int32_t c0, int32_t c1,
                                                  int32_t c2, int32_t c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// ------------------------------------------------------------------------------------ forward

__global__ void __launch_bounds__(kAttnThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnFwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nd = p.nd;
  uint8_t* sq = smem;                          // Q: nd chunks (room for 2)
  uint8_t* skv = sq + 2 * kChunk;              // stage s: K (nd chunks) then V (nd chunks)
  uint8_t* sp = skv + 2 * 2 * nd * kChunk;     // P: 2 chunks (128 keys)
  uint8_t* sob = sp + 2 * kChunk;              // O staging tile for the bulk stores: 2 chunks
  float* s_l = reinterpret_cast<float*>(sob + 2 * kChunk);  // [2][128]: the two halves' row sums
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_l + 256);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;   // Q of a query tile is free once its last S has read it
  uint64_t* k_full = bars + 2;    // [2]
  uint64_t* k_empty = bars + 4;   // [2]: K of a stage is free once S has read it
  uint64_t* v_full = bars + 6;    // [2]
  uint64_t* v_empty = bars + 8;   // [2]: V of a stage is free once P V has read it
  uint64_t* s_full = bars + 10;   // [2]
  uint64_t* s_free = bars + 12;   // [2]
  uint64_t* p_full = bars + 14;
  uint64_t* pv_done = bars + 15;
  uint64_t* o_free = bars + 16;   // [2]: an O accumulator is free once the epilogue has read it
  uint64_t* drain = bars + 18;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Persistent CTAs: unit u = (query tile, query head, sequence) runs over query tiles slowest and
  // from the last tile down (the most key tiles first); CTA c takes units c, c + grid, ... Every
  // role walks the same units; K/V stages, S buffers and P follow one tile counter over all of a
  // CTA's units, the two O accumulators alternate by unit.
  const int n_qt = (p.S + kTile - 1) / kTile;
  const int per_qt = p.hq * p.n_seq;
  const int n_units = n_qt * per_qt;
  const int hpg = p.hq / p.hkv;
  auto unit = [&](int u, int& qt, int& h, int& b) {
    qt = n_qt - 1 - u / per_qt;
    h = (u % per_qt) % p.hq;
    b = (u % per_qt) / p.hq;
  };
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], kSoftThreads);
      mbar_init(&o_free[s], kSoftThreads);
    }
    mbar_init(p_full, kSoftThreads);
    mbar_init(pv_done, 1);
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
  const uint32_t tmem = *tmem_slot;  // S buffers at columns 0 and 128, O accumulators at 256 and 384
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      // Loads in order: Q of a unit right before K of its first key tile (once the previous unit's
      // last S has read Q), K of tile t + 1 ahead of V of tile t.
      auto load_kv = [&](int t, bool is_v, int g, int kv, int b) -> bool {
        const int s = t & 1;
        uint64_t* empty = is_v ? &v_empty[s] : &k_empty[s];
        uint64_t* full = is_v ? &v_full[s] : &k_full[s];
        if (!mbar_wait(empty, ((t >> 1) & 1) ^ 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER)) return false;
        mbar_arrive_expect_tx(full, nd * kChunk);
        uint8_t* st = skv + s * 2 * nd * kChunk + (is_v ? nd * kChunk : 0);
        for (int c = 0; c < nd; ++c)
          tma_load_4d(st + c * kChunk, is_v ? &p.vmap : &p.kmap, full, 64 * c, g, kv * kTile, b);
        return true;
      };
      int nq = 0, nk = 0, nv = 0;  // Q, K and V tiles issued
      int pg = 0, pkv = 0, pb = 0;   // the tile whose V is still to load (tile nv when nk > nv)
      bool ok = true;
      for (int u = blockIdx.x, i = 0; ok && u < n_units; u += gridDim.x, ++i) {
        int qt, h, b;
        unit(u, qt, h, b);
        const int g = h / hpg;
        for (int j = 0; j <= qt; ++j) {
          if (j == 0) {
            // the previous unit's last V first (its P V does not wait for this unit), then Q
            if (nk > nv) {
              if (!load_kv(nv, true, pg, pkv, pb)) { ok = false; break; }
              ++nv;
            }
            if (i > 0 && !mbar_wait(q_empty, (i - 1) & 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER)) { ok = false; break; }
            mbar_arrive_expect_tx(q_full, nd * kChunk);
            for (int c = 0; c < nd; ++c) tma_load_4d(sq + c * kChunk, &p.qmap, q_full, 64 * c, h, qt * kTile, b);
            ++nq;
          }
          if (!load_kv(nk, false, g, j, b)) { ok = false; break; }
          ++nk;
          if (j > 0) {
            if (!load_kv(nv, true, pg, pkv, pb)) { ok = false; break; }
            ++nv;
          }
          pg = g;
          pkv = j;
          pb = b;
        }
      }
      if (ok && nk > nv && load_kv(nv, true, pg, pkv, pb)) ++nv;
      // every copy lands before the CTA may exit
      if (nq > 0) mbar_wait(q_full, (nq - 1) & 1, nullptr, p.err, DEV_TIMEOUT_DRAIN);
      for (int t = max(0, nk - 2); t < nk; ++t) mbar_wait(&k_full[t & 1], (t >> 1) & 1, nullptr, p.err, DEV_TIMEOUT_DRAIN);
      for (int t = max(0, nv - 2); t < nv; ++t) mbar_wait(&v_full[t & 1], (t >> 1) & 1, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(128, 128, 0, 0);          // S = Q K^T: both K-major over d
      const uint32_t id_pv = idesc_bf16(128, 64 * nd, 0, 1);     // O += P V: P K-major, V MN-major
      const uint32_t aq = smem_u32(sq), ap = smem_u32(sp);
      // P V of tile t (key tile j of the CTA's unit i) into the unit's O accumulator
      auto issue_pv = [&](int t, int i, int j) -> bool {
        if (!mbar_wait(p_full, t & 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) return false;
        if (!mbar_wait(&v_full[t & 1], (t >> 1) & 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) return false;
        // the first P V of a unit overwrites its accumulator: the epilogue of unit i - 2 has read it
        if (j == 0 && i >= 2 && !mbar_wait(&o_free[i & 1], ((i >> 1) & 1) ^ 1, abort_flag, p.err, DEV_TIMEOUT_MMA))
          return false;
        tc_fence_after();
        const uint32_t bv = smem_u32(skv + (t & 1) * 2 * nd * kChunk + nd * kChunk);
        for (int k = 0; k < 8; ++k)
          umma_bf16(tmem + 256 + 128 * (i & 1), kmajor_desc(ap, k), mnmajor_desc(bv, k), id_pv, (j > 0 || k > 0) ? 1u : 0u);
        umma_commit(pv_done);
        umma_commit(&v_empty[t & 1]);
        return true;
      };
      bool ok = true;
      int t = 0;
      for (int u = blockIdx.x, i = 0; ok && u < n_units; u += gridDim.x, ++i) {
        int qt, h, b;
        unit(u, qt, h, b);
        if (!mbar_wait(q_full, i & 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) { ok = false; break; }
        for (int j = 0; j <= qt; ++j, ++t) {
          const int s = t & 1;
          if (!mbar_wait(&k_full[s], (t >> 1) & 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) { ok = false; break; }
          if (t >= 2 && !mbar_wait(&s_free[s], ((t - 2) >> 1) & 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t bk = smem_u32(skv + s * 2 * nd * kChunk);
          for (int k = 0; k < 4 * nd; ++k)
            umma_bf16(tmem + 128 * s, kmajor_desc(aq, k), kmajor_desc(bk, k), id_s, k > 0 ? 1u : 0u);
          umma_commit(&s_full[s]);
          umma_commit(&k_empty[s]);
          if (j == qt) umma_commit(q_empty);
          if (j >= 1 && !issue_pv(t - 1, i, j - 1)) { ok = false; break; }
        }
        // this unit's last P V before the next unit's first S: the epilogue needs it first
        if (ok && !issue_pv(t - 1, i, qt)) ok = false;
      }
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else {
    // Eight softmax warps: warp w holds query rows 32 (w % 4) .. + 31 (its TMEM lanes) and one half
    // of the key columns of each S tile (exponentials, P) and of O (rescale, output). Both halves
    // read the whole S row for its maximum, so they keep the same running maximum without an
    // exchange; their partial row sums meet once per unit, at its end.
    const int cw = warp - 2;
    const int quarter = warp & 3;
    const int half = cw >> 2;
    const int r = quarter * 32 + lane;               // query row in the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int own0 = 64 * half, oth0 = 64 - own0;    // first key column of this half / the other
    const bool storer = cw == 0 && lane == 0;        // issues the output tile's bulk stores
    bool ok = true;
    int t = 0;
    for (int u = blockIdx.x, i = 0; u < n_units; u += gridDim.x, ++i) {
      int qt, h, b;
      unit(u, qt, h, b);
      const int qpos = qt * kTile + r;               // position in the sequence
      const uint32_t o_tm = tmem + lane_off + 256 + 128 * (i & 1);
      float m = -INFINITY, l = 0.f;                  // l: this half's share of the row sum
      for (int j = 0; j <= qt && ok; ++j, ++t) {
        const int s = t & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[s], (t >> 1) & 1, abort_flag, p.err, DEV_TIMEOUT_EPILOGUE))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t so[2][32], sx[2][32];               // this half's columns, the other half's
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tmem_ld32(tmem + lane_off + 128 * s + own0 + 32 * c, so[c]);
          tmem_ld32(tmem + lane_off + 128 * s + oth0 + 32 * c, sx[c]);
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s_free[s]);
        // causal mask within the sequence: key k is visible to query q when k <= q and k < S
        const int kbase = j * kTile;
        const int kmax = min(qpos, p.S - 1) - kbase;  // last visible column of this tile
        // Masked scores become -inf (then their exponentials are 0); tiles wholly below the
        // diagonal and inside the sequence (kmax >= 127) skip this. Column 0 is always visible.
        if (kmax < kTile - 1) {
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (own0 + 32 * c + e > kmax) so[c][e] = __float_as_uint(-INFINITY);
              if (oth0 + 32 * c + e > kmax) sx[c][e] = __float_as_uint(-INFINITY);
            }
        }
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            mx[e & 3] = fmaxf(mx[e & 3], fmaxf(__uint_as_float(so[c][e]), __uint_as_float(sx[c][e])));
        const float mj = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        // The running maximum moves only when a row's maximum grows by more than 2^8 in the
        // exponential's scale: the exponentials then stay below 256 and O and l keep one common
        // reference, so O is rescaled in TMEM rarely (after the first tiles almost never).
        const float m_cand = fmaxf(m, mj);
        const bool grow = m == -INFINITY || (m_cand - m) * p.scale_log2 > 8.0f;
        const float m_new = grow ? m_cand : m;
        const float mb = m_new * p.scale_log2;
        const float corr = (m == -INFINITY) ? 0.f : (grow ? ex2(m * p.scale_log2 - mb) : 1.f);
        float rs[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pw[2][16];
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float e0 = ex2(__uint_as_float(so[c][e]) * p.scale_log2 - mb);
            const float e1 = ex2(__uint_as_float(so[c][e + 1]) * p.scale_log2 - mb);
            rs[(e >> 1) & 3] += e0 + e1;
            pw[c][e / 2] = pack2(e0, e1);
          }
        l = l * corr + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
        if (j >= 1) {
          // the previous P V has landed in O (and read P): rescale this half of O when the maximum
          // grew (the first key tile of a unit: the previous unit's epilogue waited for its last P V)
          if (!__all_sync(0xffffffffu, mbar_wait(pv_done, (t - 1) & 1, abort_flag, p.err, DEV_TIMEOUT_EPILOGUE))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (__any_sync(0xffffffffu, corr != 1.f)) {
            for (int c = 2 * half; c < 2 * half + 2 && c < 2 * nd; ++c) {
              uint32_t ov[32];
              __syncwarp();
              tmem_ld32(o_tm + 32 * c, ov);
              tmem_ld_wait_regs(ov);
#pragma unroll
              for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
              tmem_st32(o_tm + 32 * c, ov);
            }
            tmem_st_wait();
          }
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) st_swizzled_row32(sp, r, own0 + 32 * c, pw[c]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
        m = m_new;
      }
      // this unit's last P V (tile t - 1) has landed
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(pv_done, (t - 1) & 1, abort_flag, p.err, DEV_TIMEOUT_EPILOGUE));
      // the previous unit's bulk stores have read the staging tile (rewritten below)
      if (storer) bulk_wait_read<0>();
      s_l[half * 128 + r] = l;
      // every softmax thread reaches both barriers of every unit (the loops only break)
      ok = bar_and_soft(ok);
      if (ok) {
        // O / l as bf16 into the staging tile, laid out like a loaded tile (128-byte swizzle,
        // 64-column chunks), then out by bulk tensor stores (rows past the sequence and columns
        // past head_dim are not written); the accumulator is released as soon as it is read
        tc_fence_after();
        const float lt = s_l[r] + s_l[128 + r];
        const float inv = 1.f / lt;
        for (int c = 2 * half; c < 2 * half + 2 && c < 2 * nd; ++c) {
          uint32_t ov[32];
          __syncwarp();
          tmem_ld32(o_tm + 32 * c, ov);
          tmem_ld_wait_regs(ov);
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) w[e / 2] = pack2(__uint_as_float(ov[e]) * inv, __uint_as_float(ov[e + 1]) * inv);
          st_swizzled_row32(sob, r, 32 * c, w);
        }
        tc_fence_before();
        mbar_arrive(&o_free[i & 1]);
        fence_proxy_async_smem();
        if (qpos < p.S && half == 0) p.lse[(int64_t)h * p.n_seq * p.S + (int64_t)b * p.S + qpos] = m * p.scale + logf(lt);
      }
      ok = bar_and_soft(ok);
      if (!ok) break;
      if (storer) {
        for (int c = 0; c < nd; ++c) tma_store_4d(&p.omap, sob + c * kChunk, 64 * c, h, qt * kTile, b);
        bulk_commit();
      }
    }
    if (storer) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// --------------------------------------------------------------------------- backward pieces

// delta[h][t] = sum_d dO[t, h hd + d] O[t, h hd + d], and the dQ accumulator's segment
// [t][h hd, (h + 1) hd) set to zero (the backward adds into it); half a warp per (token, head),
// eight elements (16 bytes) of each row per lane.
__global__ void attn_delta_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ d_o,
                                  int64_t ld, int64_t T, int hq, int hd, float* __restrict__ delta,
                                  float* __restrict__ dq_acc) {
  pdl_wait();
  const int64_t item = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
  const int sub = threadIdx.x & 15;
  const bool live = item < T * hq;
  const int64_t t = live ? item / hq : 0;
  const int h = live ? (int)(item % hq) : 0;
  float acc = 0.f;
  if (live) {
    if (8 * sub < hd) {
      const uint4 a = *reinterpret_cast<const uint4*>(o + t * ld + (int64_t)h * hd + 8 * sub);
      const uint4 c = *reinterpret_cast<const uint4*>(d_o + t * ld + (int64_t)h * hd + 8 * sub);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 fa = __bfloat1622float2(a2[k]), fc = __bfloat1622float2(c2[k]);
        acc += fa.x * fc.x + fa.y * fc.y;
      }
    }
    float* z = dq_acc + (t * hq + h) * (int64_t)hd;
    for (int d = 4 * sub; d < hd; d += 64) *reinterpret_cast<float4*>(z + d) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int s = 8; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (live && sub == 0) delta[(int64_t)h * T + t] = acc;
}

// dq[t * ldq + c] = bf16(acc[t * n + c]) for a [T, n] fp32 accumulator (n % 4 == 0), four
// columns per thread.
__global__ void attn_dq_cast_kernel(const float* __restrict__ acc, int64_t T, int64_t n, __nv_bfloat16* __restrict__ dq,
                                    int64_t ldq) {
  pdl_wait();
  const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= T * n) return;
  const int64_t t = i / n, c = i % n;
  const float4 v = *reinterpret_cast<const float4*>(acc + i);
  *reinterpret_cast<uint2*>(dq + t * ldq + c) = make_uint2(pack2(v.x, v.y), pack2(v.z, v.w));
}

// ----------------------------------------------------------------------------------- backward

__global__ void __launch_bounds__(kAttnBwdThreads, 1) attn_bwd_kernel(const __grid_constant__ AttnBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nd = p.nd;
  uint8_t* sk = smem;                  // K_j: nd chunks
  uint8_t* sv = sk + nd * kChunk;      // V_j
  uint8_t* sq = sv + nd * kChunk;      // Q_i
  uint8_t* sdo = sq + nd * kChunk;     // dO_i
  uint8_t* spt = sdo + nd * kChunk;    // P^T: 2 chunks (128 queries)
  uint8_t* sdst = spt + 2 * kChunk;    // dS^T: 2 chunks
  // P^T and dS^T also hold the dQ boxes (32 query rows x 32 fp32 per warp and box, 128-byte
  // swizzle) once the MMAs of an iteration have read them
  float* s_lse = reinterpret_cast<float*>(sdst + 2 * kChunk);  // [2][128] by iteration parity
  float* s_delta = s_lse + 256;                                // [2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_delta + 256);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;
  uint64_t* q_empty = bars + 2;
  uint64_t* do_full = bars + 3;
  uint64_t* do_empty = bars + 4;
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;
  uint64_t* mma2_done = bars + 7;
  uint64_t* dq_free = bars + 8;
  uint64_t* drain = bars + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Longest first, as in the forward: the linear block index runs over key tiles slowest and from
  // the first key tile up (key tile kt loops over the query tiles at or after it).
  const int lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  const int per_kt = p.hkv * p.n_seq;
  const int kt = lin / per_kt;
  const int g = (lin % per_kt) % p.hkv, b = (lin % per_kt) / p.hkv;
  const int hpg = p.hq / p.hkv;
  const int n_qt = (p.S + kTile - 1) / kTile;
  const int n_it = hpg * (n_qt - kt);  // (query head of the group, query tile >= kt)
  const int64_t T = (int64_t)p.n_seq * p.S;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(do_full, 1);
    mbar_init(do_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, kBwdComputeThreads);
    mbar_init(mma2_done, 1);
    mbar_init(dq_free, kBwdComputeThreads);
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
  // TMEM: S^T, then dQ, at 0; dP^T at 128; dV at 256; dK at 256 + 64 nd
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_dv = 256, t_dk = 256 + 64 * nd;
  pdl_wait();

  auto it_head = [&](int it) { return g * hpg + it % hpg; };
  auto it_qtile = [&](int it) { return kt + it / hpg; };

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, 2 * nd * kChunk);
      for (int c = 0; c < nd; ++c) {
        tma_load_4d(sk + c * kChunk, &p.kmap, kv_full, 64 * c, g, kt * kTile, b);
        tma_load_4d(sv + c * kChunk, &p.vmap, kv_full, 64 * c, g, kt * kTile, b);
      }
      // dO and Q have one buffer each and separate barriers: dO_(i+1) loads as soon as dV_i has
      // read dO_i, Q_(i+1) once dK_i has read Q_i
      int issued_do = 0, issued_q = 0;
      for (int it = 0; it < n_it; ++it) {
        const int h = it_head(it), qt = it_qtile(it);
        if (it > 0 && !mbar_wait(do_empty, (it - 1) & 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER)) break;
        mbar_arrive_expect_tx(do_full, nd * kChunk);
        for (int c = 0; c < nd; ++c) tma_load_4d(sdo + c * kChunk, &p.domap, do_full, 64 * c, h, qt * kTile, b);
        issued_do = it + 1;
        if (it > 0 && !mbar_wait(q_empty, (it - 1) & 1, abort_flag, p.err, DEV_TIMEOUT_PRODUCER)) break;
        mbar_arrive_expect_tx(q_full, nd * kChunk);
        for (int c = 0; c < nd; ++c) tma_load_4d(sq + c * kChunk, &p.qmap, q_full, 64 * c, h, qt * kTile, b);
        issued_q = it + 1;
      }
      mbar_wait(kv_full, 0, nullptr, p.err, DEV_TIMEOUT_DRAIN);
      if (issued_do > 0) mbar_wait(do_full, (issued_do - 1) & 1, nullptr, p.err, DEV_TIMEOUT_DRAIN);
      if (issued_q > 0) mbar_wait(q_full, (issued_q - 1) & 1, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_kq = idesc_bf16(128, 128, 0, 0);       // S^T = K Q^T, dP^T = V dO^T
      const uint32_t id_kd = idesc_bf16(128, 64 * nd, 0, 1);   // dV += P^T dO, dK += dS^T Q
      const uint32_t id_qd = idesc_bf16(128, 64 * nd, 1, 1);   // dQ = dS K (dS read MN-major from dS^T)
      const uint32_t ak = smem_u32(sk), av = smem_u32(sv), bq = smem_u32(sq), bdo = smem_u32(sdo);
      const uint32_t apt = smem_u32(spt), adst = smem_u32(sdst);
      bool ok = mbar_wait(kv_full, 0, abort_flag, p.err, DEV_TIMEOUT_MMA);
      for (int it = 0; ok && it < n_it; ++it) {
        // dP^T (columns 128..255) needs only dO: it may run while the previous dQ is drained
        if (!mbar_wait(do_full, it & 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < 4 * nd; ++t)
          umma_bf16(tmem + 128, kmajor_desc(av, t), kmajor_desc(bdo, t), id_kq, t > 0 ? 1u : 0u);
        if (!mbar_wait(q_full, it & 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) { ok = false; break; }
        if (it > 0 && !mbar_wait(dq_free, (it - 1) & 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < 4 * nd; ++t)
          umma_bf16(tmem, kmajor_desc(ak, t), kmajor_desc(bq, t), id_kq, t > 0 ? 1u : 0u);
        umma_commit(s_full);
        if (!mbar_wait(p_full, it & 1, abort_flag, p.err, DEV_TIMEOUT_MMA)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < 8; ++t)
          umma_bf16(tmem + t_dv, kmajor_desc(apt, t), mnmajor_desc(bdo, t), id_kd, (it > 0 || t > 0) ? 1u : 0u);
        umma_commit(do_empty);
        for (int t = 0; t < 8; ++t)
          umma_bf16(tmem + t_dk, kmajor_desc(adst, t), mnmajor_desc(bq, t), id_kd, (it > 0 || t > 0) ? 1u : 0u);
        umma_commit(q_empty);
        for (int t = 0; t < 8; ++t)
          umma_bf16(tmem, mnmajor_desc(adst, t), mnmajor_desc(ak, t), id_qd, t > 0 ? 1u : 0u);
        umma_commit(mma2_done);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else {
    // Eight compute warps: warp w reads TMEM lanes 32 (w % 4) .. + 31 and handles one half of the
    // columns (query columns of S^T / dP^T, head-dimension columns of dQ, dK or dV).
    const int cw = warp - 2;
    const int quarter = warp & 3;
    const int half = cw >> 2;
    const int r = quarter * 32 + lane;           // key row of the tile (S^T, dP^T, dV, dK) or query row (dQ)
    const int kpos = kt * kTile + r;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float log2e = 1.4426950408889634f;
    // This warp's dQ boxes: head-dimension columns 64 half .. + 31 over its rows of P^T chunk `half`,
    // columns 64 half + 32 .. + 63 over its rows of dS^T chunk `half`: the same shared memory the
    // warp itself rewrites next (P^T and dS^T rows r, columns 64 half .. + 63), so one wait of its
    // own bulk reads orders the two.
    uint8_t* box0 = spt + half * kChunk + quarter * 32 * 128;
    uint8_t* box1 = sdst + half * kChunk + quarter * 32 * 128;
    // LSE and delta of a query tile are staged in shared memory (two buffers by iteration parity),
    // read from global memory one iteration ahead
    float n_lse = 0.f, n_delta = 0.f;
    auto fetch = [&](int it) {
      const int qp = it_qtile(it) * kTile + r;
      const int64_t at = (int64_t)it_head(it) * T + (int64_t)b * p.S + qp;
      n_lse = qp < p.S ? p.lse[at] * log2e : 0.f;
      n_delta = qp < p.S ? p.delta[at] : 0.f;
    };
    if (half == 0 && n_it > 0) fetch(0);
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int h = it_head(it), qt = it_qtile(it);
      float* lse_it = s_lse + (it & 1) * 128;
      float* delta_it = s_delta + (it & 1) * 128;
      if (half == 0) {
        lse_it[r] = n_lse;
        delta_it[r] = n_delta;
      }
      // this iteration's LSE and delta are visible; `ok` is the same in every compute thread
      ok = bar_and_bwd(ok);
      if (!ok) break;
      if (half == 0 && it + 1 < n_it) fetch(it + 1);
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, it & 1, abort_flag, p.err, DEV_TIMEOUT_EPILOGUE));
      if (ok) {
        tc_fence_after();
        // this warp's previous dQ reductions have read its boxes (rewritten below)
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        // visible (key r, query c) pairs: kpos <= qpos = qt * 128 + c, qpos < S, kpos < S; a warp
        // whose rows all lie wholly above the diagonal and inside the sequence needs no masks (the
        // choice is the same for the whole warp: the chunks below hold warp-collective TMEM loads)
        const int cmin = kpos - qt * kTile;            // first visible query column
        const int cmax = p.S - 1 - qt * kTile;         // last query column inside the sequence
        const bool whole = __all_sync(0xffffffffu, cmin <= 0 && cmax >= kTile - 1 && kpos < p.S);
        auto soft_chunk = [&](int c, auto masked) {
          uint32_t st[32], dp[32];
          __syncwarp();
          tmem_ld32(tmem + lane_off + 32 * c, st);
          tmem_ld32(tmem + lane_off + 128 + 32 * c, dp);
          tmem_ld_wait_regs(st);
          regs_after_wait(dp);
          uint32_t pw[16], dw[16];
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lse_it + 32 * c + i);
            const float4 d4 = *reinterpret_cast<const float4*>(delta_it + 32 * c + i);
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dl[4] = {d4.x, d4.y, d4.z, d4.w};
            float pv[4], dv4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float pe = ex2(__uint_as_float(st[i + e]) * p.scale_log2 - lv[e]);
              if (decltype(masked)::value) {
                const int col = 32 * c + i + e;
                pe = (col >= cmin && col <= cmax && kpos < p.S) ? pe : 0.f;
              }
              pv[e] = pe;
              dv4[e] = pe * (__uint_as_float(dp[i + e]) - dl[e]);
            }
            pw[i / 2] = pack2(pv[0], pv[1]);
            pw[i / 2 + 1] = pack2(pv[2], pv[3]);
            dw[i / 2] = pack2(dv4[0], dv4[1]);
            dw[i / 2 + 1] = pack2(dv4[2], dv4[3]);
          }
          st_swizzled_row32(spt, r, 32 * c, pw);
          st_swizzled_row32(sdst, r, 32 * c, dw);
        };
        for (int c = 2 * half; c < 2 * half + 2; ++c) {
          if (whole) soft_chunk(c, std::false_type{});
          else soft_chunk(c, std::true_type{});
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
        ok = __all_sync(0xffffffffu, mbar_wait(mma2_done, it & 1, abort_flag, p.err, DEV_TIMEOUT_EPILOGUE));
      }
      if (ok) {
        // dQ of this (head, query tile), lane r = query row qt * 128 + r: out of TMEM (which the next
        // S^T may then overwrite), scaled into this warp's boxes, added to the accumulator by bulk
        // reductions of 32 rows x 32 columns
        tc_fence_after();
        uint32_t v0[32], v1[32];
        __syncwarp();
        tmem_ld32(tmem + lane_off + 64 * half, v0);
        tmem_ld32(tmem + lane_off + 64 * half + 32, v1);
        tmem_ld_wait_regs(v0);
        regs_after_wait(v1);
        tc_fence_before();
        mbar_arrive(dq_free);
        st_dq_box_row(box0, lane, v0, p.scale);
        st_dq_box_row(box1, lane, v1, p.scale);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && 64 * half < p.hd) {
          tma_reduce_add_4d(&p.dqmap, box0, 64 * half, h, qt * kTile + 32 * quarter, b);
          if (64 * half + 32 < p.hd) tma_reduce_add_4d(&p.dqmap, box1, 64 * half + 32, h, qt * kTile + 32 * quarter, b);
          bulk_commit();
        }
      }
    }
    // the reductions have completed before the CTA ends (and before its shared memory is reused)
    if (lane == 0) bulk_wait_all();
    // dK (half 1), dV (half 0) of this key tile: the MMAs of the last iteration have completed
    // (mma2_done); every lane takes part in the (warp-collective) loads, rows past the sequence
    // store nothing
    if (ok) {
      tc_fence_after();
      const bool kok = kpos < p.S;
      const int64_t row = (int64_t)b * p.S + kpos;
      const int which = half;
      __nv_bfloat16* out = (which ? p.dk : p.dv) + row * p.ldkv + (int64_t)g * p.hd;
      const float mul = which ? p.scale : 1.f;
      for (int c = 0; c < 2 * nd; ++c) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld32(tmem + lane_off + (which ? t_dk : t_dv) + 32 * c, v);
        tmem_ld_wait_regs(v);
        if (!kok || 32 * c >= p.hd) continue;
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) w[i / 2] = pack2(__uint_as_float(v[i]) * mul, __uint_as_float(v[i + 1]) * mul);
        uint4* dst = reinterpret_cast<uint4*>(out + 32 * c);
        const int nv = min(32, p.hd - 32 * c) / 8;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q < nv) dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// [hd, heads, S, n_seq] view of a [n_seq * S, ld] bf16 matrix whose head h occupies columns
// [h hd, (h + 1) hd); boxes of 64 x 1 x 128 x 1, 128-byte swizzle, zero fill outside.
bool head_map(CUtensorMap* m, const void* ptr, int64_t ld, int n_seq, int S, int heads, int hd) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)hd, (cuuint64_t)heads, (cuuint64_t)S, (cuuint64_t)n_seq};
  cuuint64_t strides[3] = {(cuuint64_t)hd * 2, (cuuint64_t)ld * 2, (cuuint64_t)S * ld * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [hd, heads, S, n_seq] view of the [n_seq * S, heads * hd] fp32 dQ accumulator; boxes of
// 32 x 1 x 32 x 1 (32 rows of 128 bytes: one warp's rows), 128-byte swizzle.
bool dq_acc_map(CUtensorMap* m, float* ptr, int n_seq, int S, int heads, int hd) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)hd, (cuuint64_t)heads, (cuuint64_t)S, (cuuint64_t)n_seq};
  cuuint64_t strides[3] = {(cuuint64_t)hd * 4, (cuuint64_t)heads * hd * 4, (cuuint64_t)S * heads * hd * 4};
  cuuint32_t box[4] = {32, 1, 32, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ptr, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shared memory of a launch: sized for head_dim 128 whatever the head dimension, which also keeps
// one CTA per SM (each CTA allocates all 512 TMEM columns).
int fwd_smem() { return 1024 + 2 * kChunk + 8 * kChunk + 2 * kChunk + 2 * kChunk + 1024 + 256; }
int bwd_smem() { return 1024 + 8 * kChunk + 4 * kChunk + 2 * 256 * 4 + 256; }

}  // namespace

int attention_fwd(const void* q, const void* k, const void* v, int64_t ldq, int64_t ldkv, int n_seq, int S, int hq,
                  int hkv, int hd, void* o, int64_t ldo, float* lse, int* err, cudaStream_t s) {
  AttnFwdParams p;
  memset(&p, 0, sizeof(p));
  if (!head_map(&p.qmap, q, ldq, n_seq, S, hq, hd) || !head_map(&p.kmap, k, ldkv, n_seq, S, hkv, hd) ||
      !head_map(&p.vmap, v, ldkv, n_seq, S, hkv, hd) || !head_map(&p.omap, o, ldo, n_seq, S, hq, hd))
    return 2;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.ldo = ldo;
  p.lse = lse;
  p.n_seq = n_seq;
  p.S = S;
  p.hq = hq;
  p.hkv = hkv;
  p.hd = hd;
  p.nd = (hd + 63) / 64;
  p.scale = 1.0f / std::sqrt((float)hd);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.err = err;
  const int smem = fwd_smem();
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, fwd_smem()) != cudaSuccess)
      return 5;
    attr = true;
  }
  static int n_sm = 0;
  if (!n_sm) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0)
      return 5;
  }
  const int64_t n_units = (int64_t)((S + kTile - 1) / kTile) * hq * n_seq;
  const dim3 grid((unsigned)std::min<int64_t>(n_units, n_sm));
  launch_kernel(attn_fwd_kernel, grid, kAttnThreads, smem, s, p);
  if (launch_failed("sl_attention")) return 5;
  note_launch();
  return 0;
}

size_t attention_bwd_scratch(int n_seq, int S, int hq, int hd) {
  const size_t T = (size_t)n_seq * S;
  return T * hq * hd * 4 + 256 + T * hq * 4;  // dQ accumulator, then delta
}

int attention_bwd(const void* q, const void* k, const void* v, const void* o, const void* d_o, const float* lse,
                  int64_t ldq, int64_t ldkv, int n_seq, int S, int hq, int hkv, int hd, void* dq, void* dk, void* dv,
                  void* scratch, int* err, cudaStream_t s) {
  AttnBwdParams p;
  memset(&p, 0, sizeof(p));
  if (!head_map(&p.qmap, q, ldq, n_seq, S, hq, hd) || !head_map(&p.kmap, k, ldkv, n_seq, S, hkv, hd) ||
      !head_map(&p.vmap, v, ldkv, n_seq, S, hkv, hd) || !head_map(&p.domap, d_o, ldq, n_seq, S, hq, hd))
    return 2;
  const int64_t T = (int64_t)n_seq * S;
  float* dq_acc = static_cast<float*>(scratch);
  float* delta = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + ((T * hq * hd * 4 + 255) & ~int64_t(255)));
  if (!dq_acc_map(&p.dqmap, dq_acc, n_seq, S, hq, hd)) return 2;
  {
    const int64_t items = T * hq;
    launch_kernel(attn_delta_kernel, (unsigned)((items + 15) / 16), 256, 0, s, static_cast<const __nv_bfloat16*>(o),
                  static_cast<const __nv_bfloat16*>(d_o), ldq, T, hq, hd, delta, dq_acc);
    if (launch_failed("sl_attention")) return 5;
    note_launch();
  }
  p.lse = lse;
  p.delta = delta;
  p.dq_acc = dq_acc;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.ldkv = ldkv;
  p.n_seq = n_seq;
  p.S = S;
  p.hq = hq;
  p.hkv = hkv;
  p.hd = hd;
  p.nd = (hd + 63) / 64;
  p.scale = 1.0f / std::sqrt((float)hd);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.err = err;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(attn_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bwd_smem()) != cudaSuccess)
      return 5;
    attr = true;
  }
  const dim3 grid((unsigned)((S + kTile - 1) / kTile), (unsigned)hkv, (unsigned)n_seq);
  launch_kernel(attn_bwd_kernel, grid, kAttnBwdThreads, bwd_smem(), s, p);
  if (launch_failed("sl_attention")) return 5;
  note_launch();
  // dQ: the dense [T, hq hd] accumulator to bf16 rows of leading dimension ldq
  const int64_t n = (int64_t)hq * hd;
  launch_kernel(attn_dq_cast_kernel, (unsigned)((T * n / 4 + 255) / 256), 256, 0, s, dq_acc, T, n,
                static_cast<__nv_bfloat16*>(dq), ldq);
  if (launch_failed("sl_attention")) return 5;
  note_launch();
  return 0;
}

}  // namespace sl
