// Grouped, persistent tcgen05 GEMM engine: the description of one launch.
//
// One launch runs a list of problems. A problem computes an output block
//   C[M, N] = sum over K-segments of A_seg[M, K_seg] * B_seg[N, K_seg]^T
// with bf16 operands staged by TMA (128-byte swizzle) and fp32 accumulation in
// TMEM, followed by a fused epilogue. Operands can be K-major (K contiguous) or
// MN-major (M or N contiguous); a segment can be switched off for the output
// tiles at or beyond a channel limit (the kept prefix of a channel-ordered
// output). The B tile of a segment can be assembled from up to four sources
// (e.g. the gate and up weights for the two halves of a paired SwiGLU tile), and its rows can
// be gathered through an index list straight from the full weight (tile::gather4 copies of
// the kept rows; positions past the kept count read a zero row).
#pragma once
#include <cstdint>
#include <cuda.h>

namespace sl {

constexpr int kBM = 128;          // rows per tile (TMEM lanes)
constexpr int kBN = 256;          // max accumulator columns per tile
constexpr int kBK = 64;           // K per stage (one 128-byte swizzle atom of bf16)
constexpr int kStages = 4;
constexpr int kMaxMaps = 48;
constexpr int kMaxProbs = 12;
constexpr int kMaxSegs = 6;
constexpr int kMaxBSrc = 4;
// Workspace header: error word at byte 0, a zero row of 64 bf16 at bytes 128..255 (the zero
// source of gathered B operands; cleared with the header and never written), split-tile finish
// counters from byte 256.
constexpr int kWorkspaceHeaderBytes = 65536;
constexpr int kZeroRowOffsetBytes = 128;
constexpr int kCounterOffsetInts = 64;
constexpr int kMaxSplitCounters = (kWorkspaceHeaderBytes - 256) / 4;
constexpr int kEpiWarps = 8;       // two epilogue warps per TMEM lane quarter, splitting the columns
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;  // warp 0 TMA, warp 1 MMA, warps 2.. epilogue
constexpr int kStageABytes = kBM * kBK * 2;
constexpr int kStageBBytes = kBN * kBK * 2;
// Per epilogue warp 4 KB of shared memory, 512-byte aligned: two 2 KB boxes of the bulk tensor
// stores (32 x 32 bf16, 64-byte swizzle) or one 32 x 32 fp32 transpose tile (XOR layout).
constexpr int kEpiWarpBytes = 4096;
constexpr int kEpiStageBytes = kEpiWarps * kEpiWarpBytes;
constexpr int kBarBlockBytes = 512;  // mbarriers and flags; the epilogue region follows, 512-byte aligned
constexpr int kGemmSmemBytes = kStages * (kStageABytes + kStageBBytes) + 1024 + kBarBlockBytes + kEpiStageBytes;
static_assert(kGemmSmemBytes <= 232448, "GEMM shared memory exceeds the opt-in limit");

enum Epi : int32_t {
  EPI_BF16 = 0,     // out0 bf16 = a0 * acc
  EPI_F32 = 1,      // out0 fp32 = a0 * acc (+ out0 when beta)
  EPI_XA = 2,       // out0 fp32 = a0 * acc, out1 bf16 = a1 * acc (columns < z_col0 when set; out2 fp32 past it)
  EPI_SWIGLU = 3,   // paired tile: g = acc[:, 0:128], u = acc[:, 128:256]; out0 g, out1 u, out2 h = SiLU(g) u
  EPI_DSWIGLU = 4,  // dh = acc; reads g (aux0), u (aux1); out0 dg = dh u SiLU'(g), out1 du = dh SiLU(g)
  EPI_F32_T = 5,    // out0[col, row] fp32 = a0 * acc (+ old when beta): transposed store
};

struct BSrc {
  int16_t map;       // tensor map index
  int16_t tile_off;  // first row of the B tile (K-major) / first N column (MN-major) this source fills
  int16_t rows;      // rows (K-major, = box height) / N columns (MN-major, multiple of 64) it fills
  int16_t gather;    // 1: the map is a row-gather map (box 64 x 1) read through the segment's index list
  int32_t row0;      // coordinate of that first row / column for output tile 0
  int32_t row_step;  // coordinate advance per output tile along N
};

struct Seg {
  int16_t a_map, a_mn;  // A tensor map, 1 = MN-major
  int16_t b_mn, nb;     // B majorness, number of B sources
  int32_t a_row0;       // A coordinate along M of the problem's first row
  int32_t a_k0, b_k0;   // K coordinate offsets
  int32_t nk;           // number of kBK blocks
  int32_t n_limit;      // segment runs only for tiles whose first output column < n_limit
  BSrc b[kMaxBSrc];
  // Row gather of the B operand (sources with `gather` set): the B row at position q (the N
  // coordinate for K-major B, the K coordinate for MN-major B) is row gidx[q] of the source's
  // tensor when q < g_valid, and zero from the zero map `zmap` otherwise (and for MN-major
  // column blocks at or past g_cols); g_rows = rows of the gathered tensors (checked in the
  // debug build).
  const int32_t* gidx;
  int32_t g_valid, g_rows, g_cols;
  int16_t zmap, pad_;
};

struct Prob {
  int32_t M, N;         // output rows, output columns (channels)
  int32_t tile_cols;    // output columns per tile: 256 (plain) or 128 (paired SwiGLU)
  int32_t n_mma;        // accumulator columns produced by the MMA (<= 256, multiple of 16)
  int32_t tiles_m, tiles_n, tile_begin;
  int32_t ksplit;       // K ranges computed as separate tiles (1 = none); partials go to `part`
  int32_t cnt_base;     // first finish counter of this problem's split tiles (4 per row tile)
  int32_t kblocks;      // total kBK blocks over all segments (all segments must be always-active)
  int32_t nseg;
  Seg seg[kMaxSegs];
  int32_t epi, beta;
  int32_t col_split;    // EPI_F32_T: output columns [j * col_split, (j + 1) * col_split) go to
                        // out_j (j < 3), column c - j * col_split; 0 = all columns to out0
  int32_t out_row0;     // first output row
  int32_t z_col0;       // EPI_XA: columns >= z_col0 (> 0) go to out2 (fp32, ld ld2, column c - z_col0),
  int32_t z_rows;       //   only for output rows < z_rows; 0: every column goes to out0 / out1
  int8_t omap[4];       // tensor maps (32 x 32 boxes) of out0..out2 (SwiGLU backward: dg, du, g, u)
                        // over rows [out_row0, out_row0 + M), for the epilogue's bulk tensor copies;
                        // -1: per-thread loads and stores
  int64_t ld0, ld1, ld2, ld_aux;
  void* out0;
  void* out1;
  void* out2;
  const void* aux0;
  const void* aux1;
  const int32_t* col_map;  // optional: output column j -> col_map[j]
  const int32_t* row_map;  // optional: output row i (problem-local) -> row_map[i]
  float a0, a1;
  float* part;          // split-K partials [ksplit][N][M] fp32 (workspace, column-major)
};

constexpr int kMaxSlots = 4096;

struct GemmParams {
  CUtensorMap maps[kMaxMaps];
  Prob probs[kMaxProbs];
  int32_t nprob, total_tiles;
  int32_t any_gather;   // some segment gathers its B rows (the producer warp's lanes issue those copies)
  int32_t n_slots;      // CTA-pair launches: slots of the tile order below (0: tile t runs in slot t)
  int* err;
  int* counters;        // split-tile finish counters (zero between launches)
  // Tile of each slot of the CTA-pair schedule (pair c runs slots c, c + pairs, ...), -1: none.
  // The host balances the pairs' estimated work by longest-first assignment.
  int16_t order[kMaxSlots];
};

}  // namespace sl
