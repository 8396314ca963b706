// Data-movement helpers: row gathers (weight rows of kept channels, token
// permutation), column gathers (kept columns of activations), transposes of
// frozen weights and LoRA matrices, and small fp32 adds. All bf16 traffic moves
// in 16-byte vectors where the layout allows it.
#include <cuda_bf16.h>

#include <algorithm>

#include "sl_internal.h"

namespace sl {

namespace {

// One warp copies row i of a gather: dst[drow(i), col0 + c] = src[idx ? idx[i] : i, c], c < n_cols,
// drow(i) = i, or (i / blk) * blk_stride + blk_off + i % blk when blk > 0.
// The debug build checks idx[i] against the source's rows first (and skips the row if it is out
// of range).
__device__ __forceinline__ void gather_row(const GatherJob& j, int64_t row, int lane, int* err) {
  const int64_t sr = j.idx ? (int64_t)j.idx[row] : row;
  if (!index_ok(sr, j.src_rows, err, DEV_BAD_GATHER_ROW)) return;
  const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(j.src) + sr * j.ld_src;
  const int64_t drow = j.blk ? (row / j.blk) * j.blk_stride + j.blk_off + row % j.blk : row;
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(j.dst) + drow * j.ld_dst + j.col0;
  if (j.vec) {
    const int64_t nv = j.n_cols / 8;
    for (int64_t c = lane; c < nv; c += 32)
      reinterpret_cast<uint4*>(dst)[c] = __ldg(reinterpret_cast<const uint4*>(src) + c);
  } else {
    for (int64_t c = lane; c < j.n_cols; c += 32) dst[c] = src[c];
  }
}

// Row gathers in one launch: blockIdx.y picks the job, each warp copies one row (the grid covers
// the job with the most rows; shorter jobs return early).
__global__ void gather_rows_multi_kernel(const __grid_constant__ GatherJobs p) {
  pdl_wait();
  const GatherJob& j = p.j[blockIdx.y];
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= j.n_rows) return;
  gather_row(j, row, threadIdx.x & 31, p.err);
}

// dst[t, j] = src[t, idx[j]]
__global__ void gather_cols_kernel(const __nv_bfloat16* __restrict__ src, int64_t ld_src, int64_t src_cols,
                                   int64_t n_rows, const int32_t* __restrict__ idx, int64_t n_idx,
                                   __nv_bfloat16* __restrict__ dst, int64_t ld_dst, int* err) {
  pdl_wait();
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n_idx) return;
  const int64_t c = idx[j];
  if (!index_ok(c, src_cols, err, DEV_BAD_GATHER_COL)) return;
  for (int64_t t = blockIdx.y; t < n_rows; t += gridDim.y) dst[t * ld_dst + j] = src[t * ld_src + c];
}

// dst[c, r] = src[r, c] with a 32 x 32 shared-memory tile.
__global__ void transpose_kernel(const __nv_bfloat16* __restrict__ src, int64_t rows, int64_t cols, int64_t ld_src,
                                 __nv_bfloat16* __restrict__ dst, int64_t ld_dst) {
  pdl_wait();
  __shared__ __nv_bfloat16 tile[32][34];
  const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = src[r * ld_src + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) dst[c * ld_dst + r] = tile[threadIdx.x][i];
  }
}

// Row permutation that also converts the channel order of context rows to or from the sigma
// layout (context rows store channel sigma[p] in column p), one CTA per row in a grid-stride
// loop: dst[i, :] = src[perm[i], :], except
//   to_sigma, destination row i < n_ctx:       dst[i, p] = src[perm[i], sigma[p]]
//   from the sigma layout, source row < n_ctx: dst[i, sigma[p]] = src[perm[i], p]
// A context row goes through shared memory, so the global read and write stay contiguous
// 16-byte vectors and only the shared-memory accesses follow sigma.
constexpr int kPermThreads = 256;
__global__ void __launch_bounds__(kPermThreads)
    permute_rows_sigma_kernel(const __nv_bfloat16* __restrict__ src, int64_t ld_src, int64_t src_rows,
                              const int32_t* __restrict__ perm, int64_t n_rows, int n_cols,
                              const int32_t* __restrict__ sigma, int64_t n_ctx, int to_sigma,
                              __nv_bfloat16* __restrict__ dst, int64_t ld_dst, int* err) {
  extern __shared__ __align__(16) __nv_bfloat16 rowbuf[];  // two rows of n_cols
  pdl_wait();
  __nv_bfloat16* a = rowbuf;
  __nv_bfloat16* b = rowbuf + n_cols;
  const int nv = n_cols / 8;
  for (int64_t i = blockIdx.x; i < n_rows; i += gridDim.x) {
    const int64_t sr = perm[i];
    if (!index_ok(sr, src_rows, err, DEV_BAD_GATHER_ROW)) continue;  // the whole CTA skips the row
    const uint4* s4 = reinterpret_cast<const uint4*>(src + sr * ld_src);
    uint4* d4 = reinterpret_cast<uint4*>(dst + i * ld_dst);
    const bool ctx = to_sigma ? i < n_ctx : sr < n_ctx;
    if (!ctx) {
      for (int c = threadIdx.x; c < nv; c += kPermThreads) d4[c] = __ldg(s4 + c);
      continue;
    }
    for (int c = threadIdx.x; c < nv; c += kPermThreads) reinterpret_cast<uint4*>(a)[c] = __ldg(s4 + c);
    __syncthreads();
    if (to_sigma) {
      for (int v = threadIdx.x; v < nv; v += kPermThreads) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c0 = sigma[8 * v + 2 * k], c1 = sigma[8 * v + 2 * k + 1];
          const __nv_bfloat16 lo = index_ok(c0, n_cols, err, DEV_BAD_GATHER_COL) ? a[c0] : __float2bfloat16(0.f);
          const __nv_bfloat16 hi = index_ok(c1, n_cols, err, DEV_BAD_GATHER_COL) ? a[c1] : __float2bfloat16(0.f);
          w[k] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
        }
        d4[v] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      for (int p = threadIdx.x; p < n_cols; p += kPermThreads) {
        const int c = sigma[p];
        if (index_ok(c, n_cols, err, DEV_BAD_GATHER_COL)) b[c] = a[p];
      }
      __syncthreads();
      for (int c = threadIdx.x; c < nv; c += kPermThreads) d4[c] = reinterpret_cast<const uint4*>(b)[c];
    }
    __syncthreads();  // the row buffers are refilled for the next row
  }
}

__global__ void add_f32_kernel(float* __restrict__ dst, const float* __restrict__ src, int64_t n) {
  pdl_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] += src[i];
}

}  // namespace

static int vec_ok(const void* src, int64_t ld_src, const void* dst, int64_t ld_dst, int64_t n_cols, int64_t col0) {
  return (n_cols % 8 == 0) && (ld_src % 8 == 0) && (ld_dst % 8 == 0) && (col0 % 8 == 0) &&
         ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) % 16 == 0);
}

int gather_rows_bf16(const void* src, int64_t ld_src, int64_t src_rows, const int32_t* idx, int64_t n_rows,
                     int64_t n_cols, void* dst, int64_t ld_dst, int64_t dst_col0, int* err, cudaStream_t s) {
  GatherBatch b;
  b.add(src, ld_src, src_rows, idx, n_rows, n_cols, dst, ld_dst, dst_col0);
  return b.launch(err, s);
}

int GatherBatch::add(const void* src, int64_t ld_src, int64_t src_rows, const int32_t* idx, int64_t n_rows,
                     int64_t n_cols, void* dst, int64_t ld_dst, int64_t dst_col0, int blk, int blk_stride,
                     int blk_off) {
  if (n_rows <= 0 || n_cols <= 0) return 0;
  if (jobs.n >= kMaxGatherJobs) return 1;
  GatherJob& j = jobs.j[jobs.n++];
  j.src = src;
  j.ld_src = ld_src;
  j.src_rows = src_rows;
  j.idx = idx;
  j.n_rows = n_rows;
  j.n_cols = n_cols;
  j.dst = dst;
  j.ld_dst = ld_dst;
  j.col0 = dst_col0;
  j.blk = blk;
  j.blk_stride = blk_stride;
  j.blk_off = blk_off;
  j.vec = vec_ok(src, ld_src, dst, ld_dst, n_cols, dst_col0);
  return 0;
}

int GatherBatch::launch(int* err, cudaStream_t s) {
  if (jobs.n == 0) return 0;
  int64_t rows = 0;
  for (int i = 0; i < jobs.n; ++i) rows = rows > jobs.j[i].n_rows ? rows : jobs.j[i].n_rows;
  const int rows_per_block = 8;
  jobs.err = err;
  const dim3 grid((unsigned)((rows + rows_per_block - 1) / rows_per_block), (unsigned)jobs.n);
  launch_kernel(gather_rows_multi_kernel, grid, 32 * rows_per_block, 0, s, jobs);
  jobs.n = 0;
  if (launch_failed("sl_aux")) return 5;
  note_launch();
  return 0;
}

int gather_cols_bf16(const void* src, int64_t ld_src, int64_t src_cols, int64_t n_rows, const int32_t* idx,
                     int64_t n_idx, void* dst, int64_t ld_dst, int* err, cudaStream_t s) {
  if (n_rows <= 0 || n_idx <= 0) return 0;
  dim3 grid((unsigned)((n_idx + 255) / 256), (unsigned)(n_rows < 1024 ? n_rows : 1024));
  launch_kernel(gather_cols_kernel, grid, 256, 0, s, (const __nv_bfloat16*)src, ld_src, src_cols, n_rows, idx, n_idx,
                (__nv_bfloat16*)dst, ld_dst, err);
  if (launch_failed("sl_aux")) return 5;
  note_launch();
  return 0;
}

int transpose_bf16(const void* src, int64_t rows, int64_t cols, int64_t ld_src, void* dst, int64_t ld_dst,
                   cudaStream_t s) {
  if (rows <= 0 || cols <= 0) return 0;
  dim3 grid((unsigned)((cols + 31) / 32), (unsigned)((rows + 31) / 32));
  launch_kernel(transpose_kernel, grid, dim3(32, 8), 0, s, (const __nv_bfloat16*)src, rows, cols, ld_src, (__nv_bfloat16*)dst,
                                                ld_dst);
  if (launch_failed("sl_aux")) return 5;
  note_launch();
  return 0;
}

#ifdef SL_DEBUG_BOUNDS
// The error word of the debug checks in the entries that take no workspace (one per device).
static __device__ int g_aux_debug_word;
int* aux_debug_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_aux_debug_word) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}
#else
int* aux_debug_word() { return nullptr; }
#endif

int permute_rows_sigma(const void* src, int64_t ld_src, int64_t src_rows, const int32_t* perm, int64_t n_rows,
                       int64_t n_cols, const int32_t* sigma, int64_t n_ctx, int to_sigma, void* dst, int64_t ld_dst,
                       int* err, cudaStream_t s) {
  if (n_rows <= 0) return 0;
  if (n_cols <= 0 || n_cols > kPermMaxCols || n_cols % 8 || ld_src % 8 || ld_dst % 8 ||
      (reinterpret_cast<uintptr_t>(src) & 15) || (reinterpret_cast<uintptr_t>(dst) & 15))
    return 2;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(permute_rows_sigma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             2 * kPermMaxCols * 2) != cudaSuccess)
      return 5;
    attr = true;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const unsigned grid = (unsigned)std::min<int64_t>(n_rows, (int64_t)sms * 8);
  launch_kernel(permute_rows_sigma_kernel, grid, kPermThreads, (size_t)n_cols * 4, s,
                static_cast<const __nv_bfloat16*>(src), ld_src, src_rows, perm, n_rows, (int)n_cols, sigma, n_ctx,
                to_sigma, static_cast<__nv_bfloat16*>(dst), ld_dst, err);
  if (launch_failed("sl_aux")) return 5;
  note_launch();
  return 0;
}

int add_f32(float* dst, const float* src, int64_t n, cudaStream_t s) {
  if (n <= 0) return 0;
  launch_kernel(add_f32_kernel, (unsigned)((n + 255) / 256), 256, 0, s, dst, src, n);
  if (launch_failed("sl_aux")) return 5;
  note_launch();
  return 0;
}

// ---- tensor maps

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
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
}  // namespace

bool encode_bf16_2d(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int64_t ld, int box_cols,
                    int box_rows, bool swizzle128) {
  auto enc = encode_tiled();
  if (!enc || !ptr || rows <= 0 || cols <= 0 || ld < cols || (reinterpret_cast<uintptr_t>(ptr) & 15) || (ld % 8))
    return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             swizzle128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace sl
