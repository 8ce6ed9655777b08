// Column sums for the bias gradients (dbA = colsum(dY), dbB = colsum(dZ),
// "图解Transformer并行计算" §2.2: each shard's bias gradient is the column
// sum of its own slice, so a column sum over the full width gives every
// shard's at once).  Two passes, deterministic: row chunks summed into fp32
// partials, then the partials summed in chunk order.  HBM-bound: each input
// element is read once.  On the bf16 tensor-core path dbA skips the first
// pass: the GeLU' GEMM's epilogue writes per-32-row partials of dY, and only
// colsum_final runs (launch_colsum_finish).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "tp_internal.h"

namespace tp {
namespace {

// First pass: CTA (column tile, row chunk) of 256 threads; a column tile is
// 64 groups of 8 columns (512 columns), and the CTA's 256 threads are 4 row
// phases x 64 groups.  A warp reads 32 groups of one row: 512 contiguous
// bytes of bf16 in 16-byte loads.  The 4 phases are added in order through
// shared memory, so the partial of a chunk is deterministic.
constexpr int kColGroups = 64;
constexpr int kRowPhases = 4;
constexpr int kColsumThreads = kColGroups * kRowPhases;

struct ColsumPlan {
  int64_t tiles, chunks, rows_per_chunk;
};

// About four CTAs per SM of a 148-SM B200 (a fixed target, so the scratch
// size does not depend on the device), at least 32 rows per chunk.
ColsumPlan colsum_plan(int64_t rows, int64_t cols) {
  ColsumPlan p;
  p.tiles = (cols / 8 + kColGroups - 1) / kColGroups;
  int64_t chunks = (4 * 148 + p.tiles - 1) / p.tiles;
  const int64_t most = (rows + 31) / 32;
  if (chunks > most) chunks = most;
  if (chunks > 512) chunks = 512;
  if (chunks < 1) chunks = 1;
  p.rows_per_chunk = (rows + chunks - 1) / chunks;
  p.chunks = (rows + p.rows_per_chunk - 1) / p.rows_per_chunk;
  return p;
}

template <bool F32>
__global__ void __launch_bounds__(kColsumThreads)
    colsum_partial(const void* in, int64_t rows, int64_t cols, int64_t rows_per_chunk,
                   float* part) {
  __shared__ float red[kRowPhases][kColGroups][8];
  const int g = threadIdx.x % kColGroups, ph = threadIdx.x / kColGroups;
  const int64_t c = (static_cast<int64_t>(blockIdx.x) * kColGroups + g) * 8;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_chunk;
  int64_t r1 = r0 + rows_per_chunk;
  if (r1 > rows) r1 = rows;
  float s[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  if (c < cols) {
#pragma unroll 4
    for (int64_t r = r0 + ph; r < r1; r += kRowPhases) {
      if (F32) {
        const float4* p =
            reinterpret_cast<const float4*>(static_cast<const float*>(in) + r * cols + c);
        const float4 u = p[0], w = p[1];
        s[0] += u.x; s[1] += u.y; s[2] += u.z; s[3] += u.w;
        s[4] += w.x; s[5] += w.y; s[6] += w.z; s[7] += w.w;
      } else {
        const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(in) +
                                                        r * cols + c);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(h[i]);
          s[2 * i] += f.x;
          s[2 * i + 1] += f.y;
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[ph][g][i] = s[i];
  __syncthreads();
  if (ph == 0 && c < cols) {
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i] = ((red[0][g][i] + red[1][g][i]) + red[2][g][i]) + red[3][g][i];
    float4* out = reinterpret_cast<float4*>(part + static_cast<int64_t>(blockIdx.y) * cols + c);
    out[0] = make_float4(s[0], s[1], s[2], s[3]);
    out[1] = make_float4(s[4], s[5], s[6], s[7]);
  }
}

// Second pass: out[c] = the sum of the chunk partials of column c.  A CTA of
// 1024 threads takes 32 columns: warp w adds chunks w, w + 32, w + 64, ...
// of its lane's column (128-byte rows, eight loads in flight), then the 32
// warp sums are added in warp order (deterministic).  Few columns (768 for
// a GPT-2-small bias) still give every thread only a handful of loads.
constexpr int kFinalWarps = 32;

template <bool F32>
__global__ void __launch_bounds__(kFinalWarps * 32)
    colsum_final(const float* part, int64_t chunks, int64_t cols, void* out) {
  __shared__ float red[kFinalWarps][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * 32 + lane;
  float s = 0.0f;
  if (c < cols) {
#pragma unroll 8
    for (int64_t k = w; k < chunks; k += kFinalWarps) s += part[k * cols + c];
  }
  red[w][lane] = s;
  __syncthreads();
  if (w == 0 && c < cols) {
    float t = 0.0f;
#pragma unroll
    for (int i = 0; i < kFinalWarps; ++i) t += red[i][lane];
    if (F32)
      static_cast<float*>(out)[c] = t;
    else
      static_cast<__nv_bfloat16*>(out)[c] = __float2bfloat16_rn(t);
  }
}

}  // namespace

size_t colsum_scratch_bytes(int64_t rows, int64_t cols) {
  return static_cast<size_t>(colsum_plan(rows, cols).chunks) * static_cast<size_t>(cols) *
         sizeof(float);
}

tp_status launch_colsum(const void* in, int64_t rows, int64_t cols, bool f32, void* out,
                        void* scratch, cudaStream_t stream) {
  if (rows <= 0 || cols <= 0) return TP_OK;
  if (cols % 8 != 0) return fail(TP_ERR_ALIGN, "colsum: columns must be a multiple of 8");
  const ColsumPlan p = colsum_plan(rows, cols);
  dim3 g1(static_cast<unsigned>(p.tiles), static_cast<unsigned>(p.chunks));
  dim3 g2(static_cast<unsigned>((cols + 31) / 32));
  float* part = static_cast<float*>(scratch);
  const double es = f32 ? 4.0 : 2.0;
  LaunchScope s1(TP_KIND_REDUCE, double(rows) * cols, es * rows * cols + 4.0 * p.chunks * cols,
                 stream, 2);
  if (f32) {
    colsum_partial<true><<<g1, kColsumThreads, 0, stream>>>(in, rows, cols, p.rows_per_chunk, part);
    colsum_final<true><<<g2, kFinalWarps * 32, 0, stream>>>(part, p.chunks, cols, out);
  } else {
    colsum_partial<false><<<g1, kColsumThreads, 0, stream>>>(in, rows, cols, p.rows_per_chunk,
                                                             part);
    colsum_final<false><<<g2, kFinalWarps * 32, 0, stream>>>(part, p.chunks, cols, out);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "colsum launch");
  return TP_OK;
}

tp_status launch_colsum_finish(const float* part, int64_t chunks, int64_t cols, bool f32,
                               void* out, cudaStream_t stream) {
  if (chunks <= 0 || cols <= 0) return TP_OK;
  dim3 g(static_cast<unsigned>((cols + 31) / 32));
  LaunchScope s1(TP_KIND_REDUCE, double(chunks) * cols, 4.0 * chunks * cols, stream);
  if (f32)
    colsum_final<true><<<g, kFinalWarps * 32, 0, stream>>>(part, chunks, cols, out);
  else
    colsum_final<false><<<g, kFinalWarps * 32, 0, stream>>>(part, chunks, cols, out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "colsum finish launch");
  return TP_OK;
}

}  // namespace tp
