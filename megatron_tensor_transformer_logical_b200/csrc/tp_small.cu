// Column sums for the bias gradients (dbA = colsum(dY), dbB = colsum(dZ),
// "图解Transformer并行计算" §2.2: each shard's bias gradient is the column
// sum of its own slice, so a column sum over the full width gives every
// shard's at once).  Two passes, deterministic: row chunks summed into fp32
// partials, then the partials summed in chunk order.  HBM-bound: each input
// element is read once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "tp_internal.h"

namespace tp {
namespace {

constexpr int kRowsPerChunkMin = 256;
constexpr int kMaxChunks = 64;

int64_t chunks_for(int64_t rows) {
  int64_t c = (rows + kRowsPerChunkMin - 1) / kRowsPerChunkMin;
  return c < 1 ? 1 : (c > kMaxChunks ? kMaxChunks : c);
}

template <bool F32>
__global__ void colsum_partial(const void* in, int64_t rows, int64_t cols, int64_t rows_per_chunk,
                               float* part) {
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_chunk;
  int64_t r1 = r0 + rows_per_chunk;
  if (r1 > rows) r1 = rows;
  float s = 0.0f;
  for (int64_t r = r0; r < r1; ++r) {
    if (F32)
      s += static_cast<const float*>(in)[r * cols + c];
    else
      s += __bfloat162float(static_cast<const __nv_bfloat16*>(in)[r * cols + c]);
  }
  part[static_cast<int64_t>(blockIdx.y) * cols + c] = s;
}

template <bool F32>
__global__ void colsum_final(const float* part, int64_t chunks, int64_t cols, void* out) {
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  float s = 0.0f;
  for (int64_t k = 0; k < chunks; ++k) s += part[k * cols + c];
  if (F32)
    static_cast<float*>(out)[c] = s;
  else
    static_cast<__nv_bfloat16*>(out)[c] = __float2bfloat16_rn(s);
}

}  // namespace

size_t colsum_scratch_bytes(int64_t rows, int64_t cols) {
  return static_cast<size_t>(chunks_for(rows)) * static_cast<size_t>(cols) * sizeof(float);
}

tp_status launch_colsum(const void* in, int64_t rows, int64_t cols, bool f32, void* out,
                        void* scratch, cudaStream_t stream) {
  if (rows <= 0 || cols <= 0) return TP_OK;
  const int64_t chunks = chunks_for(rows);
  const int64_t rpc = (rows + chunks - 1) / chunks;
  dim3 g1(static_cast<unsigned>((cols + 255) / 256), static_cast<unsigned>(chunks));
  dim3 g2(static_cast<unsigned>((cols + 255) / 256));
  float* part = static_cast<float*>(scratch);
  const double es = f32 ? 4.0 : 2.0;
  LaunchScope s1(TP_KIND_REDUCE, double(rows) * cols, es * rows * cols + 4.0 * chunks * cols,
                 stream, 2);
  if (f32) {
    colsum_partial<true><<<g1, 256, 0, stream>>>(in, rows, cols, rpc, part);
    colsum_final<true><<<g2, 256, 0, stream>>>(part, chunks, cols, out);
  } else {
    colsum_partial<false><<<g1, 256, 0, stream>>>(in, rows, cols, rpc, part);
    colsum_final<false><<<g2, 256, 0, stream>>>(part, chunks, cols, out);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "colsum launch");
  return TP_OK;
}

}  // namespace tp
