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

// Both bias gradients of the MLP backward on the bf16 tensor-core path in one
// launch (the two passes above cost three launches there):
// * dbB = colsum(dZ): CTA (column block of 64, row chunk) sums its rows into
//   fp32 partials (8 groups of 8 columns x 32 row phases, the phases added
//   in order through shared memory); the CTA whose arrival on the column
//   block's counter is the last adds the block's chunk partials in chunk
//   order (16 groups of 4 columns x 16 chunk phases, phases in order);
// * dbA: CTAs past those add the GeLU' GEMM's per-32-row partials of dY in
//   the same 16 x 16 arrangement.
// 64-column blocks keep many short CTAs in flight for a narrow dZ (workload
// 2's h = 768: 516 CTAs of 192 rows); 256-column blocks (a warp reading 512
// contiguous bytes of a row) measured 8% faster on a 12288-wide dZ but 2%
// slower on workload 2's MLP backward.
// Which CTA arrives last varies; the order of every sum does not, so the
// result is deterministic.  The counters are cleared on the stream before
// the launch (one atomicAdd per arrival: a compare-and-swap loop retried
// under 64-way contention costs tens of microseconds).
constexpr int kBiasCols = 64;
constexpr int kBiasThreads = 256;

struct BiasPlan {
  int64_t chunk_rows, chunks, col_blocks;
};

// At most four CTAs per SM of a 148-SM B200, one wave (a fixed target, so
// the scratch size does not depend on the device), and at most 64 row
// chunks of a multiple of 32 rows: wide inputs get few, long chunks that
// stream, narrow ones many short chunks.
BiasPlan bias_plan(int64_t rows, int64_t cols) {
  BiasPlan p;
  p.col_blocks = (cols + kBiasCols - 1) / kBiasCols;
  int64_t want = 4 * 148 / p.col_blocks;
  if (want > 64) want = 64;
  if (want < 1) want = 1;
  p.chunk_rows = ((rows + want - 1) / want + 31) / 32 * 32;
  p.chunks = (rows + p.chunk_rows - 1) / p.chunk_rows;
  return p;
}

struct BiasArgs {
  const __nv_bfloat16* dZ;  // [M, h]
  int64_t M, h, chunk_rows, chunks, col_blocks;
  int nb;                   // CTAs of the dbB part (0: no dbB)
  float* partB;             // [chunks, h]
  unsigned int* ctr;        // [col_blocks], zero at launch
  __nv_bfloat16* dbB;
  const float* partA;       // [rowsA, f]
  int64_t rowsA, f;
  __nv_bfloat16* dbA;
};

// out[0..3] = the P phases' float4 partials of group g (red[q * G + g]),
// added in phase order.
template <int P, int G>
__device__ __forceinline__ void bias_finish4(const float4* red, int g, __nv_bfloat16* out) {
  float4 t = red[g];
#pragma unroll
  for (int q = 1; q < P; ++q) {
    const float4 v = red[q * G + g];
    t.x += v.x; t.y += v.y; t.z += v.z; t.w += v.w;
  }
  __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(out);
  o[0] = __floats2bfloat162_rn(t.x, t.y);
  o[1] = __floats2bfloat162_rn(t.z, t.w);
}

__global__ void __launch_bounds__(kBiasThreads) mlp_bias_grads(const BiasArgs a) {
  __shared__ float redB[32][kBiasCols];
  __shared__ float4 red4[256];
  __shared__ int last;
  const int tid = static_cast<int>(threadIdx.x);
  if (static_cast<int>(blockIdx.x) < a.nb) {
    const int64_t cb = blockIdx.x % a.col_blocks, ch = blockIdx.x / a.col_blocks;
    const int g = tid & 7, p = tid >> 3;
    const int64_t c = cb * kBiasCols + g * 8;
    const int64_t r0 = ch * a.chunk_rows;
    const int64_t r1 = r0 + a.chunk_rows < a.M ? r0 + a.chunk_rows : a.M;
    float s[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    if (c < a.h) {
#pragma unroll 4
      for (int64_t r = r0 + p; r < r1; r += 32) {
        const uint4 u = *reinterpret_cast<const uint4*>(a.dZ + r * a.h + c);
        const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(hv[i]);
          s[2 * i] += f.x;
          s[2 * i + 1] += f.y;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) redB[p][g * 8 + i] = s[i];
    __syncthreads();
    if (tid < kBiasCols && cb * kBiasCols + tid < a.h) {
      float t = redB[0][tid];
#pragma unroll 8
      for (int k = 1; k < 32; ++k) t += redB[k][tid];
      a.partB[ch * a.h + cb * kBiasCols + tid] = t;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) last = atomicAdd(a.ctr + cb, 1u) + 1u == static_cast<unsigned>(a.chunks);
    __syncthreads();
    if (!last) return;
    __threadfence();
    const int g4 = tid & 15, q = tid >> 4;
    const int64_t c4 = cb * kBiasCols + g4 * 4;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (c4 < a.h) {
#pragma unroll 4
      for (int64_t k = q; k < a.chunks; k += 16) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(a.partB + k * a.h + c4));
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
    }
    red4[q * 16 + g4] = acc;
    __syncthreads();
    if (tid < 16 && c4 < a.h) bias_finish4<16, 16>(red4, g4, a.dbB + c4);
  } else {
    const int g4 = tid & 15, q = tid >> 4;
    const int64_t c4 = (static_cast<int64_t>(blockIdx.x) - a.nb) * kBiasCols + g4 * 4;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (c4 < a.f) {
#pragma unroll 8
      for (int64_t k = q; k < a.rowsA; k += 16) {
        const float4 v = *reinterpret_cast<const float4*>(a.partA + k * a.f + c4);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
    }
    red4[q * 16 + g4] = acc;
    __syncthreads();
    if (tid < 16 && c4 < a.f) bias_finish4<16, 16>(red4, g4, a.dbA + c4);
  }
}

}  // namespace

size_t mlp_bias_grads_scratch_bytes(int64_t M, int64_t h) {
  const BiasPlan p = bias_plan(M, h);
  return static_cast<size_t>(p.chunks) * static_cast<size_t>(h) * 4 +
         static_cast<size_t>(p.col_blocks) * 4;
}

tp_status launch_mlp_bias_grads(const void* dZ, int64_t M, int64_t h, void* dbB,
                                const float* partA, int64_t f, void* dbA, void* scratch,
                                cudaStream_t stream) {
  if (M <= 0 || (dbA == nullptr && dbB == nullptr)) return TP_OK;
  if (h % 8 != 0 || f % 8 != 0) return fail(TP_ERR_ALIGN, "bias grads: widths must be multiples of 8");
  const BiasPlan p = bias_plan(M, h);
  BiasArgs a;
  a.dZ = static_cast<const __nv_bfloat16*>(dZ);
  a.M = M; a.h = h;
  a.chunk_rows = p.chunk_rows; a.chunks = p.chunks; a.col_blocks = p.col_blocks;
  a.nb = dbB != nullptr ? static_cast<int>(p.col_blocks * p.chunks) : 0;
  a.partB = static_cast<float*>(scratch);
  a.ctr = reinterpret_cast<unsigned int*>(static_cast<char*>(scratch) +
                                          static_cast<size_t>(p.chunks) * h * 4);
  a.dbB = static_cast<__nv_bfloat16*>(dbB);
  a.partA = partA;
  a.rowsA = (M + 31) / 32;
  a.f = f;
  a.dbA = static_cast<__nv_bfloat16*>(dbA);
  const int na = dbA != nullptr ? static_cast<int>((f + kBiasCols - 1) / kBiasCols) : 0;
  LaunchScope s1(TP_KIND_REDUCE, double(M) * h + double(a.rowsA) * f,
                 2.0 * M * h + 8.0 * p.chunks * h + 4.0 * a.rowsA * f, stream);
  cudaError_t e = cudaSuccess;
  if (a.nb > 0) e = cudaMemsetAsync(a.ctr, 0, static_cast<size_t>(p.col_blocks) * 4, stream);
  if (e != cudaSuccess) return cuda_fail(e, "bias grads counters");
  mlp_bias_grads<<<a.nb + na, kBiasThreads, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bias grads launch");
  return TP_OK;
}

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
