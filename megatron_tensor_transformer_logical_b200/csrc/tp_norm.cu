// LayerNorm over the last dimension, for the Transformer block that wraps the
// partitioned attention and MLP (the PyTorch tensor-parallel tutorial, §3.3:
// x = x + attention(norm1(x)); x = x + mlp(norm2(x)), norm = nn.LayerNorm).
// LayerNorm is replicated, not partitioned: every logical shard sees the
// whole normalised row.
//
// Forward: one CTA of 512 threads per row; the row (h <= 16384, h % 8 == 0)
// stays in registers; mean, then the centred variance (two passes over the
// registers), both in fp32 with block reductions; Y written in the input
// type, mean and rstd saved in fp32.
// Backward: a CTA per group of rows; per row g = dY * gamma,
//   dX = rstd * (g - mean(g) - xhat * mean(g * xhat)) (+ dR, the residual
// path's gradient, when given); dgamma / dbeta partial column sums stay in
// shared memory across the CTA's rows and are summed over CTAs by a second,
// deterministic pass.  HBM-bound: each element of X and dY is read once,
// dX written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "tp_internal.h"

namespace tp {
namespace {

constexpr int kLnThreads = 512;
constexpr int kLnChunks = 4;  // chunks of 8 elements per thread: h <= 512 * 4 * 8 = 16384
constexpr int kLnMaxH = kLnThreads * kLnChunks * 8;

template <bool F32>
__device__ __forceinline__ void load8(const void* base, long long off, float* v) {
  if (F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + off);
    const __nv_bfloat162* q = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(q[i]);
      v[2 * i] = t.x;
      v[2 * i + 1] = t.y;
    }
  }
}

template <bool F32>
__device__ __forceinline__ void store8(void* base, long long off, const float* v) {
  if (F32) {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(base) + off);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    uint4 u;
    uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&t);
    }
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + off) = u;
  }
}

// Sum over the 512 threads of the CTA (all threads get the result).
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red is free (the previous reduction has been read)
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = lane < kLnThreads / 32 ? red[lane] : 0.0f;
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) t += __shfl_xor_sync(0xffffffffu, t, s);  // every lane: the sum
  return t;
}

template <bool F32>
__global__ void __launch_bounds__(kLnThreads)
    layernorm_fwd_kernel(const void* X, const void* gamma, const void* beta, void* Y, float* mean,
                         float* rstd, int h, float eps) {
  __shared__ float red[kLnThreads / 32];
  const long long row = blockIdx.x;
  const int nch = h / 8;
  float x[kLnChunks][8];
  float s = 0.0f;
#pragma unroll
  for (int k = 0; k < kLnChunks; ++k) {
    const int ch = threadIdx.x + k * kLnThreads;
    if (ch < nch) {
      load8<F32>(X, row * h + ch * 8, x[k]);
#pragma unroll
      for (int i = 0; i < 8; ++i) s += x[k][i];
    }
  }
  const float mu = block_sum(s, red) / h;
  float q = 0.0f;
#pragma unroll
  for (int k = 0; k < kLnChunks; ++k) {
    const int ch = threadIdx.x + k * kLnThreads;
    if (ch < nch) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float d = x[k][i] - mu;
        q += d * d;
      }
    }
  }
  const float rs = rsqrtf(block_sum(q, red) / h + eps);
#pragma unroll
  for (int k = 0; k < kLnChunks; ++k) {
    const int ch = threadIdx.x + k * kLnThreads;
    if (ch < nch) {
      float g[8], b[8], y[8];
      if (gamma != nullptr) load8<F32>(gamma, ch * 8, g);
      if (beta != nullptr) load8<F32>(beta, ch * 8, b);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        y[i] = (x[k][i] - mu) * rs;
        if (gamma != nullptr) y[i] *= g[i];
        if (beta != nullptr) y[i] += b[i];
      }
      store8<F32>(Y, row * h + ch * 8, y);
    }
  }
  if (threadIdx.x == 0) {
    if (mean != nullptr) mean[row] = mu;
    if (rstd != nullptr) rstd[row] = rs;
  }
}

// Dynamic shared memory: dgamma and dbeta partials, 2 x h floats, laid out
// [element i of a chunk][chunk] so that consecutive threads touch
// consecutive words.
template <bool F32>
__global__ void __launch_bounds__(kLnThreads)
    layernorm_bwd_kernel(const void* X, const void* gamma, const float* mean, const float* rstd,
                         const void* dY, const void* dR, void* dX, float* part_g, float* part_b,
                         int M, int h, int rows_per_cta) {
  __shared__ float red[kLnThreads / 32];
  extern __shared__ float sp[];
  const int nch = h / 8;
  float* sg = sp;      // [8][nch]
  float* sb = sp + h;  // [8][nch]
  for (int i = threadIdx.x; i < 2 * h; i += kLnThreads) sp[i] = 0.0f;
  __syncthreads();
  const int r0 = blockIdx.x * rows_per_cta;
  const int r1 = min(r0 + rows_per_cta, M);
  for (int r = r0; r < r1; ++r) {
    const long long base = static_cast<long long>(r) * h;
    const float mu = mean[r], rs = rstd[r];
    float xh[kLnChunks][8], g[kLnChunks][8];
    float s1 = 0.0f, s2 = 0.0f;
#pragma unroll
    for (int k = 0; k < kLnChunks; ++k) {
      const int ch = threadIdx.x + k * kLnThreads;
      if (ch < nch) {
        float dy[8], gm[8];
        load8<F32>(X, base + ch * 8, xh[k]);
        load8<F32>(dY, base + ch * 8, dy);
        if (gamma != nullptr) load8<F32>(gamma, ch * 8, gm);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          xh[k][i] = (xh[k][i] - mu) * rs;
          g[k][i] = gamma != nullptr ? dy[i] * gm[i] : dy[i];
          s1 += g[k][i];
          s2 += g[k][i] * xh[k][i];
          sg[i * nch + ch] += dy[i] * xh[k][i];
          sb[i * nch + ch] += dy[i];
        }
      }
    }
    const float m1 = block_sum(s1, red) / h;
    const float m2 = block_sum(s2, red) / h;
#pragma unroll
    for (int k = 0; k < kLnChunks; ++k) {
      const int ch = threadIdx.x + k * kLnThreads;
      if (ch < nch) {
        float dx[8], dr[8];
        if (dR != nullptr) load8<F32>(dR, base + ch * 8, dr);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          dx[i] = rs * (g[k][i] - m1 - xh[k][i] * m2);
          if (dR != nullptr) dx[i] += dr[i];
        }
        store8<F32>(dX, base + ch * 8, dx);
      }
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < h; c += kLnThreads) {
    const long long off = static_cast<long long>(blockIdx.x) * h + c;
    part_g[off] = sg[(c & 7) * nch + (c >> 3)];
    part_b[off] = sb[(c & 7) * nch + (c >> 3)];
  }
}

template <bool F32>
__global__ void column_total_kernel(const float* part, int parts, int h, void* out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= h) return;
  float s = 0.0f;
  for (int p = 0; p < parts; ++p) s += part[static_cast<long long>(p) * h + c];
  if (F32)
    static_cast<float*>(out)[c] = s;
  else
    static_cast<__nv_bfloat16*>(out)[c] = __float2bfloat16_rn(s);
}

constexpr int kLnMaxParts = 296;  // CTAs of the backward: about two per SM

int ln_parts(int64_t M) { return static_cast<int>(M < kLnMaxParts ? M : kLnMaxParts); }

}  // namespace

int64_t layernorm_max_h() { return kLnMaxH; }

size_t layernorm_bwd_scratch_bytes(int64_t M, int64_t h) {
  const int parts = ln_parts(M > 0 ? M : 1);
  return 2 * static_cast<size_t>(parts) * static_cast<size_t>(h) * sizeof(float);
}

tp_status launch_layernorm_fwd(const void* X, const void* gamma, const void* beta, void* Y,
                               float* mean, float* rstd, int64_t M, int64_t h, float eps,
                               bool f32, cudaStream_t stream) {
  if (M <= 0) return TP_OK;
  if (h <= 0 || h % 8 != 0 || h > kLnMaxH)
    return fail(TP_ERR_UNSUPPORTED, "layernorm: h must be a multiple of 8 and at most 16384");
  LaunchScope scope(TP_KIND_REDUCE, 0.0, (f32 ? 4.0 : 2.0) * 2.0 * double(M) * h, stream);
  if (f32)
    layernorm_fwd_kernel<true><<<static_cast<unsigned>(M), kLnThreads, 0, stream>>>(
        X, gamma, beta, Y, mean, rstd, static_cast<int>(h), eps);
  else
    layernorm_fwd_kernel<false><<<static_cast<unsigned>(M), kLnThreads, 0, stream>>>(
        X, gamma, beta, Y, mean, rstd, static_cast<int>(h), eps);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "layernorm_fwd launch");
  return TP_OK;
}

tp_status launch_layernorm_bwd(const void* X, const void* gamma, const float* mean,
                               const float* rstd, const void* dY, const void* dR, void* dX,
                               void* dgamma, void* dbeta, int64_t M, int64_t h, bool f32,
                               void* scratch, cudaStream_t stream) {
  if (M <= 0) return TP_OK;
  if (h <= 0 || h % 8 != 0 || h > kLnMaxH)
    return fail(TP_ERR_UNSUPPORTED, "layernorm: h must be a multiple of 8 and at most 16384");
  const int parts = ln_parts(M);
  const int rows_per = static_cast<int>((M + parts - 1) / parts);
  const int grid = static_cast<int>((M + rows_per - 1) / rows_per);
  float* part_g = static_cast<float*>(scratch);
  float* part_b = part_g + static_cast<size_t>(grid) * h;
  const int smem = static_cast<int>(2 * h * sizeof(float));
  cudaError_t e0 = cudaFuncSetAttribute(
      f32 ? layernorm_bwd_kernel<true> : layernorm_bwd_kernel<false>,
      cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e0 != cudaSuccess) return cuda_fail(e0, "layernorm_bwd smem attribute");
  LaunchScope scope(TP_KIND_REDUCE, 0.0, (f32 ? 4.0 : 2.0) * 3.0 * double(M) * h, stream, 3);
  if (f32)
    layernorm_bwd_kernel<true><<<grid, kLnThreads, smem, stream>>>(
        X, gamma, mean, rstd, dY, dR, dX, part_g, part_b, static_cast<int>(M), static_cast<int>(h),
        rows_per);
  else
    layernorm_bwd_kernel<false><<<grid, kLnThreads, smem, stream>>>(
        X, gamma, mean, rstd, dY, dR, dX, part_g, part_b, static_cast<int>(M), static_cast<int>(h),
        rows_per);
  const unsigned cg = static_cast<unsigned>((h + 255) / 256);
  if (dgamma != nullptr) {
    if (f32)
      column_total_kernel<true><<<cg, 256, 0, stream>>>(part_g, grid, static_cast<int>(h), dgamma);
    else
      column_total_kernel<false><<<cg, 256, 0, stream>>>(part_g, grid, static_cast<int>(h), dgamma);
  }
  if (dbeta != nullptr) {
    if (f32)
      column_total_kernel<true><<<cg, 256, 0, stream>>>(part_b, grid, static_cast<int>(h), dbeta);
    else
      column_total_kernel<false><<<cg, 256, 0, stream>>>(part_b, grid, static_cast<int>(h), dbeta);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "layernorm_bwd launch");
  return TP_OK;
}

}  // namespace tp
