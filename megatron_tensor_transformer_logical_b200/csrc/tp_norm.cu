// LayerNorm over the last dimension, for the Transformer block that wraps the
// partitioned attention and MLP (the PyTorch tensor-parallel tutorial, §3.3:
// x = x + attention(norm1(x)); x = x + mlp(norm2(x)), norm = nn.LayerNorm).
// LayerNorm is replicated, not partitioned: every logical shard sees the
// whole normalised row.
//
// Forward: one CTA of 256 threads per row (h <= 16384, h % 8 == 0); the
// shifted sums of the row give mean and variance in one block reduction
// (fp32), a second pass over the row writes Y in the input type; mean and
// rstd are saved in fp32.
// Backward: dX by one CTA per row, two passes over it (g = dY * gamma;
//   dX = rstd * (g - mean(g) - xhat * mean(g * xhat)) (+ dR, the residual
// path's gradient, when given)); dgamma / dbeta by a column kernel over row
// chunks of 32 (X and dY read a second time) whose chunk partials a third
// kernel sums in chunk order (deterministic).  HBM-bound.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "tp_internal.h"

namespace tp {
namespace {

constexpr int kLnMaxH = 16384;  // the widest row the library accepts

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

// dX of one row per CTA of 256 threads: with xhat = (x - mean) * rstd and
// g = dY * gamma, dX = rstd * (g - mean(g) - xhat * mean(g * xhat)) (+ dR).
// Two passes over the row: the first forms both row sums (one block
// reduction), the second re-reads X and dY (from L2) and writes dX, so a
// thread holds no row data in registers and several rows run per SM.
constexpr int kLnBwdThreads = 256;

__device__ __forceinline__ float2 block_sum2(float a, float b, float2* red) {
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, s);
    b += __shfl_xor_sync(0xffffffffu, b, s);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = make_float2(a, b);
  __syncthreads();
  float2 t = lane < kLnBwdThreads / 32 ? red[lane] : make_float2(0.0f, 0.0f);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) {
    t.x += __shfl_xor_sync(0xffffffffu, t.x, s);
    t.y += __shfl_xor_sync(0xffffffffu, t.y, s);
  }
  return t;
}

// Forward, one row per CTA of 256 threads, two passes over the row: the
// first forms the sums of (x - K) and (x - K)^2 with K = the row's first
// element (the shifted-data form of the variance: with K a sample of the row
// the two sums do not cancel), one block reduction for both; the second pass
// re-reads the row (from L2) and writes Y.  Each pass issues all of a
// thread's 16-byte loads (at most 8 at h = 16384) before using them, so a
// CTA keeps its whole row in flight; no row data stays in registers across
// the reduction, so several rows run per SM.
constexpr int kLnMaxChunks = kLnMaxH / 8 / kLnBwdThreads;  // 8

template <bool F32>
__global__ void __launch_bounds__(kLnBwdThreads)
    layernorm_fwd_kernel(const void* X, const void* gamma, const void* beta, void* Y, float* mean,
                         float* rstd, int h, float eps) {
  __shared__ float2 red[kLnBwdThreads / 32];
  const long long row = blockIdx.x;
  const long long base = row * h;
  const int nch = h / 8;
  const float K = F32 ? static_cast<const float*>(X)[base]
                      : __bfloat162float(static_cast<const __nv_bfloat16*>(X)[base]);
  float s1 = 0.0f, s2 = 0.0f;
  {
    // the raw 16-byte words (bf16: one per chunk, 32 registers at most)
    constexpr int kWords = F32 ? 2 : 1;
    uint4 raw[kLnMaxChunks * kWords];
#pragma unroll
    for (int k = 0; k < kLnMaxChunks; ++k) {
      const int ch = threadIdx.x + k * kLnBwdThreads;
      if (ch < nch) {
        const uint4* p =
            F32 ? reinterpret_cast<const uint4*>(static_cast<const float*>(X) + base + ch * 8)
                : reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(X) + base +
                                                 ch * 8);
#pragma unroll
        for (int w = 0; w < kWords; ++w) raw[k * kWords + w] = p[w];
      }
    }
#pragma unroll
    for (int k = 0; k < kLnMaxChunks; ++k) {
      if (threadIdx.x + k * kLnBwdThreads < nch) {
        float x[8];
        if (F32) {
          const float* f = reinterpret_cast<const float*>(&raw[k * kWords]);
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = f[i];
        } else {
          const __nv_bfloat162* q = reinterpret_cast<const __nv_bfloat162*>(&raw[k * kWords]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 t = __bfloat1622float2(q[i]);
            x[2 * i] = t.x;
            x[2 * i + 1] = t.y;
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float d = x[i] - K;
          s1 += d;
          s2 += d * d;
        }
      }
    }
  }
  const float2 m = block_sum2(s1, s2, red);
  const float d1 = m.x / h;
  const float mu = K + d1;
  const float rs = rsqrtf(fmaxf(m.y / h - d1 * d1, 0.0f) + eps);
#pragma unroll 4
  for (int ch = threadIdx.x; ch < nch; ch += kLnBwdThreads) {
    float x[8], g[8], b[8], y[8];
    load8<F32>(X, base + ch * 8, x);
    if (gamma != nullptr) load8<F32>(gamma, ch * 8, g);
    if (beta != nullptr) load8<F32>(beta, ch * 8, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      y[i] = (x[i] - mu) * rs;
      if (gamma != nullptr) y[i] *= g[i];
      if (beta != nullptr) y[i] += b[i];
    }
    store8<F32>(Y, base + ch * 8, y);
  }
  if (threadIdx.x == 0) {
    if (mean != nullptr) mean[row] = mu;
    if (rstd != nullptr) rstd[row] = rs;
  }
}

template <bool F32>
__global__ void __launch_bounds__(kLnBwdThreads)
    layernorm_bwd_dx_kernel(const void* X, const void* gamma, const float* mean,
                            const float* rstd, const void* dY, const void* dR, void* dX, int h) {
  __shared__ float2 red[kLnBwdThreads / 32];
  const long long row = blockIdx.x;
  const long long base = row * h;
  const int nch = h / 8;
  const float mu = mean[row], rs = rstd[row];
  float s1 = 0.0f, s2 = 0.0f;
#pragma unroll 2
  for (int ch = threadIdx.x; ch < nch; ch += kLnBwdThreads) {
    float x[8], dy[8], gm[8];
    load8<F32>(X, base + ch * 8, x);
    load8<F32>(dY, base + ch * 8, dy);
    if (gamma != nullptr) load8<F32>(gamma, ch * 8, gm);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float g = gamma != nullptr ? dy[i] * gm[i] : dy[i];
      s1 += g;
      s2 += g * ((x[i] - mu) * rs);
    }
  }
  const float2 m = block_sum2(s1, s2, red);
  const float m1 = m.x / h, m2 = m.y / h;
#pragma unroll 2
  for (int ch = threadIdx.x; ch < nch; ch += kLnBwdThreads) {
    float x[8], dy[8], gm[8], dr[8], dx[8];
    load8<F32>(X, base + ch * 8, x);
    load8<F32>(dY, base + ch * 8, dy);
    if (gamma != nullptr) load8<F32>(gamma, ch * 8, gm);
    if (dR != nullptr) load8<F32>(dR, base + ch * 8, dr);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float g = gamma != nullptr ? dy[i] * gm[i] : dy[i];
      dx[i] = rs * (g - m1 - ((x[i] - mu) * rs) * m2);
      if (dR != nullptr) dx[i] += dr[i];
    }
    store8<F32>(dX, base + ch * 8, dx);
  }
}

// dgamma / dbeta partial column sums: CTA (column block, row chunk), each
// thread 8 columns summed over the chunk's rows in row order; the chunk
// totals are summed in chunk order by column_total_kernel (deterministic).
constexpr int kLnColThreads = 128;
constexpr int kLnRowsPerChunk = 32;

template <bool F32>
__global__ void __launch_bounds__(kLnColThreads)
    layernorm_bwd_cols_kernel(const void* X, const float* mean, const float* rstd,
                              const void* dY, float* part_g, float* part_b, int M, int h) {
  const int c8 = blockIdx.x * kLnColThreads + threadIdx.x;  // chunk of 8 columns
  if (c8 * 8 >= h) return;
  const int r0 = blockIdx.y * kLnRowsPerChunk;
  const int r1 = min(r0 + kLnRowsPerChunk, M);
  float ag[8], ab[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) ag[i] = ab[i] = 0.0f;
#pragma unroll 4
  for (int r = r0; r < r1; ++r) {
    float x[8], dy[8];
    const long long off = static_cast<long long>(r) * h + c8 * 8;
    load8<F32>(X, off, x);
    load8<F32>(dY, off, dy);
    const float mu = mean[r], rs = rstd[r];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      ag[i] += dy[i] * ((x[i] - mu) * rs);
      ab[i] += dy[i];
    }
  }
  const long long o = static_cast<long long>(blockIdx.y) * h + c8 * 8;
  if (part_g != nullptr) {
    reinterpret_cast<float4*>(part_g + o)[0] = make_float4(ag[0], ag[1], ag[2], ag[3]);
    reinterpret_cast<float4*>(part_g + o)[1] = make_float4(ag[4], ag[5], ag[6], ag[7]);
  }
  if (part_b != nullptr) {
    reinterpret_cast<float4*>(part_b + o)[0] = make_float4(ab[0], ab[1], ab[2], ab[3]);
    reinterpret_cast<float4*>(part_b + o)[1] = make_float4(ab[4], ab[5], ab[6], ab[7]);
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

int ln_parts(int64_t M) { return static_cast<int>((M + kLnRowsPerChunk - 1) / kLnRowsPerChunk); }

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
    layernorm_fwd_kernel<true><<<static_cast<unsigned>(M), kLnBwdThreads, 0, stream>>>(
        X, gamma, beta, Y, mean, rstd, static_cast<int>(h), eps);
  else
    layernorm_fwd_kernel<false><<<static_cast<unsigned>(M), kLnBwdThreads, 0, stream>>>(
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
  if (M > 0x7fffffffLL) return fail(TP_ERR_SHAPE, "layernorm: too many rows");
  const int parts = ln_parts(M);
  const bool cols = dgamma != nullptr || dbeta != nullptr;
  float* part_g = dgamma != nullptr ? static_cast<float*>(scratch) : nullptr;
  float* part_b = dbeta != nullptr ? static_cast<float*>(scratch) + static_cast<size_t>(parts) * h
                                   : nullptr;
  const double es = f32 ? 4.0 : 2.0;
  const double bytes = es * double(M) * h * (dR != nullptr ? 4.0 : 3.0) +
                       (cols ? es * 2.0 * double(M) * h + 8.0 * parts * h : 0.0);
  LaunchScope scope(TP_KIND_REDUCE, 0.0, bytes, stream, cols ? 2 + (dgamma != nullptr) +
                                                                   (dbeta != nullptr) : 1);
  const int ih = static_cast<int>(h), im = static_cast<int>(M);
  if (f32)
    layernorm_bwd_dx_kernel<true><<<static_cast<unsigned>(M), kLnBwdThreads, 0, stream>>>(
        X, gamma, mean, rstd, dY, dR, dX, ih);
  else
    layernorm_bwd_dx_kernel<false><<<static_cast<unsigned>(M), kLnBwdThreads, 0, stream>>>(
        X, gamma, mean, rstd, dY, dR, dX, ih);
  if (cols) {
    dim3 grid(static_cast<unsigned>((h / 8 + kLnColThreads - 1) / kLnColThreads),
              static_cast<unsigned>(parts));
    if (f32)
      layernorm_bwd_cols_kernel<true><<<grid, kLnColThreads, 0, stream>>>(
          X, mean, rstd, dY, part_g, part_b, im, ih);
    else
      layernorm_bwd_cols_kernel<false><<<grid, kLnColThreads, 0, stream>>>(
          X, mean, rstd, dY, part_g, part_b, im, ih);
    const unsigned cg = static_cast<unsigned>((h + 255) / 256);
    if (dgamma != nullptr) {
      if (f32)
        column_total_kernel<true><<<cg, 256, 0, stream>>>(part_g, parts, ih, dgamma);
      else
        column_total_kernel<false><<<cg, 256, 0, stream>>>(part_g, parts, ih, dgamma);
    }
    if (dbeta != nullptr) {
      if (f32)
        column_total_kernel<true><<<cg, 256, 0, stream>>>(part_b, parts, ih, dbeta);
      else
        column_total_kernel<false><<<cg, 256, 0, stream>>>(part_b, parts, ih, dbeta);
    }
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "layernorm_bwd launch");
  return TP_OK;
}

}  // namespace tp
