// Vocabulary-parallel embedding and cross-entropy helpers
// ("图解Transformer并行计算：从矩阵乘法切分到Megatron架构设计" §4.1, §4.2).
//
// The logits GEMM and its per-chunk reductions run in the tcgen05 GEMM
// (kEpiCE epilogue); the kernels here are the HBM-bound remainder:
//   embed_fwd     the masked row lookup of §4.1 (a gather),
//   embed_bwd     its transpose, a deterministic scatter-add into dE,
//   ce_combine    §4.2 steps 2-5: chunk partials -> shard sums -> lse, loss,
//   ce_shard_loss §4.2 step 6: per-shard loss sums, then their total,
//   ce_dlogits    the softmax gradient, (exp(z - lse) - onehot) * dloss.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "tp_internal.h"

namespace tp {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ embedding

// One CTA copies whole rows, 16 bytes per thread and step.  The shard that
// owns id is id / v_shard; its local row is id - shard * v_shard, which is
// row id of the unsplit E.  Ids outside [0, V) belong to no shard: zeros.
__global__ void __launch_bounds__(256) embed_fwd_kernel(const int* __restrict__ ids,
                                                        const uint4* __restrict__ E,
                                                        uint4* __restrict__ Y, int64_t M,
                                                        int64_t V, int64_t v_shard,
                                                        int64_t row_vecs) {
  for (int64_t r = blockIdx.x; r < M; r += gridDim.x) {
    const int64_t id = ids[r];
    const bool owned = id >= 0 && id < V;
    const int64_t shard = owned ? id / v_shard : 0;
    const int64_t local = owned ? id - shard * v_shard : 0;
    const uint4* src = E + (shard * v_shard + local) * row_vecs;
    uint4* dst = Y + r * row_vecs;
#pragma unroll 4
    for (int64_t i = threadIdx.x; i < row_vecs; i += blockDim.x)
      dst[i] = owned ? src[i] : make_uint4(0u, 0u, 0u, 0u);
  }
}

// dE rows [v0, v0 + 8) x one column slice of 256 x 16 bytes per CTA.  The CTA
// scans all ids in rounds of 2048 tokens, compacts the tokens that hit its 8
// rows into a shared list in token order, and adds their dY slices into
// fp32 registers in that order; so every row's sum has a fixed order.
constexpr int kEbRows = 8;
constexpr int kEbThreads = 256;
constexpr int kEbPerThread = 8;
constexpr int kEbRound = kEbThreads * kEbPerThread;

template <bool F32>
__global__ void __launch_bounds__(kEbThreads, 2) embed_bwd_kernel(const int* __restrict__ ids,
                                                               const void* __restrict__ dY,
                                                               const void* dE_in, void* dE,
                                                               int64_t M, int64_t V, int64_t h) {
  constexpr int EPV = F32 ? 4 : 8;  // elements per 16-byte vector
  __shared__ int list[kEbRound];
  __shared__ int counts[kEbPerThread][kEbThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t v0 = static_cast<int64_t>(blockIdx.x) * kEbRows;
  const int64_t c0 = (static_cast<int64_t>(blockIdx.y) * kEbThreads + threadIdx.x) * EPV;
  const bool col_ok = c0 < h;  // h % EPV == 0: a vector is all in or all out
  float acc[kEbRows][EPV];
#pragma unroll
  for (int r = 0; r < kEbRows; ++r)
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[r][e] = 0.0f;

  for (int64_t base = 0; base < M; base += kEbRound) {
    unsigned hits[kEbPerThread];
    int rows[kEbPerThread];
#pragma unroll
    for (int k = 0; k < kEbPerThread; ++k) {
      const int64_t tok = base + k * kEbThreads + threadIdx.x;
      const int64_t id = tok < M ? ids[tok] : -1;
      const bool hit = id >= v0 && id < v0 + kEbRows && id < V;
      rows[k] = static_cast<int>(id - v0);
      hits[k] = __ballot_sync(0xffffffffu, hit);
      if (lane == 0) counts[k][warp] = __popc(hits[k]);
    }
    __syncthreads();
    // Token order is (k, warp, lane): the slot of a hit is the number of
    // hits before it in that order.
    int total = 0;  // hits of the steps before k
#pragma unroll
    for (int k = 0; k < kEbPerThread; ++k) {
      int before = 0, in_k = 0;
#pragma unroll
      for (int w = 0; w < kEbThreads / 32; ++w) {
        const int c = counts[k][w];
        before += w < warp ? c : 0;
        in_k += c;
      }
      if ((hits[k] >> lane) & 1u) {
        const int slot = total + before + __popc(hits[k] & ((1u << lane) - 1u));
        list[slot] = ((k * kEbThreads + static_cast<int>(threadIdx.x)) << 3) | rows[k];
      }
      total += in_k;
    }
    __syncthreads();
    if (col_ok) {
#pragma unroll 4
      for (int e = 0; e < total; ++e) {
        const int packed = list[e];
        const int64_t tok = base + (packed >> 3);
        const int rr = packed & 7;
        float x[EPV];
        if (F32) {
          const float4 q = *reinterpret_cast<const float4*>(static_cast<const float*>(dY) +
                                                            tok * h + c0);
          x[0] = q.x; x[1] = q.y; x[2] = q.z; x[3] = q.w;
        } else {
          const uint4 q = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(dY) +
                                                          tok * h + c0);
          const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
          for (int i = 0; i < EPV / 2; ++i) {
            const float2 f = __bfloat1622float2(p[i]);
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
          }
        }
#pragma unroll
        for (int r = 0; r < kEbRows; ++r)
          if (r == rr)
#pragma unroll
            for (int i = 0; i < EPV; ++i) acc[r][i] += x[i];
      }
    }
    __syncthreads();  // the list and counts are rewritten by the next round
  }
  if (!col_ok) return;
#pragma unroll
  for (int r = 0; r < kEbRows; ++r) {
    const int64_t v = v0 + r;
    if (v >= V) break;
    if (F32) {
      float* o = static_cast<float*>(dE) + v * h + c0;
      float4 q = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
      if (dE_in != nullptr) {
        const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(dE_in) +
                                                          v * h + c0);
        q.x += b.x; q.y += b.y; q.z += b.z; q.w += b.w;
      }
      *reinterpret_cast<float4*>(o) = q;
    } else {
      float y[EPV];
#pragma unroll
      for (int i = 0; i < EPV; ++i) y[i] = acc[r][i];
      if (dE_in != nullptr) {
        const uint4 q = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(dE_in) +
                                                        v * h + c0);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int i = 0; i < EPV / 2; ++i) {
          const float2 f = __bfloat1622float2(p[i]);
          y[2 * i] += f.x;
          y[2 * i + 1] += f.y;
        }
      }
      uint4 out;
      uint32_t* w = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
      for (int i = 0; i < EPV / 2; ++i) {
        __nv_bfloat162 t2 = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&t2);
      }
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dE) + v * h + c0) = out;
    }
  }
}

// -------------------------------------------------------------- cross-entropy

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;  // exact: every lane holds the same maximum
}

// Fixed-shape tree; lane 0's total is broadcast so every lane uses one value.
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  return __shfl_sync(0xffffffffu, v, 0);
}

// One warp per row.  Step 2: the chunks of shard i are combined into the
// shard's (max m_i, sum s_i of exp(z - m_i)).  Step 3: the shards are
// combined in shard order, each rescaled to the running maximum, into
// lse = m + log(S).  Steps 4-5: loss = lse - z[target] (0 if ignored).
__global__ void __launch_bounds__(256) ce_combine_kernel(const float2* __restrict__ part,
                                                         int64_t ldp, int cps, int t,
                                                         const int* __restrict__ target,
                                                         const float* __restrict__ tlogit,
                                                         int64_t M, int64_t V, float* lse,
                                                         float* loss) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= M) return;  // warp-uniform
  const float2* p = part + row * ldp;
  float gm = -INFINITY, gs = 0.0f;
  for (int sh = 0; sh < t; ++sh) {
    const float2* q = p + static_cast<int64_t>(sh) * cps;
    float m = -INFINITY;
    for (int j = lane; j < cps; j += 32) m = fmaxf(m, q[j].x);
    m = warp_max(m);
    float s = 0.0f;
    for (int j = lane; j < cps; j += 32) {
      const float2 c = q[j];
      s += c.y * exp2f((c.x - m) * kLog2e);
    }
    s = warp_sum(s);
    const float nm = fmaxf(gm, m);
    gs = gs * exp2f((gm - nm) * kLog2e) + s * exp2f((m - nm) * kLog2e);
    gm = nm;
  }
  if (lane == 0) {
    const float l = gm + logf(gs);
    lse[row] = l;
    const int tg = target[row];
    loss[row] = (tg >= 0 && tg < V) ? l - tlogit[row] : 0.0f;
  }
}

// Step 5-6: block i sums the losses of the rows whose target shard i owns
// (fixed per-thread order, then a fixed tree).
__global__ void __launch_bounds__(1024) ce_shard_loss_kernel(const float* __restrict__ loss,
                                                             const int* __restrict__ target,
                                                             int64_t M, int64_t v_shard,
                                                             float* shard_tot) {
  __shared__ float red[32];
  const int64_t lo = static_cast<int64_t>(blockIdx.x) * v_shard, hi = lo + v_shard;
  float s = 0.0f;
  for (int64_t r = threadIdx.x; r < M; r += blockDim.x) {
    const int64_t tg = target[r];
    if (tg >= lo && tg < hi) s += loss[r];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) shard_tot[blockIdx.x] = v;
  }
}

// Step 6: the AllReduce of the t local losses, in shard order.
__global__ void ce_total_kernel(const float* __restrict__ shard_tot, int t, float* total) {
  if (threadIdx.x != 0) return;
  float s = 0.0f;
  for (int i = 0; i < t; ++i) s += shard_tot[i];
  *total = s;
}

// dlogits = (exp(z - lse) - [col == target]) * dloss over [M, V] bf16, 8
// columns per thread; rows with an ignored target get zeros.
__global__ void __launch_bounds__(256) ce_dlogits_kernel(const __nv_bfloat16* logits,
                                                         const float* __restrict__ lse,
                                                         const int* __restrict__ target,
                                                         const float* __restrict__ dloss,
                                                         __nv_bfloat16* dlogits, int64_t M,
                                                         int64_t V) {
  const int64_t nvec = V / 8;
  for (int64_t row = blockIdx.y; row < M; row += gridDim.y) {
    const int64_t tg = target[row];
    const bool ok = tg >= 0 && tg < V;
    const float dl = ok ? (dloss != nullptr ? dloss[row] : 1.0f) : 0.0f;
    const float l2 = lse[row] * kLog2e;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const uint4 q = *reinterpret_cast<const uint4*>(logits + row * V + 8 * i);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
      uint4 out;
      uint32_t* w = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 z = __bfloat1622float2(p[k]);
        const int64_t c = 8 * i + 2 * k;
        const float g0 = (exp2f(fmaf(z.x, kLog2e, -l2)) - (c == tg ? 1.0f : 0.0f)) * dl;
        const float g1 = (exp2f(fmaf(z.y, kLog2e, -l2)) - (c + 1 == tg ? 1.0f : 0.0f)) * dl;
        __nv_bfloat162 t2 = __floats2bfloat162_rn(g0, g1);
        w[k] = *reinterpret_cast<uint32_t*>(&t2);
      }
      *reinterpret_cast<uint4*>(dlogits + row * V + 8 * i) = out;
    }
  }
}

}  // namespace

tp_status launch_embed_fwd(const int* ids, const void* E, void* Y, int64_t M, int64_t V,
                           int64_t h, int t, bool f32, cudaStream_t stream) {
  if (M <= 0) return TP_OK;
  const int64_t row_vecs = h * (f32 ? 4 : 2) / 16;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  const int grid = static_cast<int>(M < cap ? M : cap);
  {
    LaunchScope scope(TP_KIND_VOCAB, 0.0, 2.0 * M * h * (f32 ? 4 : 2) + 4.0 * M, stream, 1,
                      kVocabEmbedFwd);
    embed_fwd_kernel<<<grid, 256, 0, stream>>>(ids, static_cast<const uint4*>(E),
                                               static_cast<uint4*>(Y), M, V, V / t, row_vecs);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "embed_fwd launch");
}

tp_status launch_embed_bwd(const int* ids, const void* dY, const void* dE_in, void* dE,
                           int64_t M, int64_t V, int64_t h, bool f32, cudaStream_t stream) {
  const int epv = f32 ? 4 : 8;
  const int64_t gx = (V + kEbRows - 1) / kEbRows;
  const int64_t gy = (h + int64_t(kEbThreads) * epv - 1) / (int64_t(kEbThreads) * epv);
  if (gx > 0x7fffffffLL || gy > 65535) return fail(TP_ERR_SHAPE, "embedding backward: V or h too large");
  const double es = f32 ? 4.0 : 2.0;
  const double bytes = es * (double(V) * h * (dE_in ? 2.0 : 1.0) + double(M) * h) + 4.0 * M;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  {
    LaunchScope scope(TP_KIND_VOCAB, double(M) * h, bytes, stream, 1, kVocabEmbedBwd);
    if (f32)
      embed_bwd_kernel<true><<<grid, kEbThreads, 0, stream>>>(ids, dY, dE_in, dE, M, V, h);
    else
      embed_bwd_kernel<false><<<grid, kEbThreads, 0, stream>>>(ids, dY, dE_in, dE, M, V, h);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "embed_bwd launch");
}

tp_status launch_ce_finish(const CEOut& ce, int t, int64_t M, int64_t V, float* lse, float* loss,
                           float* total, float* shard_tot, cudaStream_t stream) {
  if (M <= 0) return TP_OK;
  const int64_t blocks = (M + 7) / 8;
  {
    LaunchScope scope(TP_KIND_VOCAB, 0.0, 8.0 * M * ce.ldp + 20.0 * M, stream,
                      total != nullptr ? 3 : 1, kVocabLossCombine);
    ce_combine_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        reinterpret_cast<const float2*>(ce.part), ce.ldp, ce.cps, t, ce.target, ce.tlogit, M, V,
        lse, loss);
    if (total != nullptr) {
      ce_shard_loss_kernel<<<t, 1024, 0, stream>>>(loss, ce.target, M, V / t, shard_tot);
      ce_total_kernel<<<1, 32, 0, stream>>>(shard_tot, t, total);
    }
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "cross-entropy combine launch");
}

tp_status launch_ce_dlogits(const void* logits, const float* lse, const int* target,
                            const float* dloss, void* dlogits, int64_t M, int64_t V,
                            cudaStream_t stream) {
  if (M <= 0) return TP_OK;
  const int64_t nvec = V / 8;
  const int64_t gx64 = (nvec + 255) / 256;
  const unsigned gx = static_cast<unsigned>(gx64 < 1024 ? gx64 : 1024);
  const unsigned gy = static_cast<unsigned>(M < 65535 ? M : 65535);
  {
    LaunchScope scope(TP_KIND_VOCAB, 0.0, 4.0 * M * V + 12.0 * M, stream, 1, kVocabSoftmaxGrad);
    ce_dlogits_kernel<<<dim3(gx, gy), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(logits), lse, target, dloss,
        static_cast<__nv_bfloat16*>(dlogits), M, V);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "cross-entropy gradient launch");
}

}  // namespace tp
