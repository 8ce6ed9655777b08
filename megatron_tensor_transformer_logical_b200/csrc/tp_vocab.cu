// Vocabulary-parallel embedding and cross-entropy helpers
// ("图解Transformer并行计算：从矩阵乘法切分到Megatron架构设计" §4.1, §4.2).
//
// The logits GEMM and its per-chunk reductions run in the tcgen05 GEMM
// (kEpiCE epilogue); the kernels here are the HBM-bound remainder:
//   embed_fwd     the masked row lookup of §4.1 (a gather),
//   embed_bwd     its transpose: dE = dE_in or 0, then a deterministic
//                 scatter-add of dY into the rows that tokens hit (tokens
//                 sorted by id, one CTA per run of equal ids; or, for more
//                 than 16384 tokens, a scan of the ids per 8-row group),
//   ce_combine    §4.2 steps 2-5: chunk partials -> shard sums -> lse, loss,
//   ce_shard_loss §4.2 step 6: per-shard loss sums, then their total,
//   ce_dlogits    the softmax gradient, (exp(z - lse) - onehot) * dloss.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx_sm100.cuh"
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

// The embedding backward in two kernels.  embed_bwd_init writes every row of
// dE once: dE = dE_in, or zeros (skipped when dE_in is dE itself, the
// accumulate-in-place case).  embed_bwd_scatter then adds the dY rows into
// the rows that tokens hit, and touches no other row.
__global__ void __launch_bounds__(256) embed_bwd_init_kernel(const uint4* __restrict__ src,
                                                             uint4* __restrict__ dst,
                                                             int64_t n_vec) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_vec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = src != nullptr ? src[i] : make_uint4(0u, 0u, 0u, 0u);
}

// One CTA per group of 8 rows of dE.  It scans the ids in rounds of 2048
// tokens, compacts the tokens that hit its rows into a shared list in token
// order (ballots + per-warp counts), and for each 256 x 16-byte column slice
// adds their dY slices into fp32 registers in that order, then adds the sums
// to the hit rows of dE (read-modify-write).  The order of every row's sum is
// fixed, so the result is deterministic without atomics.  A group no token
// hits exits after one scan.
constexpr int kEbRows = 8;
constexpr int kEbThreads = 256;
constexpr int kEbPerThread = 8;
constexpr int kEbRound = kEbThreads * kEbPerThread;

struct EbList {
  int entries[kEbRound];
  int counts[kEbPerThread][kEbThreads / 32];
  int total;
  int rowmask;
};

// Builds the list of hits among tokens [base, base + 2048); returns its length.
__device__ __forceinline__ int eb_build_list(const int* __restrict__ ids, int64_t base, int64_t M,
                                             int64_t v0, int64_t V, EbList& L) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned hits[kEbPerThread];
  int rows[kEbPerThread];
  int mask = 0;
#pragma unroll
  for (int k = 0; k < kEbPerThread; ++k) {
    const int64_t tok = base + k * kEbThreads + threadIdx.x;
    const int64_t id = tok < M ? ids[tok] : -1;
    const bool hit = id >= v0 && id < v0 + kEbRows && id < V;
    rows[k] = static_cast<int>(id - v0);
    if (hit) mask |= 1 << rows[k];
    hits[k] = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) L.counts[k][warp] = __popc(hits[k]);
  }
  if (mask) atomicOr(&L.rowmask, mask);
  __syncthreads();
  // Token order is (k, warp, lane): a hit's slot is the number of hits before it.
  int total = 0;
#pragma unroll
  for (int k = 0; k < kEbPerThread; ++k) {
    int before = 0, in_k = 0;
#pragma unroll
    for (int w = 0; w < kEbThreads / 32; ++w) {
      const int c = L.counts[k][w];
      before += w < warp ? c : 0;
      in_k += c;
    }
    if ((hits[k] >> lane) & 1u) {
      const int slot = total + before + __popc(hits[k] & ((1u << lane) - 1u));
      L.entries[slot] = ((k * kEbThreads + static_cast<int>(threadIdx.x)) << 3) | rows[k];
    }
    total += in_k;
  }
  __syncthreads();
  return total;
}

template <bool F32>
__device__ __forceinline__ void eb_accumulate(const EbList& L, int n, int64_t base,
                                              const void* __restrict__ dY, int64_t h, int64_t c0,
                                              float (&acc)[kEbRows][F32 ? 4 : 8]) {
  constexpr int EPV = F32 ? 4 : 8;
#pragma unroll 2
  for (int e = 0; e < n; ++e) {
    const int packed = L.entries[e];
    const int64_t tok = base + (packed >> 3);
    const int rr = packed & 7;
    float x[EPV];
    if (F32) {
      const float4 q = *reinterpret_cast<const float4*>(static_cast<const float*>(dY) + tok * h +
                                                        c0);
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

template <bool F32>
__device__ __forceinline__ void eb_add_rows(void* dE, int64_t v0, int64_t h, int64_t c0,
                                            int rowmask, const float (&acc)[kEbRows][F32 ? 4 : 8]) {
  constexpr int EPV = F32 ? 4 : 8;
#pragma unroll
  for (int r = 0; r < kEbRows; ++r) {
    if (!((rowmask >> r) & 1)) continue;
    if (F32) {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(dE) + (v0 + r) * h + c0);
      float4 q = *o;
      q.x += acc[r][0]; q.y += acc[r][1]; q.z += acc[r][2]; q.w += acc[r][3];
      *o = q;
    } else {
      uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dE) + (v0 + r) * h + c0);
      const uint4 q = *o;
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
      uint4 out;
      uint32_t* w = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
      for (int i = 0; i < EPV / 2; ++i) {
        const float2 f = __bfloat1622float2(p[i]);
        __nv_bfloat162 t2 = __floats2bfloat162_rn(f.x + acc[r][2 * i], f.y + acc[r][2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&t2);
      }
      *o = out;
    }
  }
}

template <bool F32>
__global__ void __launch_bounds__(kEbThreads, 1) embed_bwd_scatter_kernel(
    const int* __restrict__ ids, const void* __restrict__ dY, void* dE, int64_t M, int64_t V,
    int64_t h) {
  constexpr int EPV = F32 ? 4 : 8;
  constexpr int64_t kSlice = int64_t(kEbThreads) * EPV;
  __shared__ EbList L;
  const int64_t v0 = static_cast<int64_t>(blockIdx.x) * kEbRows;
  if (threadIdx.x == 0) L.rowmask = 0;
  __syncthreads();
  float acc[kEbRows][EPV];
  if (M <= kEbRound) {
    // One round: the list is built once and serves every column slice.
    const int n = eb_build_list(ids, 0, M, v0, V, L);
    if (n == 0) return;
    const int rowmask = L.rowmask;
    for (int64_t c0 = threadIdx.x * EPV; c0 < h; c0 += kSlice) {
#pragma unroll
      for (int r = 0; r < kEbRows; ++r)
#pragma unroll
        for (int i = 0; i < EPV; ++i) acc[r][i] = 0.0f;
      eb_accumulate<F32>(L, n, 0, dY, h, c0, acc);
      eb_add_rows<F32>(dE, v0, h, c0, rowmask, acc);
    }
    return;
  }
  // Several rounds: the lists are rebuilt for every column slice.
  for (int64_t s0 = 0; s0 < h; s0 += kSlice) {
    const int64_t c0 = s0 + threadIdx.x * EPV;
    const bool col_ok = c0 < h;
#pragma unroll
    for (int r = 0; r < kEbRows; ++r)
#pragma unroll
      for (int i = 0; i < EPV; ++i) acc[r][i] = 0.0f;
    for (int64_t base = 0; base < M; base += kEbRound) {
      const int n = eb_build_list(ids, base, M, v0, V, L);
      if (col_ok) eb_accumulate<F32>(L, n, base, dY, h, c0, acc);
      __syncthreads();  // the list is rewritten by the next round
    }
    if (col_ok) eb_add_rows<F32>(dE, v0, h, c0, L.rowmask, acc);
  }
}

// Sorted form (M <= kSortMax tokens).  embed_sort_kernel, one CTA, sorts the
// (id, token) pairs by id with a bitonic network in shared memory (keys are
// unique, so equal ids keep token order), then lists the runs of equal valid
// ids: run r covers sorted positions [run_start[r], run_start[r + 1]) and
// has id run_id[r]; ids outside [0, V) sort to the end and form no run.
constexpr int kSortMax = 16384;
constexpr int kSortThreads = 1024;

__global__ void __launch_bounds__(kSortThreads) embed_sort_kernel(
    const int* __restrict__ ids, int M, int n_pow2, int64_t V, int* sorted_tok, int* run_start,
    int* run_id, int* n_runs) {
  extern __shared__ unsigned long long keys[];
  __shared__ int warp_sums[kSortThreads / 32];
  for (int i = threadIdx.x; i < n_pow2; i += blockDim.x)
    keys[i] = i < M ? (static_cast<unsigned long long>(static_cast<unsigned>(ids[i])) << 32) |
                          static_cast<unsigned>(i)
                    : ~0ull;
  __syncthreads();
  for (int k = 2; k <= n_pow2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n_pow2; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = keys[i], b = keys[ixj];
          const bool up = (i & k) == 0;
          if ((a > b) == up) {
            keys[i] = b;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // Runs: thread t owns the contiguous positions [t*per, (t+1)*per).
  const int per = (M + kSortThreads - 1) / kSortThreads;
  const int p0 = threadIdx.x * per, p1 = min(p0 + per, M);
  int count = 0;
  for (int p = p0; p < p1; ++p) {
    const unsigned long long id = keys[p] >> 32;
    sorted_tok[p] = static_cast<int>(keys[p] & 0xffffffffu);
    if (id < static_cast<unsigned long long>(V) && (p == 0 || (keys[p - 1] >> 32) != id)) ++count;
  }
  // Block-wide exclusive scan of the run counts (warp scans, then warp totals).
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = count;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += v;
    }
    warp_sums[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int r = incl - count + (warp > 0 ? warp_sums[warp - 1] : 0);
  for (int p = p0; p < p1; ++p) {
    const unsigned long long id = keys[p] >> 32;
    if (id < static_cast<unsigned long long>(V) && (p == 0 || (keys[p - 1] >> 32) != id)) {
      run_start[r] = p;
      run_id[r] = static_cast<int>(id);
      ++r;
    }
  }
  if (threadIdx.x == kSortThreads - 1) {
    const int total = warp_sums[kSortThreads / 32 - 1];
    *n_runs = total;
    // End of the last valid run: the first position whose id is not valid.
    int end = M;
    for (int p = M - 1; p >= 0 && (keys[p] >> 32) >= static_cast<unsigned long long>(V); --p)
      end = p;
    run_start[total] = end;
  }
}

// One CTA per (run, 2048-column slice): sums the run's dY rows in token
// order in fp32 (eight loads in flight per thread) and adds the sum to its
// row of dE.
template <bool F32>
__global__ void __launch_bounds__(256) embed_run_scatter_kernel(
    const int* __restrict__ sorted_tok, const int* __restrict__ run_start,
    const int* __restrict__ run_id, const int* __restrict__ n_runs, const void* __restrict__ dY,
    void* dE, int64_t h) {
  constexpr int EPV = F32 ? 4 : 8;
  const int64_t c0 = (static_cast<int64_t>(blockIdx.y) * blockDim.x + threadIdx.x) * EPV;
  if (c0 >= h) return;
  const int nr = *n_runs;
  for (int r = blockIdx.x; r < nr; r += gridDim.x) {
    const int e0 = run_start[r], e1 = run_start[r + 1];
    float acc[EPV];
#pragma unroll
    for (int i = 0; i < EPV; ++i) acc[i] = 0.0f;
    // Batches of eight rows: the eight loads are issued before any is added,
    // so a long run (a frequent token) costs one round trip per batch.
    for (int e = e0; e < e1; e += 8) {
      uint4 q[8];
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        if (e + b < e1) {
          const int64_t tok = sorted_tok[e + b];
          q[b] = F32 ? *reinterpret_cast<const uint4*>(static_cast<const float*>(dY) + tok * h + c0)
                     : *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(dY) +
                                                       tok * h + c0);
        } else {
          q[b] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        if (e + b >= e1) break;  // adds stay in token order; zeros are never added
        if (F32) {
          const float* f = reinterpret_cast<const float*>(&q[b]);
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i] += f[i];
        } else {
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&q[b]);
#pragma unroll
          for (int i = 0; i < EPV / 2; ++i) {
            const float2 f = __bfloat1622float2(p2[i]);
            acc[2 * i] += f.x;
            acc[2 * i + 1] += f.y;
          }
        }
      }
    }
    const int64_t v = run_id[r];
    if (F32) {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(dE) + v * h + c0);
      float4 q = *o;
      q.x += acc[0]; q.y += acc[1]; q.z += acc[2]; q.w += acc[3];
      *o = q;
    } else {
      uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dE) + v * h + c0);
      const uint4 q = *o;
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
      uint4 out;
      uint32_t* w = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
      for (int i = 0; i < EPV / 2; ++i) {
        const float2 f = __bfloat1622float2(p[i]);
        __nv_bfloat162 t2 = __floats2bfloat162_rn(f.x + acc[2 * i], f.y + acc[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&t2);
      }
      *o = out;
    }
  }
}

// -------------------------------------------------------------- cross-entropy

// Folds the pair (m2, s2) into the running pair (m, s), both meaning
// s * exp(m) = the sum of exp(z) over what was folded in so far.  Commutative
// bit for bit (one max, two products, one sum), so an xor-shuffle tree leaves
// every lane with the same pair.
__device__ __forceinline__ void ms_fold(float& m, float& s, float m2, float s2) {
  const float nm = fmaxf(m, m2);
  if (nm == -INFINITY) return;  // both empty
  s = s * exp2f((m - nm) * kLog2e) + s2 * exp2f((m2 - nm) * kLog2e);
  m = nm;
}

constexpr int kCombineThreads = 256;
constexpr int kCombineBatch = 4;

// One block per row.  Steps 2-3: the row's chunk pairs (max m_c, sum of
// exp(z - m_c)) over all shards are folded into one (max, sum) -- each thread
// a fixed strided share, then a fixed xor tree in the warp and across the
// block's warps -- and lse = m + log(S); the grouping of a log-sum-exp's terms
// changes it only by rounding.  Steps 4-5: loss = lse - z[target] (0 if the
// target is ignored).
__global__ void __launch_bounds__(kCombineThreads) ce_combine_kernel(
    const float2* __restrict__ part, int64_t ldp, const int* __restrict__ target,
    const float* __restrict__ tlogit, int64_t V, float* lse, float* loss) {
  __shared__ float2 red[kCombineThreads / 32];
  const int64_t row = blockIdx.x;
  const float2* p = part + row * ldp;
  float m = -INFINITY, s = 0.0f;
  for (int64_t j0 = threadIdx.x; j0 < ldp; j0 += kCombineBatch * kCombineThreads) {
    float2 c[kCombineBatch];
#pragma unroll
    for (int u = 0; u < kCombineBatch; ++u) {
      const int64_t j = j0 + u * kCombineThreads;
      c[u] = j < ldp ? p[j] : make_float2(-INFINITY, 0.0f);
    }
#pragma unroll
    for (int u = 0; u < kCombineBatch; ++u) ms_fold(m, s, c[u].x, c[u].y);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    ms_fold(m, s, m2, s2);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) red[warp] = make_float2(m, s);
  __syncthreads();
  if (warp != 0) return;
  const float2 w = lane < kCombineThreads / 32 ? red[lane] : make_float2(-INFINITY, 0.0f);
  m = w.x;
  s = w.y;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    ms_fold(m, s, m2, s2);
  }
  if (lane == 0) {
    const float l = m + logf(s);
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

// dlogits = (exp(z - lse) - [col == target]) * dloss over [M, V] bf16 in
// 8-column vectors, each thread's four loads issued before its first store
// (dlogits may alias logits: every vector is read before the same thread
// overwrites it); rows with an ignored target get zeros.
constexpr int kGradThreads = 256;
constexpr int kGradBatch = 4;  // 16-byte vectors in flight per thread

__global__ void __launch_bounds__(kGradThreads) ce_dlogits_kernel(
    const __nv_bfloat16* logits, const float* __restrict__ lse, const int* __restrict__ target,
    const float* __restrict__ dloss, __nv_bfloat16* dlogits, int64_t M, int64_t V) {
  const int64_t nvec = V / 8;
  const int64_t span = static_cast<int64_t>(kGradBatch) * kGradThreads;
  for (int64_t row = blockIdx.y; row < M; row += gridDim.y) {
    const int64_t tg = target[row];
    const bool ok = tg >= 0 && tg < V;
    const float dl = ok ? (dloss != nullptr ? dloss[row] : 1.0f) : 0.0f;
    const float l2 = lse[row] * kLog2e;
    const uint4* zr = reinterpret_cast<const uint4*>(logits + row * V);
    uint4* gr = reinterpret_cast<uint4*>(dlogits + row * V);
    for (int64_t i0 = blockIdx.x * span + threadIdx.x; i0 < nvec; i0 += gridDim.x * span) {
      uint4 q[kGradBatch];
#pragma unroll
      for (int u = 0; u < kGradBatch; ++u) {
        const int64_t i = i0 + u * kGradThreads;
        if (i < nvec) q[u] = zr[i];
      }
#pragma unroll
      for (int u = 0; u < kGradBatch; ++u) {
        const int64_t i = i0 + u * kGradThreads;
        if (i >= nvec) break;
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q[u]);
        uint4 out;
        uint32_t* w = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 z = __bfloat1622float2(p[k]);
          const int64_t c = 8 * i + 2 * k;
          const float g0 = (ex2_approx(fmaf(z.x, kLog2e, -l2)) - (c == tg ? 1.0f : 0.0f)) * dl;
          const float g1 =
              (ex2_approx(fmaf(z.y, kLog2e, -l2)) - (c + 1 == tg ? 1.0f : 0.0f)) * dl;
          __nv_bfloat162 t2 = __floats2bfloat162_rn(g0, g1);
          w[k] = *reinterpret_cast<uint32_t*>(&t2);
        }
        gr[i] = out;
      }
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

size_t embed_bwd_scratch_bytes(int64_t M) {
  if (M > kSortMax) return 0;
  return static_cast<size_t>(3 * M + 2) * sizeof(int);
}

tp_status launch_embed_bwd(const int* ids, const void* dY, const void* dE_in, void* dE,
                           int64_t M, int64_t V, int64_t h, bool f32, void* scratch,
                           cudaStream_t stream) {
  const int64_t gx = (V + kEbRows - 1) / kEbRows;
  if (gx > 0x7fffffffLL) return fail(TP_ERR_SHAPE, "embedding backward: V too large");
  const double es = f32 ? 4.0 : 2.0;
  const bool init = dE_in != dE;  // in place: only the hit rows change
  const bool sorted = M > 0 && M <= kSortMax;
  const int64_t hit_rows = M < V ? M : V;
  // Bytes: the init pass (all of dE written, dE_in read) and at most
  // min(M, V) rows read and written by the scatter, plus dY and the ids.
  const double bytes = (init ? es * double(V) * h * (dE_in ? 2.0 : 1.0) : 0.0) +
                       es * (double(M) * h + 2.0 * double(hit_rows) * h) + 4.0 * M;
  const int kernels = (init ? 1 : 0) + (M > 0 ? (sorted ? 2 : 1) : 0);
  const int64_t slices = (h + 256 * (f32 ? 4 : 8) - 1) / (256 * (f32 ? 4 : 8));
  if (sorted) {
    static unsigned long long configured = 0;  // one bit per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (!(configured & (1ull << (dev & 63)))) {
      cudaError_t e = cudaFuncSetAttribute(embed_sort_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kSortMax * 8);
      if (e != cudaSuccess) return cuda_fail(e, "embed_sort smem attribute");
      configured |= 1ull << (dev & 63);
    }
    if (scratch == nullptr) return fail(TP_ERR_WORKSPACE, "embedding backward: workspace missing");
    if (slices > 65535) return fail(TP_ERR_SHAPE, "embedding backward: h too large");
  }
  {
    LaunchScope scope(TP_KIND_VOCAB, double(M) * h, bytes, stream, kernels, kVocabEmbedBwd);
    if (init) {
      const int64_t n_vec = V * h * static_cast<int64_t>(es) / 16;
      const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
      const int64_t blocks = (n_vec + 255) / 256;
      embed_bwd_init_kernel<<<static_cast<unsigned>(blocks < cap ? blocks : cap), 256, 0,
                              stream>>>(static_cast<const uint4*>(dE_in), static_cast<uint4*>(dE),
                                        n_vec);
    }
    if (sorted) {
      int* sorted_tok = static_cast<int*>(scratch);
      int* run_start = sorted_tok + M;
      int* run_id = run_start + M + 1;
      int* n_runs = run_id + M;
      int n_pow2 = 2;
      while (n_pow2 < M) n_pow2 <<= 1;
      embed_sort_kernel<<<1, kSortThreads, static_cast<size_t>(n_pow2) * 8, stream>>>(
          ids, static_cast<int>(M), n_pow2, V, sorted_tok, run_start, run_id, n_runs);
      const int64_t runs_cap = M < 8192 ? M : 8192;
      dim3 grid(static_cast<unsigned>(runs_cap), static_cast<unsigned>(slices));
      if (f32)
        embed_run_scatter_kernel<true><<<grid, 256, 0, stream>>>(sorted_tok, run_start, run_id,
                                                                 n_runs, dY, dE, h);
      else
        embed_run_scatter_kernel<false><<<grid, 256, 0, stream>>>(sorted_tok, run_start, run_id,
                                                                  n_runs, dY, dE, h);
    } else if (M > 0) {
      if (f32)
        embed_bwd_scatter_kernel<true><<<static_cast<unsigned>(gx), kEbThreads, 0, stream>>>(
            ids, dY, dE, M, V, h);
      else
        embed_bwd_scatter_kernel<false><<<static_cast<unsigned>(gx), kEbThreads, 0, stream>>>(
            ids, dY, dE, M, V, h);
    }
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "embed_bwd launch");
}

tp_status launch_ce_finish(const CEOut& ce, int t, int64_t M, int64_t V, float* lse, float* loss,
                           float* total, float* shard_tot, cudaStream_t stream) {
  if (M <= 0) return TP_OK;
  if (M > 0x7fffffffLL) return fail(TP_ERR_SHAPE, "cross-entropy combine: M too large");
  {
    LaunchScope scope(TP_KIND_VOCAB, 0.0, 8.0 * M * ce.ldp + 20.0 * M, stream,
                      total != nullptr ? 3 : 1, kVocabLossCombine);
    ce_combine_kernel<<<static_cast<unsigned>(M), kCombineThreads, 0, stream>>>(
        reinterpret_cast<const float2*>(ce.part), ce.ldp, ce.target, ce.tlogit, V, lse, loss);
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
  const int64_t span = static_cast<int64_t>(kGradBatch) * kGradThreads;
  const int64_t gx64 = (nvec + span - 1) / span;
  const unsigned gx = static_cast<unsigned>(gx64 < 1024 ? gx64 : 1024);
  const unsigned gy = static_cast<unsigned>(M < 65535 ? M : 65535);
  {
    LaunchScope scope(TP_KIND_VOCAB, 0.0, 4.0 * M * V + 12.0 * M, stream, 1, kVocabSoftmaxGrad);
    ce_dlogits_kernel<<<dim3(gx, gy), kGradThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(logits), lse, target, dloss,
        static_cast<__nv_bfloat16*>(dlogits), M, V);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "cross-entropy gradient launch");
}

}  // namespace tp
