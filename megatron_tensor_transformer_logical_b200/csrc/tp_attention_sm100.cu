// Attention core forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Per head ("图解Transformer并行计算" §3.1): O = softmax(Q K^T / sqrt(d)) V with
// the causal mask hiding key c from query r when c > r; each head group of
// §3.2 runs its own heads, so the core runs per (batch, head).
//
// One CTA per (batch element, head, pair of adjacent 128-row query tiles);
// blockIdx.x is the (batch element, head) and blockIdx.y the pair, longest
// rows first, so the CTAs launch in order of decreasing work over all heads.
// The two tiles share each K / V block and take turns on the tensor core: one
// tile's softmax runs while the other tile's products are computed.
//   warp 0      TMA: both Q tiles once, then K_j and V_j (128 keys each) into
//               two-deep rings (fp16, 128-byte swizzle);
//   warp 1      allocates 512 TMEM columns; one thread issues, per key block,
//               P_0 V_j, S_0 = Q_0 K_{j+1}^T, P_1 V_j, S_1 = Q_1 K_{j+1}^T;
//   warps 4-7   softmax of tile 0, warps 8-11 of tile 1: thread i owns query
//               row i = TMEM lane i, so row max and sum need no shuffles;
//               P_j (fp16) is written back into tensor memory over its S
//               columns and is the tensor-memory A operand of P V, which
//               accumulates O in tensor memory.
// O and the row sum are kept relative to a row maximum that is raised only
// when the new maximum exceeds it by more than 2^8 (then O is rescaled in
// tensor memory); P stays below 2^8, and the final O / l uses the same
// maximum, so the result does not depend on when the maximum was raised.
// The maximum of a block after the first is formed only when its row sum of
// P exceeds 255 (which any key more than 2^8 above the maximum in use
// forces), so the common block costs the exponentials and the sum alone.
// Scores are kept in the log2 domain (scaled by log2(e)/sqrt(d)); the saved
// LSE is the natural log of the softmax denominator.  Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cudaTypedefs.h>

#include "ptx_sm100.cuh"
#include "tp_internal.h"

namespace tp {
namespace {

constexpr int kD = 128;           // head dimension
constexpr int kBM = 128;          // query rows per CTA
constexpr int kBN = 128;          // keys per block
constexpr int kTile = 128 * 128 * 2;  // one [128 x 128] fp16 tile: 32 KB
constexpr int kHalf = kTile / 2;      // one 64-column half: 16 KB
constexpr int kThreadsA = 384;
// Q of both tiles, K[2], V[2], barriers.
constexpr int kSmemA = 1024 + 6 * kTile + 256;
// O and the row sum keep the scale of a stale row maximum until the maximum
// has risen by more than 2^8 (log2 units); the final 1/l uses the same
// maximum, so the result is exact either way, and P stays below 2^8.
constexpr float kRescaleLog2 = 8.0f;
// A block's row sum of P above this may hide a key more than 2^8 above the
// maximum in use (that key's P alone is 2^8 up to the rounding of its
// exponent), so the exact block maximum is formed and compared.
constexpr float kCheckSum = 255.0f;
constexpr float kLog2eA = 1.4426950408889634f;
constexpr float kLn2A = 0.69314718055994531f;

struct FwdArgs {
  int s, h, heads, causal;
  float scale_log2;
  __nv_bfloat16* out;  // O [M, h]
  float* lse;          // [b, heads, s]
  WaitCtl status;
};

// kind::f16 instruction descriptor with fp16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int m, int n, bool a_mn, bool b_mn) {
  return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((static_cast<uint32_t>(n) >> 3) << 17) | ((static_cast<uint32_t>(m) >> 4) << 24);
}


__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 t = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// max(m, v[0..31]) by three-input maxima: 16 instructions, depth 4.
__device__ __forceinline__ float max32(const float (&v)[32], float m) {
  float w[12];
#pragma unroll
  for (int k = 0; k < 10; ++k) w[k] = max3f(v[3 * k], v[3 * k + 1], v[3 * k + 2]);
  w[10] = v[30];
  w[11] = v[31];
  float x[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) x[k] = max3f(w[3 * k], w[3 * k + 1], w[3 * k + 2]);
  return max3f(max3f(x[0], x[1], x[2]), x[3], m);
}

// The raw-score maximum over this row's visible keys [0, vis) of one block.
__device__ __forceinline__ float row_max_visible(uint32_t srow, int vis) {
  float mx = -INFINITY;
#pragma unroll
  for (int c = 0; c < kBN; c += 32) {
    float v[32];
    tmem_ld32(srow + c, v);
    if (vis < c + 32) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = (c + i < vis) ? v[i] : -INFINITY;
    }
    mx = max32(v, mx);
  }
  return mx;
}

// P = 2^(s * scale_log2 - m) over one block row (masked keys 0), packed to
// fp16 pairs in registers; returns the row sum of P.  The softmax is bound by
// instruction issue, so the arithmetic is paired where sm_100 allows it: the
// scale-and-shift as two-wide fused multiply-adds, the row sum as two-wide
// adds.  The block's maximum is not formed here: a sum above kCheckSum is
// what sends the caller to the exact maximum (a key 2^8 above m alone makes
// the sum exceed it).
__device__ __forceinline__ float exp_row(uint32_t srow, int vis, float scale_log2, float m,
                                         uint32_t (&pk)[kBN / 2]) {
  const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-m, -m);
  float2 acc = make_float2(0.0f, 0.0f);
  // The next chunk's tensor-memory load is in flight while this one is
  // computed (one wait per chunk, after the computation).
  uint32_t nx[32];
  tmem_ld32_nowait(srow, nx);
  tmem_wait_ld(nx);
#pragma unroll
  for (int c = 0; c < kBN; c += 32) {
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(nx[i]);
    if (c + 32 < kBN) tmem_ld32_nowait(srow + c + 32, nx);
    float2 u[16];
    if (vis >= c + 32) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 t = __ffma2_rn(make_float2(v[2 * i], v[2 * i + 1]), sc2, nm2);
        u[i] = make_float2(ex2_approx(t.x), ex2_approx(t.y));
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 t = __ffma2_rn(make_float2(v[2 * i], v[2 * i + 1]), sc2, nm2);
        u[i] = make_float2(c + 2 * i < vis ? ex2_approx(t.x) : 0.0f,
                           c + 2 * i + 1 < vis ? ex2_approx(t.y) : 0.0f);
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) pk[c / 2 + i] = pack_half2(u[i].x, u[i].y);
#pragma unroll
    for (int k = 8; k >= 1; k >>= 1)
#pragma unroll
      for (int i = 0; i < k; ++i) u[i] = __fadd2_rn(u[i], u[i + k]);
    acc = __fadd2_rn(acc, u[0]);
    if (c + 32 < kBN) tmem_wait_ld(nx);
  }
  return acc.x + acc.y;
}

__global__ void __launch_bounds__(kThreadsA, 1)
    attn_fwd_tcgen05(const __grid_constant__ CUtensorMap tmQKV, const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;              // [2] query tiles
  uint8_t* sK = smem + 2 * kTile;  // [2] stages
  uint8_t* sV = smem + 4 * kTile;  // [2] stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 6 * kTile);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [2] stages
  uint64_t* k_empty = bars + 3;   // [2]
  uint64_t* v_full = bars + 5;    // [2]
  uint64_t* v_empty = bars + 7;   // [2]
  uint64_t* s_full = bars + 9;    // [2] tiles: S ready (and the previous P V done)
  uint64_t* p_full = bars + 11;   // [2] tiles: P stored (and O rescaled)
  uint64_t* o_full = bars + 13;   // [2] tiles: P V done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (a.s + kBM - 1) / kBM;
  const int npairs = (nqb + 1) / 2;
  const int pair = npairs - 1 - static_cast<int>(blockIdx.y);  // longest rows first
  const int head = blockIdx.x % a.heads, bi = blockIdx.x / a.heads;
  const int qb0 = 2 * pair;  // query tiles qb0 and qb0 + 1
  const bool valid1 = qb0 + 1 < nqb;
  const int n0 = a.causal ? qb0 + 1 : nqb;                      // key blocks of tile 0
  const int n1 = valid1 ? (a.causal ? qb0 + 2 : nqb) : 0;       // and of tile 1
  const int n_max = max(n0, n1);
  const int row0 = bi * a.s;  // first row of this batch element in QKV
  const int qcol = head * kD, kcol = a.h + head * kD, vcol = 2 * a.h + head * kD;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);  // one arrival per warp of the tile's softmax group
      mbar_init(&o_full[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Tile x: S_x at columns [256 x, 256 x + 128) (P_x, fp16 pairs, over its
  // first 64 columns), O_x at [256 x + 128, 256 x + 256).
  auto tS = [tmem](int x) { return tmem + static_cast<uint32_t>(256 * x); };
  auto tO = [tmem](int x) { return tmem + static_cast<uint32_t>(256 * x + 128); };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------- TMA producer
      bool ok = true;
      tma_prefetch_desc(&tmQKV);
      mbar_arrive_expect_tx(q_full, (valid1 ? 2 : 1) * kTile);
      for (int x = 0; x < (valid1 ? 2 : 1); ++x) {
        tma_load_2d(sQ + x * kTile, &tmQKV, q_full, qcol, row0 + (qb0 + x) * kBM);
        tma_load_2d(sQ + x * kTile + kHalf, &tmQKV, q_full, qcol + 64, row0 + (qb0 + x) * kBM);
      }
      for (int j = 0; j < n_max && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1u;
        const int krow = row0 + j * kBN;
        if (!(ok = mbar_wait(&k_empty[st], ph ^ 1u, a.status, kStatusAttnTimeout))) break;
        mbar_arrive_expect_tx(&k_full[st], kTile);
        tma_load_2d(sK + st * kTile, &tmQKV, &k_full[st], kcol, krow);
        tma_load_2d(sK + st * kTile + kHalf, &tmQKV, &k_full[st], kcol + 64, krow);
        if (!(ok = mbar_wait(&v_empty[st], ph ^ 1u, a.status, kStatusAttnTimeout))) break;
        mbar_arrive_expect_tx(&v_full[st], kTile);
        tma_load_2d(sV + st * kTile, &tmQKV, &v_full[st], vcol, krow);
        tma_load_2d(sV + st * kTile + kHalf, &tmQKV, &v_full[st], vcol + 64, krow);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      // Per key block j: P_a V_j, S_a(j+1), P_b V_j, S_b(j+1).  The MMAs of
      // this thread run in issue order, so S_x(j+1) overwrites P_x(j) only
      // after P_x(j) V_j has read it, and the commit of S_x(j+1) also covers
      // P_x(j) V_j (the softmax may rescale O_x once S_x(j+1) is ready).
      constexpr uint32_t kIdS = idesc_f16_f32(128, 128, false, false);  // Q K^T
      constexpr uint32_t kIdO = idesc_f16_f32(128, 128, false, true);   // P V
      auto issue_s = [&](int x, int j) {
        const uint32_t q_addr = smem_u32(sQ + x * kTile);
        const uint32_t k_addr = smem_u32(sK + (j & 1) * kTile);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_bf16(tS(x), sw128_desc(q_addr + off, 16, 1024), sw128_desc(k_addr + off, 16, 1024),
                    kIdS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[x]);
      };
      auto issue_pv = [&](int x, int j) {
        const uint32_t v_addr = smem_u32(sV + (j & 1) * kTile);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)  // 16 keys: 8 columns of fp16 pairs
          umma_f16_ts(tO(x), tS(x) + static_cast<uint32_t>(kk * 8),
                      sw128_desc(v_addr + kk * 16 * 128, kHalf, 1024), kIdO,
                      (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&o_full[x]);
      };
      bool ok = mbar_wait(q_full, 0, a.status, kStatusAttnTimeout) &&
                mbar_wait(&k_full[0], 0, a.status, kStatusAttnTimeout);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        if (n1 > 0) issue_s(1, 0);
        umma_commit(&k_empty[0]);
      }
      for (int j = 0; j < n_max && ok; ++j) {
        const int st = j & 1;
        if (!(ok = mbar_wait(&v_full[st], static_cast<uint32_t>(j >> 1) & 1u, a.status,
                             kStatusAttnTimeout)))
          break;
        bool k_next = false;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int nx = x ? n1 : n0;
          if (!ok || j >= nx) continue;
          if (!(ok = mbar_wait(&p_full[x], static_cast<uint32_t>(j) & 1u, a.status,
                               kStatusAttnTimeout)))
            break;
          tc_fence_after();
          issue_pv(x, j);
          if (j + 1 < nx) {
            if (!k_next) {
              if (!(ok = mbar_wait(&k_full[(j + 1) & 1], static_cast<uint32_t>((j + 1) >> 1) & 1u,
                                   a.status, kStatusAttnTimeout)))
                break;
              tc_fence_after();
              k_next = true;
            }
            issue_s(x, j + 1);
          }
        }
        if (!ok) break;
        if (k_next) umma_commit(&k_empty[(j + 1) & 1]);
        umma_commit(&v_empty[st]);
      }
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------- softmax
    // Warps 4-7 take tile 0, warps 8-11 tile 1; thread i of a group owns
    // query row i of its tile = tensor-memory lane i.
    const int x = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int qrow = (qb0 + x) * kBM + r;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t srow = tS(x) + lane_off, orow_t = tO(x) + lane_off;
    const int nx = x ? n1 : n0;
    // Keys [0, limit) are visible to this row (causal: up to the row itself).
    const int limit = a.causal ? min(a.s, qrow + 1) : a.s;
    float m_used = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < nx; ++j) {
      if (!(ok = mbar_wait(&s_full[x], static_cast<uint32_t>(j) & 1u, a.status,
                           kStatusAttnTimeout)))
        break;
      tc_fence_after();
      const int vis = limit - j * kBN;  // visible keys of this block: [0, vis), vis >= 1
      if (j == 0) m_used = row_max_visible(srow, vis) * a.scale_log2;
      uint32_t pk[kBN / 2];
      float rs = exp_row(srow, vis, a.scale_log2, m_used, pk);
      // Block 0 set the maximum in use, so its P <= 1.  Later blocks: a row
      // sum above kCheckSum (rare) sends the warp to the exact maximum.
      if (j > 0 && __any_sync(0xffffffffu, rs > kCheckSum)) {
        const float m_new = row_max_visible(srow, vis) * a.scale_log2;
        const bool need = m_new > m_used + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          // The maximum rose by more than 2^8.  Recompute P at the new
          // maximum (S is still intact: P has not been stored yet) and
          // rescale O (P_{j-1} V_{j-1} completed before S_j) and l.
          const float alpha = need ? ex2_approx(m_used - m_new) : 1.0f;
          if (need) m_used = m_new;
          rs = exp_row(srow, vis, a.scale_log2, m_used, pk);
#pragma unroll 1
          for (int c = 0; c < kD; c += 32) {
            float o[32];
            tmem_ld32(orow_t + c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(orow_t + c, o);
          }
          l_run *= alpha;
        }
      }
      l_run += rs;
#pragma unroll
      for (int c = 0; c < kBN / 2; c += 16) {
        uint32_t q16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) q16[i] = pk[c + i];
        tmem_st16(srow + c, q16);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[x]);
    }
    if (ok && nx > 0 &&
        mbar_wait(&o_full[x], static_cast<uint32_t>(nx - 1) & 1u, a.status, kStatusAttnTimeout)) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      __nv_bfloat16* orow = a.out + static_cast<long long>(row0 + qrow) * a.h + head * kD;
#pragma unroll 1
      for (int c = 0; c < kD; c += 32) {
        float v[32];
        tmem_ld32(orow_t + c, v);
        if (qrow < a.s) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 8 * q + 2 * e;
              __nv_bfloat162 t = __floats2bfloat162_rn(v[i] * inv, v[i + 1] * inv);
              w[e] = *reinterpret_cast<uint32_t*>(&t);
            }
            *reinterpret_cast<uint4*>(orow + c + 8 * q) = u;
          }
        }
      }
      if (qrow < a.s)
        a.lse[(static_cast<long long>(bi) * a.heads + head) * a.s + qrow] =
            (m_used + log2f(l_run)) * kLn2A;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}


// ------------------------------------------------------------------ backward
// Two kernels, no atomics (deterministic), both on tcgen05; P and dS are
// recomputed from the saved LSE:
//   P = 2^(S * scale_log2 - LSE * log2e),  dS = P * (dP - D),  D = rowsum(dO * O).
// dQ kernel (per pair of 128-row query tiles of one head, 64-key blocks; the
// two tiles share each K / V block and take turns on the tensor core):
//   S = Q K^T, dP = dO V^T (TMEM) -> dS (fp16, written back into tensor
//   memory over S) -> dQ += dS K (dS the tensor-memory A operand); dQ is
//   scaled by 1/sqrt(d) at the end.
// dK/dV kernel (per 128 keys, 64-query blocks; persistent, one CTA per SM
// taking its key tiles in turn):
//   S^T = K Q^T, dP^T = V dO^T (TMEM, two buffers) -> P^T, dS^T (fp16, back
//   into tensor memory over S^T and dP^T) -> dV += P^T dO, dK += dS^T Q
//   (tensor-memory A operands); dK is scaled by 1/sqrt(d) at the end.
constexpr int kB64 = 64;
constexpr int kTile64 = 64 * 128 * 2;   // [64 rows x 128] fp16: 16 KB (two 8 KB halves)
constexpr int kHalf64 = kTile64 / 2;

constexpr int kThreadsB = 384;
constexpr int kEwWarpsB = 8;

struct BwdArgs {
  int s, h, heads, causal;
  int bh, kv_items;  // b * heads; dK/dV work items (key tiles of all heads)
  float scale_log2, scale;
  // Row terms of the backward, [b * heads] rows of sp floats (s rounded up
  // to 4, zero beyond s, 64 zeros after the last row): -LSE * log2(e) and
  // -D with D = rowsum(dO * O).
  const float* nlse;
  const float* nd;
  int sp;
  __nv_bfloat16* dqkv;  // [M, 3h]
  WaitCtl status;
};

// Two warp-collective loads of 32 lanes x 32 columns with a single wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, float (&va)[32], uint32_t tb,
                                            float (&vb)[32]) {
  uint32_t a[32], b[32];
#define TP_LD32(dst, addr)                                                                  \
  asm volatile(                                                                            \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                            \
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "            \
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "  \
      "[%32];"                                                                             \
      : "=r"(dst[0]), "=r"(dst[1]), "=r"(dst[2]), "=r"(dst[3]), "=r"(dst[4]),             \
        "=r"(dst[5]), "=r"(dst[6]), "=r"(dst[7]), "=r"(dst[8]), "=r"(dst[9]),             \
        "=r"(dst[10]), "=r"(dst[11]), "=r"(dst[12]), "=r"(dst[13]), "=r"(dst[14]),        \
        "=r"(dst[15]), "=r"(dst[16]), "=r"(dst[17]), "=r"(dst[18]), "=r"(dst[19]),        \
        "=r"(dst[20]), "=r"(dst[21]), "=r"(dst[22]), "=r"(dst[23]), "=r"(dst[24]),        \
        "=r"(dst[25]), "=r"(dst[26]), "=r"(dst[27]), "=r"(dst[28]), "=r"(dst[29]),        \
        "=r"(dst[30]), "=r"(dst[31])                                                       \
      : "r"(addr)                                                                          \
      : "memory")
  TP_LD32(a, ta);
  TP_LD32(b, tb);
#undef TP_LD32
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  // The wait orders the loads; the copies below cannot move above it (the
  // asm is volatile with a memory clobber).
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    va[i] = __uint_as_float(a[i]);
    vb[i] = __uint_as_float(b[i]);
  }
}

// dQ kernel.  Shared memory: Q[2] 32K each | dO[2] 32K each | KV ring of
// kKvStages stages (K 16K + V 16K) | barriers.
constexpr int kKvStages = 3;
constexpr int kSmemDQ = 1024 + 4 * kTile + kKvStages * (2 * kTile64) + 256;

__global__ void __launch_bounds__(kThreadsB, 1)
    attn_bwd_dq_tcgen05(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKV,
                        const __grid_constant__ CUtensorMap tmdO, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                  // [2] tiles
  uint8_t* sdO = smem + 2 * kTile;     // [2] tiles
  uint8_t* sKV = smem + 4 * kTile;     // stage st: K at +0, V at +kTile64
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + kKvStages * (2 * kTile64));
  uint64_t* qd_full = bars + 0;
  uint64_t* kv_full = bars + 1;                   // [kKvStages]
  uint64_t* kv_empty = kv_full + kKvStages;       // [kKvStages]
  uint64_t* s_full = kv_empty + kKvStages;        // [2] tiles: S, dP ready
  uint64_t* ds_full = s_full + 2;                 // [2] tiles: dS stored
  uint64_t* dq_done = ds_full + 2;                // [2] tiles
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dq_done + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (a.s + kBM - 1) / kBM;
  const int npairs = (nqb + 1) / 2;
  const int pair = npairs - 1 - static_cast<int>(blockIdx.y);  // longest rows first
  const int head = blockIdx.x % a.heads, bi = blockIdx.x / a.heads;
  const int qb0 = 2 * pair;
  const bool valid1 = qb0 + 1 < nqb;
  const int nkb_all = (a.s + kB64 - 1) / kB64;
  const int n0 = a.causal ? min(2 * qb0 + 2, nkb_all) : nkb_all;
  const int n1 = valid1 ? (a.causal ? min(2 * qb0 + 4, nkb_all) : nkb_all) : 0;
  const int n_max = max(n0, n1);
  const int row0 = bi * a.s;

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    for (int i = 0; i < kKvStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&ds_full[i], 4);  // the tile's four element-wise warps
      mbar_init(&dq_done[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Tile x: S_x at [256 x, +64) (dS_x, fp16 pairs, over its first 32
  // columns), dP_x at [256 x + 64, +64), dQ_x at [256 x + 128, +128).
  auto tS = [tmem](int x) { return tmem + static_cast<uint32_t>(256 * x); };
  auto tP = [tmem](int x) { return tmem + static_cast<uint32_t>(256 * x + 64); };
  auto tQ = [tmem](int x) { return tmem + static_cast<uint32_t>(256 * x + 128); };

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmKV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(qd_full, (valid1 ? 2 : 1) * 2 * kTile);
      for (int x = 0; x < (valid1 ? 2 : 1); ++x) {
        const int qr = row0 + (qb0 + x) * kBM;
        tma_load_2d(sQ + x * kTile, &tmQ, qd_full, head * kD, qr);
        tma_load_2d(sQ + x * kTile + kHalf, &tmQ, qd_full, head * kD + 64, qr);
        tma_load_2d(sdO + x * kTile, &tmdO, qd_full, head * kD, qr);
        tma_load_2d(sdO + x * kTile + kHalf, &tmdO, qd_full, head * kD + 64, qr);
      }
      for (int j = 0; j < n_max && ok; ++j) {
        const int ks = j % kKvStages;
        const uint32_t kph = static_cast<uint32_t>(j / kKvStages) & 1u;
        if (!(ok = mbar_wait(&kv_empty[ks], kph ^ 1u, a.status, kStatusAttnTimeout))) break;
        mbar_arrive_expect_tx(&kv_full[ks], 2 * kTile64);
        uint8_t* k_dst = sKV + ks * (2 * kTile64);
        const int krow = row0 + j * kB64;
        tma_load_2d(k_dst, &tmKV, &kv_full[ks], a.h + head * kD, krow);
        tma_load_2d(k_dst + kHalf64, &tmKV, &kv_full[ks], a.h + head * kD + 64, krow);
        tma_load_2d(k_dst + kTile64, &tmKV, &kv_full[ks], 2 * a.h + head * kD, krow);
        tma_load_2d(k_dst + kTile64 + kHalf64, &tmKV, &kv_full[ks], 2 * a.h + head * kD + 64, krow);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // Per key block j: dQ_0 += dS_0 K_j, S_0 / dP_0 of block j + 1, then the
      // same for tile 1.  The MMAs run in issue order, so S_x(j + 1)
      // overwrites dS_x(j) only after dQ_x's product has read it.
      constexpr uint32_t kIdSP = idesc_f16_f32(128, 64, false, false);  // Q K^T, dO V^T
      constexpr uint32_t kIdQ = idesc_f16_f32(128, 128, false, true);   // dS K
      auto issue_sp = [&](int x, int j) {
        const uint32_t q_addr = smem_u32(sQ + x * kTile), do_addr = smem_u32(sdO + x * kTile);
        const uint32_t k_addr = smem_u32(sKV + (j % kKvStages) * (2 * kTile64));
        const uint32_t v_addr = k_addr + kTile64;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t a_off = (kk >> 2) * kHalf + (kk & 3) * 32;
          const uint32_t b_off = (kk >> 2) * kHalf64 + (kk & 3) * 32;
          umma_bf16(tS(x), sw128_desc(q_addr + a_off, 16, 1024),
                    sw128_desc(k_addr + b_off, 16, 1024), kIdSP, kk > 0 ? 1u : 0u);
          umma_bf16(tP(x), sw128_desc(do_addr + a_off, 16, 1024),
                    sw128_desc(v_addr + b_off, 16, 1024), kIdSP, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[x]);
      };
      bool ok = mbar_wait(qd_full, 0, a.status, kStatusAttnTimeout) &&
                mbar_wait(&kv_full[0], 0, a.status, kStatusAttnTimeout);
      if (ok) {
        tc_fence_after();
        issue_sp(0, 0);
        if (n1 > 0) issue_sp(1, 0);
      }
      for (int j = 0; j < n_max && ok; ++j) {
        bool kv_next = false;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int nx = x ? n1 : n0;
          if (!ok || j >= nx) continue;
          if (!(ok = mbar_wait(&ds_full[x], static_cast<uint32_t>(j) & 1u, a.status,
                               kStatusAttnTimeout)))
            break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sKV + (j % kKvStages) * (2 * kTile64));
#pragma unroll
          for (int kk = 0; kk < kB64 / 16; ++kk)  // 16 keys: 8 columns of fp16 pairs
            umma_f16_ts(tQ(x), tS(x) + static_cast<uint32_t>(kk * 8),
                        sw128_desc(k_addr + kk * 2048, kHalf64, 1024), kIdQ,
                        (j | kk) != 0 ? 1u : 0u);
          if (j + 1 < nx) {
            if (!kv_next) {
              const int ks = (j + 1) % kKvStages;
              if (!(ok = mbar_wait(&kv_full[ks], static_cast<uint32_t>((j + 1) / kKvStages) & 1u,
                                   a.status, kStatusAttnTimeout)))
                break;
              tc_fence_after();
              kv_next = true;
            }
            issue_sp(x, j + 1);
          } else {
            umma_commit(&dq_done[x]);
          }
        }
        if (!ok) break;
        umma_commit(&kv_empty[j % kKvStages]);
      }
    }
  } else if (warp >= 4) {
    // Warps 4-7 take tile 0, warps 8-11 tile 1; thread i owns query row i.
    const int x = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int qrow = (qb0 + x) * kBM + r;
    const int nx = x ? n1 : n0;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const long long stat = (static_cast<long long>(bi) * a.heads + head) * a.sp;
    const int qc = min(qrow, a.s - 1);
    const float nl = a.nlse[stat + qc], ndd = a.nd[stat + qc];
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
    const float2 nl2 = make_float2(nl, nl), nd2 = make_float2(ndd, ndd);
    const int limit = a.causal ? min(a.s, qrow + 1) : a.s;
    bool ok = true;
    for (int j = 0; j < nx && ok; ++j) {
      if (!(ok = mbar_wait(&s_full[x], static_cast<uint32_t>(j) & 1u, a.status,
                           kStatusAttnTimeout)))
        break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kB64; c += 32) {
        const int vis = limit - j * kB64 - c;  // columns c + i with i < vis are visible
        float sv[32], pv[32];
        tmem_ld32x2(tS(x) + lane_off + c, sv, tP(x) + lane_off + c, pv);
        uint32_t pk[16];
        // dS = P (dP - D), P = 2^(S scale_log2 - lse2), two entries per step
        // (two-wide fused multiply-add, add and multiply: the same roundings
        // as the one-wide forms).
        if (vis >= 32) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 t = __ffma2_rn(make_float2(sv[i], sv[i + 1]), sc2, nl2);
            const float2 p = make_float2(ex2_approx(t.x), ex2_approx(t.y));
            const float2 g = __fmul2_rn(p, __fadd2_rn(make_float2(pv[i], pv[i + 1]), nd2));
            pk[i >> 1] = pack_half2(g.x, g.y);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 t = __ffma2_rn(make_float2(sv[i], sv[i + 1]), sc2, nl2);
            const float2 p = make_float2(i < vis ? ex2_approx(t.x) : 0.0f,
                                         i + 1 < vis ? ex2_approx(t.y) : 0.0f);
            const float2 g = __fmul2_rn(p, __fadd2_rn(make_float2(pv[i], pv[i + 1]), nd2));
            pk[i >> 1] = pack_half2(g.x, g.y);
          }
        }
        // dS columns [c / 2, c / 2 + 16): S columns this thread has read.
        tmem_st16(tS(x) + lane_off + c / 2, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_full[x]);
    }
    if (ok && nx > 0 && mbar_wait(&dq_done[x], 0, a.status, kStatusAttnTimeout)) {
      tc_fence_after();
      __nv_bfloat16* out = a.dqkv + static_cast<long long>(row0 + qrow) * (3LL * a.h) + head * kD;
#pragma unroll 1
      for (int cc = 0; cc < kD; cc += 32) {
        float v[32];
        tmem_ld32(tQ(x) + lane_off + cc, v);
        if (qrow < a.s) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 t = __floats2bfloat162_rn(v[8 * q + 2 * e] * a.scale,
                                                       v[8 * q + 2 * e + 1] * a.scale);
              w[e] = *reinterpret_cast<uint32_t*>(&t);
            }
            *reinterpret_cast<uint4*>(out + cc + 8 * q) = u;
          }
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// K, V (128 rows, once), then Q_i, dO_i (64 rows) with the block's row
// terms -LSE * log2(e) and -D in a ring of kQdStages stages, all of a stage
// copied asynchronously (tensor loads and two 256-byte bulk copies on the
// stage's barrier), so the TMA warp never waits on a load itself.
// Shared memory: K 32K | V 32K | QdO[4] (Q 16K + dO 16K) | barriers | stats[4]
// (128 floats).  P^T and dS^T live in tensor memory: element-wise group g
// (query columns [32 g, 32 g + 32) of a block) writes its fp16 pairs over
// the 16 columns starting at column 32 g of the S^T (P^T) and dP^T (dS^T)
// buffers, columns only it has read.
constexpr int kQdStages = 4;
constexpr int kSmemKV = 1024 + 2 * kTile + kQdStages * (2 * kTile64) + 256 + kQdStages * 2 * kB64 * 4;

// Work item k of the dK/dV kernel (k = 0 the longest): key tile k / (b *
// heads) of one (batch element, head); under the causal mask the early key
// tiles see the most query blocks.
struct KvItem {
  int bi, head, k0, i0, n_qb;  // first key, first query block, query blocks
};

__device__ __forceinline__ KvItem kv_item(int k, const BwdArgs& a) {
  KvItem it;
  const int bh = k % a.bh, kb = k / a.bh;
  it.head = bh % a.heads;
  it.bi = bh / a.heads;
  it.k0 = kb * kBN;
  const int nqb_all = (a.s + kB64 - 1) / kB64;
  it.i0 = a.causal ? it.k0 / kB64 : 0;
  it.n_qb = nqb_all - it.i0;  // >= 1: k0 < s
  return it;
}

// The r-th item of this CTA, or -1: rounds of gridDim.x items in snake order
// (even rounds from CTA 0 up, odd rounds down), so long and short key tiles
// even out over the CTAs.
__device__ __forceinline__ int kv_item_index(int r, const BwdArgs& a) {
  const long long g = gridDim.x, c = blockIdx.x;
  const long long k = r * g + ((r & 1) ? g - 1 - c : c);
  return k < a.kv_items ? static_cast<int>(k) : -1;
}

// Persistent: one CTA per SM walks its key tiles.  The Q / dO ring runs on
// across items; an item's K and V are loaded once the previous item's last
// S^T / dP^T products are done (kv_empty), and its first dV, dK products
// wait until the previous item's epilogue has read the accumulators
// (acc_empty), so the next key tile's loads and first products overlap the
// current one's epilogue.
__global__ void __launch_bounds__(kThreadsB, 1)
    attn_bwd_dkdv_tcgen05(const __grid_constant__ CUtensorMap tmKV128,
                          const __grid_constant__ CUtensorMap tmQ64,
                          const __grid_constant__ CUtensorMap tmdO64, const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + kTile;
  uint8_t* sQdO = smem + 2 * kTile;                     // stage q: Q at +0, dO at +kTile64
  uint64_t* bars = reinterpret_cast<uint64_t*>(sQdO + kQdStages * (2 * kTile64));
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;                // the item's last S^T / dP^T done
  uint64_t* qd_full = bars + 2;                 // [kQdStages]
  uint64_t* qd_empty = qd_full + kQdStages;     // [kQdStages]
  uint64_t* s_full = qd_empty + kQdStages;      // [2]
  uint64_t* p_full = s_full + 2;                // [2]
  uint64_t* acc_done = p_full + 2;              // the item's last dV, dK products done
  uint64_t* acc_empty = acc_done + 1;           // the epilogue has read dV, dK
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  // stage q: -LSE * log2(e) of the block's 64 queries at [0, 64), -D at [64, 128)
  float* s_stat = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < kQdStages; ++i) {
      mbar_init(&qd_full[i], 1);  // the TMA warp's arrival; the copies count as transactions
      mbar_init(&qd_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kEwWarpsB);
    }
    mbar_init(acc_done, 1);
    mbar_init(acc_empty, kEwWarpsB);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // S^T buffers at columns 0 and 64, dP^T at 128 and 192, dV at 256, dK at 384.
  auto tS = [tmem](int st) { return tmem + static_cast<uint32_t>(64 * st); };
  auto tP = [tmem](int st) { return tmem + static_cast<uint32_t>(128 + 64 * st); };
  const uint32_t tdV = tmem + 256, tdK = tmem + 384;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmKV128);
      tma_prefetch_desc(&tmQ64);
      tma_prefetch_desc(&tmdO64);
      bool ok = true;
      long long g = 0;  // query blocks loaded so far: the ring position
      for (int r = 0; ok; ++r) {
        const int k = kv_item_index(r, a);
        if (k < 0) break;
        const KvItem it = kv_item(k, a);
        const int row0 = it.bi * a.s;
        if (!(ok = mbar_wait(kv_empty, static_cast<uint32_t>(r & 1) ^ 1u, a.status,
                             kStatusAttnTimeout)))
          break;
        mbar_arrive_expect_tx(kv_full, 2 * kTile);
        tma_load_2d(sK, &tmKV128, kv_full, a.h + it.head * kD, row0 + it.k0);
        tma_load_2d(sK + kHalf, &tmKV128, kv_full, a.h + it.head * kD + 64, row0 + it.k0);
        tma_load_2d(sV, &tmKV128, kv_full, 2 * a.h + it.head * kD, row0 + it.k0);
        tma_load_2d(sV + kHalf, &tmKV128, kv_full, 2 * a.h + it.head * kD + 64, row0 + it.k0);
        const long long stat = (static_cast<long long>(it.bi) * a.heads + it.head) * a.sp;
        for (int j = 0; j < it.n_qb && ok; ++j, ++g) {
          const int qs = static_cast<int>(g % kQdStages);
          const uint32_t qph = static_cast<uint32_t>(g / kQdStages) & 1u;
          if (!(ok = mbar_wait(&qd_empty[qs], qph ^ 1u, a.status, kStatusAttnTimeout))) break;
          const int q0 = (it.i0 + j) * kB64;
          // Q, dO and the block's 64 row terms of each kind (256 bytes from
          // a 16-byte aligned row offset; past s they are zeros or the next
          // row's finite values, which the mask never lets through).
          mbar_arrive_expect_tx(&qd_full[qs], 2 * kTile64 + 2 * kB64 * 4);
          uint8_t* dst = sQdO + qs * (2 * kTile64);
          const int qrow = row0 + q0;
          tma_load_2d(dst, &tmQ64, &qd_full[qs], it.head * kD, qrow);
          tma_load_2d(dst + kHalf64, &tmQ64, &qd_full[qs], it.head * kD + 64, qrow);
          tma_load_2d(dst + kTile64, &tmdO64, &qd_full[qs], it.head * kD, qrow);
          tma_load_2d(dst + kTile64 + kHalf64, &tmdO64, &qd_full[qs], it.head * kD + 64, qrow);
          float* st_dst = s_stat + qs * (2 * kB64);
          bulk_load(st_dst, a.nlse + stat + q0, kB64 * 4, &qd_full[qs]);
          bulk_load(st_dst + kB64, a.nd + stat + q0, kB64 * 4, &qd_full[qs]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdSP = idesc_f16_f32(128, 64, false, false);  // K Q^T, V dO^T
      constexpr uint32_t kIdAcc = idesc_f16_f32(128, 128, false, true);  // P^T dO, dS^T Q
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      // S^T / dP^T of ring position gg into buffer gg & 1, whose P^T / dS^T
      // the products of position gg - 2 (issued before) have read.
      auto issue_sp = [&](long long gg) -> bool {
        const int st = static_cast<int>(gg & 1);
        const int qs = static_cast<int>(gg % kQdStages);
        if (!mbar_wait(&qd_full[qs], static_cast<uint32_t>(gg / kQdStages) & 1u, a.status,
                       kStatusAttnTimeout))
          return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQdO + qs * (2 * kTile64));
        const uint32_t do_addr = q_addr + kTile64;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t a_off = (kk >> 2) * kHalf + (kk & 3) * 32;
          const uint32_t b_off = (kk >> 2) * kHalf64 + (kk & 3) * 32;
          umma_bf16(tS(st), sw128_desc(k_addr + a_off, 16, 1024),
                    sw128_desc(q_addr + b_off, 16, 1024), kIdSP, kk > 0 ? 1u : 0u);
          umma_bf16(tP(st), sw128_desc(v_addr + a_off, 16, 1024),
                    sw128_desc(do_addr + b_off, 16, 1024), kIdSP, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[st]);
        return true;
      };
      bool ok = true;
      long long g = 0;  // query blocks of the items before this one
      for (int r = 0; ok; ++r) {
        const int k = kv_item_index(r, a);
        if (k < 0) break;
        const KvItem it = kv_item(k, a);
        if (!(ok = mbar_wait(kv_full, static_cast<uint32_t>(r & 1), a.status,
                             kStatusAttnTimeout)))
          break;
        if (!(ok = issue_sp(g))) break;
        if (it.n_qb == 1) umma_commit(kv_empty);
        for (int j = 0; j < it.n_qb && ok; ++j) {
          const long long gj = g + j;
          if (j + 1 < it.n_qb) {
            if (!(ok = issue_sp(gj + 1))) break;
            if (j + 2 == it.n_qb) umma_commit(kv_empty);  // the item's last S^T / dP^T
          }
          const int st = static_cast<int>(gj & 1);
          if (!(ok = mbar_wait(&p_full[st], static_cast<uint32_t>(gj >> 1) & 1u, a.status,
                               kStatusAttnTimeout)))
            break;
          // The item's first dV, dK products overwrite the accumulators: the
          // previous item's epilogue must have read them.
          if (j == 0 && r > 0 &&
              !(ok = mbar_wait(acc_empty, static_cast<uint32_t>((r - 1) & 1), a.status,
                               kStatusAttnTimeout)))
            break;
          tc_fence_after();
          const int qs = static_cast<int>(gj % kQdStages);
          const uint32_t q_addr = smem_u32(sQdO + qs * (2 * kTile64));
          const uint32_t do_addr = q_addr + kTile64;
#pragma unroll
          for (int kk = 0; kk < kB64 / 16; ++kk) {
            // queries [16 kk, 16 kk + 16): group kk / 2's columns, 8 columns each
            const uint32_t col = static_cast<uint32_t>(32 * (kk >> 1) + 8 * (kk & 1));
            const uint32_t acc = (j | kk) != 0 ? 1u : 0u;
            umma_f16_ts(tdV, tS(st) + col, sw128_desc(do_addr + kk * 2048, kHalf64, 1024),
                        kIdAcc, acc);
            umma_f16_ts(tdK, tP(st) + col, sw128_desc(q_addr + kk * 2048, kHalf64, 1024),
                        kIdAcc, acc);
          }
          umma_commit(&qd_empty[qs]);
        }
        if (ok) umma_commit(acc_done);
        g += it.n_qb;
      }
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    const int grp = (warp - 4) >> 2;  // this warp's column half
    const int c = grp * 32;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
    bool ok = true;
    long long gb = 0;  // query blocks of the items before this one
    for (int ri = 0; ok; ++ri) {
      const int k = kv_item_index(ri, a);
      if (k < 0) break;
      const KvItem it = kv_item(k, a);
      const int key = it.k0 + r;
      for (int j = 0; j < it.n_qb; ++j) {
        const long long gj = gb + j;
        const int st = static_cast<int>(gj & 1);
        const int qs = static_cast<int>(gj % kQdStages);
        const int q0 = (it.i0 + j) * kB64;
        if (!(ok = mbar_wait(&s_full[st], static_cast<uint32_t>(gj >> 1) & 1u, a.status,
                             kStatusAttnTimeout)))
          break;
        // The block's statistics were staged with its Q / dO stage; the stage
        // cannot be refilled before this block's products are done.
        if (!(ok = mbar_wait(&qd_full[qs], static_cast<uint32_t>(gj / kQdStages) & 1u, a.status,
                             kStatusAttnTimeout)))
          break;
        tc_fence_after();
        const float* wstat = s_stat + qs * (2 * kB64) + c;
        // query q = q0 + c + i is visible to this key when key <= q (causal)
        // and q < s: lo <= i < hi
        const int lo = (a.causal ? max(key - q0, 0) : 0) - c;
        const int hi = (key < a.s ? min(a.s - q0, kB64) : 0) - c;
        float sv[32], pv[32];
        tmem_ld32x2(tS(st) + lane_off + c, sv, tP(st) + lane_off + c, pv);
        uint32_t pk[16], dk[16];
        // P^T = 2^(S^T scale_log2 - lse2) and dS^T = P^T (dP^T - D), two
        // entries per step (two-wide arithmetic, the one-wide roundings); the
        // staged statistics are negated.  Blocks off the diagonal skip the mask.
        const bool full = lo <= 0 && hi >= 32;
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 nl = *reinterpret_cast<const float2*>(wstat + i);
          const float2 nd = *reinterpret_cast<const float2*>(wstat + kB64 + i);
          const float2 t = __ffma2_rn(make_float2(sv[i], sv[i + 1]), sc2, nl);
          float2 p = make_float2(ex2_approx(t.x), ex2_approx(t.y));
          if (!full) {
            p.x = (i >= lo && i < hi) ? p.x : 0.0f;
            p.y = (i + 1 >= lo && i + 1 < hi) ? p.y : 0.0f;
          }
          pk[i >> 1] = pack_half2(p.x, p.y);
          const float2 g = __fmul2_rn(p, __fadd2_rn(make_float2(pv[i], pv[i + 1]), nd));
          dk[i >> 1] = pack_half2(g.x, g.y);
        }
        tmem_st16(tS(st) + lane_off + c, pk);  // P^T over this group's S^T columns
        tmem_st16(tP(st) + lane_off + c, dk);  // dS^T over its dP^T columns
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[st]);
      }
      if (!ok) break;
      gb += it.n_qb;
      if (!(ok = mbar_wait(acc_done, static_cast<uint32_t>(ri & 1), a.status, kStatusAttnTimeout)))
        break;
      tc_fence_after();
      __nv_bfloat16* out = a.dqkv + (static_cast<long long>(it.bi) * a.s + key) * (3LL * a.h);
#pragma unroll
      for (int cc = grp * (kD / 2); cc < (grp + 1) * (kD / 2); cc += 32) {
        float vk[32], vv[32];
        tmem_ld32(tdK + lane_off + cc, vk);
        tmem_ld32(tdV + lane_off + cc, vv);
        if (key < a.s) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 uk, uv;
            uint32_t* wk = reinterpret_cast<uint32_t*>(&uk);
            uint32_t* wv = reinterpret_cast<uint32_t*>(&uv);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 8 * q + 2 * e;
              __nv_bfloat162 tk = __floats2bfloat162_rn(vk[i] * a.scale, vk[i + 1] * a.scale);
              __nv_bfloat162 tv = __floats2bfloat162_rn(vv[i], vv[i + 1]);
              wk[e] = *reinterpret_cast<uint32_t*>(&tk);
              wv[e] = *reinterpret_cast<uint32_t*>(&tv);
            }
            *reinterpret_cast<uint4*>(out + a.h + it.head * kD + cc + 8 * q) = uk;
            *reinterpret_cast<uint4*>(out + 2 * a.h + it.head * kD + cc + 8 * q) = uv;
          }
        }
      }

      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_attn() {
  // Initialised once, thread-safely (a function-local static).
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

}  // namespace

tp_status launch_attn_core_fwd_tc(const AttnShape& sh, const void* QKV, void* O, float* LSE,
                                  cudaStream_t stream) {
  if (sh.h / sh.heads != kD) return fail(TP_ERR_UNSUPPORTED, "attention: head dimension must be 128");
  if ((sh.s + kBM - 1) / kBM > 65535 || sh.b * sh.heads > 0x7fffffffLL)
    return fail(TP_ERR_SHAPE, "attention: sequence or b * heads too large");
  auto fn = encode_fn_attn();
  if (fn == nullptr) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  CUtensorMap map;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(3 * sh.h), static_cast<cuuint64_t>(sh.b * sh.s)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(3 * sh.h) * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(QKV), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled failed (attention)");
  FwdArgs a;
  a.s = static_cast<int>(sh.s);
  a.h = static_cast<int>(sh.h);
  a.heads = sh.heads;
  a.causal = sh.causal;
  a.scale_log2 = kLog2eA / std::sqrt(static_cast<float>(kD));
  a.out = static_cast<__nv_bfloat16*>(O);
  a.lse = LSE;
  a.status = wait_ctl();
  if (a.status.st == nullptr) return fail(TP_ERR_CUDA, "device status unavailable");
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_tcgen05, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemA);
  if (e != cudaSuccess) return cuda_fail(e, "attention fwd smem attribute");
  const int64_t nqb = (sh.s + kBM - 1) / kBM;
  dim3 grid(static_cast<unsigned>(sh.b * sh.heads), static_cast<unsigned>((nqb + 1) / 2));
  const double pairs = sh.causal ? 0.5 * double(sh.s) * sh.s : double(sh.s) * sh.s;
  {
    LaunchScope scope(TP_KIND_ATTN_FWD, 4.0 * kD * pairs * double(sh.b) * sh.heads,
                      2.0 * double(sh.b * sh.s) * 4 * sh.h, stream);
    attn_fwd_tcgen05<<<grid, kThreadsA, kSmemA, stream>>>(map, a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention fwd (tcgen05) launch");
  return TP_OK;
}

namespace {
bool make_map_f16(CUtensorMap* m, const void* ptr, int64_t cols, int64_t rows, int box_rows) {
  auto fn = encode_fn_attn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

// The row terms -LSE * log2(e) and -D must already be in `nlse` and `nd`.
tp_status launch_attn_core_bwd_tc(const AttnShape& sh, const void* QKV, const void* dO,
                                  const float* nlse, const float* nd, void* dQKV,
                                  cudaStream_t stream) {
  if (sh.h / sh.heads != kD) return fail(TP_ERR_UNSUPPORTED, "attention: head dimension must be 128");
  if ((sh.s + kBM - 1) / kBM > 65535 || sh.b * sh.heads > 0x7fffffffLL)
    return fail(TP_ERR_SHAPE, "attention: sequence or b * heads too large");
  const int64_t M = sh.b * sh.s;
  CUtensorMap qkv128, qkv64, do128, do64;
  if (!make_map_f16(&qkv128, QKV, 3 * sh.h, M, 128) || !make_map_f16(&qkv64, QKV, 3 * sh.h, M, 64) ||
      !make_map_f16(&do128, dO, sh.h, M, 128) || !make_map_f16(&do64, dO, sh.h, M, 64))
    return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled failed (attention backward)");
  BwdArgs a;
  a.s = static_cast<int>(sh.s);
  a.h = static_cast<int>(sh.h);
  a.heads = sh.heads;
  a.causal = sh.causal;
  a.scale = 1.0f / std::sqrt(static_cast<float>(kD));
  a.scale_log2 = a.scale * kLog2eA;
  a.nlse = nlse;
  a.nd = nd;
  a.sp = static_cast<int>(attn_stat_stride(sh.s));
  a.dqkv = static_cast<__nv_bfloat16*>(dQKV);
  a.status = wait_ctl();
  if (a.status.st == nullptr) return fail(TP_ERR_CUDA, "device status unavailable");
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_dq_tcgen05,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemDQ);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_bwd_dkdv_tcgen05, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemKV);
  if (e != cudaSuccess) return cuda_fail(e, "attention bwd smem attribute");
  // (batch element, head) fastest: the CTAs launch in order of decreasing work
  const int64_t nqb = (sh.s + kBM - 1) / kBM;
  dim3 gq(static_cast<unsigned>(sh.b * sh.heads), static_cast<unsigned>((nqb + 1) / 2));
  const int64_t kv_items = sh.b * sh.heads * ((sh.s + kBN - 1) / kBN);
  if (kv_items > 0x7fffffffLL) return fail(TP_ERR_SHAPE, "attention: too many key tiles");
  a.bh = static_cast<int>(sh.b * sh.heads);
  a.kv_items = static_cast<int>(kv_items);
  const unsigned gk = static_cast<unsigned>(std::min<int64_t>(kv_items, sm_count()));
  attn_bwd_dq_tcgen05<<<gq, kThreadsB, kSmemDQ, stream>>>(qkv128, qkv64, do128, a);
  attn_bwd_dkdv_tcgen05<<<gk, kThreadsB, kSmemKV, stream>>>(qkv128, qkv64, do64, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention bwd (tcgen05) launch");
  return TP_OK;
}

}  // namespace tp
