// Per-head causal softmax attention for the head-wise partitioned layer
// ("图解Transformer并行计算" §3.1: softmax(Q K^T / sqrt(d_k)) V per head;
// §3.2: each head group computes its own heads with no exchange, so the
// core runs per (batch, head) and the grouping only decides which Wqkv /
// Wo slices feed it).  The causal mask hides key c from query r when c > r
// ("5.1 Tensor并行与算子拆分", masked_fill(mask == 0, -inf)).
//
// Layout: QKV [M = b*s, 3h] row-major; head j of batch element bi uses
// rows [bi*s, (bi+1)*s) and columns j*d (Q), h + j*d (K), 2h + j*d (V),
// d = 128.  O [M, h] holds head j at columns j*d.  LSE [b, heads, s] is the
// natural log of each row's softmax denominator.
//
// The forward runs on tcgen05 (tp_attention_sm100.cu).  The backward kernels
// here use mma.sync m16n8k16 with fp16 operands and fp32 accumulation: Q, K,
// V, dO arrive in fp16 (written so by the GEMMs that produce them) and P, dS
// are rounded to fp16 for the products.  fp16 keeps three more mantissa bits
// than bf16, which halves the backward's rounding error; dQKV is written in
// bf16 for the linears.
//
// Backward, without atomics: D = rowsum(dO * O) per row and head; one kernel
// per key block accumulates dK and dV over the query blocks that see it;
// another per query block accumulates dQ over the key blocks it sees.
//   P = exp(S*scale - LSE); dV = P^T dO; dP = dO V^T; dS = P * (dP - D);
//   dQ = scale * dS K; dK = scale * dS^T Q.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "tp_internal.h"

namespace tp {
namespace {

constexpr int D = 128;            // head dimension
constexpr int ROW_BYTES = D * 2;  // 256 bytes per row of a [rows][128] bf16 tile
constexpr float kLog2e = 1.4426950408889634f;

struct AttnArgs {
  const __half* qkv;         // [M, 3h] fp16
  const __nv_bfloat16* o;    // [M, h] bf16
  const __half* dout;        // [M, h] fp16
  const float* lse;          // [b, heads, s]
  const float* dsum;         // [b, heads, s]: rowsum(dO * O)
  __nv_bfloat16* out;        // O (fwd) or dQKV (bwd)
  float* lse_out;
  int s, h, heads, causal;
  float scale_log2;          // log2(e) / sqrt(d)
  float scale;               // 1 / sqrt(d)
};

// ------------------------------------------------------------- primitives
__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of 16-byte chunk `c` of row `r` in a swizzled [rows][128] tile.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return static_cast<uint32_t>(r * ROW_BYTES + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 t = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

// A fragment (16 x 16) of a row-major swizzled tile at rows r0.., k chunk kc
// (k = 16*kk -> chunks 2kk, 2kk+1).
__device__ __forceinline__ void lda(uint32_t tile, int r0, int kk, int lane, uint32_t (&a)[4]) {
  const int r = r0 + (lane & 15);
  const int c = 2 * kk + (lane >> 4);
  ldsm_x4(tile + swz(r, c), a[0], a[1], a[2], a[3]);
}

// B fragments of two n-tiles (n0..n0+15) for k16 step kk, from a tile stored
// [n][k] (k contiguous): b[0],b[1] for n-tile n0, b[2],b[3] for n0+8.
__device__ __forceinline__ void ldb_nk(uint32_t tile, int n0, int kk, int lane, uint32_t (&b)[4]) {
  const int n = n0 + (lane & 7) + ((lane >> 4) << 3);
  const int c = 2 * kk + ((lane >> 3) & 1);
  ldsm_x4(tile + swz(n, c), b[0], b[1], b[2], b[3]);
}

// B fragments of two n-tiles (n columns n0..n0+15, n0 % 16 == 0) for k rows
// k0..k0+15, from a tile stored [k][n] (n contiguous), via ldmatrix.trans.
__device__ __forceinline__ void ldb_kn(uint32_t tile, int k0, int n0, int lane, uint32_t (&b)[4]) {
  const int k = k0 + (lane & 7) + (((lane >> 3) & 1) << 3);
  const int c = (n0 >> 3) + (lane >> 4);
  ldsm_x4_t(tile + swz(k, c), b[0], b[1], b[2], b[3]);
}

// Loads `rows` rows x 128 columns (bf16) starting at global row g0 of a
// matrix with leading dimension ld (elements) and column offset col into a
// swizzled tile; rows at or beyond row_end are zero-filled.
template <int ROWS, int THREADS>
__device__ __forceinline__ void load_tile(uint32_t tile, const __half* base, long long ld,
                                          int g0, int row_end, int col) {
  constexpr int CHUNKS = ROWS * 16;
#pragma unroll
  for (int i = threadIdx.x; i < CHUNKS; i += THREADS) {
    const int r = i >> 4, c = i & 15;
    const int gr = g0 + r;
    const bool ok = gr < row_end;
    const __half* src = base + static_cast<long long>(ok ? gr : 0) * ld + col + c * 8;
    cp_async16(tile + swz(r, c), src, ok);
  }
}

// ------------------------------------------------------- backward: D term
// D[bi, head, r] = sum_e dO[row, head*d + e] * O[row, head*d + e]; one warp
// per (row, head).
__global__ void attn_bwd_dsum_kernel(const AttnArgs a, float* dsum, long long M) {
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= M * a.heads) return;
  const long long row = wid / a.heads;
  const int head = static_cast<int>(wid - row * a.heads);
  const long long off = row * a.h + head * D + lane * 4;
  const uint2 ov = *reinterpret_cast<const uint2*>(a.o + off);
  const uint2 dv = *reinterpret_cast<const uint2*>(a.dout + off);
  const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
  const __half2* d2 = reinterpret_cast<const __half2*>(&dv);
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float2 x = __bfloat1622float2(o2[i]), y = __half22float2(d2[i]);
    acc += x.x * y.x + x.y * y.y;
  }
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
  if (lane == 0) {
    const long long bi = row / a.s, r = row - bi * a.s;
    dsum[(bi * a.heads + head) * a.s + r] = acc;
  }
}

// ------------------------------------------------------ backward: dQ pass
// One CTA per (64 query rows, batch, head); warp w owns 16 query rows.
constexpr int DQ_BM = 64, DQ_BN = 64, DQ_THREADS = 128;
constexpr int DQ_SMEM = (2 * DQ_BM + 4 * DQ_BN) * ROW_BYTES;  // Q, dO + 2 x (K, V)

__global__ void __launch_bounds__(DQ_THREADS) attn_bwd_dq_kernel(const AttnArgs a) {
  extern __shared__ __align__(128) uint8_t sm[];
  const uint32_t sQ = saddr(sm);
  const uint32_t sdO = sQ + DQ_BM * ROW_BYTES;
  const uint32_t sK[2] = {sQ + 2 * DQ_BM * ROW_BYTES, sQ + (2 * DQ_BM + 2 * DQ_BN) * ROW_BYTES};
  const uint32_t sV[2] = {sQ + (2 * DQ_BM + DQ_BN) * ROW_BYTES,
                          sQ + (2 * DQ_BM + 3 * DQ_BN) * ROW_BYTES};

  const int nqb = (a.s + DQ_BM - 1) / DQ_BM;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x);
  const int head = blockIdx.y % a.heads, bi = blockIdx.y / a.heads;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long ld = 3LL * a.h;
  const __half* base = a.qkv + static_cast<long long>(bi) * a.s * ld;
  const __half* dbase = a.dout + static_cast<long long>(bi) * a.s * a.h;
  const int q0 = qb * DQ_BM;
  const int n_kb = a.causal ? (min(q0 + DQ_BM, a.s) + DQ_BN - 1) / DQ_BN
                            : (a.s + DQ_BN - 1) / DQ_BN;

  load_tile<DQ_BM, DQ_THREADS>(sQ, base, ld, q0, a.s, head * D);
  load_tile<DQ_BM, DQ_THREADS>(sdO, dbase, a.h, q0, a.s, head * D);
  load_tile<DQ_BN, DQ_THREADS>(sK[0], base, ld, 0, a.s, a.h + head * D);
  load_tile<DQ_BN, DQ_THREADS>(sV[0], base, ld, 0, a.s, 2 * a.h + head * D);
  cp_commit();

  const int g = lane >> 2, tq = lane & 3;
  const int row_a = q0 + warp * 16 + g;
  const long long stat = (static_cast<long long>(bi) * a.heads + head) * a.s;
  float lse2[2], dsv[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = min(row_a + 8 * r, a.s - 1);
    lse2[r] = a.lse[stat + row] * kLog2e;
    dsv[r] = a.dsum[stat + row];
  }
  float dq[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.0f;

  for (int kb = 0; kb < n_kb; ++kb) {
    const int buf = kb & 1;
    if (kb + 1 < n_kb) {
      load_tile<DQ_BN, DQ_THREADS>(sK[buf ^ 1], base, ld, (kb + 1) * DQ_BN, a.s, a.h + head * D);
      load_tile<DQ_BN, DQ_THREADS>(sV[buf ^ 1], base, ld, (kb + 1) * DQ_BN, a.s,
                                   2 * a.h + head * D);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();

    float sc[8][4], dp[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[j][e] = dp[j][e] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t aq[4], ad[4];
      lda(sQ, warp * 16, kk, lane, aq);
      lda(sdO, warp * 16, kk, lane, ad);
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        uint32_t bk[4], bv[4];
        ldb_nk(sK[buf], j * 8, kk, lane, bk);
        ldb_nk(sV[buf], j * 8, kk, lane, bv);
        mma16816(sc[j], aq[0], aq[1], aq[2], aq[3], bk[0], bk[1]);
        mma16816(sc[j + 1], aq[0], aq[1], aq[2], aq[3], bk[2], bk[3]);
        mma16816(dp[j], ad[0], ad[1], ad[2], ad[3], bv[0], bv[1]);
        mma16816(dp[j + 1], ad[0], ad[1], ad[2], ad[3], bv[2], bv[3]);
      }
    }
    // dS = P * (dP - D), P = exp2(S * scale_log2 - LSE_log2).
    const int k0 = kb * DQ_BN;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = k0 + j * 8 + 2 * tq + (e & 1);
        const int row = row_a + ((e >> 1) << 3);
        const bool masked = col >= a.s || (a.causal && col > row);
        const float p = masked ? 0.0f : exp2f(sc[j][e] * a.scale_log2 - lse2[e >> 1]);
        sc[j][e] = p * (dp[j][e] - dsv[e >> 1]);
      }
    }
    // dQ += dS K (K stored [key][d]: k = key rows, n = d contiguous).
#pragma unroll
    for (int kk = 0; kk < DQ_BN / 16; ++kk) {
      const uint32_t a0 = pack_f16(sc[2 * kk][0], sc[2 * kk][1]);
      const uint32_t a1 = pack_f16(sc[2 * kk][2], sc[2 * kk][3]);
      const uint32_t a2 = pack_f16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
      const uint32_t a3 = pack_f16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
      for (int n = 0; n < 16; n += 2) {
        uint32_t bf[4];
        ldb_kn(sK[buf], kk * 16, n * 8, lane, bf);
        mma16816(dq[n], a0, a1, a2, a3, bf[0], bf[1]);
        mma16816(dq[n + 1], a0, a1, a2, a3, bf[2], bf[3]);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = row_a + 8 * r;
    if (row >= a.s) continue;
    __nv_bfloat16* out = a.out + (static_cast<long long>(bi) * a.s + row) * (3LL * a.h) + head * D;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      const int col = n * 8 + 2 * tq;
      *reinterpret_cast<uint32_t*>(out + col) =
          pack_bf16(dq[n][2 * r] * a.scale, dq[n][2 * r + 1] * a.scale);
    }
  }
}

// --------------------------------------------------- backward: dK, dV pass
// One CTA per (64 keys, batch, head); warp w owns 16 keys.  Query blocks of
// 32 rows stream through a double-buffered pipeline (Q and dO tiles).
constexpr int KV_BN = 64, KV_BM = 32, KV_THREADS = 128;
constexpr int KV_SMEM = (2 * KV_BN + 4 * KV_BM) * ROW_BYTES;  // K, V + 2 x (Q, dO)

__global__ void __launch_bounds__(KV_THREADS) attn_bwd_dkdv_kernel(const AttnArgs a) {
  extern __shared__ __align__(128) uint8_t sm[];
  const uint32_t sK = saddr(sm);
  const uint32_t sV = sK + KV_BN * ROW_BYTES;
  const uint32_t sQ[2] = {sK + 2 * KV_BN * ROW_BYTES, sK + (2 * KV_BN + 2 * KV_BM) * ROW_BYTES};
  const uint32_t sdO[2] = {sK + (2 * KV_BN + KV_BM) * ROW_BYTES,
                           sK + (2 * KV_BN + 3 * KV_BM) * ROW_BYTES};
  __shared__ float s_lse2[2][KV_BM], s_ds[2][KV_BM];

  const int nkb = (a.s + KV_BN - 1) / KV_BN;
  const int kb = static_cast<int>(blockIdx.x);  // early keys see the most queries: run them first
  const int head = blockIdx.y % a.heads, bi = blockIdx.y / a.heads;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long ld = 3LL * a.h;
  const __half* base = a.qkv + static_cast<long long>(bi) * a.s * ld;
  const __half* dbase = a.dout + static_cast<long long>(bi) * a.s * a.h;
  const long long stat = (static_cast<long long>(bi) * a.heads + head) * a.s;
  const int k0 = kb * KV_BN;
  const int qb_first = a.causal ? k0 / KV_BM : 0;
  const int nqb = (a.s + KV_BM - 1) / KV_BM;
  (void)nkb;

  load_tile<KV_BN, KV_THREADS>(sK, base, ld, k0, a.s, a.h + head * D);
  load_tile<KV_BN, KV_THREADS>(sV, base, ld, k0, a.s, 2 * a.h + head * D);
  auto load_q = [&](int qb, int buf) {
    load_tile<KV_BM, KV_THREADS>(sQ[buf], base, ld, qb * KV_BM, a.s, head * D);
    load_tile<KV_BM, KV_THREADS>(sdO[buf], dbase, a.h, qb * KV_BM, a.s, head * D);
    if (threadIdx.x < KV_BM) {
      const int r = min(qb * KV_BM + static_cast<int>(threadIdx.x), a.s - 1);
      s_lse2[buf][threadIdx.x] = a.lse[stat + r] * kLog2e;
      s_ds[buf][threadIdx.x] = a.dsum[stat + r];
    }
  };
  load_q(qb_first, 0);
  cp_commit();

  const int g = lane >> 2, tq = lane & 3;
  const int key_a = k0 + warp * 16 + g;  // keys of c0/c1 rows; c2/c3 at key_a + 8
  float dk[16][4], dv[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.0f;

  for (int qb = qb_first; qb < nqb; ++qb) {
    const int buf = (qb - qb_first) & 1;
    if (qb + 1 < nqb) {
      __syncthreads();  // the statistics buffer being refilled is no longer read
      load_q(qb + 1, buf ^ 1);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();

    // S^T = K Q^T and dP^T = V dO^T for this warp's 16 keys x 32 queries.
    float st[4][4], dpt[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[j][e] = dpt[j][e] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ak[4], av[4];
      lda(sK, warp * 16, kk, lane, ak);
      lda(sV, warp * 16, kk, lane, av);
#pragma unroll
      for (int j = 0; j < 4; j += 2) {
        uint32_t bq[4], bd[4];
        ldb_nk(sQ[buf], j * 8, kk, lane, bq);
        ldb_nk(sdO[buf], j * 8, kk, lane, bd);
        mma16816(st[j], ak[0], ak[1], ak[2], ak[3], bq[0], bq[1]);
        mma16816(st[j + 1], ak[0], ak[1], ak[2], ak[3], bq[2], bq[3]);
        mma16816(dpt[j], av[0], av[1], av[2], av[3], bd[0], bd[1]);
        mma16816(dpt[j + 1], av[0], av[1], av[2], av[3], bd[2], bd[3]);
      }
    }
    // P^T and dS^T (columns are queries).
    const int qrow0 = qb * KV_BM;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ql = j * 8 + 2 * tq + (e & 1);
        const int q = qrow0 + ql;
        const int key = key_a + ((e >> 1) << 3);
        const bool masked = q >= a.s || key >= a.s || (a.causal && key > q);
        const float p = masked ? 0.0f : exp2f(st[j][e] * a.scale_log2 - s_lse2[buf][ql]);
        st[j][e] = p;
        dpt[j][e] = p * (dpt[j][e] - s_ds[buf][ql]);
      }
    }
    // dV += P^T dO and dK += dS^T Q (dO, Q stored [query][d]: k = query rows).
#pragma unroll
    for (int kk = 0; kk < KV_BM / 16; ++kk) {
      const uint32_t p0 = pack_f16(st[2 * kk][0], st[2 * kk][1]);
      const uint32_t p1 = pack_f16(st[2 * kk][2], st[2 * kk][3]);
      const uint32_t p2 = pack_f16(st[2 * kk + 1][0], st[2 * kk + 1][1]);
      const uint32_t p3 = pack_f16(st[2 * kk + 1][2], st[2 * kk + 1][3]);
      const uint32_t s0 = pack_f16(dpt[2 * kk][0], dpt[2 * kk][1]);
      const uint32_t s1 = pack_f16(dpt[2 * kk][2], dpt[2 * kk][3]);
      const uint32_t s2 = pack_f16(dpt[2 * kk + 1][0], dpt[2 * kk + 1][1]);
      const uint32_t s3 = pack_f16(dpt[2 * kk + 1][2], dpt[2 * kk + 1][3]);
#pragma unroll
      for (int n = 0; n < 16; n += 2) {
        uint32_t bd[4], bq[4];
        ldb_kn(sdO[buf], kk * 16, n * 8, lane, bd);
        ldb_kn(sQ[buf], kk * 16, n * 8, lane, bq);
        mma16816(dv[n], p0, p1, p2, p3, bd[0], bd[1]);
        mma16816(dv[n + 1], p0, p1, p2, p3, bd[2], bd[3]);
        mma16816(dk[n], s0, s1, s2, s3, bq[0], bq[1]);
        mma16816(dk[n + 1], s0, s1, s2, s3, bq[2], bq[3]);
      }
    }
  }

#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int key = key_a + 8 * r;
    if (key >= a.s) continue;
    __nv_bfloat16* row = a.out + (static_cast<long long>(bi) * a.s + key) * (3LL * a.h);
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      const int col = n * 8 + 2 * tq;
      *reinterpret_cast<uint32_t*>(row + a.h + head * D + col) =
          pack_bf16(dk[n][2 * r] * a.scale, dk[n][2 * r + 1] * a.scale);
      *reinterpret_cast<uint32_t*>(row + 2 * a.h + head * D + col) =
          pack_bf16(dv[n][2 * r], dv[n][2 * r + 1]);
    }
  }
}

template <typename K>
cudaError_t set_smem(K kern, int bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// Algorithmic FLOPs of the forward core: Q K^T and P V over the unmasked
// score pairs (s^2 / 2 per head under the causal mask), 2d FLOPs each.
double core_flops(const AttnShape& sh) {
  const double pairs = sh.causal ? 0.5 * double(sh.s) * sh.s : double(sh.s) * sh.s;
  return 4.0 * D * pairs * double(sh.b) * sh.heads;
}

AttnArgs base_args(const AttnShape& sh) {
  AttnArgs a{};
  a.s = static_cast<int>(sh.s);
  a.h = static_cast<int>(sh.h);
  a.heads = sh.heads;
  a.causal = sh.causal;
  a.scale = 1.0f / std::sqrt(static_cast<float>(D));
  a.scale_log2 = a.scale * kLog2e;
  return a;
}

}  // namespace

tp_status launch_attn_core_fwd(const AttnShape& sh, const void* QKV, void* O, float* LSE,
                               cudaStream_t stream) {
  return launch_attn_core_fwd_tc(sh, QKV, O, LSE, stream);
}

size_t attn_core_bwd_scratch_bytes(const AttnShape& sh) {
  return static_cast<size_t>(sh.b * sh.s) * static_cast<size_t>(sh.heads) * sizeof(float);
}

tp_status launch_attn_core_bwd(const AttnShape& sh, const void* QKV, const void* O,
                               const float* LSE, const void* dO, void* dQKV, void* scratch,
                               cudaStream_t stream) {
  if (sh.h / sh.heads != D) return fail(TP_ERR_UNSUPPORTED, "attention: head dimension must be 128");
  if (sh.b * sh.heads > 65535) return fail(TP_ERR_SHAPE, "attention: b * heads too large");
  AttnArgs a = base_args(sh);
  a.qkv = static_cast<const __half*>(QKV);
  a.o = static_cast<const __nv_bfloat16*>(O);
  a.dout = static_cast<const __half*>(dO);
  a.lse = LSE;
  float* dsum = static_cast<float*>(scratch);
  a.dsum = dsum;
  a.out = static_cast<__nv_bfloat16*>(dQKV);
  const long long M = sh.b * sh.s;
  const long long warps = M * sh.heads;
  LaunchScope scope(TP_KIND_ATTN_BWD, 2.5 * core_flops(sh), 2.0 * double(M) * 8 * sh.h, stream,
                    3);
  attn_bwd_dsum_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, stream>>>(a, dsum, M);
  cudaError_t e = set_smem(attn_bwd_dq_kernel, DQ_SMEM);
  if (e == cudaSuccess) e = set_smem(attn_bwd_dkdv_kernel, KV_SMEM);
  if (e != cudaSuccess) return cuda_fail(e, "attention bwd smem attribute");
  dim3 gq(static_cast<unsigned>((sh.s + DQ_BM - 1) / DQ_BM), static_cast<unsigned>(sh.b * sh.heads));
  attn_bwd_dq_kernel<<<gq, DQ_THREADS, DQ_SMEM, stream>>>(a);
  dim3 gk(static_cast<unsigned>((sh.s + KV_BN - 1) / KV_BN), static_cast<unsigned>(sh.b * sh.heads));
  attn_bwd_dkdv_kernel<<<gk, KV_THREADS, KV_SMEM, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention bwd launch");
  return TP_OK;
}

}  // namespace tp
