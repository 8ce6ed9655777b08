// tcgen05 GEMM for sm_100a: D[M,N] = sum_k A(m,k) B(k,n), bf16 inputs,
// fp32 accumulation in tensor memory, fused epilogue, bf16 or fp32 output.
//
// This one kernel carries every contraction of the partitioned layer:
// * column-split linears ("图解Transformer并行计算" §1.2, §2.1 step 1): the
//   column tiles are laid out shard by shard, so no tile straddles two
//   shards, and each shard's tiles write its own column slice of the output;
//   the concatenation (the pages' All-Gather) is the output layout itself.
// * row-split linears (same page, §1.1, §2.1 step 3): the K loop walks the
//   shards' K ranges in order and every partial product lands in the same
//   tensor-memory accumulator, so the sum of partials (the pages' AllReduce)
//   costs no memory traffic and no extra pass.
// * the backward mirror (same page, §2.2, §3.2): dgrad GEMMs read the weight
//   K-major (B^T without a transpose in memory), wgrad GEMMs read both
//   operands MN-major (X^T, H^T likewise).
//
// Structure (one CTA per SM, persistent over output tiles of 128 x BN):
//   warp 0      one thread issues TMA loads of A/B K-blocks (64 deep) into a
//               ring of shared-memory stages (128-byte swizzle);
//   warp 1      allocates tensor memory; one thread issues tcgen05.mma
//               (128 x BN x 16 each) into one of two accumulator buffers;
//   warps 4-11  epilogue: tcgen05.ld the accumulator (warp w reads lanes
//               32*(w%4)..+31, i.e. one output row per thread), apply
//               bias / GeLU / GeLU' in fp32 and store; the other buffer is
//               being filled meanwhile.  Two-byte outputs go through a
//               32 x 32 shared-memory box per warp and a TMA store (whole
//               128-byte lines, four shared-memory wavefronts per 512 bytes
//               instead of one per row), and the operand the epilogue reads
//               (Y for GeLU', the residual) arrives the same way, so the
//               epilogue leaves the shared-memory datapath to the tensor
//               core's operand reads.
// Every wait is bounded (see mbar_wait): on expiry the kernel records an
// error code in the device status word and unwinds.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "ptx_sm100.cuh"
#include "tp_internal.h"

namespace tp {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 384;
constexpr int kEpiWarps = 8;
constexpr int kFirstEpiWarp = 4;

// Epilogue staging: per epilogue warp two boxes of 32 rows x 32 two-byte
// columns (64-byte rows, 64-byte swizzle).
constexpr int kEpiBoxBytes = 32 * 64;
constexpr int kEpiStageBytes = kEpiWarps * 2 * kEpiBoxBytes;  // 32 KB
constexpr int kBarBytes = 256;

template <int BN>
struct Cfg {
  static constexpr int kStages = (BN == 128) ? 6 : 4;
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kTmemCols = (2 * BN > 256) ? 512 : 256;  // a power of two
  static constexpr int kSmemBytes =
      1024 + kStages * (kABytes + kBBytes) + kEpiStageBytes + kBarBytes;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

// Shared-memory layout of a single-SM kernel: the operand ring, the epilogue
// staging boxes, the aux boxes fetched ahead, the barriers.
// * Epilogues that read an operand (`aux`: Y for GeLU', the residual) fetch
//   it one 32-column chunk ahead into two more boxes per epilogue warp where
//   shared memory has room for them (BN = 192: four 40 KB stages), so the
//   fetch of the next chunk's rows overlaps the current chunk instead of
//   being waited for at the start of every chunk; elsewhere the aux rows
//   come into the output box at the start of their own chunk.
// * Epilogues with one output and no aux need one staging box per warp; at
//   BN = 192 the 16 KB this frees and the spare room hold a fifth 40 KB
//   stage, so more operand bytes are in flight per SM.
template <int BN, int EPI>
struct Layout {
  static constexpr bool kAux = (EPI == kEpiResidual || EPI == kEpiDGelu);
  static constexpr bool kOut2 = (EPI == kEpiBiasGelu || EPI == kEpiDGelu);
  static constexpr bool kAhead = BN == 192 && kAux;
  static constexpr bool kOneBox = BN == 192 && !kAux && !kOut2;
  static constexpr int kStages = kOneBox ? 5 : Cfg<BN>::kStages;
  static constexpr int kBoxes = kOneBox ? 1 : 2;  // output boxes per epilogue warp
  static constexpr int kBoxBytes = kEpiWarps * kBoxes * kEpiBoxBytes;
  static constexpr int kAuxBytes = kAhead ? kEpiWarps * 2 * kEpiBoxBytes : 0;
  static constexpr int kBars = kAhead ? 2 * kEpiWarps : kEpiWarps;
  static constexpr int kSmemBytes = 1024 + kStages * (Cfg<BN>::kABytes + Cfg<BN>::kBBytes) +
                                    kBoxBytes + kAuxBytes + kBarBytes;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static_assert((4 + 2 * kStages + kBars) * 8 + 8 <= kBarBytes, "barrier area");
};

struct Args {
  int M, N, K;
  int m_tiles, n_tiles, k_blocks, group_m;
  int n_shard, n_tiles_per_shard;
  int kr_range_blocks, kr_t, kr_width, kr_h;
  void* out;
  long long ldo;
  const void* bias;
  __nv_bfloat16* out2;
  long long ldo2;
  const __nv_bfloat16* aux;
  long long ldaux;
  float2* ce_part;
  long long ce_ldp;
  int ce_cps;
  const int* ce_target;
  float* ce_tlogit;
  // Work units: tiles [0, tail0) whole; each later tile split into
  // tail_split slices of its K blocks, whose fp32 partial tiles go to
  // tail_part; the CTA that stores a tile's last slice adds them (slice
  // order) and applies the epilogue (tail_ctr: one arrival counter per split
  // tile, per CTA of a pair).
  int units, tail0, tail_split;
  float* tail_part;
  unsigned long long* tail_ctr;
  // Whole 32-column chunks of a two-byte output go through the shared-memory
  // boxes and the tensor maps tmO (out), tmO2 (out2) and tmX (aux).
  int tma_out;
  // kEpiDGelu only: column sums of the output (fp32, before rounding) per
  // 32-row group, csum_part[(row / 32) * csum_ld + col]; nullptr: none.
  float* csum_part;
  long long csum_ld;
  WaitCtl status;
};

struct Unit {
  int tile, kb0, kb1;
  int part;  // index of the partial tile, -1 for a whole tile
};

__host__ __device__ __forceinline__ Unit unit_of(int u, const Args& a) {
  Unit w;
  if (u < a.tail0) {
    w.tile = u;
    w.kb0 = 0;
    w.kb1 = a.k_blocks;
    w.part = -1;
  } else {
    const int v = u - a.tail0;
    const int ks = v % a.tail_split;
    w.tile = a.tail0 + v / a.tail_split;
    w.kb0 = ks * a.k_blocks / a.tail_split;
    w.kb1 = (ks + 1) * a.k_blocks / a.tail_split;
    w.part = v;
  }
  return w;
}

// 32 fp32 accumulator values of one row into a partial tile (row-major,
// `ld` floats per row).
// A split tile's fp32 partial of TM x TN is laid out as [TN / 4][TM][4]
// (four columns of one row together, rows next to each other), so a warp,
// whose lanes hold 32 consecutive rows, stores and loads 512 contiguous
// bytes per instruction.  Columns [cl, cl + 32) of row lrow:
template <int TM>
__device__ __forceinline__ void store_partial32(const float (&v)[32], float* slice, int lrow,
                                                int cl) {
  float4* d = reinterpret_cast<float4*>(slice) + (cl >> 2) * TM + lrow;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    d[i * TM] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

struct TileCoord {
  int m0, n0, n_end;
};

// Grouped raster: bands of group_m row tiles; inside a band the row tile
// varies fastest, so the CTAs running at one time share B tiles and the
// band's A rows stay in L2.
template <int BN>
__host__ __device__ __forceinline__ TileCoord tile_coord(int tile, const Args& a) {
  const int band = a.group_m * a.n_tiles;
  const int g = tile / band;
  const int first_m = g * a.group_m;
  const int gm = min(a.m_tiles - first_m, a.group_m);
  const int local = tile - g * band;
  const int mt = first_m + local % gm;
  const int nt = local / gm;
  TileCoord c;
  c.m0 = mt * BM;
  if (a.n_shard > 0) {
    const int sh = nt / a.n_tiles_per_shard;
    const int j = nt - sh * a.n_tiles_per_shard;
    c.n0 = sh * a.n_shard + j * BN;
    c.n_end = min(c.n0 + BN, (sh + 1) * a.n_shard);
  } else {
    c.n0 = nt * BN;
    c.n_end = min(c.n0 + BN, a.N);
  }
  return c;
}

// K coordinate (in elements) of K-block kb.
__device__ __forceinline__ int k_coord(int kb, const Args& a) {
  if (a.kr_range_blocks == 0) return kb * BK;
  const int r = kb / a.kr_range_blocks;   // range index in visiting order
  const int within = kb - r * a.kr_range_blocks;
  const int g = r / 3, which = r - 3 * (r / 3);
  return which * a.kr_h + g * a.kr_width + within * BK;
}

constexpr float kLog2e = 1.4426950408889634f;

// The standard normal distribution at x: Phi(x) = (1 + erf(x / sqrt 2)) / 2
// and phi(x) = exp(-x^2 / 2) / sqrt(2 pi), with erf by Abramowitz & Stegun,
// "Handbook of Mathematical Functions", formula 7.1.26: for z >= 0,
// erf z = 1 - t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-z^2),
// t = 1 / (1 + p z), |error| <= 1.5e-7, and erf(-z) = -erf z.  With
// z = |x| / sqrt 2 the factor exp(-z^2) is the exp(-x^2 / 2) of phi, so one
// reciprocal and one exponential give both.  GeLU(x) = x Phi(x) (the erf
// form) and GeLU'(x) = Phi(x) + x phi(x).  Two values at a time, on sm_100's
// two-wide fp32 instructions (each lane rounded as the one-wide form): on
// short-K GEMMs the epilogue's instruction issue, not the tensor core, sets
// the pace.
__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }

__device__ __forceinline__ void normal_cdf_pdf2(float2 x, float2& cdf, float2& pdf) {
  const float2 z = __fmul2_rn(make_float2(fabsf(x.x), fabsf(x.y)), f2(0.70710678118654752f));
  const float2 d = __ffma2_rn(f2(0.3275911f), z, f2(1.0f));
  const float2 t = make_float2(rcp_approx(d.x), rcp_approx(d.y));
  float2 p = __ffma2_rn(t, f2(1.061405429f), f2(-1.453152027f));
  p = __ffma2_rn(t, p, f2(1.421413741f));
  p = __ffma2_rn(t, p, f2(-0.284496736f));
  p = __ffma2_rn(t, p, f2(0.254829592f));
  const float2 poly = __fmul2_rn(t, p);
  const float2 arg = __fmul2_rn(__fmul2_rn(x, f2(-0.5f * kLog2e)), x);
  const float2 e = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));  // exp(-x^2 / 2)
  const float2 q = __fmul2_rn(__fmul2_rn(f2(0.5f), poly), e);         // (1 - erf z) / 2
  const float2 r = __fadd2_rn(f2(1.0f), make_float2(-q.x, -q.y));
  cdf = make_float2(x.x >= 0.0f ? r.x : q.x, x.y >= 0.0f ? r.y : q.y);
  pdf = __fmul2_rn(f2(0.39894228040143268f), e);
}

// GeLU on eight values, in pairs.
__device__ __forceinline__ void gelu8(float* x) {
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 v = make_float2(x[i], x[i + 1]);
    float2 cdf, pdf;
    normal_cdf_pdf2(v, cdf, pdf);
    const float2 g = __fmul2_rn(v, cdf);
    x[i] = g.x;
    x[i + 1] = g.y;
  }
}

// x *= GeLU'(y) on eight values, in pairs; with hh, also hh = GeLU(y).
__device__ __forceinline__ void dgelu8(float* x, const float* y, float* hh) {
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 v = make_float2(y[i], y[i + 1]);
    float2 cdf, pdf;
    normal_cdf_pdf2(v, cdf, pdf);
    if (hh != nullptr) {
      const float2 g = __fmul2_rn(v, cdf);
      hh[i] = g.x;
      hh[i + 1] = g.y;
    }
    const float2 r = __fmul2_rn(make_float2(x[i], x[i + 1]), __ffma2_rn(v, pdf, cdf));
    x[i] = r.x;
    x[i + 1] = r.y;
  }
}

// x += b on eight values, in pairs.
__device__ __forceinline__ void add8(float* x, const float* b) {
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 r = __fadd2_rn(make_float2(x[i], x[i + 1]), make_float2(b[i], b[i + 1]));
    x[i] = r.x;
    x[i + 1] = r.y;
  }
}

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Output element types of the epilogue.
enum Out : int { kOutBF16 = 0, kOutF32 = 1, kOutF16 = 2 };

constexpr float kF16Max = 65504.0f;

// Eight fp32 values to fp16, saturated to the finite range; returns whether
// any finite value had to be clamped.
__device__ __forceinline__ uint4 pack8_f16(float* f, bool& clamped) {
  uint4 u;
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (fabsf(f[i]) > kF16Max) {
      clamped = true;
      f[i] = copysignf(kF16Max, f[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 t = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&t);
  }
  return u;
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  uint4 u;
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 t = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&t);
  }
  return u;
}

// Applies the epilogue to 32 consecutive columns of one row and stores them.
// col_end is a multiple of 8, so each group of 8 columns is all in or all out.
template <int EPI, int OUT, bool BIAS_F32>
__device__ __forceinline__ void epilogue_row32(float (&v)[32], int row, int col0, int col_end,
                                               const Args& a) {
  if (row >= a.M) return;
  bool clamped = false;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int col = col0 + 8 * g;
    if (col + 8 > col_end) continue;
    float* x = v + 8 * g;
    if (EPI != kEpiDGelu && a.bias != nullptr) {
      float bb[8];
      if (BIAS_F32) {
        const float4* bp = reinterpret_cast<const float4*>(static_cast<const float*>(a.bias) + col);
        const float4 b0 = bp[0], b1 = bp[1];
        bb[0] = b0.x; bb[1] = b0.y; bb[2] = b0.z; bb[3] = b0.w;
        bb[4] = b1.x; bb[5] = b1.y; bb[6] = b1.z; bb[7] = b1.w;
      } else {
        unpack8(*reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.bias) + col),
                bb);
      }
      add8(x, bb);
    }
    if (EPI == kEpiResidual) {
      float rr[8];
      unpack8(*reinterpret_cast<const uint4*>(a.aux + (long long)row * a.ldaux + col), rr);
      add8(x, rr);
    }
    if (EPI == kEpiBiasGelu) {
      if (a.out2 != nullptr)
        *reinterpret_cast<uint4*>(a.out2 + (long long)row * a.ldo2 + col) = pack8(x);
      gelu8(x);
    } else if (EPI == kEpiDGelu) {
      float y[8];
      unpack8(*reinterpret_cast<const uint4*>(a.aux + (long long)row * a.ldaux + col), y);
      if (a.out2 != nullptr) {
        float hh[8];
        dgelu8(x, y, hh);
        *reinterpret_cast<uint4*>(a.out2 + (long long)row * a.ldo2 + col) = pack8(hh);
      } else {
        dgelu8(x, y, nullptr);
      }
    }
    if (OUT == kOutF32) {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(a.out) + (long long)row * a.ldo + col);
      o[0] = make_float4(x[0], x[1], x[2], x[3]);
      o[1] = make_float4(x[4], x[5], x[6], x[7]);
    } else if (OUT == kOutF16) {
      *reinterpret_cast<uint4*>(static_cast<__half*>(a.out) + (long long)row * a.ldo + col) =
          pack8_f16(x, clamped);
    } else {
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + (long long)row * a.ldo + col) =
          pack8(x);
    }
  }
  if (OUT == kOutF16 && clamped) status_flag(a.status, kFlagF16Range);
}

// Column sums of one warp's 32 rows x 32 columns (thread = row, v = its 32
// columns): five butterfly steps, after which lane c holds the sum of column
// c over the warp's rows (a fixed order, so the result is deterministic).
// Destroys v.  Every lane of the warp must call it with the same columns.
__device__ __forceinline__ float warp_colsum32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = up ? v[i] : v[i + w];
      const float keep = up ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}

// The bias gradient of a GeLU' epilogue: after the epilogue has left the
// output values of rows row0 + lane (row0 a multiple of 32) and columns
// [col0, col0 + 32) in v, adds this warp's 32-row column sums to the
// partial array (rows past M and columns past col_end count as zero).
template <int EPI>
__device__ __forceinline__ void epilogue_colsum(float (&v)[32], int row, int col0, int col_end,
                                                int lane, const Args& a) {
  if constexpr (EPI == kEpiDGelu) {
    if (a.csum_part == nullptr) return;
    if (row >= a.M) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.0f;
    }
    const float sum = warp_colsum32(v, lane);
    if (col0 + lane < col_end)
      a.csum_part[static_cast<long long>(row >> 5) * a.csum_ld + col0 + lane] = sum;
  }
}

// Byte offset of 16-byte chunk j (0-3) of row r in a 32-row x 64-byte box
// under the 64-byte swizzle (chunk index XOR address bits 7-8; the boxes are
// 1024-byte aligned).
__device__ __forceinline__ uint32_t sw64_off(int r, int j) {
  return static_cast<uint32_t>(r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}

// The bias of a warp's half tile, fetched when the tile starts (before its
// accumulator is ready): lane l holds columns [8 l, 8 l + 8) of the half
// (zeros past the tile's column range); a chunk takes its four groups from
// lanes bl0 .. bl0 + 3 by shuffles, instead of four global loads whose
// latency would open every chunk.
template <int EPI, int HALF>
__device__ __forceinline__ uint4 bias_half(const Args& a, int col0, int col_end, int lane) {
  uint4 q = make_uint4(0u, 0u, 0u, 0u);
  if (EPI != kEpiDGelu && EPI != kEpiCE && a.bias != nullptr) {
    const int col = col0 + 8 * lane;
    if (lane < HALF / 8 && col + 8 <= col_end)
      q = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.bias) + col);
  }
  return q;
}

// The epilogue of one row's 32 consecutive columns, all inside the tile's
// column range, written to the warp's staging boxes (row r of a box = this
// thread's lane): abox holds the row of `aux` for the epilogues that read
// one (it may be box0), box0 receives `out` and box1 out2.  The bias of the
// columns comes from lanes bl0 .. bl0 + 3 of the warp's bias_half `bq`.
// Rows past M are computed too and dropped by the TMA store.
template <int EPI, int OUT>
__device__ __forceinline__ void epilogue_box32(float (&v)[32], int r, uint8_t* box0,
                                               uint8_t* box1, const uint8_t* abox,
                                               const uint4& bq, int bl0, const Args& a) {
  constexpr bool kAux = (EPI == kEpiResidual || EPI == kEpiDGelu);
  bool clamped = false;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float* x = v + 8 * g;
    if (EPI != kEpiDGelu && a.bias != nullptr) {
      uint4 b;
      b.x = __shfl_sync(0xffffffffu, bq.x, bl0 + g);
      b.y = __shfl_sync(0xffffffffu, bq.y, bl0 + g);
      b.z = __shfl_sync(0xffffffffu, bq.z, bl0 + g);
      b.w = __shfl_sync(0xffffffffu, bq.w, bl0 + g);
      float bb[8];
      unpack8(b, bb);
      add8(x, bb);
    }
    float y[8];
    if (kAux) unpack8(*reinterpret_cast<const uint4*>(abox + sw64_off(r, g)), y);
    if (EPI == kEpiResidual) add8(x, y);
    if (EPI == kEpiBiasGelu) {
      if (a.out2 != nullptr) *reinterpret_cast<uint4*>(box1 + sw64_off(r, g)) = pack8(x);
      gelu8(x);
    } else if (EPI == kEpiDGelu) {
      if (a.out2 != nullptr) {
        float hh[8];
        dgelu8(x, y, hh);
        *reinterpret_cast<uint4*>(box1 + sw64_off(r, g)) = pack8(hh);
      } else {
        dgelu8(x, y, nullptr);
      }
    }
    *reinterpret_cast<uint4*>(box0 + sw64_off(r, g)) =
        (OUT == kOutF16) ? pack8_f16(x, clamped) : pack8(x);
  }
  if (OUT == kOutF16 && clamped) status_flag(a.status, kFlagF16Range);
}

// Cross-entropy epilogue on 32 consecutive columns (vocabulary entries) of
// one row: "图解Transformer并行计算" §4.2 steps 1-2 for one chunk of a
// shard.  The logits are rounded to bf16 first, so that the saved logits, the
// chunk statistics and the target logit all see the same values; the chunk's
// maximum and its sum of exp(z - max) over its valid columns go to the
// partial array.  col0 is 32-aligned within its shard and col_end - col0 is
// a multiple of 8.  With a staging box (whole chunks only) the logits go to
// row `r` of the box instead of global memory.
__device__ __forceinline__ void epilogue_ce32(float (&v)[32], int row, int col0, int col_end,
                                              int tg, const Args& a, uint8_t* box = nullptr,
                                              int r = 0) {
  if (row >= a.M) return;
  const int nv = min(32, col_end - col0);
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
    if (i < nv) mx = fmaxf(mx, v[i]);
  }
  if (box != nullptr) {
#pragma unroll
    for (int g = 0; g < 4; ++g) *reinterpret_cast<uint4*>(box + sw64_off(r, g)) = pack8(v + 8 * g);
  } else if (a.out != nullptr) {
#pragma unroll
    for (int g = 0; g < 4; ++g)
      if (8 * g < nv)
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + (long long)row * a.ldo +
                                  col0 + 8 * g) = pack8(v + 8 * g);
  }
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (i < nv) s += exp2f((v[i] - mx) * kLog2e);
  const int sh = col0 / a.n_shard;
  const int j = (col0 - sh * a.n_shard) >> 5;
  a.ce_part[(long long)row * a.ce_ldp + (long long)sh * a.ce_cps + j] = make_float2(mx, s);
  if (tg >= col0 && tg < col0 + nv) {
    // v[tg - col0] by a select tree on the index bits (keeps v in registers).
    const int idx = tg - col0;
    float w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = (idx & 16) ? v[i + 16] : v[i];
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = (idx & 8) ? w[i + 8] : w[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = (idx & 4) ? w[i + 4] : w[i];
#pragma unroll
    for (int i = 0; i < 2; ++i) w[i] = (idx & 2) ? w[i + 2] : w[i];
    a.ce_tlogit[row] = (idx & 1) ? w[1] : w[0];
  }
}

// One 32-column chunk of a whole tile through the warp's staging boxes:
// wait until the previous chunk's TMA stores have read the boxes, fetch the
// aux rows (TMA, counted on the warp's own barrier) while the accumulator
// is read from tensor memory, apply the epilogue into the boxes and store
// them with TMA.  Rows row0..row0+31 of the output are this warp's lanes.
// Returns false if the wait for the aux box gave up.
template <int EPI, int OUT>
__device__ __forceinline__ bool epilogue_chunk_boxed(uint32_t taddr, int lane, int row, int row0,
                                                     int col, int col_end, int tg, uint8_t* box0,
                                                     uint8_t* box1, uint64_t* auxbar,
                                                     uint32_t& aux_phase, const CUtensorMap* tmO,
                                                     const CUtensorMap* tmO2,
                                                     const CUtensorMap* tmX, const uint4& bq,
                                                     int bl0, const Args& a) {
  constexpr bool kAux = (EPI == kEpiResidual || EPI == kEpiDGelu);
  constexpr bool kOut2 = (EPI == kEpiBiasGelu || EPI == kEpiDGelu);
  if (lane == 0) bulk_wait_read<0>();
  __syncwarp();
  if (kAux && lane == 0) {
    mbar_arrive_expect_tx(auxbar, kEpiBoxBytes);
    tma_load_2d(box0, tmX, auxbar, col, row0);
  }
  float v[32];
  tmem_ld32(taddr, v);
  if (kAux) {
    const bool got = mbar_wait(auxbar, aux_phase, a.status, kStatusEpilogueTimeout);
    aux_phase ^= 1u;
    if (!__all_sync(0xffffffffu, got)) return false;
  }
  if constexpr (EPI == kEpiCE)
    epilogue_ce32(v, row, col, col_end, tg, a, box0, lane);
  else
    epilogue_box32<EPI, OUT>(v, lane, box0, box1, box0, bq, bl0, a);
  epilogue_colsum<EPI>(v, row, col, col_end, lane, a);
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmO, box0, col, row0);
    if (kOut2 && a.out2 != nullptr) tma_store_2d(tmO2, box1, col, row0);
    bulk_commit();
  }
  return true;
}

// One 32-column chunk of a whole tile for an epilogue that reads `aux`,
// whose rows were requested earlier into `abox` (counted on `abar`, wait
// parity `aphase`): as epilogue_chunk_boxed, without fetching them here.
// Returns false if the wait for the aux box gave up.
template <int EPI, int OUT>
__device__ __forceinline__ bool epilogue_chunk_ahead(uint32_t taddr, int lane, int row, int row0,
                                                     int col, int col_end, uint8_t* box0,
                                                     uint8_t* box1, const uint8_t* abox,
                                                     uint64_t* abar, uint32_t aphase,
                                                     const CUtensorMap* tmO,
                                                     const CUtensorMap* tmO2, const uint4& bq,
                                                     int bl0, const Args& a) {
  constexpr bool kOut2 = (EPI == kEpiBiasGelu || EPI == kEpiDGelu);
  if (lane == 0) bulk_wait_read<0>();
  __syncwarp();
  float v[32];
  tmem_ld32(taddr, v);
  const bool got = mbar_wait(abar, aphase, a.status, kStatusEpilogueTimeout);
  if (!__all_sync(0xffffffffu, got)) return false;
  epilogue_box32<EPI, OUT>(v, lane, box0, box1, abox, bq, bl0, a);
  epilogue_colsum<EPI>(v, row, col, col_end, lane, a);
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmO, box0, col, row0);
    if (kOut2 && a.out2 != nullptr) tma_store_2d(tmO2, box1, col, row0);
    bulk_commit();
  }
  return true;
}

// The final pass over a split tile, run by the CTA that stored its last
// slice: each epilogue thread adds its row's 32-column chunks of the
// tile's slices in slice order (L2 loads: other SMs wrote them) and applies
// the epilogue, as a whole tile's epilogue would; `lrow` is the row within
// the TM x TN partial tile, `half` the epilogue warp's half of the columns.
template <int TM, int TN, int EPI, int OUT>
__device__ __forceinline__ void tail_finish(const Args& a, const TileCoord& tc, int ti, int lrow,
                                            int row, int half, int lane) {
  const float* base = a.tail_part + static_cast<long long>(ti) * a.tail_split * TM * TN;
#pragma unroll 1
  for (int c = 0; c < TN / 2; c += 32) {
    const int cl = half * (TN / 2) + c;
    const int col = tc.n0 + cl;
    if (col >= tc.n_end) break;  // warp-uniform
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0.0f;
#pragma unroll 2
    for (int ks = 0; ks < a.tail_split; ++ks) {
      const float4* src = reinterpret_cast<const float4*>(base + static_cast<long long>(ks) * TM * TN) +
                          (cl >> 2) * TM + lrow;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 q = __ldcg(src + i * TM);
        v[4 * i] += q.x;
        v[4 * i + 1] += q.y;
        v[4 * i + 2] += q.z;
        v[4 * i + 3] += q.w;
      }
    }
    epilogue_row32<EPI, OUT, false>(v, row, col, tc.n_end, a);
    epilogue_colsum<EPI>(v, row, col, tc.n_end, lane, a);
  }
}

// After a CTA's epilogue warps stored their parts of a slice of split tile
// ti (counter slot `slot`): the last CTA to do so for that tile finishes it
// and clears the counter, so that a CUDA graph replaying this launch (the
// same generation baked into its arguments) counts from zero again.
// Called by all epilogue warps of the CTA together (named barrier 1).
template <int TM, int TN, int EPI, int OUT>
__device__ __forceinline__ void tail_arrive(const Args& a, const TileCoord& tc, int ti, int slot,
                                            int lrow, int row, int half, int lane, int ew,
                                            int* flag) {
  __threadfence();
  named_sync(1, kEpiWarps * 32);
  if (ew == 0 && lane == 0) {
    const bool last = gen_ticket(a.tail_ctr + slot, a.status.gen, a.tail_split);
    if (last) atomicExch(a.tail_ctr + slot, 0ull);
    *flag = last ? 1 : 0;
  }
  named_sync(1, kEpiWarps * 32);
  if (*reinterpret_cast<volatile int*>(flag)) {
    __threadfence();
    tail_finish<TM, TN, EPI, OUT>(a, tc, ti, lrow, row, half, lane);
  }
}

template <int BN, bool A_KMAJ, bool B_KMAJ, int EPI, int OUT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_bf16_tcgen05(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmO,
                      const __grid_constant__ CUtensorMap tmO2,
                      const __grid_constant__ CUtensorMap tmX, const Args args) {
  using C = Cfg<BN>;
  using LY = Layout<BN, EPI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + LY::kStages * C::kABytes;
  uint8_t* sE = sB + LY::kStages * C::kBBytes;  // epilogue boxes, 1024-byte aligned
  uint8_t* sX = sE + LY::kBoxBytes;             // aux boxes fetched ahead (LY::kAhead)
  uint64_t* full = reinterpret_cast<uint64_t*>(sX + LY::kAuxBytes);
  uint64_t* empty = full + LY::kStages;
  uint64_t* tfull = empty + LY::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* auxbar = tempty + 2;  // one (two with LY::kAhead) per epilogue warp
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(auxbar + LY::kBars);
  int* tail_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < LY::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiWarps);
    }
    for (int i = 0; i < LY::kBars; ++i) mbar_init(&auxbar[i], 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (args.tma_out) tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
        const Unit w = unit_of(u, args);
        const TileCoord tc = tile_coord<BN>(w.tile, args);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, args.status, kStatusProducerTimeout)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::kABytes + C::kBBytes);
          const int kc = k_coord(kb, args);
          uint8_t* a_dst = sA + stage * C::kABytes;
          uint8_t* b_dst = sB + stage * C::kBBytes;
          if (A_KMAJ) {
            tma_load_2d(a_dst, &tmA, &full[stage], kc, tc.m0);
          } else {
#pragma unroll
            for (int c = 0; c < BM / 64; ++c)
              tma_load_2d(a_dst + c * (BK * 128), &tmA, &full[stage], tc.m0 + 64 * c, kc);
          }
          if (B_KMAJ) {
            tma_load_2d(b_dst, &tmB, &full[stage], kc, tc.n0);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_2d(b_dst + c * (BK * 128), &tmB, &full[stage], tc.n0 + 64 * c, kc);
          }
          if (++stage == LY::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t kIdesc = idesc_bf16_f32(BM, BN, !A_KMAJ, !B_KMAJ);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
        const Unit w = unit_of(u, args);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, args.status, kStatusMmaTimeout)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, args.status, kStatusMmaTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::kABytes);
          const uint32_t b0 = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = A_KMAJ ? sw128_desc(a0 + k * 32, 16, 1024)
                                       : sw128_desc(a0 + k * 2048, BK * 128, 1024);
            const uint64_t bd = B_KMAJ ? sw128_desc(b0 + k * 32, 16, 1024)
                                       : sw128_desc(b0 + k * 2048, BK * 128, 1024);
            umma_bf16(d_tmem, ad, bd, kIdesc, (kb != w.kb0 || k != 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == LY::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else if (warp >= kFirstEpiWarp) {
    // -------------------------------------------------------- epilogue
    const int ew = warp - kFirstEpiWarp;
    const int quarter = warp & 3;  // tensor-memory lanes this warp may read
    const int half = ew >> 2;      // which half of the tile's columns
    uint8_t* box0 = sE + ew * (LY::kBoxes * kEpiBoxBytes);
    uint8_t* box1 = box0 + (LY::kBoxes - 1) * kEpiBoxBytes;  // box0 when there is one
    uint32_t aux_phase = 0;
    // Aux fetched ahead (LY::kAhead): the chunk (unit ax_u, column offset ax_c)
    // whose rows are on their way into aux box ax_slot (ax_u < 0: none);
    // ax_par holds each box's wait parity.
    uint8_t* xbox = sX + ew * (2 * kEpiBoxBytes);
    int ax_u = -1, ax_c = 0, ax_slot = 0;
    uint32_t ax_par = 0;
    auto ax_fetch = [&](int slot, int col, int row0) {
      if (lane == 0) {
        mbar_arrive_expect_tx(&auxbar[2 * ew + slot], kEpiBoxBytes);
        tma_load_2d(xbox + slot * kEpiBoxBytes, &tmX, &auxbar[2 * ew + slot], col, row0);
      }
    };
    bool ok = true;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
      const Unit w = unit_of(u, args);
      const TileCoord tc = tile_coord<BN>(w.tile, args);
      const uint4 bq = bias_half<EPI, BN / 2>(args, tc.n0 + half * (BN / 2), tc.n_end, lane);
      if (!mbar_wait(&tfull[acc], acc_phase, args.status, kStatusEpilogueTimeout)) break;
      tc_fence_after();
      const int lrow = quarter * 32 + lane;
      const int row = tc.m0 + lrow;
      const int tg = (EPI == kEpiCE && row < args.M) ? args.ce_target[row] : -1;
#pragma unroll 1
      for (int c = 0; c < BN / 2; c += 32) {
        const int cl = half * (BN / 2) + c;
        const int col = tc.n0 + cl;
        if (col >= tc.n_end) break;  // warp-uniform
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                               static_cast<uint32_t>(acc * BN + cl);
        if constexpr (OUT != kOutF32) {
          if (args.tma_out && w.part < 0 && col + 32 <= tc.n_end) {
            if constexpr (LY::kAhead) {
              // This chunk's aux rows: requested by the previous chunk, else now.
              const int slot = ax_slot;
              if (ax_u != u || ax_c != c) ax_fetch(slot, col, tc.m0 + quarter * 32);
              // Request the next chunk's: the next one of this tile, or the
              // first one of this CTA's next unit.
              ax_u = -1;
              if (c + 32 < BN / 2) {
                if (col + 64 <= tc.n_end) {
                  ax_fetch(slot ^ 1, col + 32, tc.m0 + quarter * 32);
                  ax_u = u;
                  ax_c = c + 32;
                }
              } else if (u + static_cast<int>(gridDim.x) < args.units) {
                const int un = u + static_cast<int>(gridDim.x);
                const Unit wn = unit_of(un, args);
                const TileCoord tn = tile_coord<BN>(wn.tile, args);
                const int coln = tn.n0 + half * (BN / 2);
                if (wn.part < 0 && coln + 32 <= tn.n_end) {
                  ax_fetch(slot ^ 1, coln, tn.m0 + quarter * 32);
                  ax_u = un;
                  ax_c = 0;
                }
              }
              ax_slot = slot ^ 1;
              ok = epilogue_chunk_ahead<EPI, OUT>(
                  taddr, lane, row, tc.m0 + quarter * 32, col, tc.n_end, box0, box1,
                  xbox + slot * kEpiBoxBytes, &auxbar[2 * ew + slot], (ax_par >> slot) & 1u,
                  &tmO, &tmO2, bq, c / 8, args);
              ax_par ^= 1u << slot;
            } else {
              ok = epilogue_chunk_boxed<EPI, OUT>(taddr, lane, row, tc.m0 + quarter * 32, col,
                                                  tc.n_end, tg, box0, box1, &auxbar[ew],
                                                  aux_phase, &tmO, &tmO2, &tmX, bq, c / 8, args);
            }
            if (!ok) break;
            continue;
          }
        }
        float v[32];
        tmem_ld32(taddr, v);
        if (w.part >= 0)  // a K slice of a tail tile: raw partial sums
          store_partial32<BM>(v, args.tail_part + static_cast<long long>(w.part) * BM * BN, lrow, cl);
        else if constexpr (EPI == kEpiCE)
          epilogue_ce32(v, row, col, tc.n_end, tg, args);
        else {
          epilogue_row32<EPI, OUT, false>(v, row, col, tc.n_end, args);
          epilogue_colsum<EPI>(v, row, col, tc.n_end, lane, args);
        }
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (w.part >= 0)
        tail_arrive<BM, BN, EPI, OUT>(args, tc, w.tile - args.tail0, w.tile - args.tail0, lrow,
                                      row, half, lane, ew, tail_flag);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    // An aux fetch still in flight (only after a wait gave up): let it land
    // before the CTA's shared memory goes away.
    if (LY::kAhead && ax_u >= 0)
      mbar_wait(&auxbar[2 * ew + ax_slot], (ax_par >> ax_slot) & 1u, args.status,
                kStatusEpilogueTimeout);
    if (lane == 0) bulk_wait<0>();  // this warp's TMA stores have landed
  }

  __syncwarp();  // lane 0 of the producer / MMA warps rejoins its warp
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}


// ------------------------------------------------------- two-SM (CTA pair)
// The same GEMM on 256 x 256 output tiles computed by a pair of CTAs on two
// SMs with tcgen05.mma.cta_group::2: each CTA loads 128 rows of the A tile
// and 128 columns of the B tile (a plain TMA load into its own shared memory,
// counted on the even CTA's barrier); one thread of the even CTA issues the
// 256 x 256 x 16 MMAs; each CTA's tensor memory receives its 128 output rows.
// Per SM this halves the B bytes pulled from L2 per FLOP.
constexpr int kPairStages = 6;
constexpr int kPairABytes = 128 * BK * 2;  // 16 KB: this CTA's half of A
constexpr int kPairBBytes = 128 * BK * 2;  // 16 KB: this CTA's half of B
constexpr int kPairSmemBytes =
    1024 + kPairStages * (kPairABytes + kPairBBytes) + kEpiStageBytes + kBarBytes;
static_assert(kPairSmemBytes <= 232448, "shared memory per CTA");
constexpr int kPairTM = 256, kPairTN = 256;

__host__ __device__ __forceinline__ TileCoord tile_coord_pair(int tile, const Args& a) {
  const int band = a.group_m * a.n_tiles;
  const int g = tile / band;
  const int first_m = g * a.group_m;
  const int gm = min(a.m_tiles - first_m, a.group_m);
  const int local = tile - g * band;
  const int mt = first_m + local % gm;
  const int nt = local / gm;
  TileCoord c;
  c.m0 = mt * kPairTM;
  if (a.n_shard > 0) {
    const int sh = nt / a.n_tiles_per_shard;
    const int j = nt - sh * a.n_tiles_per_shard;
    c.n0 = sh * a.n_shard + j * kPairTN;
    c.n_end = min(c.n0 + kPairTN, (sh + 1) * a.n_shard);
  } else {
    c.n0 = nt * kPairTN;
    c.n_end = min(c.n0 + kPairTN, a.N);
  }
  return c;
}

template <bool A_KMAJ, bool B_KMAJ, int EPI, int OUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_bf16_tcgen05_pair(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmO,
                           const __grid_constant__ CUtensorMap tmO2,
                           const __grid_constant__ CUtensorMap tmX, const Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPairStages * kPairABytes;
  uint8_t* sE = sB + kPairStages * kPairBBytes;  // epilogue boxes, 1024-byte aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(sE + kEpiStageBytes);
  uint64_t* empty = full + kPairStages;
  uint64_t* tfull = empty + kPairStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* auxbar = tempty + 2;  // one per epilogue warp
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(auxbar + kEpiWarps);
  int* tail_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs, 1: its peer
  const uint32_t peer = rank ^ 1u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * kEpiWarps);  // both CTAs' epilogue warps
    }
    for (int i = 0; i < kEpiWarps; ++i) mbar_init(&auxbar[i], 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (args.tma_out) tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers initialised and tensor memory allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int cluster_id = static_cast<int>(blockIdx.x >> 1);
  const int num_clusters = static_cast<int>(gridDim.x >> 1);

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = cluster_id; u < args.units && ok; u += num_clusters) {
        const Unit w = unit_of(u, args);
        const TileCoord tc = tile_coord_pair(w.tile, args);
        const int am0 = tc.m0 + 128 * static_cast<int>(rank);
        const int bn0 = tc.n0 + 128 * static_cast<int>(rank);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, args.status, kStatusProducerTimeout)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (kPairABytes + kPairBBytes));
          const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
          const int kc = k_coord(kb, args);
          uint8_t* a_dst = sA + stage * kPairABytes;
          uint8_t* b_dst = sB + stage * kPairBBytes;
          if (A_KMAJ) {
            tma_load_2d_pair(a_dst, &tmA, bar, kc, am0);
          } else {
            tma_load_2d_pair(a_dst, &tmA, bar, am0, kc);
            tma_load_2d_pair(a_dst + BK * 128, &tmA, bar, am0 + 64, kc);
          }
          if (B_KMAJ) {
            tma_load_2d_pair(b_dst, &tmB, bar, kc, bn0);
          } else {
            tma_load_2d_pair(b_dst, &tmB, bar, bn0, kc);
            tma_load_2d_pair(b_dst + BK * 128, &tmB, bar, bn0 + 64, kc);
          }
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------- MMA issuer (even CTA only)
      constexpr uint32_t kIdesc = idesc_bf16_f32(kPairTM, kPairTN, !A_KMAJ, !B_KMAJ);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int u = cluster_id; u < args.units && ok; u += num_clusters) {
        const Unit w = unit_of(u, args);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, args.status, kStatusMmaTimeout)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kPairTN);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, args.status, kStatusMmaTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * kPairABytes);
          const uint32_t b0 = smem_u32(sB + stage * kPairBBytes);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = A_KMAJ ? sw128_desc(a0 + k * 32, 16, 1024)
                                       : sw128_desc(a0 + k * 2048, BK * 128, 1024);
            const uint64_t bd = B_KMAJ ? sw128_desc(b0 + k * 32, 16, 1024)
                                       : sw128_desc(b0 + k * 2048, BK * 128, 1024);
            umma_bf16_pair(d_tmem, ad, bd, kIdesc, (kb != w.kb0 || k != 0) ? 1u : 0u);
          }
          // Free the stage in both CTAs once these MMAs have read it.
          umma_commit_pair(mapa_shared(smem_u32(&empty[stage]), 0));
          umma_commit_pair(mapa_shared(smem_u32(&empty[stage]), 1));
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(mapa_shared(smem_u32(&tfull[acc]), 0));
        umma_commit_pair(mapa_shared(smem_u32(&tfull[acc]), 1));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else if (warp >= kFirstEpiWarp) {
    // ------------------------------------------------ epilogue (both CTAs)
    const int ew = warp - kFirstEpiWarp;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    const uint32_t tempty_leader[2] = {mapa_shared(smem_u32(&tempty[0]), 0),
                                       mapa_shared(smem_u32(&tempty[1]), 0)};
    uint8_t* box0 = sE + ew * (2 * kEpiBoxBytes);
    uint8_t* box1 = box0 + kEpiBoxBytes;
    uint32_t aux_phase = 0;
    bool ok = true;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = cluster_id; u < args.units && ok; u += num_clusters) {
      const Unit w = unit_of(u, args);
      const TileCoord tc = tile_coord_pair(w.tile, args);
      const uint4 bq =
          bias_half<EPI, kPairTN / 2>(args, tc.n0 + half * (kPairTN / 2), tc.n_end, lane);
      if (!mbar_wait(&tfull[acc], acc_phase, args.status, kStatusEpilogueTimeout)) break;
      tc_fence_after();
      const int lrow = 128 * static_cast<int>(rank) + quarter * 32 + lane;
      const int row = tc.m0 + lrow;
      const int tg = (EPI == kEpiCE && row < args.M) ? args.ce_target[row] : -1;
#pragma unroll 1
      for (int c = 0; c < kPairTN / 2; c += 32) {
        const int cl = half * (kPairTN / 2) + c;
        const int col = tc.n0 + cl;
        if (col >= tc.n_end) break;  // warp-uniform
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                               static_cast<uint32_t>(acc * kPairTN + cl);
        if constexpr (OUT != kOutF32) {
          if (args.tma_out && w.part < 0 && col + 32 <= tc.n_end) {
            ok = epilogue_chunk_boxed<EPI, OUT>(
                taddr, lane, row, tc.m0 + 128 * static_cast<int>(rank) + quarter * 32, col,
                tc.n_end, tg, box0, box1, &auxbar[ew], aux_phase, &tmO, &tmO2, &tmX, bq, c / 8,
                args);
            if (!ok) break;
            continue;
          }
        }
        float v[32];
        tmem_ld32(taddr, v);
        if (w.part >= 0)  // a K slice of a tail tile: raw partial sums
          store_partial32<kPairTM>(
              v, args.tail_part + static_cast<long long>(w.part) * kPairTM * kPairTN, lrow, cl);
        else if constexpr (EPI == kEpiCE)
          epilogue_ce32(v, row, col, tc.n_end, tg, args);
        else {
          epilogue_row32<EPI, OUT, false>(v, row, col, tc.n_end, args);
          epilogue_colsum<EPI>(v, row, col, tc.n_end, lane, args);
        }
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader[acc]);
      if (w.part >= 0)  // each CTA of the pair finishes its own 128 rows
        tail_arrive<kPairTM, kPairTN, EPI, OUT>(args, tc, w.tile - args.tail0,
                                                2 * (w.tile - args.tail0) + static_cast<int>(rank),
                                                lrow, row, half, lane, ew, tail_flag);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait<0>();  // this warp's TMA stores have landed
  }
  (void)peer;

  __syncwarp();  // lane 0 of the producer / MMA warps rejoins its warp
  tc_fence_before();
  cluster_sync();  // no CTA frees tensor memory while its pair may still use it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 512);
}

// Splitting tiles along K when the tiles alone would leave SMs idle:
// * the last, partial wave: with T tiles on G persistent CTAs (or CTA pairs)
//   and R = T mod G tiles left for the last wave (at most half a wave),
//   those R tiles are cut into S = min(G / R, K blocks / B) K slices, so
//   the last wave keeps R * S of the G workers busy for 1/S of a tile's time;
// * fewer tiles than workers (T < G): all T tiles are cut into
//   S = min(G / T, K blocks / B) slices, so T * S workers share them.
// The CTA that stores a tile's last slice adds the slices (tail_finish).
// B = 32 K blocks (shorter slices cost more in partial traffic than they
// save), or 16 for a GEMM of fewer than four waves, whose last wave is a
// large share of its time; and only when the caller gave scratch for the
// R * S fp32 partial tiles.  The result of a
// split tile differs from the unsplit one only in the grouping of its fp32
// sums.
constexpr int kMinSliceBlocks = 32;
// The split tiles' arrival counters sit at the start of the scratch (at most
// one tile per worker, two counters per tile for a CTA pair), the partial
// tiles after them.
constexpr size_t kTailCtrBytes = 4096;

struct TailPlan {
  int units, tail0, split;
};

TailPlan plan_tail(long long tiles, int workers, int k_blocks, size_t part_bytes,
                   size_t scratch_bytes, int epi) {
  TailPlan tp{static_cast<int>(tiles), static_cast<int>(tiles), 1};
  if (epi == kEpiCE || scratch_bytes <= kTailCtrBytes || tiles == 0) return tp;
  scratch_bytes -= kTailCtrBytes;
  long long R;
  if (tiles < workers) {
    R = tiles;
  } else {
    R = tiles % workers;
    if (R == 0 || 2 * R > workers) return tp;
  }
  // A GEMM of fewer than 4 waves loses a large share of its time to the
  // short last wave, so its slices may be as short as 16 K blocks.
  const int min_slice = tiles < 4LL * workers ? kMinSliceBlocks / 2 : kMinSliceBlocks;
  int S = static_cast<int>(workers / R);
  if (S > k_blocks / min_slice) S = k_blocks / min_slice;
  if (S < 2 || static_cast<size_t>(R) * S * part_bytes > scratch_bytes) return tp;
  tp.tail0 = static_cast<int>(tiles - R);
  tp.split = S;
  tp.units = tp.tail0 + static_cast<int>(R) * S;
  return tp;
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map of a row-major bf16 matrix with `inner` columns (contiguous),
// `outer` rows, leading dimension `ld`; boxes of box_inner x box_outer with
// the 128-byte swizzle; out-of-range elements read as zero.
bool make_map(CUtensorMap* m, const void* ptr, int64_t inner, int64_t outer, int64_t ld,
              int box_inner, int box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map of the epilogue's 32 x 32 boxes of a row-major two-byte matrix
// with `cols` columns, `rows` rows and leading dimension `ld`, 64-byte
// swizzle (the layout sw64_off addresses).
bool make_box_map(CUtensorMap* m, const void* ptr, int64_t cols, int64_t rows, int64_t ld) {
  auto fn = encode_fn();
  if (fn == nullptr || ptr == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The epilogue's tensor maps: output, second output, operand read.
struct EpiMaps {
  CUtensorMap o, o2, x;
};

// Encodes the maps the boxed epilogue needs; false (the epilogue then stores
// directly) for fp32 outputs, a missing output, or a matrix a tensor map
// cannot describe.
template <int EPI, int OUT>
bool make_epi_maps(const Gemm& g, EpiMaps& e) {
  std::memset(&e, 0, sizeof(e));
  if (OUT == kOutF32 || g.out == nullptr) return false;
  if (!make_box_map(&e.o, g.out, g.N, g.M, g.ldo)) return false;
  if ((EPI == kEpiBiasGelu || EPI == kEpiDGelu) && g.out2 != nullptr &&
      !make_box_map(&e.o2, g.out2, g.N, g.M, g.ldo2))
    return false;
  if ((EPI == kEpiResidual || EPI == kEpiDGelu) && !make_box_map(&e.x, g.aux, g.N, g.M, g.ldaux))
    return false;
  return true;
}

struct Plan {
  int bn;
  int m_tiles, n_tiles, n_tiles_per_shard;
};

Plan plan_for(const Gemm& g, int bn) {
  Plan p;
  p.bn = bn;
  p.m_tiles = static_cast<int>((g.M + BM - 1) / BM);
  if (g.n_shard > 0) {
    p.n_tiles_per_shard = static_cast<int>((g.n_shard + bn - 1) / bn);
    p.n_tiles = static_cast<int>(g.N / g.n_shard) * p.n_tiles_per_shard;
  } else {
    p.n_tiles_per_shard = 0;
    p.n_tiles = static_cast<int>((g.N + bn - 1) / bn);
  }
  return p;
}

// The tile grid and raster of one GEMM in kernel arguments: 128 x bn tiles
// on one SM, or 256 x 256 tiles on an SM pair (pair = true, bn = 256).
// Shared by the launchers and tp_gemm_plan.
Args plan_args(const Gemm& g, int bn, bool pair) {
  const Plan p = plan_for(g, bn);
  Args a{};
  a.M = static_cast<int>(g.M);
  a.N = static_cast<int>(g.N);
  a.K = static_cast<int>(g.K);
  a.m_tiles = pair ? static_cast<int>((g.M + kPairTM - 1) / kPairTM) : p.m_tiles;
  a.n_tiles = p.n_tiles;
  a.k_blocks = static_cast<int>((g.K + BK - 1) / BK);
  a.group_m = pair ? 8 : 16;
  a.n_shard = static_cast<int>(g.n_shard);
  a.n_tiles_per_shard = p.n_tiles_per_shard;
  a.kr_range_blocks = g.korder.range_blocks;
  a.kr_t = g.korder.t;
  a.kr_width = g.korder.width;
  a.kr_h = g.korder.h;
  a.units = a.tail0 = static_cast<int>(static_cast<long long>(a.m_tiles) * a.n_tiles);
  a.tail_split = 1;
  return a;
}

// The last-wave K split of `a`'s tiles on `workers` persistent CTAs (or
// pairs) with partial tiles of `part_bytes` in `scratch_bytes` of caller
// scratch (0: none), written into a.
TailPlan plan_tail_args(Args& a, int workers, size_t part_bytes, size_t scratch_bytes, int epi) {
  const long long tiles = static_cast<long long>(a.m_tiles) * a.n_tiles;
  const TailPlan tp = plan_tail(tiles, workers, a.k_blocks, part_bytes, scratch_bytes, epi);
  a.units = tp.units;
  a.tail0 = tp.tail0;
  a.tail_split = tp.split;
  return tp;
}

size_t tail_bytes(const Gemm& g) { return g.tail_ws != nullptr ? g.tail_ws_bytes : 0; }

// Tile override for tests and tuning: TP_GEMM_TILE = 128 | 256 | pair.
int tile_override() {
  const char* e = std::getenv("TP_GEMM_TILE");
  if (e == nullptr) return 0;
  if (std::strcmp(e, "pair") == 0) return 512;
  const int v = std::atoi(e);
  return (v == 128 || v == 192 || v == 256) ? v : 0;
}

// Estimated time of T tiles of `tile_work` each on `workers` persistent CTAs
// (or pairs): whole waves, except that a GEMM with fewer tiles than workers
// counts the K slices plan_tail cuts every tile into (a short last wave's
// split is left out of the estimate: measured, it does not repay the
// narrower tiles it would displace).
double est_tiles(const Gemm& g, long long T, int workers, size_t part_bytes, double tile_work) {
  if (T < workers) {
    const int k_blocks = static_cast<int>((g.K + BK - 1) / BK);
    const TailPlan tp = plan_tail(T, workers, k_blocks, part_bytes, tail_bytes(g), g.epi);
    if (tp.split > 1) return tile_work / tp.split;
  }
  return std::ceil(double(T) / workers) * tile_work;
}

// Tile kind: 128, 192 or 256 columns on one SM, or 512 = 256 x 256 on an SM
// pair.  Picks the least estimated time, est_tiles with the work per tile
// divided by a relative rate.  The rates are throughputs relative to the 256-wide
// single-SM tile, measured on the 175B-shaped layer's twelve GEMMs under the
// sustained power cap with the tile kinds interleaved step by step: with A
// K-major and B MN-major (the forward linears) the single-SM tile is 3-5%
// faster than the pair; with both operands MN-major (wgrads) the pair is
// 6-12% faster; with both K-major (dgrads) the single-SM tile is 3-6% faster
// in natural K order and the pair 7% faster in the attention's head-group K
// order.  The 192- and 128-wide tiles run 15% and 30% slower per tile and
// only pay where they fill the last wave far better.  With at most 16 K
// blocks the per-tile epilogue, not the main loop, sets the pace and the
// narrower tiles lose only 4% and 10% (workload 2's K = 768 GEMMs: 60 us on
// 192-wide tiles against 66 us on 256-wide ones).
int choose_tile(const Gemm& g) {
  const int ov = tile_override();
  if (ov != 0) return ov;
  const double sms = sm_count();
  double best = 1e300;
  int kind = 256;
  const int widths[3] = {256, 192, 128};
  const bool short_k = (g.K + BK - 1) / BK <= 16;
  const double rate[3] = {1.0, short_k ? 0.96 : 0.85, short_k ? 0.90 : 0.68};
  for (int i = 0; i < 3; ++i) {
    const Plan p = plan_for(g, widths[i]);
    const double t = est_tiles(g, static_cast<long long>(p.m_tiles) * p.n_tiles,
                               static_cast<int>(sms), size_t(BM) * widths[i] * 4,
                               128.0 * widths[i] / rate[i]);
    if (t < best * 0.999) {
      best = t;
      kind = widths[i];
    }
  }
  double pair_rate;
  if (g.a.k_major && !g.b.k_major)
    pair_rate = 0.96;                                 // forward
  else if (g.a.k_major && g.b.k_major)
    pair_rate = g.korder.range_blocks > 0 ? 1.07 : 0.96;  // dgrad
  else
    pair_rate = 1.10;                                 // wgrad
  const Plan pp = plan_for(g, kPairTN);
  const long long pair_tiles = (g.M + kPairTM - 1) / kPairTM * pp.n_tiles;
  const double tp = est_tiles(g, pair_tiles, static_cast<int>(sms) / 2,
                              size_t(kPairTM) * kPairTN * 4, 256.0 * 256.0 / 2.0 / pair_rate);
  if (tp < best * 0.999) kind = 512;
  return kind;
}

template <int BN, bool AK, bool BKM, int EPI, int OUT>
tp_status launch_impl(const Gemm& g, cudaStream_t stream) {
  using C = Cfg<BN>;
  CUtensorMap ta, tb;
  const bool ok_a = AK ? make_map(&ta, g.a.ptr, g.K, g.M, g.a.ld, BK, BM)
                       : make_map(&ta, g.a.ptr, g.M, g.K, g.a.ld, 64, BK);
  const bool ok_b = BKM ? make_map(&tb, g.b.ptr, g.K, g.N, g.b.ld, BK, BN)
                        : make_map(&tb, g.b.ptr, g.N, g.K, g.b.ld, 64, BK);
  if (!ok_a || !ok_b) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled failed");

  Args a = plan_args(g, BN, false);
  a.out = g.out;
  a.ldo = g.ldo;
  a.bias = g.bias;
  a.out2 = static_cast<__nv_bfloat16*>(g.out2);
  a.ldo2 = g.ldo2;
  a.aux = static_cast<const __nv_bfloat16*>(g.aux);
  a.ldaux = g.ldaux;
  a.ce_part = reinterpret_cast<float2*>(g.ce.part);
  a.ce_ldp = g.ce.ldp;
  a.ce_cps = g.ce.cps;
  a.ce_target = g.ce.target;
  a.ce_tlogit = g.ce.tlogit;
  a.csum_part = EPI == kEpiDGelu ? g.csum_part : nullptr;
  a.csum_ld = g.N;
  a.status = wait_ctl();
  if (a.status.st == nullptr) return fail(TP_ERR_CUDA, "device status unavailable");
  EpiMaps em;
  a.tma_out = make_epi_maps<EPI, OUT>(g, em) ? 1 : 0;

  auto kern = gemm_bf16_tcgen05<BN, AK, BKM, EPI, OUT>;
  // Shared-memory opt-in once per device (devices past 31 every launch);
  // two threads may both set it, which is harmless.
  static std::atomic<unsigned> configured{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned bit = (dev >= 0 && dev < 32) ? (1u << dev) : 0u;
  if (bit == 0 || !(configured.load(std::memory_order_acquire) & bit)) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Layout<BN, EPI>::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm)");
    configured.fetch_or(bit, std::memory_order_release);
  }
  const long long tiles = static_cast<long long>(a.m_tiles) * a.n_tiles;
  if (tiles == 0) return TP_OK;
  const TailPlan tp = plan_tail_args(a, sm_count(), size_t(BM) * BN * 4, tail_bytes(g), EPI);
  const int grid = static_cast<int>(tp.units < sm_count() ? tp.units : sm_count());
  a.tail_ctr = static_cast<unsigned long long*>(g.tail_ws);
  a.tail_part = reinterpret_cast<float*>(static_cast<char*>(g.tail_ws) + kTailCtrBytes);
  const double flops = 2.0 * double(g.M) * double(g.N) * double(g.K);
  const double bytes = 2.0 * (double(g.M) * g.K + double(g.K) * g.N) +
                       (OUT == kOutF32 ? 4.0 : 2.0) * double(g.M) * g.N +
                       (g.out2 ? 2.0 * double(g.M) * g.N : 0.0) +
                       (g.aux ? 2.0 * double(g.M) * g.N : 0.0) +
                       (EPI == kEpiCE ? 8.0 * double(g.M) * g.N / 32.0 : 0.0);
  {
    LaunchScope scope(TP_KIND_GEMM_TCGEN05, flops, bytes, stream, 1, BN, g.M, g.N, g.K);
    kern<<<grid, kThreads, Layout<BN, EPI>::kSmemBytes, stream>>>(ta, tb, em.o, em.o2, em.x, a);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "gemm_bf16_tcgen05 launch");
  return TP_OK;
}

template <int BN, bool AK, bool BKM, int EPI>
tp_status by_out(const Gemm& g, cudaStream_t s) {
  if (g.out_f32) return launch_impl<BN, AK, BKM, EPI, kOutF32>(g, s);
  if (g.out_f16) return launch_impl<BN, AK, BKM, EPI, kOutF16>(g, s);
  return launch_impl<BN, AK, BKM, EPI, kOutBF16>(g, s);
}

template <int BN>
tp_status dispatch(const Gemm& g, cudaStream_t s) {
  const bool ak = g.a.k_major, bk = g.b.k_major;
  const bool plain_out = !g.out_f32 && !g.out_f16;
  if (g.epi == kEpiBiasGelu) {
    if (ak && !bk && plain_out) return launch_impl<BN, true, false, kEpiBiasGelu, kOutBF16>(g, s);
  } else if (g.epi == kEpiResidual) {
    if (ak && !bk && plain_out) return launch_impl<BN, true, false, kEpiResidual, kOutBF16>(g, s);
  } else if (g.epi == kEpiDGelu) {
    if (ak && bk && plain_out) return launch_impl<BN, true, true, kEpiDGelu, kOutBF16>(g, s);
  } else if (g.epi == kEpiCE) {
    if (ak && bk && plain_out) return launch_impl<BN, true, true, kEpiCE, kOutBF16>(g, s);
  } else {
    if (ak && !bk) return by_out<BN, true, false, kEpiStore>(g, s);
    if (ak && bk) return by_out<BN, true, true, kEpiStore>(g, s);
    if (!ak && !bk && !g.out_f16) {
      return g.out_f32 ? launch_impl<BN, false, false, kEpiStore, kOutF32>(g, s)
                       : launch_impl<BN, false, false, kEpiStore, kOutBF16>(g, s);
    }
  }
  return fail(TP_ERR_UNSUPPORTED, "gemm: operand layout / epilogue combination not built");
}


template <bool AK, bool BKM, int EPI, int OUT>
tp_status launch_pair(const Gemm& g, cudaStream_t stream) {
  CUtensorMap ta, tb;
  const bool ok_a = AK ? make_map(&ta, g.a.ptr, g.K, g.M, g.a.ld, BK, 128)
                       : make_map(&ta, g.a.ptr, g.M, g.K, g.a.ld, 64, BK);
  const bool ok_b = BKM ? make_map(&tb, g.b.ptr, g.K, g.N, g.b.ld, BK, 128)
                        : make_map(&tb, g.b.ptr, g.N, g.K, g.b.ld, 64, BK);
  if (!ok_a || !ok_b) return fail(TP_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  Args a = plan_args(g, kPairTN, true);
  a.out = g.out;
  a.ldo = g.ldo;
  a.bias = g.bias;
  a.out2 = static_cast<__nv_bfloat16*>(g.out2);
  a.ldo2 = g.ldo2;
  a.aux = static_cast<const __nv_bfloat16*>(g.aux);
  a.ldaux = g.ldaux;
  a.ce_part = reinterpret_cast<float2*>(g.ce.part);
  a.ce_ldp = g.ce.ldp;
  a.ce_cps = g.ce.cps;
  a.ce_target = g.ce.target;
  a.ce_tlogit = g.ce.tlogit;
  a.csum_part = EPI == kEpiDGelu ? g.csum_part : nullptr;
  a.csum_ld = g.N;
  a.status = wait_ctl();
  if (a.status.st == nullptr) return fail(TP_ERR_CUDA, "device status unavailable");
  EpiMaps em;
  a.tma_out = make_epi_maps<EPI, OUT>(g, em) ? 1 : 0;

  auto kern = gemm_bf16_tcgen05_pair<AK, BKM, EPI, OUT>;
  // Shared-memory opt-in and the number of co-resident pairs, once per
  // device (devices past 31 every launch); concurrent first calls compute
  // the same values.
  static std::atomic<unsigned> configured{0};
  static std::atomic<int> max_clusters[32];
  int dev = 0;
  cudaGetDevice(&dev);
  const unsigned bit = (dev >= 0 && dev < 32) ? (1u << dev) : 0u;
  int mc = 0;
  if (bit != 0 && (configured.load(std::memory_order_acquire) & bit)) {
    mc = max_clusters[dev].load(std::memory_order_relaxed);
  } else {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm pair)");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kPairSmemBytes;
    if (cudaOccupancyMaxActiveClusters(&mc, kern, &cfg) != cudaSuccess || mc <= 0) {
      cudaGetLastError();
      mc = sm_count() / 2;
    }
    if (bit != 0) {
      max_clusters[dev].store(mc, std::memory_order_relaxed);
      configured.fetch_or(bit, std::memory_order_release);
    }
  }
  const long long tiles = static_cast<long long>(a.m_tiles) * a.n_tiles;
  if (tiles == 0) return TP_OK;
  const TailPlan tp = plan_tail_args(a, mc, size_t(kPairTM) * kPairTN * 4, tail_bytes(g), EPI);
  const int clusters = static_cast<int>(tp.units < mc ? tp.units : mc);
  a.tail_ctr = static_cast<unsigned long long*>(g.tail_ws);
  a.tail_part = reinterpret_cast<float*>(static_cast<char*>(g.tail_ws) + kTailCtrBytes);
  const double flops = 2.0 * double(g.M) * double(g.N) * double(g.K);
  const double bytes = 2.0 * (double(g.M) * g.K + double(g.K) * g.N) +
                       (OUT == kOutF32 ? 4.0 : 2.0) * double(g.M) * g.N +
                       (g.out2 ? 2.0 * double(g.M) * g.N : 0.0) +
                       (g.aux ? 2.0 * double(g.M) * g.N : 0.0) +
                       (EPI == kEpiCE ? 8.0 * double(g.M) * g.N / 32.0 : 0.0);
  {
    LaunchScope scope(TP_KIND_GEMM_TCGEN05, flops, bytes, stream, 1, 512, g.M, g.N, g.K);
    kern<<<2 * clusters, kThreads, kPairSmemBytes, stream>>>(ta, tb, em.o, em.o2, em.x, a);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "gemm_bf16_tcgen05_pair launch");
  return TP_OK;
}

template <bool AK, bool BKM, int EPI>
tp_status pair_by_out(const Gemm& g, cudaStream_t s) {
  if (g.out_f32) return launch_pair<AK, BKM, EPI, kOutF32>(g, s);
  if (g.out_f16) return launch_pair<AK, BKM, EPI, kOutF16>(g, s);
  return launch_pair<AK, BKM, EPI, kOutBF16>(g, s);
}

tp_status dispatch_pair(const Gemm& g, cudaStream_t s) {
  const bool ak = g.a.k_major, bk = g.b.k_major;
  const bool plain_out = !g.out_f32 && !g.out_f16;
  if (g.epi == kEpiBiasGelu) {
    if (ak && !bk && plain_out) return launch_pair<true, false, kEpiBiasGelu, kOutBF16>(g, s);
  } else if (g.epi == kEpiResidual) {
    if (ak && !bk && plain_out) return launch_pair<true, false, kEpiResidual, kOutBF16>(g, s);
  } else if (g.epi == kEpiDGelu) {
    if (ak && bk && plain_out) return launch_pair<true, true, kEpiDGelu, kOutBF16>(g, s);
  } else if (g.epi == kEpiCE) {
    if (ak && bk && plain_out) return launch_pair<true, true, kEpiCE, kOutBF16>(g, s);
  } else {
    if (ak && !bk) return pair_by_out<true, false, kEpiStore>(g, s);
    if (ak && bk) return pair_by_out<true, true, kEpiStore>(g, s);
    if (!ak && !bk && !g.out_f16) {
      return g.out_f32 ? launch_pair<false, false, kEpiStore, kOutF32>(g, s)
                       : launch_pair<false, false, kEpiStore, kOutBF16>(g, s);
    }
  }
  return fail(TP_ERR_UNSUPPORTED, "gemm: operand layout / epilogue combination not built");
}

}  // namespace

size_t gemm_tail_scratch_bytes() {
  // The arrival counters, then at most one partial tile per persistent CTA
  // (128 x 256 fp32) or per CTA pair (256 x 256 fp32, half as many pairs).
  return kTailCtrBytes + static_cast<size_t>(sm_count()) * 128 * 256 * 4;
}

int64_t gemm_plan_units(int64_t M, int64_t N, int64_t K, int64_t n_shard, int kind, int sms,
                        bool tail_scratch, GemmPlanUnit* out, int64_t cap) {
  if (M <= 0 || N <= 0 || K <= 0 || sms < 2 || n_shard < 0 || cap < 0 ||
      (kind != 128 && kind != 192 && kind != 256 && kind != 512))
    return -1;
  if (M > (1ll << 31) - BM || N > (1ll << 31) - 256 || K > (1ll << 31) - BK) return -1;
  Gemm g;
  g.M = M;
  g.N = N;
  g.K = K;
  // the same shard normalisation as launch_gemm_bf16
  g.n_shard = (n_shard > 0 && n_shard % 8 == 0 && N % n_shard == 0) ? n_shard : 0;
  const bool pair = kind == 512;
  const int bn = pair ? kPairTN : kind;
  Args a = plan_args(g, bn, pair);
  const int slots = pair ? sms / 2 : sms;  // persistent CTAs, or pairs
  const size_t scratch =
      tail_scratch ? kTailCtrBytes + static_cast<size_t>(sms) * 128 * 256 * 4 : 0;
  plan_tail_args(a, slots, size_t(pair ? kPairTM : BM) * bn * 4, scratch, kEpiStore);
  for (int u = 0; u < a.units && u < cap && out != nullptr; ++u) {
    const Unit w = unit_of(u, a);
    TileCoord tc;
    if (pair)
      tc = tile_coord_pair(w.tile, a);
    else if (bn == 128)
      tc = tile_coord<128>(w.tile, a);
    else if (bn == 192)
      tc = tile_coord<192>(w.tile, a);
    else
      tc = tile_coord<256>(w.tile, a);
    out[u] = GemmPlanUnit{tc.m0, pair ? kPairTM : BM, tc.n0, tc.n_end, w.kb0, w.kb1, w.part,
                          w.tile};
  }
  return a.units;
}

tp_status launch_gemm_bf16(const Gemm& g, cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return TP_OK;
  if (g.M > (1ll << 31) - BM || g.N > (1ll << 31) - 256 || g.K > (1ll << 31) - BK)
    return fail(TP_ERR_SHAPE, "gemm: dimension too large");
  if (g.a.ld % 8 != 0 || g.b.ld % 8 != 0 || g.ldo % 8 != 0 ||
      (g.out2 != nullptr && g.ldo2 % 8 != 0) || (g.aux != nullptr && g.ldaux % 8 != 0))
    return fail(TP_ERR_ALIGN, "gemm: leading dimensions must be multiples of 8 elements");
  if (g.korder.range_blocks > 0 &&
      (g.korder.width % BK != 0 || g.korder.h % 8 != 0 ||
       static_cast<int64_t>(g.korder.t) * 3 * g.korder.width != g.K))
    return fail(TP_ERR_SHAPE, "gemm: inconsistent shard K order");
  Gemm gg = g;
  // A shard-aligned column tile starts at shard * n_shard; the TMA x
  // coordinate must be a multiple of 8 elements (16 bytes) and the epilogue
  // stores whole groups of 8 columns, so other shard widths tile plainly
  // (every column is still computed by the same K loop).
  if (gg.n_shard > 0 && (gg.n_shard % 8 != 0 || gg.N % gg.n_shard != 0)) gg.n_shard = 0;
  if (gg.epi == kEpiCE &&
      (gg.n_shard <= 0 || gg.ce.part == nullptr || gg.ce.target == nullptr ||
       gg.ce.tlogit == nullptr || gg.ce.cps != (gg.n_shard + 31) / 32 ||
       gg.ce.ldp != gg.ce.cps * (gg.N / gg.n_shard)))
    return fail(TP_ERR_SHAPE, "gemm: inconsistent cross-entropy partial layout");
  switch (choose_tile(gg)) {
    case 512: return dispatch_pair(gg, stream);
    case 128: return dispatch<128>(gg, stream);
    case 192: return dispatch<192>(gg, stream);
    default: return dispatch<256>(gg, stream);
  }
}

}  // namespace tp
