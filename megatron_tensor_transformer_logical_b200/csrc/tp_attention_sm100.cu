// Attention core forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Per head ("图解Transformer并行计算" §3.1): O = softmax(Q K^T / sqrt(d)) V with
// the causal mask hiding key c from query r when c > r; each head group of
// §3.2 runs its own heads, so the core runs per (batch, head).
//
// One CTA per (batch element, head, 128 query rows), longest rows first:
//   warp 0     TMA: the Q tile once, then K_j and V_j (128 keys each) into a
//              two-deep ring (fp16, 128-byte swizzle);
//   warp 1     allocates 512 TMEM columns; one thread issues
//              S_j = Q K_j^T (128 x 128, K = d = 128) into one of two S
//              buffers, so S_{j+1} is computed while S_j is being
//              normalised, and O_j = P_j V_j into an O buffer;
//   warps 4-7  softmax: thread i owns query row i = TMEM lane i, so the
//              row max and sum need no shuffles; P_j (fp16) is written to
//              shared memory in the MMA's K-major swizzled layout; the
//              output is accumulated and rescaled in registers:
//                O <- (O + P_{j-1} V_{j-1}) * 2^(m_{j-1} - m_j).
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
constexpr int kThreadsA = 256;
constexpr int kSmemA = 1024 + 6 * kTile + 256;  // Q, K[2], V[2], P, barriers
constexpr float kLog2eA = 1.4426950408889634f;
constexpr float kLn2A = 0.69314718055994531f;

struct FwdArgs {
  int s, h, heads, causal;
  float scale_log2;
  __nv_bfloat16* out;  // O [M, h]
  float* lse;          // [b, heads, s]
  int* status;
};

// kind::f16 instruction descriptor with fp16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int m, int n, bool a_mn, bool b_mn) {
  return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((static_cast<uint32_t>(n) >> 3) << 17) | ((static_cast<uint32_t>(m) >> 4) << 24);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 t = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}

__global__ void __launch_bounds__(kThreadsA, 1)
    attn_fwd_tcgen05(const __grid_constant__ CUtensorMap tmQKV, const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTile;          // 2 stages
  uint8_t* sV = smem + 3 * kTile;      // 2 stages
  uint8_t* sP = smem + 5 * kTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 6 * kTile);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* v_full = bars + 3;   // [2]
  uint64_t* k_empty = bars + 5;  // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2]
  uint64_t* p_full = bars + 11;
  uint64_t* o_full = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (a.s + kBM - 1) / kBM;
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x);  // longest rows first
  const int head = blockIdx.y % a.heads, bi = blockIdx.y / a.heads;
  const int q0 = qb * kBM;
  const int n_kb = a.causal ? qb + 1 : nqb;
  const int row0 = bi * a.s;  // first row of this batch element in QKV
  const int qcol = head * kD, kcol = a.h + head * kD, vcol = 2 * a.h + head * kD;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
    }
    mbar_init(p_full, 4);  // one arrival per softmax warp
    mbar_init(o_full, 1);
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
  const uint32_t tS[2] = {tmem, tmem + 128};
  const uint32_t tO = tmem + 256;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------- TMA producer
      bool ok = true;
      tma_prefetch_desc(&tmQKV);
      mbar_arrive_expect_tx(q_full, kTile);
      tma_load_2d(sQ, &tmQKV, q_full, qcol, row0 + q0);
      tma_load_2d(sQ + kHalf, &tmQKV, q_full, qcol + 64, row0 + q0);
      for (int j = 0; j < n_kb && ok; ++j) {
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
      constexpr uint32_t kIdS = idesc_f16_f32(128, 128, false, false);  // Q K^T
      constexpr uint32_t kIdO = idesc_f16_f32(128, 128, false, true);   // P V
      const uint32_t q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0, a.status, kStatusAttnTimeout);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&k_full[st], static_cast<uint32_t>(j >> 1) & 1u, a.status,
                       kStatusAttnTimeout))
          return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + st * kTile);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_bf16(tS[st], sw128_desc(q_addr + off, 16, 1024), sw128_desc(k_addr + off, 16, 1024),
                    kIdS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[st]);
        umma_commit(&k_empty[st]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < n_kb && ok; ++j) {
        if (j + 1 < n_kb && !(ok = issue_s(j + 1))) break;
        // P_j written by the softmax warps (which also read O_{j-1} already).
        if (!(ok = mbar_wait(p_full, static_cast<uint32_t>(j) & 1u, a.status, kStatusAttnTimeout)))
          break;
        const int st = j & 1;
        if (!(ok = mbar_wait(&v_full[st], static_cast<uint32_t>(j >> 1) & 1u, a.status,
                             kStatusAttnTimeout)))
          break;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + st * kTile);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint32_t poff = (kk >> 2) * kHalf + (kk & 3) * 32;  // P: K-major over keys
          const uint32_t voff = kk * 16 * 128;                       // V: MN-major, 16 key rows
          umma_bf16(tO, sw128_desc(p_addr + poff, 16, 1024),
                    sw128_desc(v_addr + voff, kHalf, 1024), kIdO, kk > 0 ? 1u : 0u);
        }
        umma_commit(o_full);
        umma_commit(&v_empty[st]);
      }
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row within the tile = TMEM lane
    const int qrow = q0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    float o[kD];
#pragma unroll
    for (int i = 0; i < kD; ++i) o[i] = 0.0f;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    uint8_t* prow = sP + (r >> 3) * 1024 + (r & 7) * 128;  // row r in the SW128 layout
    // Keys [0, limit) are visible to this row (causal: up to the row itself).
    const int limit = a.causal ? min(a.s, qrow + 1) : a.s;
    for (int j = 0; j < n_kb; ++j) {
      const int st = j & 1;
      if (!(ok = mbar_wait(&s_full[st], static_cast<uint32_t>(j >> 1) & 1u, a.status,
                           kStatusAttnTimeout)))
        break;
      tc_fence_after();
      const int vis = limit - j * kBN;  // visible keys of this block: [0, vis)
      // pass 1: row max of the raw scores (the scale is positive, so the max
      // of the scaled scores is the scaled max)
      float mraw = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN; c += 32) {
        float v[32];
        tmem_ld32(tS[st] + lane_off + c, v);
        if (vis < c + 32) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = (c + i < vis) ? v[i] : -INFINITY;
        }
#pragma unroll
        for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
          for (int i = 0; i < w; ++i) v[i] = fmaxf(v[i], v[i + w]);
        mraw = fmaxf(mraw, v[0]);
      }
      const float mx = fmaxf(m_run, mraw * a.scale_log2);
      const float alpha = (m_run == -INFINITY) ? 0.0f : exp2f(m_run - mx);
      m_run = mx;
      // fold in O_{j-1} (scaled at m_{j-1}) and rescale to m_j
      if (j > 0) {
        if (!(ok = mbar_wait(o_full, static_cast<uint32_t>(j - 1) & 1u, a.status,
                             kStatusAttnTimeout)))
          break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kD; c += 32) {
          float v[32];
          tmem_ld32(tO + lane_off + c, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[c + i] = (o[c + i] + v[i]) * alpha;
        }
      }
      // pass 2: P = 2^(s * scale - m), row sum, fp16 into the P tile
      float rs = 0.0f;
#pragma unroll
      for (int c = 0; c < kBN; c += 32) {
        float v[32];
        tmem_ld32(tS[st] + lane_off + c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = exp2f(fmaf(v[i], a.scale_log2, -mx));
        if (vis < c + 32) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = (c + i < vis) ? v[i] : 0.0f;
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_half2(v[2 * i], v[2 * i + 1]);
#pragma unroll
        for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
          for (int i = 0; i < w; ++i) v[i] += v[i + w];
        rs += v[0];
        // 32 keys = 64 bytes = four 16-byte chunks of the row's 128-byte line
        // in the 64-key half c / 64; the chunk index is swizzled by (row & 7).
        uint8_t* line = prow + (c >> 6) * kHalf;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = ((c & 63) >> 3) + q;
          *reinterpret_cast<uint4*>(line + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      l_run = l_run * alpha + rs;
      fence_proxy_async_smem();  // P stores visible to the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && mbar_wait(o_full, static_cast<uint32_t>(n_kb - 1) & 1u, a.status,
                        kStatusAttnTimeout)) {
      tc_fence_after();
      const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
      __nv_bfloat16* orow = a.out + static_cast<long long>(row0 + qrow) * a.h + head * kD;
#pragma unroll
      for (int c = 0; c < kD; c += 32) {
        float v[32];
        tmem_ld32(tO + lane_off + c, v);
        if (qrow < a.s) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 8 * q + 2 * e;
              __nv_bfloat162 t = __floats2bfloat162_rn((o[c + i] + v[i]) * inv,
                                                       (o[c + i + 1] + v[i + 1]) * inv);
              w[e] = *reinterpret_cast<uint32_t*>(&t);
            }
            *reinterpret_cast<uint4*>(orow + c + 8 * q) = u;
          }
        }
      }
      if (qrow < a.s)
        a.lse[(static_cast<long long>(bi) * a.heads + head) * a.s + qrow] =
            (m_run + log2f(l_run)) * kLn2A;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_attn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

tp_status launch_attn_core_fwd_tc(const AttnShape& sh, const void* QKV, void* O, float* LSE,
                                  cudaStream_t stream) {
  if (sh.h / sh.heads != kD) return fail(TP_ERR_UNSUPPORTED, "attention: head dimension must be 128");
  if (sh.b * sh.heads > 65535) return fail(TP_ERR_SHAPE, "attention: b * heads too large");
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
  a.status = device_status_ptr();
  if (a.status == nullptr) return fail(TP_ERR_CUDA, "device status word unavailable");
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_tcgen05, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemA);
  if (e != cudaSuccess) return cuda_fail(e, "attention fwd smem attribute");
  dim3 grid(static_cast<unsigned>((sh.s + kBM - 1) / kBM), static_cast<unsigned>(sh.b * sh.heads));
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

}  // namespace tp
