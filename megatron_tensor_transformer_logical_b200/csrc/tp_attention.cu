// Per-head causal softmax attention for the head-wise partitioned layer
// ("图解Transformer并行计算" §3.1: softmax(Q K^T / sqrt(d_k)) V per head;
// §3.2: each head group computes its own heads with no exchange, so the
// core runs per (batch, head) and the grouping only decides which Wqkv /
// Wo slices feed it).  The causal mask hides key c from query r when c > r
// ("5.1 Tensor并行与算子拆分", masked_fill(mask == 0, -inf)).
//
// Layout: QKV [M = b*s, 3h] fp16 row-major; head j of batch element bi uses
// rows [bi*s, (bi+1)*s) and columns j*d (Q), h + j*d (K), 2h + j*d (V),
// d = 128.  O [M, h] bf16 holds head j at columns j*d.  LSE [b, heads, s] is
// the natural log of each row's softmax denominator.
//
// The forward and the dQ and dK/dV backward kernels run on tcgen05
// (tp_attention_sm100.cu).  This file holds the backward's row term
// D = rowsum(dO * O) and the launchers.  Q, K, V and dO are fp16 (the GEMMs
// that produce them write fp16), which keeps three more mantissa bits than
// bf16 and halves the backward's rounding error; O and dQKV are bf16 for the
// linears that consume them.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "tp_internal.h"

namespace tp {
namespace {

constexpr int D = 128;            // head dimension
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
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention bwd (D term) launch");
  return launch_attn_core_bwd_tc(sh, QKV, dO, LSE, dsum, dQKV, stream);
}

}  // namespace tp
