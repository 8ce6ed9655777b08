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

#include <algorithm>
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
  __nv_bfloat16* out;        // O (fwd) or dQKV (bwd)
  float* lse_out;
  int s, h, heads, causal;
  float scale_log2;          // log2(e) / sqrt(d)
  float scale;               // 1 / sqrt(d)
};

// ------------------------------------------------------- backward: D term
// D[bi, head, r] = sum_e dO[row, head*d + e] * O[row, head*d + e].  Sixteen
// threads per (row, head), each with 16-byte loads of 8 elements of O and
// dO (a warp reads two heads' 512 contiguous bytes of each), the 16 partial
// sums added by four shuffle steps.  HBM-bound: 4 bytes read per element.
// Writes the backward's row terms in the form the tcgen05 kernels take:
// nd = -D and nlse = -LSE * log2(e), rows of sp floats per (batch element,
// head); the same threads also zero the row padding and the 64-float tail.
__global__ void __launch_bounds__(256) attn_bwd_dsum_kernel(const AttnArgs a, float* nlse,
                                                             float* nd, long long M,
                                                             long long rows, int sp) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long pair = t >> 4;  // (row, head), head fastest
  const int l16 = threadIdx.x & 15;
  const bool in = pair < M * a.heads;
  float acc = 0.0f, lse = 0.0f;
  long long dst = 0;
  if (in) {
    const long long row = pair / a.heads;
    const int head = static_cast<int>(pair - row * a.heads);
    const long long bi = row / a.s, r = row - bi * a.s;
    const long long q = bi * a.heads + head;
    dst = q * sp + r;
    // The group's LSE load goes out with its O and dO loads.
    if (l16 == 0) lse = a.lse[q * a.s + r];
    const long long off = row * a.h + head * D + l16 * 8;
    const uint4 ov = *reinterpret_cast<const uint4*>(a.o + off);
    const uint4 dv = *reinterpret_cast<const uint4*>(a.dout + off);
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
    const __half2* d2 = reinterpret_cast<const __half2*>(&dv);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(o2[i]), y = __half22float2(d2[i]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int sh = 8; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
  if (in && l16 == 0) {
    nd[dst] = -acc;
    nlse[dst] = -(lse * kLog2e);
  }
  const int padr = sp - a.s;
  if (t < rows * padr) {
    const long long i = t / padr * sp + a.s + t % padr;
    nd[i] = 0.0f;
    nlse[i] = 0.0f;
  } else if (t < rows * padr + 64) {
    const long long i = rows * sp + (t - rows * padr);
    nd[i] = 0.0f;
    nlse[i] = 0.0f;
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

// Two arrays of row terms, each [b * heads] rows of attn_stat_stride(s)
// floats and a 64-float tail, 256-byte aligned.
size_t attn_core_bwd_scratch_bytes(const AttnShape& sh) {
  const size_t n = static_cast<size_t>(sh.b * sh.heads) * attn_stat_stride(sh.s) + 64;
  return 2 * ((n * sizeof(float) + 255) / 256 * 256);
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
  a.out = static_cast<__nv_bfloat16*>(dQKV);
  const int64_t sp = attn_stat_stride(sh.s);
  const size_t half = attn_core_bwd_scratch_bytes(sh) / 2;
  float* nlse = static_cast<float*>(scratch);
  float* nd = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + half);
  const long long M = sh.b * sh.s;
  const long long pad = sh.b * sh.heads * (sp - sh.s) + 64;
  const long long threads = std::max(M * sh.heads * 16, pad);
  LaunchScope scope(TP_KIND_ATTN_BWD, 2.5 * core_flops(sh), 2.0 * double(M) * 8 * sh.h, stream,
                    3);
  attn_bwd_dsum_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
      a, nlse, nd, M, sh.b * sh.heads, static_cast<int>(sp));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attention bwd (D term) launch");
  return launch_attn_core_bwd_tc(sh, QKV, dO, nlse, nd, dQKV, stream);
}

}  // namespace tp
