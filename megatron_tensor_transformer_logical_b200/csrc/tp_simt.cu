// fp32 contractions on the CUDA cores.  The tensor cores offer no exact-fp32
// product (tf32 keeps a 10-bit mantissa), so fp32 work runs here: 64 x 64
// output tiles, K staged through shared memory 16 at a time, each thread
// accumulating a 4 x 4 block with fp32 FMAs in natural K order (shard 0's K
// range first, which is the order of the row-split sum).
//
// Same epilogues as the tensor-core path (bias, GeLU, GeLU'), in fp32.
#include <cuda_runtime.h>

#include "tp_internal.h"

namespace tp {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

struct ArgsF32 {
  int M, N, K;
  const float* A;
  long long lda;
  bool a_kmaj;
  const float* B;
  long long ldb;
  bool b_kmaj;
  float* out;
  long long ldo;
  const float* bias;
  float* out2;
  long long ldo2;
  const float* aux;
  long long ldaux;
};

__device__ __forceinline__ float gelu32(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}
__device__ __forceinline__ float gelu32_prime(float x) {
  return 0.5f * (1.0f + erff(x * 0.70710678118654752f)) +
         x * 0.39894228040143268f * expf(-0.5f * x * x);
}

template <int EPI>
__global__ void __launch_bounds__(256) gemm_f32_simt(const ArgsF32 a) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

  for (int k0 = 0; k0 < a.K; k0 += TK) {
    for (int i = threadIdx.x; i < TM * TK; i += 256) {
      int mm, kk;
      if (a.a_kmaj) { mm = i / TK; kk = i % TK; } else { mm = i % TM; kk = i / TM; }
      const int gm = m0 + mm, gk = k0 + kk;
      float v = 0.0f;
      if (gm < a.M && gk < a.K)
        v = a.a_kmaj ? a.A[(long long)gm * a.lda + gk] : a.A[(long long)gk * a.lda + gm];
      As[kk][mm] = v;
    }
    for (int i = threadIdx.x; i < TN * TK; i += 256) {
      int nn, kk;
      if (a.b_kmaj) { nn = i / TK; kk = i % TK; } else { nn = i % TN; kk = i / TN; }
      const int gn = n0 + nn, gk = k0 + kk;
      float v = 0.0f;
      if (gn < a.N && gk < a.K)
        v = a.b_kmaj ? a.B[(long long)gn * a.ldb + gk] : a.B[(long long)gk * a.ldb + gn];
      Bs[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = m0 + ty * 4 + i;
    if (r >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx * 4 + j;
      if (c >= a.N) continue;
      float x = acc[i][j];
      if (EPI != kEpiDGelu && a.bias != nullptr) x += a.bias[c];
      if (EPI == kEpiResidual) x += a.aux[(long long)r * a.ldaux + c];
      if (EPI == kEpiBiasGelu) {
        if (a.out2 != nullptr) a.out2[(long long)r * a.ldo2 + c] = x;
        x = gelu32(x);
      } else if (EPI == kEpiDGelu) {
        const float y = a.aux[(long long)r * a.ldaux + c];
        if (a.out2 != nullptr) a.out2[(long long)r * a.ldo2 + c] = gelu32(y);
        x *= gelu32_prime(y);
      }
      a.out[(long long)r * a.ldo + c] = x;
    }
  }
}

}  // namespace

tp_status launch_gemm_f32(const Gemm& g, cudaStream_t stream) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return TP_OK;
  if (g.M > (1ll << 31) - TM || g.N > (1ll << 31) - TN || g.K > (1ll << 31) - TK)
    return fail(TP_ERR_SHAPE, "gemm_f32: dimension too large");
  if (!g.out_f32) return fail(TP_ERR_DTYPE, "gemm_f32: output must be fp32");
  if ((g.N + TN - 1) / TN > 2147483647ll || (g.M + TM - 1) / TM > 65535)
    return fail(TP_ERR_SHAPE, "gemm_f32: grid too large");
  ArgsF32 a;
  a.M = static_cast<int>(g.M);
  a.N = static_cast<int>(g.N);
  a.K = static_cast<int>(g.K);
  a.A = static_cast<const float*>(g.a.ptr);
  a.lda = g.a.ld;
  a.a_kmaj = g.a.k_major;
  a.B = static_cast<const float*>(g.b.ptr);
  a.ldb = g.b.ld;
  a.b_kmaj = g.b.k_major;
  a.out = static_cast<float*>(g.out);
  a.ldo = g.ldo;
  a.bias = static_cast<const float*>(g.bias);
  a.out2 = static_cast<float*>(g.out2);
  a.ldo2 = g.ldo2;
  a.aux = static_cast<const float*>(g.aux);
  a.ldaux = g.ldaux;
  dim3 grid(static_cast<unsigned>((g.N + TN - 1) / TN), static_cast<unsigned>((g.M + TM - 1) / TM));
  {
    LaunchScope scope(TP_KIND_GEMM_SIMT, 2.0 * double(g.M) * g.N * g.K,
                      4.0 * (double(g.M) * g.K + double(g.K) * g.N + double(g.M) * g.N), stream);
    switch (g.epi) {
      case kEpiBiasGelu: gemm_f32_simt<kEpiBiasGelu><<<grid, 256, 0, stream>>>(a); break;
      case kEpiDGelu: gemm_f32_simt<kEpiDGelu><<<grid, 256, 0, stream>>>(a); break;
      case kEpiResidual: gemm_f32_simt<kEpiResidual><<<grid, 256, 0, stream>>>(a); break;
      default: gemm_f32_simt<kEpiStore><<<grid, 256, 0, stream>>>(a); break;
    }
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "gemm_f32_simt launch");
  return TP_OK;
}

}  // namespace tp
