// Host-side interface between libtp's C entry points and its kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>

#include "../../include/libtp.h"
#include "ptx_sm100.cuh"

namespace tp {

// Records a message for tp_last_error() and returns the status.
tp_status fail(tp_status st, const std::string& msg);
tp_status cuda_fail(cudaError_t e, const char* where);

// Status of the current device (kernels record bounded-wait expiry and
// flags there); resolved once per device with cudaGetSymbolAddress.
DeviceStatus* device_status_ptr();
// Bounded-wait control for one kernel launch on the current device: its
// status, a fresh generation and the default wait limit.  st is nullptr if
// the status could not be resolved.
WaitCtl wait_ctl();
int sm_count();
// Unique id of the current CUDA context (cuCtxGetId), 0 if there is none or
// it cannot be queried.  Caches of device-symbol addresses key on it.
unsigned long long current_context_id();

// Brackets one kernel launch: counts it and, while profiling is enabled,
// records a start/stop event pair on `stream` with its kind and work.
class LaunchScope {
 public:
  // `kernels`: how many kernels the bracketed region launches.
  // `tile`, m, n, k describe a GEMM launch for the per-launch trace.
  LaunchScope(tp_kernel_kind kind, double flops, double bytes, cudaStream_t stream,
              int kernels = 1, int tile = 0, int64_t m = 0, int64_t n = 0, int64_t k = 0);
  ~LaunchScope();
  LaunchScope(const LaunchScope&) = delete;
  LaunchScope& operator=(const LaunchScope&) = delete;

 private:
  int slot_ = -1;
  cudaStream_t stream_;
};

// Epilogue applied to each fp32 accumulator value before it is stored.
enum Epi : int {
  kEpiStore = 0,     // out = acc (+ bias[col])
  kEpiBiasGelu = 1,  // v = acc + bias[col]; out = GeLU(v); out2 = v (if out2)
  kEpiDGelu = 2,     // y = aux[row,col]; out = acc * GeLU'(y); out2 = GeLU(y) (if out2)
  kEpiResidual = 3,  // out = acc (+ bias[col]) + aux[row,col]: a residual addition
  kEpiCE = 4,        // z = bf16(acc); out = z (if out); per 32-column chunk of a
                     // shard: (max z, sum exp(z - max)) to ce_part; the target's z
};

// Cross-entropy outputs of a kEpiCE GEMM (columns are vocabulary entries).
// Chunk j of shard i (columns i*n_shard + [32 j, 32 j + 32)) of row r is
// part[r * ldp + i * cps + j] = (max, sum of exp(z - max)) over its columns;
// tlogit[r] = z[r, target[r]] when the target is a column of the GEMM.
struct CEOut {
  float* part = nullptr;  // float pairs
  int64_t ldp = 0;        // pairs per row = shards * cps
  int cps = 0;            // chunks per shard = ceil(n_shard / 32)
  const int* target = nullptr;
  float* tlogit = nullptr;
};

// One operand of D[M,N] = sum_k A(m,k) B(k,n) stored as a row-major matrix.
// k_major: A stored [M, K] / B stored [N, K] (K contiguous).
// otherwise: A stored [K, M] / B stored [K, N] (M or N contiguous).
struct Operand {
  const void* ptr = nullptr;
  int64_t ld = 0;  // leading dimension (elements) of the stored matrix
  bool k_major = true;
};

// K-block visiting order for a reduction whose shards are not one contiguous
// K range.  With range_blocks > 0, the K extent is t shards of 3 ranges of
// `width` columns each (the q, k and v columns of one head group); shard g's
// ranges start at 0*h + g*width, 1*h + g*width, 2*h + g*width.  The K loop
// visits shard 0's three ranges, then shard 1's, and so on.
struct KOrder {
  int range_blocks = 0;  // 64-column blocks per range (0: natural order)
  int t = 1;
  int width = 0;
  int h = 0;
};

struct Gemm {
  int64_t M = 0, N = 0, K = 0;
  Operand a, b;
  int epi = kEpiStore;
  void* out = nullptr;
  int64_t ldo = 0;
  bool out_f32 = false;
  bool out_f16 = false;        // fp16 output (saturating; range errors are flagged)
  const void* bias = nullptr;  // [N] bf16 / f32 (same type as inputs)
  void* out2 = nullptr;        // second output (bf16), ldo2
  int64_t ldo2 = 0;
  const void* aux = nullptr;   // auxiliary input (bf16), ldaux
  int64_t ldaux = 0;
  int64_t n_shard = 0;         // columns per shard: column tiles never straddle shards
  KOrder korder;
  CEOut ce;                    // kEpiCE only (requires n_shard % 8 == 0)
  // kEpiDGelu on the tensor-core path: per-32-row column sums of the output
  // (fp32, before rounding) to csum_part[(row / 32) * N + col], ceil(M / 32)
  // rows; finish with launch_colsum_finish.  nullptr: none.
  float* csum_part = nullptr;
  // Scratch for splitting the last partial wave of tiles along K (optional;
  // gemm_tail_scratch_bytes() is always enough).
  void* tail_ws = nullptr;
  size_t tail_ws_bytes = 0;
};

// Scratch that lets a tcgen05 GEMM split its last wave along K.
size_t gemm_tail_scratch_bytes();

// One unit of a GEMM work plan: output rows [m0, m0 + rows), columns
// [n0, n_end), K blocks [kb0, kb1) of 64; part = partial-tile index of a K
// slice, -1 for a whole tile; tile = the output tile's index.
struct GemmPlanUnit {
  int m0, rows, n0, n_end, kb0, kb1, part, tile;
};

// The units the tcgen05 GEMM would run for D[M, N] = A[M, K] B[K, N] with
// tile kind 128 / 192 / 256 (one SM) or 512 (256 x 256 on an SM pair), column
// shards of width n_shard (0: none) and `sms` SMs, with or without the
// last-wave scratch; host only.  Writes up to cap units to out; returns the
// number of units, -1 for invalid arguments.
int64_t gemm_plan_units(int64_t M, int64_t N, int64_t K, int64_t n_shard, int kind, int sms,
                        bool tail_scratch, GemmPlanUnit* out, int64_t cap);

// The smallest workspace tp_mlp_fwd accepts (without the optional GEMM tail
// scratch that tp_workspace_size() adds).
size_t mlp_fwd_ws_min(int64_t M, int64_t f, tp_dtype d);

// bf16 x bf16 -> fp32 accumulate on tcgen05; out bf16, fp16 or fp32.
tp_status launch_gemm_bf16(const Gemm& g, cudaStream_t stream);
// fp32 SIMT path (exact fp32 products and sums).
tp_status launch_gemm_f32(const Gemm& g, cudaStream_t stream);

// Column sums: out[c] = sum_r in[r, c] for in [rows, cols] (bf16 or f32),
// written in the same type.  `scratch` holds `colsum_scratch_bytes` bytes.
size_t colsum_scratch_bytes(int64_t rows, int64_t cols);
tp_status launch_colsum(const void* in, int64_t rows, int64_t cols, bool f32, void* out,
                        void* scratch, cudaStream_t stream);
// out[c] = sum over k < chunks of part[k * cols + c], in k order (bf16 or f32).
tp_status launch_colsum_finish(const float* part, int64_t chunks, int64_t cols, bool f32,
                               void* out, cudaStream_t stream);
// Both bias gradients of the bf16 MLP backward in one launch: dbB =
// colsum(dZ) for dZ [M, h], and dbA from partA, the GeLU' GEMM's per-32-row
// partials ([ceil(M / 32), f] fp32).  Either output may be nullptr (then its
// part is skipped).  `scratch` holds mlp_bias_grads_scratch_bytes(M, h)
// bytes (chunk partials and arrival counters, cleared here on `stream`).
size_t mlp_bias_grads_scratch_bytes(int64_t M, int64_t h);
tp_status launch_mlp_bias_grads(const void* dZ, int64_t M, int64_t h, void* dbB,
                                const float* partA, int64_t f, void* dbA, void* scratch,
                                cudaStream_t stream);

// LayerNorm over rows of [M, h] (h % 8 == 0, h <= layernorm_max_h()).
int64_t layernorm_max_h();
tp_status launch_layernorm_fwd(const void* X, const void* gamma, const void* beta, void* Y,
                               float* mean, float* rstd, int64_t M, int64_t h, float eps,
                               bool f32, cudaStream_t stream);
size_t layernorm_bwd_scratch_bytes(int64_t M, int64_t h);
tp_status launch_layernorm_bwd(const void* X, const void* gamma, const float* mean,
                               const float* rstd, const void* dY, const void* dR, void* dX,
                               void* dgamma, void* dbeta, int64_t M, int64_t h, bool f32,
                               void* scratch, cudaStream_t stream);

// Vocabulary-parallel embedding and loss helpers (HBM-bound kernels).  Their
// trace records carry one of these codes in the `tile` field.
enum VocabKernel : int {
  kVocabEmbedFwd = 1,     // embedding gather
  kVocabEmbedBwd = 2,     // embedding scatter-add
  kVocabLossCombine = 3,  // chunk partials -> lse, loss, total
  kVocabSoftmaxGrad = 4,  // dlogits
};
tp_status launch_embed_fwd(const int* ids, const void* E, void* Y, int64_t M, int64_t V,
                           int64_t h, int t, bool f32, cudaStream_t stream);
size_t embed_bwd_scratch_bytes(int64_t M);
tp_status launch_embed_bwd(const int* ids, const void* dY, const void* dE_in, void* dE,
                           int64_t M, int64_t V, int64_t h, bool f32, void* scratch,
                           cudaStream_t stream);
// From the chunk partials of a kEpiCE GEMM: lse, loss and (if not NULL) the
// total.  `shard_tot` holds t floats of scratch.
tp_status launch_ce_finish(const CEOut& ce, int t, int64_t M, int64_t V, float* lse, float* loss,
                           float* total, float* shard_tot, cudaStream_t stream);
// dlogits = (exp(logits - lse) - onehot(target)) * dloss, bf16, in place allowed.
tp_status launch_ce_dlogits(const void* logits, const float* lse, const int* target,
                            const float* dloss, void* dlogits, int64_t M, int64_t V,
                            cudaStream_t stream);

// Attention core (per head causal softmax attention), bf16 with d = 128.
struct AttnShape {
  int64_t b = 0, s = 0, h = 0;
  int heads = 0;
  int causal = 1;
};
// Q, K, V are column blocks of QKV [M, 3h]; O [M, h]; LSE [b, heads, s] fp32.
tp_status launch_attn_core_fwd(const AttnShape& sh, const void* QKV, void* O, float* LSE,
                               cudaStream_t stream);
// The tcgen05 / TMEM forward that launch_attn_core_fwd runs.
tp_status launch_attn_core_fwd_tc(const AttnShape& sh, const void* QKV, void* O, float* LSE,
                                  cudaStream_t stream);
// Row stride of the backward's row terms: s rounded up to 4 floats, so each
// row starts 16-byte aligned for the bulk copies of the dK/dV kernel.
inline int64_t attn_stat_stride(int64_t s) { return (s + 3) / 4 * 4; }
// The tcgen05 dQ and dK/dV kernels, given the row terms -LSE * log2(e) in
// `nlse` and -D = -rowsum(dO * O) in `nd`: [b * heads] rows of
// attn_stat_stride(s) floats, zero beyond s, and 64 zeros after the last row.
tp_status launch_attn_core_bwd_tc(const AttnShape& sh, const void* QKV, const void* dO,
                                  const float* nlse, const float* nd, void* dQKV,
                                  cudaStream_t stream);
// dO [M, h]; writes dQKV [M, 3h] (bf16).  `scratch` holds
// attn_core_bwd_scratch_bytes bytes (the two arrays of row terms).
size_t attn_core_bwd_scratch_bytes(const AttnShape& sh);
tp_status launch_attn_core_bwd(const AttnShape& sh, const void* QKV, const void* O,
                               const float* LSE, const void* dO, void* dQKV, void* scratch,
                               cudaStream_t stream);

}  // namespace tp
