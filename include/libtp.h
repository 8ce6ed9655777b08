/*
 * libtp — the Megatron-style partitioned Transformer layer on one B200.
 *
 * The layer is split into t *logical* shards that all live on one GPU.  What
 * the pages do with an AllReduce across GPUs (the sum of row-shard partials)
 * happens here inside the kernel: the partial products of every shard are
 * accumulated in tensor memory, shard after shard, and never written to HBM.
 *
 * Sources (page title, then section):
 *   [P3] "图解Transformer并行计算：从矩阵乘法切分到Megatron架构设计"
 *        §1.1 row split, §1.2 column split, §2.1/§2.2 MLP, §3.1/§3.2 attention.
 *   [P2] PyTorch tensor-parallel tutorial (page title "企业官网建设流程全解析"),
 *        §2.2 ParallelAttention, §3.2 ColumnParallelLinear, §3.3 the block.
 *   [P4] "5.1 Tensor并行与算子拆分" §1.1 tensor_parallel_split (divisibility).
 *   [P3] §4.1 vocabulary-parallel embedding, §4.2 vocabulary-parallel loss.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every tensor is row-major and dense; a [rows, cols] tensor has leading
 *   dimension cols.  Weights are stored [in, out] ([P3] §1: W is [h, h']).
 * - Every pointer is a DEVICE pointer owned by the caller; the library keeps
 *   no reference after the call returns and allocates no device memory.
 *   Scratch space comes from the caller's workspace `ws` of `ws_bytes`
 *   bytes, sized with tp_workspace_size().
 * - Each call validates its arguments on the host, synchronously, before any
 *   launch, and then enqueues its kernels on `stream` (a cudaStream_t; NULL is
 *   the legacy default stream) and returns without waiting.
 * - Calls other than tp_device_status() and the profiling reads never
 *   synchronise the host, so a sequence of them may be captured in a CUDA
 *   graph and replayed (after one ordinary call of each, so one-time set-up
 *   is done outside the capture); the graph replays the same pointers, so the
 *   tensors and workspaces must outlive it.  Arrival counters in a workspace
 *   are left cleared by every launch, so replays count from zero.  A replay
 *   keeps the launch generations of its capture, so after a bounded wait of
 *   a later launch has expired, the replays' waits give up as well until
 *   tp_device_status() has read and cleared the record.
 * - Alignment: every pointer must be 16-byte aligned and every row length
 *   (number of columns) a multiple of 8 elements, otherwise TP_ERR_ALIGN.
 * - Shard i of a column split owns columns [i*n/t, (i+1)*n/t); shard i of a
 *   row split owns rows [i*k/t, (i+1)*k/t) ([P4] §1.1: contiguous, equal
 *   shards; a size that t does not divide is an error, TP_ERR_SHAPE).
 *   t must be in [1, 64].
 * - bf16 work multiplies in bf16 and accumulates in fp32 on the tensor cores
 *   (tcgen05); outputs are rounded to the output type round-to-nearest-even.
 *   fp32 work runs on the CUDA cores in fp32.
 * - No C++ exception crosses this interface.  A non-TP_OK status leaves a
 *   message for tp_last_error().  TP_ERR_CUDA reports a launch error.  Errors
 *   that kernels detect while running (a bounded wait that expired) and
 *   conditions they flag (an fp16 intermediate saturated) are recorded in a
 *   per-device status, read by tp_device_status().  Neither stops a later
 *   call: a flag is never read by a kernel, and a timeout makes only the
 *   other waits of its own launch give up early (each launch carries its own
 *   generation number).  No call checks or clears the status on entry; the
 *   record stays until tp_device_status() reads it.
 */
#ifndef LIBTP_H_
#define LIBTP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tp_status {
  TP_OK = 0,
  TP_ERR_NULL = 1,         /* a required pointer is NULL                         */
  TP_ERR_SHAPE = 2,        /* a size <= 0, or t / heads does not divide a size   */
  TP_ERR_ALIGN = 3,        /* pointer not 16B aligned or row length % 8 != 0     */
  TP_ERR_DTYPE = 4,        /* unknown dtype or a disallowed dtype combination    */
  TP_ERR_UNSUPPORTED = 5,  /* valid request outside what is implemented          */
  TP_ERR_CUDA = 6,         /* CUDA runtime error (launch or query)               */
  TP_ERR_KERNEL = 7,       /* a kernel recorded an error in the status word      */
  TP_ERR_WORKSPACE = 8     /* ws is NULL or smaller than tp_workspace_size()     */
} tp_status;

typedef enum tp_dtype { TP_F32 = 0, TP_BF16 = 1 } tp_dtype;

typedef enum tp_op {
  TP_OP_MLP_FWD = 0,
  TP_OP_MLP_BWD = 1,
  TP_OP_ATTN_FWD = 2,
  TP_OP_ATTN_BWD = 3,
  TP_OP_LN_BWD = 4,
  TP_OP_BLOCK_FWD = 5,
  TP_OP_BLOCK_BWD = 6,
  TP_OP_VOCAB_CE_FWD = 7,   /* f is the vocabulary size V */
  TP_OP_VOCAB_EMBED_BWD = 8 /* depends on M only */
} tp_op;

/*
 * Column-parallel linear ([P3] §1.2; [P2] §3.2 ColumnParallelLinear):
 * W = [W_0 | ... | W_{t-1}] split on its output columns, X whole,
 * Y_i = X @ W_i + bias_i, Y = concat_i Y_i (the All-Gather is the layout:
 * shard i's tiles write columns [i*N/t, (i+1)*N/t) of Y).
 *   X    [M, K]  dtype          W [K, N] dtype          bias [N] dtype or NULL
 *   Y    shard <  0: [M, N] out_dtype, every shard
 *        shard >= 0: [M, N/t] out_dtype, shard `shard` only (its columns)
 *   dtype TP_BF16 allows out_dtype TP_BF16 or TP_F32; dtype TP_F32 needs TP_F32.
 * Errors: NULL X/W/Y; M, K, N <= 0; N % t; shard >= t; alignment; dtypes.
 */
tp_status tp_linear_col(const void* X, const void* W, const void* bias, void* Y,
                        int64_t M, int64_t K, int64_t N, int t, int shard,
                        tp_dtype dtype, tp_dtype out_dtype, void* stream);

/*
 * Row-parallel linear ([P3] §1.1): W = [W_0; ...; W_{t-1}] split on its
 * input rows, X split on its last dimension (the library slices the full X
 * itself), Z = sum_i X_i @ W_i + bias.  The partials are summed in the
 * accumulator, shard 0 first; none is written to memory.  The bias is added
 * once, after the sum.
 *   X [M, K] dtype; W [K, N] dtype; bias [N] dtype or NULL; Z [M, N] out_dtype.
 *   shard >= 0: Z receives the partial X_shard @ W_shard alone (the bias is
 *   added to shard 0's partial only, so that the t partials sum to the full
 *   result); use out_dtype TP_F32 to keep partials unrounded.
 * Errors: as tp_linear_col, with K % t instead of N % t.
 */
tp_status tp_linear_row(const void* X, const void* W, const void* bias, void* Z,
                        int64_t M, int64_t K, int64_t N, int t, int shard,
                        tp_dtype dtype, tp_dtype out_dtype, void* stream);

/*
 * Partitioned MLP forward ([P3] §2.1 steps 1-3, §2.2 MLP_forward_TP):
 *   shard i: Y_i = X @ A_i + bA_i;  H_i = GeLU(Y_i)  (the erf GeLU, [P2] §3.3:
 *   fp32 erff for TP_F32; for TP_BF16 erf to within 1.5e-7 (Abramowitz &
 *   Stegun 7.1.26), far below the bf16 rounding of H);
 *   Z = sum_i H_i @ B_i + bB   (A split by columns, B by rows, f = 4h typically).
 *   X [M, h]; A [h, f]; bA [f] or NULL; B [f, h]; bB [h] or NULL; Z [M, h];
 *   Ysave [M, f] or NULL: receives the pre-activation Y for the backward.
 *   All tensors in `dtype`.  H lives in the workspace.
 * Errors: NULL X/A/B/Z/ws; f % t; alignment; TP_ERR_WORKSPACE.
 */
tp_status tp_mlp_fwd(const void* X, const void* A, const void* bA, const void* B,
                     const void* bB, void* Z, void* Ysave, int64_t M, int64_t h,
                     int64_t f, int t, tp_dtype dtype, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * tp_mlp_fwd without a workspace, for callers that cannot allocate device
 * memory (a host that owns all device memory and forbids allocation on its
 * inference path, a latency-critical loop that cannot afford cudaMalloc's
 * synchronisation, a plugin interface that passes only inputs and outputs).
 * The source pages have no counterpart: this is a deployment variant.
 *   Same arguments, arithmetic and kernels as tp_mlp_fwd; the intermediate
 *   H [M, f] lives in a fixed array of 64 MiB + 256 bytes compiled into
 *   libtp, which every GPU that loads the library holds until the process
 *   exits.  M * f * element size must not exceed 64 MiB = 67108864 bytes
 *   (H alone; so M * f <= 33554432 for bf16, 16777216 for fp32; exactly
 *   that much is accepted), otherwise TP_ERR_SHAPE with a message saying so.
 *   Allocates nothing and calls no allocator.
 *   The first call on each device looks up the array's device address with
 *   cudaGetSymbolAddress (that device must be current); make that first call
 *   before any stream capture.  The address is cached per device and CUDA
 *   context: after cudaDeviceReset (or with another context current) the
 *   next call looks it up again, so that call, too, should come before any
 *   stream capture.  Every call shares the one array and it keeps
 *   the previous call's contents; nothing in it needs to start at zero (H is
 *   fully written before it is read).  Calls whose executions overlap on the
 *   GPU (on different streams, or on several host threads) race on it.
 * Errors: those of tp_mlp_fwd (without TP_ERR_WORKSPACE), plus TP_ERR_SHAPE
 * for sizes beyond the array and TP_ERR_CUDA if the lookup fails.
 */
tp_status tp_mlp_fwd_noalloc(const void* X, const void* A, const void* bA, const void* B,
                             const void* bB, void* Z, void* Ysave, int64_t M, int64_t h,
                             int64_t f, int t, tp_dtype dtype, void* stream);

/*
 * Partitioned MLP backward, the pages' mirror rule ([P3] §2.2):
 *   dY_i = (dZ @ B_i^T) * GeLU'(Y_i);  dB_i = H_i^T @ dZ;  dA_i = X^T @ dY_i
 *   (weight gradients per shard, no exchange);  dX = sum_i dY_i @ A_i^T (the
 *   partials summed in the accumulator);  dbA = colsum(dY);  dbB = colsum(dZ).
 *   Ysave: the forward's pre-activation, or NULL to recompute it from X, A, bA.
 *   Outputs dX [M, h], dA [h, f], dB [f, h] in `dtype`; dbA [f], dbB [h] in
 *   `dtype`, each computed only when its pointer is not NULL.
 * Errors: NULL X/A/B/dZ/dX/dA/dB/ws; f % t; alignment; TP_ERR_WORKSPACE.
 */
tp_status tp_mlp_bwd(const void* X, const void* A, const void* bA, const void* B,
                     const void* Ysave, const void* dZ, void* dX, void* dA, void* dbA,
                     void* dB, void* dbB, int64_t M, int64_t h, int64_t f, int t,
                     tp_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Head-wise partitioned attention forward ([P3] §3.1, §3.2 forward steps 1-3;
 * [P2] §2.2 ParallelAttention):
 *   Wqkv = [Wq | Wk | Wv] ([h, 3h]); head j owns columns [j*d, (j+1)*d) of
 *   each block, d = h/heads; head group g owns heads [g*heads/t, (g+1)*heads/t)
 *   and so three column ranges of Wqkv.  QKV_g = X @ Wqkv_g;  per head
 *   O_j = softmax(Q_j K_j^T / sqrt(d) + mask) V_j with the causal mask hiding
 *   key c from query r when c > r ([P4] masked_fill(mask == 0, -inf));
 *   Z = sum_g O_g @ Wo_g with Wo split by rows (no concatenation before Wo).
 *   X [M = b*s, h]; Wqkv [h, 3h]; Wo [h, h]; Z [M, h]; all bf16.
 *   QKVsave [M, 3h] fp16 or NULL; Osave [M, h] bf16 or NULL (heads in column
 *   order); LSEsave [b, heads, s] fp32 or NULL: natural-log softmax
 *   denominators of the scaled, masked scores.
 *   Precision: the linears multiply bf16 with fp32 accumulation; the
 *   attention core takes Q, K, V (and, in the backward, dO) as fp16, which
 *   the QKV (dO) GEMM writes, and rounds P and dS to fp16 for its products
 *   (fp32 accumulation).  A QKV or dO value beyond the fp16 range is
 *   saturated and reported by tp_device_status() as TP_ERR_KERNEL.
 *   d must be 128.  dtype must be TP_BF16 (else TP_ERR_UNSUPPORTED).
 * Errors: NULL X/Wqkv/Wo/Z/ws; heads % t; h % heads; s < 1; TP_ERR_WORKSPACE.
 */
tp_status tp_attn_fwd(const void* X, const void* Wqkv, const void* Wo, void* Z,
                      void* QKVsave, void* Osave, void* LSEsave, int64_t b, int64_t s,
                      int64_t h, int heads, int t, int causal, tp_dtype dtype, void* ws,
                      size_t ws_bytes, void* stream);

/*
 * Head-wise attention backward ([P3] §3.2 backward steps 1-3):
 *   dO_g = dZ @ Wo_g^T;  dWo_g = O_g^T @ dZ;  per head the softmax backward
 *   gives dQ, dK, dV;  dWqkv_g = X^T @ dQKV_g;  dX = sum_g dQKV_g @ Wqkv_g^T
 *   with the group partials summed in the accumulator, group 0 first.
 *   Osave, LSEsave: from tp_attn_fwd (required).  QKVsave (fp16): from
 *   tp_attn_fwd, or NULL to recompute QKV = X @ Wqkv.  Outputs dX [M, h], dWqkv [h, 3h],
 *   dWo [h, h], all bf16.
 * Errors: as tp_attn_fwd, plus NULL Osave/LSEsave/dZ/dX/dWqkv/dWo.
 */
tp_status tp_attn_bwd(const void* X, const void* Wqkv, const void* Wo, const void* QKVsave,
                      const void* Osave, const void* LSEsave, const void* dZ, void* dX,
                      void* dWqkv, void* dWo, int64_t b, int64_t s, int64_t h, int heads,
                      int t, int causal, tp_dtype dtype, void* ws, size_t ws_bytes,
                      void* stream);

/*
 * LayerNorm over the last dimension, as nn.LayerNorm in the tutorial's block
 * ([P2] §3.3): Y = (X - mean) * rstd * gamma + beta per row, with mean and
 * the biased variance over the row, rstd = 1 / sqrt(var + eps); statistics
 * in fp32.  Replicated across the logical shards (not partitioned).
 *   X, Y [M, h] dtype; gamma, beta [h] dtype or NULL (1 and 0); mean, rstd
 *   [M] fp32 or NULL (saved for the backward).  h % 8 == 0, h <= 16384.
 * Errors: NULL X/Y; M, h <= 0; alignment; h > 16384 is TP_ERR_UNSUPPORTED.
 */
tp_status tp_layernorm_fwd(const void* X, const void* gamma, const void* beta, void* Y,
                           float* mean, float* rstd, int64_t M, int64_t h, float eps,
                           tp_dtype dtype, void* stream);

/*
 * LayerNorm backward: with xhat = (X - mean) * rstd and g = dY * gamma,
 *   dX = rstd * (g - rowmean(g) - xhat * rowmean(g * xhat)) (+ dR if not NULL:
 *   the gradient of a residual path that joins here), dgamma = colsum(dY * xhat),
 *   dbeta = colsum(dY) (each only if its pointer is not NULL).
 *   mean, rstd: from tp_layernorm_fwd (required).  ws: tp_workspace_size(TP_OP_LN_BWD).
 */
tp_status tp_layernorm_bwd(const void* X, const void* gamma, const float* mean,
                           const float* rstd, const void* dY, const void* dR, void* dX,
                           void* dgamma, void* dbeta, int64_t M, int64_t h, tp_dtype dtype,
                           void* ws, size_t ws_bytes, void* stream);

/* Weights of one Transformer block (bf16; biases and LayerNorm affines may be NULL). */
typedef struct tp_block_weights {
  const void* ln1_g;
  const void* ln1_b;
  const void* Wqkv; /* [h, 3h] */
  const void* Wo;   /* [h, h]  */
  const void* ln2_g;
  const void* ln2_b;
  const void* A;    /* [h, f]  */
  const void* bA;   /* [f]     */
  const void* B;    /* [f, h]  */
  const void* bB;   /* [h]     */
} tp_block_weights;

/* Activations the block forward keeps for its backward (all required). */
typedef struct tp_block_saves {
  void* Xn1;    /* [M, h] bf16: LN1(X)                 */
  float* mean1; /* [M]                                  */
  float* rstd1; /* [M]                                  */
  void* QKV;    /* [M, 3h] fp16                         */
  void* O;      /* [M, h] bf16                          */
  float* LSE;   /* [b, heads, s]                        */
  void* X1;     /* [M, h] bf16: X + Attn(LN1(X))        */
  void* Xn2;    /* [M, h] bf16: LN2(X1)                 */
  float* mean2; /* [M]                                  */
  float* rstd2; /* [M]                                  */
  void* Y;      /* [M, f] bf16: MLP pre-activation      */
} tp_block_saves;

/* Weight gradients of one block (bf16; the bias / affine ones may be NULL). */
typedef struct tp_block_grads {
  void* dln1_g;
  void* dln1_b;
  void* dWqkv;
  void* dWo;
  void* dln2_g;
  void* dln2_b;
  void* dA;
  void* dbA;
  void* dB;
  void* dbB;
} tp_block_grads;

/*
 * One Transformer block, the tutorial's ParallelTransformerBlock.forward
 * ([P2] §3.3):  X1 = X + Attn(LN1(X));  X2 = X1 + MLP(LN2(X1)),
 * with the attention and the MLP partitioned exactly as tp_attn_fwd and
 * tp_mlp_fwd (t logical shards, causal attention) and each residual addition
 * fused into the epilogue of the row-split GEMM that ends its sublayer.
 *   X, X2 [M = b*s, h] bf16; weights, saves as above; eps for both norms.
 *   ws: tp_workspace_size(TP_OP_BLOCK_FWD, M, h, f, heads, t, TP_BF16).
 * Errors: those of the parts; a NULL save is TP_ERR_NULL; dtype must be bf16.
 */
tp_status tp_block_fwd(const void* X, const tp_block_weights* w, void* X2, tp_block_saves* saves,
                       int64_t b, int64_t s, int64_t h, int64_t f, int heads, int t, float eps,
                       tp_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Backward of tp_block_fwd (the mirror rule for each sublayer, residual paths
 * passing the gradient through):  dX1 = dX2 + LN2'(MLP'(dX2));
 * dX = dX1 + LN1'(Attn'(dX1)).  Writes dX [M, h] and every gradient in g.
 *   ws: tp_workspace_size(TP_OP_BLOCK_BWD, M, h, f, heads, t, TP_BF16).
 */
tp_status tp_block_bwd(const void* X, const tp_block_weights* w, const tp_block_saves* saves,
                       const void* dX2, void* dX, const tp_block_grads* g, int64_t b, int64_t s,
                       int64_t h, int64_t f, int heads, int t, float eps, tp_dtype dtype,
                       void* ws, size_t ws_bytes, void* stream);

/*
 * Vocabulary-parallel input embedding ([P3] §4.1).  E [V, h] is split by rows
 * into t vocabulary shards of V/t rows.  For each token, the shard whose range
 * holds ids[r] supplies row ids[r] - i*V/t of its slice and every other shard
 * supplies a zero row; the shards' rows are summed (the page's AllReduce).
 * Exactly one shard contributes, so Y[r] = E[ids[r]] exactly; an id outside
 * [0, V) belongs to no shard and gives a zero row.
 *   ids [M] int32; E [V, h] dtype; Y [M, h] dtype.  M == 0 is a no-op.
 * Errors: NULL ids / E / Y; M < 0 or V, h <= 0; V % t != 0 (TP_ERR_SHAPE);
 *   alignment (h % 8, 16-byte pointers).
 */
tp_status tp_vocab_embed_fwd(const int32_t* ids, const void* E, void* Y, int64_t M, int64_t V,
                             int64_t h, int t, tp_dtype dtype, void* stream);

/*
 * Backward of tp_vocab_embed_fwd: dE[v] = sum of dY[r] over the rows r with
 * ids[r] == v (zero for a row of E no token used), plus dE_in[v] when dE_in
 * is not NULL (the tied output layer's gradient, accumulated; dE_in may be
 * dE itself, and then only the rows that tokens use are touched).  Each
 * shard writes only its own V/t rows of dE.  Deterministic: the terms of a
 * row are added in token order, in fp32.
 *   ids [M] int32; dY [M, h]; dE_in, dE [V, h] dtype; M < 2^28.
 *   ws: tp_workspace_size(TP_OP_VOCAB_EMBED_BWD, M, h, V, 0, t, dtype)
 *   (may be NULL when M == 0).
 * Errors: as tp_vocab_embed_fwd; NULL dY (when M > 0) or dE; workspace.
 */
tp_status tp_vocab_embed_bwd(const int32_t* ids, const void* dY, const void* dE_in, void* dE,
                             int64_t M, int64_t V, int64_t h, int t, tp_dtype dtype, void* ws,
                             size_t ws_bytes, void* stream);

/*
 * Vocabulary-parallel cross-entropy, the output layer tied to the input
 * embedding E ([P3] §4.2), bf16.  With logits = X @ E^T:
 *   1. shard i computes its logits X @ E_i^T (columns [i*V/t, (i+1)*V/t)) in
 *      the GEMM; its epilogue rounds them to bf16 (stored in `logits` when
 *      not NULL) and reduces every 32-column chunk to (max, sum of
 *      exp(z - max)) over those rounded values;
 *   2. the chunks of a shard are combined into the shard's local sum;
 *   3. the shards' sums are combined, each rescaled to the common maximum:
 *      lse[r] = log sum_v exp(logits[r, v]);
 *   4-5. the shard owning targets[r] supplies its logit and
 *      loss[r] = lse[r] - logits[r, targets[r]];
 *   6. total = sum over shards of the losses of the rows whose target they
 *      own, i.e. the sum of loss[r].
 * A row whose target lies outside [0, V) is ignored: loss 0 (its lse is
 * still written).  Results are deterministic and independent of the GEMM
 * tile shape.
 *   X [M, h] bf16; E [V, h] bf16; targets [M] int32; logits [M, V] bf16 or
 *   NULL (needed by tp_vocab_ce_bwd); lse, loss [M] fp32; total: one fp32 or
 *   NULL.  V % (8 t) == 0.
 *   ws: tp_workspace_size(TP_OP_VOCAB_CE_FWD, M, h, V, 0, t, TP_BF16).
 * Errors: NULL X / E / targets / lse / loss; sizes; alignment; dtype must be
 *   TP_BF16; workspace.
 */
tp_status tp_vocab_ce_fwd(const void* X, const void* E, const int32_t* targets, void* logits,
                          float* lse, float* loss, float* total, int64_t M, int64_t h, int64_t V,
                          int t, tp_dtype dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * Backward of tp_vocab_ce_fwd for the objective sum_r dloss[r] * loss[r]
 * (dloss NULL: every dloss[r] = 1, the gradient of `total`):
 *   dlogits[r, v] = (exp(logits[r, v] - lse[r]) - [v == targets[r]]) * dloss[r]
 *     (zero on ignored rows), stored in bf16;
 *   dX = dlogits @ E  (the sum over the vocabulary shards of dlogits_i @ E_i,
 *     accumulated in one fp32 accumulator: the mirror of the column split);
 *   dE = dlogits^T @ X  (each shard's own rows; overwritten, not accumulated:
 *     add the input embedding's gradient afterwards with tp_vocab_embed_bwd
 *     and dE_in = dE).
 *   logits, lse: from tp_vocab_ce_fwd; dlogits [M, V] bf16 (may be `logits`
 *   itself, which is then overwritten); dX [M, h], dE [V, h] bf16, each
 *   skipped when NULL.
 */
tp_status tp_vocab_ce_bwd(const void* X, const void* E, const int32_t* targets,
                          const void* logits, const float* lse, const float* dloss,
                          void* dlogits, void* dX, void* dE, int64_t M, int64_t h, int64_t V,
                          int t, tp_dtype dtype, void* stream);

/*
 * Workspace bytes that `op` needs for these sizes (M = b*s tokens; f is
 * ignored by the attention and LayerNorm ops, heads by the MLP and LayerNorm
 * ops).  Returns 0 for invalid arguments.  The size covers the worst case
 * (recomputed Y / QKV) and, for the MLP, attention and block ops, scratch of
 * one fp32 partial tile per SM (about 19 MB on a B200) with which a GEMM
 * splits its last, partial wave of tiles along K.  Those ops also accept a
 * workspace without that scratch (the size minus it); their GEMMs then run
 * the last wave whole.
 */
size_t tp_workspace_size(tp_op op, int64_t M, int64_t h, int64_t f, int heads, int t,
                         tp_dtype dtype);

/*
 * Launch profiling (tracing).  While enabled, every kernel that libtp
 * launches is bracketed by a pair of CUDA events recorded on the launching
 * stream, tagged with its kind and its algorithmic work (2*M*N*K FLOPs for a
 * contraction; unmasked score pairs for attention; bytes read + written for
 * the memory-bound helpers).  tp_profile_read() waits for the recorded
 * events and returns the totals of one kind.  Independently of profiling,
 * tp_launch_count() counts every launch libtp has made since it was loaded.
 */
typedef enum tp_kernel_kind {
  TP_KIND_GEMM_TCGEN05 = 0,  /* bf16 tensor-core GEMM (all linear layers)   */
  TP_KIND_GEMM_SIMT = 1,     /* fp32 CUDA-core GEMM                          */
  TP_KIND_ATTN_FWD = 2,      /* attention core forward                       */
  TP_KIND_ATTN_BWD = 3,      /* attention core backward (all its kernels)    */
  TP_KIND_REDUCE = 4,        /* column sums, row terms                       */
  TP_KIND_VOCAB = 5,         /* embedding gather / scatter, loss reductions  */
  TP_KIND_COUNT = 6
} tp_kernel_kind;

typedef struct tp_profile_stats {
  int64_t launches;   /* launches of this kind while profiling was on */
  double total_ms;    /* sum of their event-timed durations           */
  double flops;       /* sum of their algorithmic FLOPs                */
  double bytes;       /* sum of their algorithmic HBM bytes            */
} tp_profile_stats;

/* Turns launch profiling on (1) or off (0); turning it on clears the totals. */
tp_status tp_profile_enable(int on);
/* Synchronizes on the recorded events and fills *out for `kind`. */
tp_status tp_profile_read(tp_kernel_kind kind, tp_profile_stats* out);
/* Kernels launched by libtp since the library was loaded. */
int64_t tp_launch_count(void);

/* One traced launch (or launch group) recorded while profiling was on. */
typedef struct tp_launch_record {
  int kind;            /* tp_kernel_kind                                        */
  int tile;            /* GEMM tile: 128/192/256 columns on one SM, 512 = 256x256 */
                       /* on an SM pair.  TP_KIND_VOCAB: 1 embedding gather,    */
                       /* 2 embedding scatter-add, 3 loss combination, 4 the    */
                       /* softmax gradient.  0 for other kernels                */
  int64_t m, n, k;     /* GEMM problem size (0 for other kernels)               */
  double ms;           /* event-timed duration                                  */
  double flops, bytes; /* algorithmic work                                      */
} tp_launch_record;

/* Records taken since profiling was last turned on. */
int64_t tp_profile_count(void);
/* Synchronizes on record `index`'s events and fills *out. */
tp_status tp_profile_record(int64_t index, tp_launch_record* out);

/* Message for the last non-TP_OK status returned on this host thread. */
const char* tp_last_error(void);

/*
 * Synchronizes `stream`, then reads and clears the status of the current
 * device.  TP_OK, TP_ERR_KERNEL (a kernel gave up a bounded wait since the
 * last read, or an fp16 attention intermediate was saturated; the message
 * says which, a timeout first) or TP_ERR_CUDA.  Outputs of the launch that
 * gave up a wait are incomplete; outputs of every other launch are not
 * affected.  The same launch replayed from a captured CUDA graph keeps its
 * generation, so after a timeout read this before replaying the graph.
 */
tp_status tp_device_status(void* stream);

/*
 * Self-test of the kernels' bounded waits (failure detection without a GPU
 * fault): launches one small kernel on `stream` in which one warp waits on an
 * mbarrier that nothing ever completes, giving up after `limit_ns`
 * nanoseconds, and a second warp waits on it with the default 2 s limit and
 * must be released by the first one's abort.  No copy or tensor-core work is
 * in flight, so the kernel returns normally; the following
 * tp_device_status() then returns TP_ERR_KERNEL ("bounded-wait self-test").
 * limit_ns must be in [1e3, 2e9] (else TP_ERR_SHAPE).
 */
tp_status tp_selftest_bounded_wait(int64_t limit_ns, void* stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int tp_version(void);

/*
 * Work plan of the tensor-core GEMM, for tests of its tile scheduler (host
 * only: no device, no CUDA call).  For D[M, N] = A[M, K] B[K, N] with tile
 * kind `kind` (128, 192 or 256 output columns per tile on one SM with 128
 * rows, or 512 = 256 x 256 tiles on an SM pair), column shards of width
 * `n_shard` (0: none; a width the GEMM cannot align to 8 columns tiles
 * plainly, as in every entry point), a device of `sms` SMs, and with
 * (tail_scratch = 1) or without the optional last-wave scratch of the
 * workspaces, the units the persistent kernel hands out in order: unit u
 * runs on CTA (or pair) u mod workers.  A whole tile is one unit (part = -1);
 * the tiles of a short last wave may be split into K slices (part >= 0, the
 * index of the slice's fp32 partial tile), summed afterwards in slice order.
 *   out   up to `cap` units (may be NULL to count only), caller-owned HOST memory
 * Returns the number of units, or -1 for invalid arguments (a size <= 0,
 * sms < 2, an unknown kind).
 */
typedef struct tp_gemm_unit {
  int32_t m0, rows;    /* output rows [m0, m0 + rows) (clipped to M)            */
  int32_t n0, n_end;   /* output columns [n0, n_end)                            */
  int32_t kb0, kb1;    /* K blocks [kb0, kb1), 64 deep                          */
  int32_t part;        /* partial-tile index of a K slice, -1 for a whole tile  */
  int32_t tile;        /* output tile index                                     */
} tp_gemm_unit;
int64_t tp_gemm_plan(int64_t M, int64_t N, int64_t K, int64_t n_shard, int kind, int sms,
                     int tail_scratch, tp_gemm_unit* out, int64_t cap);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* LIBTP_H_ */
