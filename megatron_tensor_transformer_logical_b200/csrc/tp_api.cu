// libtp C entry points: host-side validation, the shard planner (how each
// partitioned operation of the pages maps onto kernel launches), workspace
// carving and the device status word.  Nothing here computes on the host.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <exception>
#include <atomic>
#include <chrono>
#include <cstdint>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "../../include/libtp.h"
#include "ptx_sm100.cuh"
#include "tp_internal.h"

namespace tp {

namespace {
thread_local std::string g_last_error;
constexpr int kMaxDevices = 64;
}  // namespace

// Device status: kernels that give up a bounded wait record a code here, and
// the fp16-saturating epilogue sets a flag (DeviceStatus in ptx_sm100.cuh).
__device__ DeviceStatus g_tp_status;

tp_status fail(tp_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

tp_status cuda_fail(cudaError_t e, const char* where) {
  g_last_error = std::string(where) + ": " + cudaGetErrorString(e);
  return TP_ERR_CUDA;
}

unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static const std::pair<GetCurrent, GetId> fns = [] {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    const bool ok =
        cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &q1) == cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &q2) == cudaSuccess &&
        q2 == cudaDriverEntryPointSuccess;
    return ok ? std::make_pair(reinterpret_cast<GetCurrent>(a), reinterpret_cast<GetId>(b))
              : std::make_pair(static_cast<GetCurrent>(nullptr), static_cast<GetId>(nullptr));
  }();
  if (fns.first == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (fns.first(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (fns.second(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

DeviceStatus* device_status_ptr() {
  // Cached per device together with the context it was resolved in: a new
  // context on the device (after cudaDeviceReset, say) loads libtp's device
  // code again, possibly elsewhere, so the address is looked up again.
  static DeviceStatus* ptrs[kMaxDevices] = {};
  static unsigned long long ctx_ids[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long id = current_context_id();
  if (ptrs[dev] == nullptr || id == 0 || id != ctx_ids[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_tp_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<DeviceStatus*>(p);
    ctx_ids[dev] = current_context_id();  // the lookup made the context current
  }
  return ptrs[dev];
}

namespace {
// Launch generations start from a value drawn when the library loads (the
// clock and an address, below 2^47), so arrival counters left in reused
// device memory by another process, or by another load of this library,
// carry no current generation; they are never 0, so a cleared status
// (abort_gen 0) stops no wait.
unsigned long long first_launch_gen() {
  const unsigned long long t = static_cast<unsigned long long>(
      std::chrono::steady_clock::now().time_since_epoch().count());
  const unsigned long long a = static_cast<unsigned long long>(
      reinterpret_cast<uintptr_t>(&first_launch_gen));
  return ((t * 0x9E3779B97F4A7C15ull) ^ (a >> 4)) & ((1ull << 47) - 1);
}
std::atomic<unsigned long long> g_launch_gen{first_launch_gen()};
}  // namespace

WaitCtl wait_ctl() {
  WaitCtl w;
  w.st = device_status_ptr();
  w.gen = g_launch_gen.fetch_add(1, std::memory_order_relaxed) + 1;
  w.limit_ns = kWaitLimitNs;
  return w;
}

int sm_count() {
  static std::atomic<int> counts[kMaxDevices];  // 0 until queried
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = counts[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    counts[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}


// ------------------------------------------------------------ launch profiling
namespace {
struct ProfRecord {
  cudaEvent_t start = nullptr, stop = nullptr;
  tp_kernel_kind kind = TP_KIND_GEMM_TCGEN05;
  double flops = 0, bytes = 0;
  int tile = 0;
  int64_t m = 0, n = 0, k = 0;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof;  // events are created once and reused
size_t g_prof_used = 0;
std::atomic<int64_t> g_launches{0};
}  // namespace

LaunchScope::LaunchScope(tp_kernel_kind kind, double flops, double bytes, cudaStream_t stream,
                         int kernels, int tile, int64_t m, int64_t n, int64_t k)
    : stream_(stream) {
  g_launches.fetch_add(kernels, std::memory_order_relaxed);
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (!g_prof_on) return;
  if (g_prof_used == g_prof.size()) {
    ProfRecord r;
    if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess)
      return;
    g_prof.push_back(r);
  }
  ProfRecord& r = g_prof[g_prof_used];
  r.kind = kind;
  r.flops = flops;
  r.bytes = bytes;
  r.tile = tile;
  r.m = m;
  r.n = n;
  r.k = k;
  if (cudaEventRecord(r.start, stream) != cudaSuccess) return;
  slot_ = static_cast<int>(g_prof_used++);
}

LaunchScope::~LaunchScope() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  cudaEventRecord(g_prof[slot_].stop, stream_);
}

namespace {

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t esize(tp_dtype d) { return d == TP_F32 ? 4 : 2; }

// Every size is below 2^31 - 256 (the kernels index rows and columns with
// 32-bit integers), which also keeps every byte count below 2^63.
constexpr int64_t kMaxDim = (1ll << 31) - 256;
inline bool dims_ok(std::initializer_list<int64_t> ds) {
  for (int64_t d : ds)
    if (d > kMaxDim) return false;
  return true;
}

// Bump allocator over the caller's workspace.
struct Carve {
  char* base;
  size_t cap, off = 0;
  Carve(void* b, size_t c) : base(static_cast<char*>(b)), cap(c) {}
  void* take(size_t bytes) {
    off = align_up(off, 256);
    void* p = base + off;
    off += bytes;
    return p;
  }
  // `bytes` more if the workspace has room for them, else nullptr.
  void* take_optional(size_t bytes) {
    const size_t o = align_up(off, 256);
    if (o + bytes > cap) return nullptr;
    off = o + bytes;
    return base + o;
  }
};

// The optional part of a workspace: scratch for splitting a GEMM's last
// partial wave along K.  tp_workspace_size() includes it; a workspace of
// only the minimum size works without it.
size_t tail_ws() { return align_up(gemm_tail_scratch_bytes(), 256) + 256; }

struct Tail {
  void* p = nullptr;
  size_t bytes = 0;
  explicit Tail(Carve& c) {
    p = c.take_optional(gemm_tail_scratch_bytes());
    bytes = p ? gemm_tail_scratch_bytes() : 0;
  }
  void to(Gemm& g) const {
    g.tail_ws = p;
    g.tail_ws_bytes = bytes;
  }
};

tp_status check_dtype(tp_dtype d) {
  if (d != TP_F32 && d != TP_BF16) return fail(TP_ERR_DTYPE, "unknown dtype");
  return TP_OK;
}

tp_status check_t(int t) {
  if (t < 1 || t > 64) return fail(TP_ERR_SHAPE, "shard count t must be in [1, 64]");
  return TP_OK;
}

tp_status check_ptrs_aligned(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p != nullptr && !aligned16(p)) return fail(TP_ERR_ALIGN, "pointer not 16-byte aligned");
  return TP_OK;
}

tp_status check_rows(std::initializer_list<int64_t> lens) {
  for (int64_t n : lens)
    if (n % 8 != 0) return fail(TP_ERR_ALIGN, "row length not a multiple of 8 elements");
  return TP_OK;
}

inline tp_status run(const Gemm& g, bool f32, cudaStream_t s) {
  return f32 ? launch_gemm_f32(g, s) : launch_gemm_bf16(g, s);
}

#define TP_TRY(expr)                   \
  do {                                 \
    tp_status _st = (expr);            \
    if (_st != TP_OK) return _st;      \
  } while (0)

// ------------------------------------------------------------------ linear

tp_status linear_common(const void* X, const void* W, const void* bias, void* Y, int64_t M,
                        int64_t K, int64_t N, int t, int shard, tp_dtype dtype,
                        tp_dtype out_dtype, bool col, cudaStream_t stream) {
  if (X == nullptr || W == nullptr || Y == nullptr) return fail(TP_ERR_NULL, "X, W and Y are required");
  TP_TRY(check_dtype(dtype));
  TP_TRY(check_dtype(out_dtype));
  if (dtype == TP_F32 && out_dtype != TP_F32)
    return fail(TP_ERR_DTYPE, "fp32 inputs need an fp32 output");
  if (M <= 0 || K <= 0 || N <= 0) return fail(TP_ERR_SHAPE, "M, K and N must be positive");
  if (!dims_ok({M, K, N})) return fail(TP_ERR_SHAPE, "M, K and N must be below 2^31 - 256");
  TP_TRY(check_t(t));
  if (shard >= t) return fail(TP_ERR_SHAPE, "shard must be < t");
  const int64_t split = col ? N : K;
  if (split % t != 0)
    return fail(TP_ERR_SHAPE, col ? "N must be divisible by t (column split)"
                                  : "K must be divisible by t (row split)");
  TP_TRY(check_ptrs_aligned({X, W, bias, Y}));
  TP_TRY(check_rows({K, N}));
  const int64_t part = split / t;
  if (shard >= 0) TP_TRY(check_rows({part}));

  const bool f32 = dtype == TP_F32;
  const size_t es = esize(dtype);
  Gemm g;
  g.M = M;
  g.N = N;
  g.K = K;
  g.a = {X, K, true};
  g.b = {W, N, false};
  g.epi = kEpiStore;
  g.out = Y;
  g.ldo = N;
  g.out_f32 = out_dtype == TP_F32;
  g.bias = bias;
  if (col) {
    if (shard < 0) {
      g.n_shard = part;  // tiles of shard i cover columns [i*N/t, (i+1)*N/t) only
    } else {
      g.N = part;
      g.b.ptr = static_cast<const char*>(W) + shard * part * es;
      if (bias) g.bias = static_cast<const char*>(bias) + shard * part * es;
      g.ldo = part;
    }
  } else if (shard >= 0) {
    // Partial of row shard `shard`: X[:, K_i] @ W[K_i, :]; bias on shard 0 only.
    g.K = part;
    g.a.ptr = static_cast<const char*>(X) + shard * part * es;
    g.b.ptr = static_cast<const char*>(W) + shard * part * N * es;
    if (shard != 0) g.bias = nullptr;
  }
  return run(g, f32, stream);
}

// --------------------------------------------------------------------- MLP

}  // namespace

size_t mlp_fwd_ws_min(int64_t M, int64_t f, tp_dtype d) {
  return align_up(M * f * esize(d), 256) + 256;
}

namespace {

size_t mlp_fwd_ws(int64_t M, int64_t f, tp_dtype d) { return mlp_fwd_ws_min(M, f, d) + tail_ws(); }

// The GeLU' GEMM's per-32-row partials of dY: ceil(M / 32) x f floats.
size_t dba_partial_bytes(int64_t M, int64_t f) {
  return static_cast<size_t>((M + 31) / 32) * static_cast<size_t>(f) * 4;
}

// Column-sum scratch of the MLP backward: the two-pass sums of dY and dZ
// (fp32 path), or the GeLU' GEMM's partials of dY followed by the scratch of
// the one-launch bias gradients (bf16 path).
size_t mlp_bwd_colsum_bytes(int64_t M, int64_t h, int64_t f) {
  size_t cs = colsum_scratch_bytes(M, f);
  const size_t cs2 = colsum_scratch_bytes(M, h);
  const size_t cs3 = align_up(dba_partial_bytes(M, f), 256) + mlp_bias_grads_scratch_bytes(M, h);
  if (cs2 > cs) cs = cs2;
  if (cs3 > cs) cs = cs3;
  return cs;
}

size_t mlp_bwd_ws_min(int64_t M, int64_t h, int64_t f, tp_dtype d) {
  const size_t mf = align_up(M * f * esize(d), 256);
  return 3 * mf + align_up(mlp_bwd_colsum_bytes(M, h, f), 256) + 1024;
}

size_t mlp_bwd_ws(int64_t M, int64_t h, int64_t f, tp_dtype d) {
  return mlp_bwd_ws_min(M, h, f, d) + tail_ws();
}

tp_status mlp_fwd(const void* X, const void* A, const void* bA, const void* B, const void* bB,
                  void* Z, void* Ysave, int64_t M, int64_t h, int64_t f, int t, tp_dtype dtype,
                  void* ws, size_t ws_bytes, cudaStream_t stream, const void* residual = nullptr) {
  if (!X || !A || !B || !Z) return fail(TP_ERR_NULL, "X, A, B and Z are required");
  TP_TRY(check_dtype(dtype));
  if (M <= 0 || h <= 0 || f <= 0) return fail(TP_ERR_SHAPE, "M, h and f must be positive");
  if (!dims_ok({M, h, f})) return fail(TP_ERR_SHAPE, "M, h and f must be below 2^31 - 256");
  TP_TRY(check_t(t));
  if (f % t != 0) return fail(TP_ERR_SHAPE, "f must be divisible by t");
  TP_TRY(check_ptrs_aligned({X, A, bA, B, bB, Z, Ysave, ws}));
  TP_TRY(check_rows({h, f}));
  if (ws == nullptr || ws_bytes < mlp_fwd_ws_min(M, f, dtype))
    return fail(TP_ERR_WORKSPACE, "workspace missing or smaller than tp_workspace_size()");
  const bool f32 = dtype == TP_F32;
  Carve c(ws, ws_bytes);
  void* H = c.take(M * f * esize(dtype));
  const Tail tail(c);

  // Column-split first linear with GeLU per shard ([P3] §2.1 steps 1-2).
  Gemm g1;
  g1.M = M; g1.N = f; g1.K = h;
  g1.a = {X, h, true};
  g1.b = {A, f, false};
  g1.epi = kEpiBiasGelu;
  g1.out = H; g1.ldo = f; g1.out_f32 = f32;
  g1.bias = bA;
  g1.out2 = Ysave; g1.ldo2 = f;
  g1.n_shard = f / t;
  tail.to(g1);
  TP_TRY(run(g1, f32, stream));

  // Row-split second linear; the t partials are summed in the accumulator
  // (K walks shard 0's rows of B first) and bB is added once.
  Gemm g2;
  g2.M = M; g2.N = h; g2.K = f;
  g2.a = {H, f, true};
  g2.b = {B, h, false};
  g2.epi = residual ? kEpiResidual : kEpiStore;  // Z = residual + MLP(X) when given
  g2.aux = residual; g2.ldaux = h;
  g2.out = Z; g2.ldo = h; g2.out_f32 = f32;
  g2.bias = bB;
  tail.to(g2);
  return run(g2, f32, stream);
}

tp_status mlp_bwd(const void* X, const void* A, const void* bA, const void* B, const void* Ysave,
                  const void* dZ, void* dX, void* dA, void* dbA, void* dB, void* dbB, int64_t M,
                  int64_t h, int64_t f, int t, tp_dtype dtype, void* ws, size_t ws_bytes,
                  cudaStream_t stream) {
  if (!X || !A || !B || !dZ || !dX || !dA || !dB)
    return fail(TP_ERR_NULL, "X, A, B, dZ, dX, dA and dB are required");
  TP_TRY(check_dtype(dtype));
  if (M <= 0 || h <= 0 || f <= 0) return fail(TP_ERR_SHAPE, "M, h and f must be positive");
  if (!dims_ok({M, h, f})) return fail(TP_ERR_SHAPE, "M, h and f must be below 2^31 - 256");
  TP_TRY(check_t(t));
  if (f % t != 0) return fail(TP_ERR_SHAPE, "f must be divisible by t");
  TP_TRY(check_ptrs_aligned({X, A, bA, B, Ysave, dZ, dX, dA, dbA, dB, dbB, ws}));
  TP_TRY(check_rows({h, f}));
  if (ws == nullptr || ws_bytes < mlp_bwd_ws_min(M, h, f, dtype))
    return fail(TP_ERR_WORKSPACE, "workspace missing or smaller than tp_workspace_size()");
  const bool f32 = dtype == TP_F32;
  const size_t es = esize(dtype);
  Carve c(ws, ws_bytes);
  void* dY = c.take(M * f * es);
  void* H = c.take(M * f * es);
  void* Yrec = c.take(M * f * es);
  void* scratch = c.take(mlp_bwd_colsum_bytes(M, h, f));
  const Tail tail(c);

  const void* Y = Ysave;
  if (Y == nullptr) {
    // Recompute the pre-activation (and H from it, as in the forward).
    Gemm gr;
    gr.M = M; gr.N = f; gr.K = h;
    gr.a = {X, h, true};
    gr.b = {A, f, false};
    gr.epi = kEpiBiasGelu;
    gr.out = H; gr.ldo = f; gr.out_f32 = f32;
    gr.bias = bA;
    gr.out2 = Yrec; gr.ldo2 = f;
    gr.n_shard = f / t;
    tail.to(gr);
    TP_TRY(run(gr, f32, stream));
    Y = Yrec;
  }

  // dY_i = (dZ @ B_i^T) * GeLU'(Y_i) per column shard; H_i = GeLU(Y_i) too.
  Gemm g3;
  g3.M = M; g3.N = f; g3.K = h;
  g3.a = {dZ, h, true};
  g3.b = {B, h, true};  // B [f, h] read as B^T: n = f index, K contiguous
  g3.epi = kEpiDGelu;
  g3.aux = Y; g3.ldaux = f;
  g3.out = dY; g3.ldo = f; g3.out_f32 = f32;
  g3.out2 = (Ysave != nullptr) ? H : nullptr; g3.ldo2 = f;
  g3.n_shard = f / t;
  // dbA_i = colsum(dY_i): on the tensor-core path the epilogue writes the
  // column sums of each 32-row group of dY (fp32, before rounding).
  const bool fused_dba = dbA != nullptr && !f32;
  if (fused_dba) g3.csum_part = static_cast<float*>(scratch);
  tail.to(g3);
  TP_TRY(run(g3, f32, stream));

  // dB_i = H_i^T @ dZ: shard i's rows of dB, no exchange.
  Gemm g4;
  g4.M = f; g4.N = h; g4.K = M;
  g4.a = {H, f, false};
  g4.b = {dZ, h, false};
  g4.epi = kEpiStore;
  g4.out = dB; g4.ldo = h; g4.out_f32 = f32;
  tail.to(g4);
  TP_TRY(run(g4, f32, stream));

  // dA_i = X^T @ dY_i: shard i's columns of dA, no exchange.
  Gemm g5;
  g5.M = h; g5.N = f; g5.K = M;
  g5.a = {X, h, false};
  g5.b = {dY, f, false};
  g5.epi = kEpiStore;
  g5.out = dA; g5.ldo = f; g5.out_f32 = f32;
  g5.n_shard = f / t;
  tail.to(g5);
  TP_TRY(run(g5, f32, stream));

  // dX = sum_i dY_i @ A_i^T: shard partials summed in the accumulator.
  Gemm g6;
  g6.M = M; g6.N = h; g6.K = f;
  g6.a = {dY, f, true};
  g6.b = {A, f, true};  // A [h, f] read as A^T: n = h index, K contiguous
  g6.epi = kEpiStore;
  g6.out = dX; g6.ldo = h; g6.out_f32 = f32;
  tail.to(g6);
  TP_TRY(run(g6, f32, stream));

  if (!f32)  // one launch: dbA from the partials, dbB = colsum(dZ)
    TP_TRY(launch_mlp_bias_grads(
        dZ, M, h, dbB, static_cast<const float*>(scratch), f, dbA,
        static_cast<char*>(scratch) + align_up(dba_partial_bytes(M, f), 256), stream));
  else {
    if (dbA) TP_TRY(launch_colsum(dY, M, f, f32, dbA, scratch, stream));
    if (dbB) TP_TRY(launch_colsum(dZ, M, h, f32, dbB, scratch, stream));
  }
  return TP_OK;
}

// --------------------------------------------------------------- attention

size_t attn_fwd_ws_min(int64_t M, int64_t h, int heads) {
  return align_up(M * 3 * h * 2, 256) + align_up(M * h * 2, 256) +
         align_up(static_cast<size_t>(M) * heads * 4, 256) + 1024;
}

size_t attn_fwd_ws(int64_t M, int64_t h, int heads) { return attn_fwd_ws_min(M, h, heads) + tail_ws(); }

size_t attn_bwd_ws_min(int64_t M, int64_t h, int heads) {
  // The row terms take the most room with one token per sequence (every row
  // padded to 4 floats): b = M, s = 1 bounds every split of M.
  AttnShape sh;
  sh.b = M; sh.s = 1; sh.h = h; sh.heads = heads;
  return 2 * align_up(M * 3 * h * 2, 256) + align_up(M * h * 2, 256) +
         align_up(attn_core_bwd_scratch_bytes(sh), 256) + 1024;
}

size_t attn_bwd_ws(int64_t M, int64_t h, int heads) { return attn_bwd_ws_min(M, h, heads) + tail_ws(); }

tp_status attn_check(const void* X, const void* Wqkv, const void* Wo, int64_t b, int64_t s,
                     int64_t h, int heads, int t, tp_dtype dtype) {
  if (!X || !Wqkv || !Wo) return fail(TP_ERR_NULL, "X, Wqkv and Wo are required");
  TP_TRY(check_dtype(dtype));
  if (dtype != TP_BF16) return fail(TP_ERR_UNSUPPORTED, "attention is implemented for bf16 only");
  if (b <= 0 || s <= 0 || h <= 0 || heads <= 0)
    return fail(TP_ERR_SHAPE, "b, s, h and heads must be positive");
  TP_TRY(check_t(t));
  if (h % heads != 0) return fail(TP_ERR_SHAPE, "h must be divisible by heads");
  if (heads % t != 0) return fail(TP_ERR_SHAPE, "heads must be divisible by t");
  if (h / heads != 128) return fail(TP_ERR_UNSUPPORTED, "head dimension must be 128");
  if (!dims_ok({b, s, 3 * h}) || b * s > kMaxDim) return fail(TP_ERR_SHAPE, "too many tokens");
  TP_TRY(check_rows({h}));
  return TP_OK;
}

tp_status attn_fwd(const void* X, const void* Wqkv, const void* Wo, void* Z, void* QKVsave,
                   void* Osave, void* LSEsave, int64_t b, int64_t s, int64_t h, int heads, int t,
                   int causal, tp_dtype dtype, void* ws, size_t ws_bytes, cudaStream_t stream,
                   const void* residual = nullptr) {
  TP_TRY(attn_check(X, Wqkv, Wo, b, s, h, heads, t, dtype));
  if (!Z) return fail(TP_ERR_NULL, "Z is required");
  TP_TRY(check_ptrs_aligned({X, Wqkv, Wo, Z, QKVsave, Osave, LSEsave, ws}));
  const int64_t M = b * s;
  if (ws == nullptr || ws_bytes < attn_fwd_ws_min(M, h, heads))
    return fail(TP_ERR_WORKSPACE, "workspace missing or smaller than tp_workspace_size()");
  Carve c(ws, ws_bytes);
  void* QKVw = c.take(M * 3 * h * 2);
  void* Ow = c.take(M * h * 2);
  void* LSEw = c.take(static_cast<size_t>(M) * heads * 4);
  const Tail tail(c);
  void* QKV = QKVsave ? QKVsave : QKVw;
  void* O = Osave ? Osave : Ow;
  float* LSE = static_cast<float*>(LSEsave ? LSEsave : LSEw);

  // QKV_g = X @ Wqkv_g: column tiles aligned to the head groups' ranges.
  Gemm gq;
  gq.M = M; gq.N = 3 * h; gq.K = h;
  gq.a = {X, h, true};
  gq.b = {Wqkv, 3 * h, false};
  gq.out = QKV; gq.ldo = 3 * h; gq.out_f16 = true;  // the attention core reads fp16
  gq.n_shard = h / t;
  tail.to(gq);
  TP_TRY(launch_gemm_bf16(gq, stream));

  AttnShape sh;
  sh.b = b; sh.s = s; sh.h = h; sh.heads = heads; sh.causal = causal ? 1 : 0;
  TP_TRY(launch_attn_core_fwd(sh, QKV, O, LSE, stream));

  // Z = sum_g O_g @ Wo_g: group partials summed in the accumulator.
  Gemm go;
  go.M = M; go.N = h; go.K = h;
  go.a = {O, h, true};
  go.b = {Wo, h, false};
  go.out = Z; go.ldo = h;
  go.epi = residual ? kEpiResidual : kEpiStore;  // Z = residual + Attn(X) when given
  go.aux = residual; go.ldaux = h;
  tail.to(go);
  return launch_gemm_bf16(go, stream);
}

tp_status attn_bwd(const void* X, const void* Wqkv, const void* Wo, const void* QKVsave,
                   const void* Osave, const void* LSEsave, const void* dZ, void* dX, void* dWqkv,
                   void* dWo, int64_t b, int64_t s, int64_t h, int heads, int t, int causal,
                   tp_dtype dtype, void* ws, size_t ws_bytes, cudaStream_t stream) {
  TP_TRY(attn_check(X, Wqkv, Wo, b, s, h, heads, t, dtype));
  if (!Osave || !LSEsave || !dZ || !dX || !dWqkv || !dWo)
    return fail(TP_ERR_NULL, "Osave, LSEsave, dZ, dX, dWqkv and dWo are required");
  TP_TRY(check_ptrs_aligned({X, Wqkv, Wo, QKVsave, Osave, LSEsave, dZ, dX, dWqkv, dWo, ws}));
  const int64_t M = b * s;
  if (ws == nullptr || ws_bytes < attn_bwd_ws_min(M, h, heads))
    return fail(TP_ERR_WORKSPACE, "workspace missing or smaller than tp_workspace_size()");
  Carve c(ws, ws_bytes);
  void* QKVw = c.take(M * 3 * h * 2);
  void* dO = c.take(M * h * 2);
  void* dQKV = c.take(M * 3 * h * 2);
  AttnShape sh;
  sh.b = b; sh.s = s; sh.h = h; sh.heads = heads; sh.causal = causal ? 1 : 0;
  void* scratch = c.take(attn_core_bwd_scratch_bytes(sh));
  const Tail tail(c);

  const void* QKV = QKVsave;
  if (QKV == nullptr) {
    Gemm gq;
    gq.M = M; gq.N = 3 * h; gq.K = h;
    gq.a = {X, h, true};
    gq.b = {Wqkv, 3 * h, false};
    gq.out = QKVw; gq.ldo = 3 * h; gq.out_f16 = true;
    gq.n_shard = h / t;
    tail.to(gq);
  TP_TRY(launch_gemm_bf16(gq, stream));
    QKV = QKVw;
  }

  // dO_g = dZ @ Wo_g^T: group g's columns of dO.
  Gemm g1;
  g1.M = M; g1.N = h; g1.K = h;
  g1.a = {dZ, h, true};
  g1.b = {Wo, h, true};
  g1.out = dO; g1.ldo = h; g1.out_f16 = true;  // the attention core reads fp16
  g1.n_shard = h / t;
  tail.to(g1);
  TP_TRY(launch_gemm_bf16(g1, stream));

  // dWo_g = O_g^T @ dZ: group g's rows of dWo, no exchange.
  Gemm g2;
  g2.M = h; g2.N = h; g2.K = M;
  g2.a = {Osave, h, false};
  g2.b = {dZ, h, false};
  g2.out = dWo; g2.ldo = h;
  tail.to(g2);
  TP_TRY(launch_gemm_bf16(g2, stream));

  TP_TRY(launch_attn_core_bwd(sh, QKV, Osave, static_cast<const float*>(LSEsave), dO, dQKV,
                              scratch, stream));

  // dWqkv_g = X^T @ dQKV_g: group g's three column ranges, no exchange.
  Gemm g3;
  g3.M = h; g3.N = 3 * h; g3.K = M;
  g3.a = {X, h, false};
  g3.b = {dQKV, 3 * h, false};
  g3.out = dWqkv; g3.ldo = 3 * h;
  g3.n_shard = h / t;
  tail.to(g3);
  TP_TRY(launch_gemm_bf16(g3, stream));

  // dX = sum_g dQKV_g @ Wqkv_g^T: the K loop visits group 0's q, k and v
  // ranges, then group 1's, ..., all into one accumulator.
  Gemm g4;
  g4.M = M; g4.N = h; g4.K = 3 * h;
  g4.a = {dQKV, 3 * h, true};
  g4.b = {Wqkv, 3 * h, true};
  g4.out = dX; g4.ldo = h;
  const int64_t width = h / t;
  if (width % 64 == 0) {
    g4.korder.range_blocks = static_cast<int>(width / 64);
    g4.korder.t = t;
    g4.korder.width = static_cast<int>(width);
    g4.korder.h = static_cast<int>(h);
  }
  tail.to(g4);
  return launch_gemm_bf16(g4, stream);
}

// -------------------------------------------------------------- LayerNorm

tp_status ln_check(const void* X, const void* Y, int64_t M, int64_t h, tp_dtype dtype) {
  if (!X || !Y) return fail(TP_ERR_NULL, "X and Y are required");
  TP_TRY(check_dtype(dtype));
  if (M <= 0 || h <= 0) return fail(TP_ERR_SHAPE, "M and h must be positive");
  if (!dims_ok({M, h})) return fail(TP_ERR_SHAPE, "M and h must be below 2^31 - 256");
  TP_TRY(check_rows({h}));
  if (h > layernorm_max_h()) return fail(TP_ERR_UNSUPPORTED, "layernorm: h must be at most 16384");
  return TP_OK;
}

size_t ln_bwd_ws(int64_t M, int64_t h) { return align_up(layernorm_bwd_scratch_bytes(M, h), 256) + 256; }

// ------------------------------------------------------------------- block

size_t block_fwd_ws(int64_t M, int64_t h, int64_t f, int heads) {
  const size_t a = attn_fwd_ws(M, h, heads), m = mlp_fwd_ws(M, f, TP_BF16);
  return a > m ? a : m;
}

size_t block_bwd_ws(int64_t M, int64_t h, int64_t f, int heads) {
  size_t inner = mlp_bwd_ws(M, h, f, TP_BF16);
  if (attn_bwd_ws(M, h, heads) > inner) inner = attn_bwd_ws(M, h, heads);
  if (ln_bwd_ws(M, h) > inner) inner = ln_bwd_ws(M, h);
  return 3 * align_up(M * h * 2, 256) + inner + 1024;
}

tp_status block_check(const void* X, const tp_block_weights* w, int64_t b, int64_t s, int64_t h,
                      int64_t f, int heads, int t, tp_dtype dtype) {
  if (!X || !w) return fail(TP_ERR_NULL, "X and the weights are required");
  if (!w->Wqkv || !w->Wo || !w->A || !w->B) return fail(TP_ERR_NULL, "Wqkv, Wo, A and B are required");
  TP_TRY(attn_check(X, w->Wqkv, w->Wo, b, s, h, heads, t, dtype));
  if (f <= 0 || f % t != 0) return fail(TP_ERR_SHAPE, "f must be positive and divisible by t");
  TP_TRY(check_rows({f}));
  if (h > layernorm_max_h()) return fail(TP_ERR_UNSUPPORTED, "layernorm: h must be at most 16384");
  TP_TRY(check_ptrs_aligned({X, w->ln1_g, w->ln1_b, w->Wqkv, w->Wo, w->ln2_g, w->ln2_b, w->A,
                             w->bA, w->B, w->bB}));
  return TP_OK;
}

tp_status block_fwd(const void* X, const tp_block_weights* w, void* X2, tp_block_saves* sv,
                    int64_t b, int64_t s, int64_t h, int64_t f, int heads, int t, float eps,
                    tp_dtype dtype, void* ws, size_t ws_bytes, cudaStream_t stream) {
  TP_TRY(block_check(X, w, b, s, h, f, heads, t, dtype));
  if (!X2 || !sv) return fail(TP_ERR_NULL, "X2 and the saves are required");
  if (!sv->Xn1 || !sv->mean1 || !sv->rstd1 || !sv->QKV || !sv->O || !sv->LSE || !sv->X1 ||
      !sv->Xn2 || !sv->mean2 || !sv->rstd2 || !sv->Y)
    return fail(TP_ERR_NULL, "every tp_block_saves pointer is required");
  TP_TRY(check_ptrs_aligned({X2, sv->Xn1, sv->QKV, sv->O, sv->LSE, sv->X1, sv->Xn2, sv->Y, ws}));
  const int64_t M = b * s;
  if (ws == nullptr || ws_bytes < block_fwd_ws(M, h, f, heads))
    return fail(TP_ERR_WORKSPACE, "workspace missing or smaller than tp_workspace_size()");
  // X1 = X + Attn(LN1(X))
  TP_TRY(launch_layernorm_fwd(X, w->ln1_g, w->ln1_b, sv->Xn1, sv->mean1, sv->rstd1, M, h, eps,
                              false, stream));
  TP_TRY(attn_fwd(sv->Xn1, w->Wqkv, w->Wo, sv->X1, sv->QKV, sv->O, sv->LSE, b, s, h, heads, t, 1,
                  dtype, ws, ws_bytes, stream, X));
  // X2 = X1 + MLP(LN2(X1))
  TP_TRY(launch_layernorm_fwd(sv->X1, w->ln2_g, w->ln2_b, sv->Xn2, sv->mean2, sv->rstd2, M, h,
                              eps, false, stream));
  return mlp_fwd(sv->Xn2, w->A, w->bA, w->B, w->bB, X2, sv->Y, M, h, f, t, dtype, ws, ws_bytes,
                 stream, sv->X1);
}

tp_status block_bwd(const void* X, const tp_block_weights* w, const tp_block_saves* sv,
                    const void* dX2, void* dX, const tp_block_grads* g, int64_t b, int64_t s,
                    int64_t h, int64_t f, int heads, int t, float eps, tp_dtype dtype, void* ws,
                    size_t ws_bytes, cudaStream_t stream) {
  (void)eps;
  TP_TRY(block_check(X, w, b, s, h, f, heads, t, dtype));
  if (!sv || !dX2 || !dX || !g) return fail(TP_ERR_NULL, "saves, dX2, dX and the grads are required");
  if (!sv->Xn1 || !sv->mean1 || !sv->rstd1 || !sv->QKV || !sv->O || !sv->LSE || !sv->X1 ||
      !sv->Xn2 || !sv->mean2 || !sv->rstd2 || !sv->Y)
    return fail(TP_ERR_NULL, "every tp_block_saves pointer is required");
  if (!g->dWqkv || !g->dWo || !g->dA || !g->dB)
    return fail(TP_ERR_NULL, "dWqkv, dWo, dA and dB are required");
  TP_TRY(check_ptrs_aligned({dX2, dX, g->dln1_g, g->dln1_b, g->dWqkv, g->dWo, g->dln2_g, g->dln2_b,
                             g->dA, g->dbA, g->dB, g->dbB, ws}));
  const int64_t M = b * s;
  if (ws == nullptr || ws_bytes < block_bwd_ws(M, h, f, heads))
    return fail(TP_ERR_WORKSPACE, "workspace missing or smaller than tp_workspace_size()");
  Carve c(ws, ws_bytes);
  void* dXn2 = c.take(M * h * 2);
  void* dX1 = c.take(M * h * 2);
  void* dXn1 = c.take(M * h * 2);
  void* inner = c.take(0);
  const size_t inner_bytes = ws_bytes - (static_cast<char*>(inner) - static_cast<char*>(ws));
  // MLP sublayer, then LN2 with the residual path's gradient joining: dX1.
  TP_TRY(mlp_bwd(sv->Xn2, w->A, w->bA, w->B, sv->Y, dX2, dXn2, g->dA, g->dbA, g->dB, g->dbB, M, h,
                 f, t, dtype, inner, inner_bytes, stream));
  TP_TRY(launch_layernorm_bwd(sv->X1, w->ln2_g, sv->mean2, sv->rstd2, dXn2, dX2, dX1, g->dln2_g,
                              g->dln2_b, M, h, false, inner, stream));
  // Attention sublayer, then LN1 with the residual gradient: dX.
  TP_TRY(attn_bwd(sv->Xn1, w->Wqkv, w->Wo, sv->QKV, sv->O, sv->LSE, dX1, dXn1, g->dWqkv, g->dWo, b,
                  s, h, heads, t, 1, dtype, inner, inner_bytes, stream));
  return launch_layernorm_bwd(X, w->ln1_g, sv->mean1, sv->rstd1, dXn1, dX1, dX, g->dln1_g,
                              g->dln1_b, M, h, false, inner, stream);
}

// -------------------------------------------------------------- vocabulary

tp_status vocab_common(int64_t M, int64_t V, int64_t h, int t, tp_dtype dtype) {
  TP_TRY(check_dtype(dtype));
  if (M < 0 || V <= 0 || h <= 0) return fail(TP_ERR_SHAPE, "M must be >= 0, V and h positive");
  TP_TRY(check_t(t));
  if (V % t != 0) return fail(TP_ERR_SHAPE, "V must be divisible by t (vocabulary split)");
  if (V > 0x7fffffffLL) return fail(TP_ERR_SHAPE, "V must fit the int32 token ids");
  TP_TRY(check_rows({h}));
  return TP_OK;
}

tp_status vocab_embed_fwd(const int32_t* ids, const void* E, void* Y, int64_t M, int64_t V,
                          int64_t h, int t, tp_dtype dtype, cudaStream_t stream) {
  if (ids == nullptr || E == nullptr || Y == nullptr)
    return fail(TP_ERR_NULL, "ids, E and Y are required");
  TP_TRY(vocab_common(M, V, h, t, dtype));
  TP_TRY(check_ptrs_aligned({E, Y}));
  return launch_embed_fwd(ids, E, Y, M, V, h, t, dtype == TP_F32, stream);
}

size_t embed_bwd_ws(int64_t M) { return align_up(embed_bwd_scratch_bytes(M), 256) + 256; }

tp_status vocab_embed_bwd(const int32_t* ids, const void* dY, const void* dE_in, void* dE,
                          int64_t M, int64_t V, int64_t h, int t, tp_dtype dtype, void* ws,
                          size_t ws_bytes, cudaStream_t stream) {
  if (dE == nullptr || (M > 0 && (ids == nullptr || dY == nullptr)))
    return fail(TP_ERR_NULL, "dE is required, and ids and dY when M > 0");
  TP_TRY(vocab_common(M, V, h, t, dtype));
  if (M >= (1ll << 28)) return fail(TP_ERR_SHAPE, "embedding backward: M must be below 2^28");
  TP_TRY(check_ptrs_aligned({dY, dE_in, dE, ws}));
  if (M > 0 && (ws == nullptr || ws_bytes < embed_bwd_ws(M)))
    return fail(TP_ERR_WORKSPACE, "workspace missing or smaller than tp_workspace_size()");
  return launch_embed_bwd(ids, dY, dE_in, dE, M, V, h, dtype == TP_F32, ws, stream);
}

int64_t ce_chunks_per_shard(int64_t V, int t) { return (V / t + 31) / 32; }

size_t ce_fwd_ws(int64_t M, int64_t V, int t) {
  const int64_t ldp = t * ce_chunks_per_shard(V, t);
  return align_up(static_cast<size_t>(M) * ldp * 8, 256) + align_up(M * 4, 256) +
         align_up(static_cast<size_t>(t) * 4, 256) + 1024;
}

tp_status ce_check(int64_t M, int64_t h, int64_t V, int t, tp_dtype dtype) {
  TP_TRY(vocab_common(M, V, h, t, dtype));
  if (dtype != TP_BF16) return fail(TP_ERR_DTYPE, "the vocabulary cross-entropy is bf16 only");
  if ((V / t) % 8 != 0) return fail(TP_ERR_ALIGN, "V / t must be a multiple of 8");
  return TP_OK;
}

tp_status vocab_ce_fwd(const void* X, const void* E, const int32_t* targets, void* logits,
                       float* lse, float* loss, float* total, int64_t M, int64_t h, int64_t V,
                       int t, tp_dtype dtype, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (X == nullptr || E == nullptr || targets == nullptr || lse == nullptr || loss == nullptr)
    return fail(TP_ERR_NULL, "X, E, targets, lse and loss are required");
  TP_TRY(ce_check(M, h, V, t, dtype));
  TP_TRY(check_ptrs_aligned({X, E, logits, ws}));
  if (M == 0) {
    if (total == nullptr) return TP_OK;
    cudaError_t e = cudaMemsetAsync(total, 0, sizeof(float), stream);
    return e == cudaSuccess ? TP_OK : cuda_fail(e, "cudaMemsetAsync(total)");
  }
  if (ws == nullptr || ws_bytes < ce_fwd_ws(M, V, t))
    return fail(TP_ERR_WORKSPACE, "workspace missing or smaller than tp_workspace_size()");
  Carve c(ws, ws_bytes);
  CEOut ce;
  ce.cps = static_cast<int>(ce_chunks_per_shard(V, t));
  ce.ldp = static_cast<int64_t>(t) * ce.cps;
  ce.part = static_cast<float*>(c.take(static_cast<size_t>(M) * ce.ldp * 8));
  ce.tlogit = static_cast<float*>(c.take(M * 4));
  ce.target = targets;
  float* shard_tot = static_cast<float*>(c.take(static_cast<size_t>(t) * 4));
  // Step 1: every shard's logits X @ E_i^T in one GEMM whose column tiles
  // never straddle a shard; the epilogue reduces each 32-column chunk.
  Gemm g;
  g.M = M;
  g.N = V;
  g.K = h;
  g.a = {X, h, true};
  g.b = {E, h, true};  // B(k, v) = E[v, k]
  g.epi = kEpiCE;
  g.out = logits;
  g.ldo = V;
  g.n_shard = V / t;
  g.ce = ce;
  TP_TRY(launch_gemm_bf16(g, stream));
  // Steps 2-6.
  return launch_ce_finish(ce, t, M, V, lse, loss, total, shard_tot, stream);
}

tp_status vocab_ce_bwd(const void* X, const void* E, const int32_t* targets, const void* logits,
                       const float* lse, const float* dloss, void* dlogits, void* dX, void* dE,
                       int64_t M, int64_t h, int64_t V, int t, tp_dtype dtype,
                       cudaStream_t stream) {
  if (X == nullptr || E == nullptr || targets == nullptr || logits == nullptr || lse == nullptr ||
      dlogits == nullptr)
    return fail(TP_ERR_NULL, "X, E, targets, logits, lse and dlogits are required");
  TP_TRY(ce_check(M, h, V, t, dtype));
  TP_TRY(check_ptrs_aligned({X, E, logits, dlogits, dX, dE}));
  if (M == 0) {
    if (dE == nullptr) return TP_OK;
    cudaError_t e = cudaMemsetAsync(dE, 0, static_cast<size_t>(V) * h * 2, stream);
    return e == cudaSuccess ? TP_OK : cuda_fail(e, "cudaMemsetAsync(dE)");
  }
  TP_TRY(launch_ce_dlogits(logits, lse, targets, dloss, dlogits, M, V, stream));
  if (dX != nullptr) {
    // dX = sum over shards of dlogits_i @ E_i: one K loop over all V.
    Gemm g;
    g.M = M;
    g.N = h;
    g.K = V;
    g.a = {dlogits, V, true};
    g.b = {E, h, false};
    g.out = dX;
    g.ldo = h;
    TP_TRY(launch_gemm_bf16(g, stream));
  }
  if (dE != nullptr) {
    // dE = dlogits^T @ X: row v of dE needs only column v of dlogits, so each
    // shard's rows come from its own logits.
    Gemm g;
    g.M = V;
    g.N = h;
    g.K = M;
    g.a = {dlogits, V, false};
    g.b = {X, h, false};
    g.out = dE;
    g.ldo = h;
    TP_TRY(launch_gemm_bf16(g, stream));
  }
  return TP_OK;
}

}  // namespace
}  // namespace tp

using namespace tp;

#define TP_GUARD(body)                                              \
  try {                                                             \
    body                                                            \
  } catch (const std::exception& e) {                               \
    return fail(TP_ERR_UNSUPPORTED, std::string("internal: ") + e.what()); \
  } catch (...) {                                                   \
    return fail(TP_ERR_UNSUPPORTED, "internal error");              \
  }

namespace tp {
namespace {
// The bounded-wait self-test: an mbarrier that nothing ever arrives on.
// Warp 0 waits on it with the short limit `short_ns` and gives up, recording
// kStatusSelftestTimeout; warp 1 waits with the default limit and must be
// released early by warp 0's abort (same launch generation).  No copy or
// tensor-core work is in flight, so giving up leaves nothing behind.
__global__ void bounded_wait_selftest_kernel(WaitCtl w, unsigned long long short_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) {
    WaitCtl mine = w;
    if (threadIdx.x == 0) mine.limit_ns = short_ns;
    mbar_wait(&bar, 0, mine, kStatusSelftestTimeout);
  }
  __syncwarp();
}
}  // namespace
}  // namespace tp

extern "C" {

tp_status tp_linear_col(const void* X, const void* W, const void* bias, void* Y, int64_t M,
                        int64_t K, int64_t N, int t, int shard, tp_dtype dtype,
                        tp_dtype out_dtype, void* stream) {
  TP_GUARD(return linear_common(X, W, bias, Y, M, K, N, t, shard, dtype, out_dtype, true,
                                static_cast<cudaStream_t>(stream));)
}

tp_status tp_linear_row(const void* X, const void* W, const void* bias, void* Z, int64_t M,
                        int64_t K, int64_t N, int t, int shard, tp_dtype dtype,
                        tp_dtype out_dtype, void* stream) {
  TP_GUARD(return linear_common(X, W, bias, Z, M, K, N, t, shard, dtype, out_dtype, false,
                                static_cast<cudaStream_t>(stream));)
}

tp_status tp_mlp_fwd(const void* X, const void* A, const void* bA, const void* B, const void* bB,
                     void* Z, void* Ysave, int64_t M, int64_t h, int64_t f, int t, tp_dtype dtype,
                     void* ws, size_t ws_bytes, void* stream) {
  TP_GUARD(return mlp_fwd(X, A, bA, B, bB, Z, Ysave, M, h, f, t, dtype, ws, ws_bytes,
                          static_cast<cudaStream_t>(stream));)
}

tp_status tp_mlp_bwd(const void* X, const void* A, const void* bA, const void* B,
                     const void* Ysave, const void* dZ, void* dX, void* dA, void* dbA, void* dB,
                     void* dbB, int64_t M, int64_t h, int64_t f, int t, tp_dtype dtype, void* ws,
                     size_t ws_bytes, void* stream) {
  TP_GUARD(return mlp_bwd(X, A, bA, B, Ysave, dZ, dX, dA, dbA, dB, dbB, M, h, f, t, dtype, ws,
                          ws_bytes, static_cast<cudaStream_t>(stream));)
}

tp_status tp_attn_fwd(const void* X, const void* Wqkv, const void* Wo, void* Z, void* QKVsave,
                      void* Osave, void* LSEsave, int64_t b, int64_t s, int64_t h, int heads,
                      int t, int causal, tp_dtype dtype, void* ws, size_t ws_bytes,
                      void* stream) {
  TP_GUARD(return attn_fwd(X, Wqkv, Wo, Z, QKVsave, Osave, LSEsave, b, s, h, heads, t, causal,
                           dtype, ws, ws_bytes, static_cast<cudaStream_t>(stream));)
}

tp_status tp_attn_bwd(const void* X, const void* Wqkv, const void* Wo, const void* QKVsave,
                      const void* Osave, const void* LSEsave, const void* dZ, void* dX,
                      void* dWqkv, void* dWo, int64_t b, int64_t s, int64_t h, int heads, int t,
                      int causal, tp_dtype dtype, void* ws, size_t ws_bytes, void* stream) {
  TP_GUARD(return attn_bwd(X, Wqkv, Wo, QKVsave, Osave, LSEsave, dZ, dX, dWqkv, dWo, b, s, h,
                           heads, t, causal, dtype, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream));)
}

tp_status tp_layernorm_fwd(const void* X, const void* gamma, const void* beta, void* Y,
                           float* mean, float* rstd, int64_t M, int64_t h, float eps,
                           tp_dtype dtype, void* stream) {
  TP_GUARD(TP_TRY(ln_check(X, Y, M, h, dtype));
           TP_TRY(check_ptrs_aligned({X, gamma, beta, Y, mean, rstd}));
           return launch_layernorm_fwd(X, gamma, beta, Y, mean, rstd, M, h, eps, dtype == TP_F32,
                                       static_cast<cudaStream_t>(stream));)
}

tp_status tp_layernorm_bwd(const void* X, const void* gamma, const float* mean,
                           const float* rstd, const void* dY, const void* dR, void* dX,
                           void* dgamma, void* dbeta, int64_t M, int64_t h, tp_dtype dtype,
                           void* ws, size_t ws_bytes, void* stream) {
  TP_GUARD(TP_TRY(ln_check(X, dX, M, h, dtype));
           if (!mean || !rstd || !dY) return fail(TP_ERR_NULL, "mean, rstd and dY are required");
           TP_TRY(check_ptrs_aligned({X, gamma, dY, dR, dX, dgamma, dbeta, ws}));
           if (ws == nullptr || ws_bytes < ln_bwd_ws(M, h))
             return fail(TP_ERR_WORKSPACE, "workspace missing or smaller than tp_workspace_size()");
           return launch_layernorm_bwd(X, gamma, mean, rstd, dY, dR, dX, dgamma, dbeta, M, h,
                                       dtype == TP_F32, ws, static_cast<cudaStream_t>(stream));)
}

tp_status tp_block_fwd(const void* X, const tp_block_weights* w, void* X2, tp_block_saves* saves,
                       int64_t b, int64_t s, int64_t h, int64_t f, int heads, int t, float eps,
                       tp_dtype dtype, void* ws, size_t ws_bytes, void* stream) {
  TP_GUARD(return block_fwd(X, w, X2, saves, b, s, h, f, heads, t, eps, dtype, ws, ws_bytes,
                            static_cast<cudaStream_t>(stream));)
}

tp_status tp_block_bwd(const void* X, const tp_block_weights* w, const tp_block_saves* saves,
                       const void* dX2, void* dX, const tp_block_grads* g, int64_t b, int64_t s,
                       int64_t h, int64_t f, int heads, int t, float eps, tp_dtype dtype,
                       void* ws, size_t ws_bytes, void* stream) {
  TP_GUARD(return block_bwd(X, w, saves, dX2, dX, g, b, s, h, f, heads, t, eps, dtype, ws,
                            ws_bytes, static_cast<cudaStream_t>(stream));)
}

tp_status tp_vocab_embed_fwd(const int32_t* ids, const void* E, void* Y, int64_t M, int64_t V,
                             int64_t h, int t, tp_dtype dtype, void* stream) {
  TP_GUARD(return vocab_embed_fwd(ids, E, Y, M, V, h, t, dtype,
                                  static_cast<cudaStream_t>(stream));)
}

tp_status tp_vocab_embed_bwd(const int32_t* ids, const void* dY, const void* dE_in, void* dE,
                             int64_t M, int64_t V, int64_t h, int t, tp_dtype dtype, void* ws,
                             size_t ws_bytes, void* stream) {
  TP_GUARD(return vocab_embed_bwd(ids, dY, dE_in, dE, M, V, h, t, dtype, ws, ws_bytes,
                                  static_cast<cudaStream_t>(stream));)
}

tp_status tp_vocab_ce_fwd(const void* X, const void* E, const int32_t* targets, void* logits,
                          float* lse, float* loss, float* total, int64_t M, int64_t h, int64_t V,
                          int t, tp_dtype dtype, void* ws, size_t ws_bytes, void* stream) {
  TP_GUARD(return vocab_ce_fwd(X, E, targets, logits, lse, loss, total, M, h, V, t, dtype, ws,
                               ws_bytes, static_cast<cudaStream_t>(stream));)
}

tp_status tp_vocab_ce_bwd(const void* X, const void* E, const int32_t* targets,
                          const void* logits, const float* lse, const float* dloss,
                          void* dlogits, void* dX, void* dE, int64_t M, int64_t h, int64_t V,
                          int t, tp_dtype dtype, void* stream) {
  TP_GUARD(return vocab_ce_bwd(X, E, targets, logits, lse, dloss, dlogits, dX, dE, M, h, V, t,
                               dtype, static_cast<cudaStream_t>(stream));)
}

size_t tp_workspace_size(tp_op op, int64_t M, int64_t h, int64_t f, int heads, int t,
                         tp_dtype dtype) {
  try {
    if (M <= 0 || h <= 0 || t < 1 || (dtype != TP_F32 && dtype != TP_BF16)) return 0;
    if (!dims_ok({M, h, f})) return 0;
    switch (op) {
      case TP_OP_MLP_FWD: return f > 0 ? mlp_fwd_ws(M, f, dtype) : 0;
      case TP_OP_MLP_BWD: return f > 0 ? mlp_bwd_ws(M, h, f, dtype) : 0;
      case TP_OP_ATTN_FWD: return heads > 0 ? attn_fwd_ws(M, h, heads) : 0;
      case TP_OP_ATTN_BWD: return heads > 0 ? attn_bwd_ws(M, h, heads) : 0;
      case TP_OP_LN_BWD: return ln_bwd_ws(M, h);
      case TP_OP_BLOCK_FWD: return (heads > 0 && f > 0) ? block_fwd_ws(M, h, f, heads) : 0;
      case TP_OP_BLOCK_BWD: return (heads > 0 && f > 0) ? block_bwd_ws(M, h, f, heads) : 0;
      case TP_OP_VOCAB_CE_FWD: return (f > 0 && f % t == 0) ? ce_fwd_ws(M, f, t) : 0;
      case TP_OP_VOCAB_EMBED_BWD: return embed_bwd_ws(M);
    }
  } catch (...) {
  }
  return 0;
}

const char* tp_last_error(void) { return g_last_error.c_str(); }

tp_status tp_device_status(void* stream) {
  try {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    DeviceStatus* p = device_status_ptr();
    if (p == nullptr) return fail(TP_ERR_CUDA, "device status unavailable");
    DeviceStatus v{};
    e = cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status");
    if (v.code == 0 && v.flags == 0 && v.abort_gen == 0) return TP_OK;
    const DeviceStatus zero{};
    e = cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status");
    const char* sat = (v.flags & kFlagF16Range) ? "; an fp16 attention intermediate (QKV or dO) "
                                                  "exceeded the fp16 range and was saturated"
                                                : "";
    char buf[256];
    if (v.code != 0) {
      const char* who = v.code == kStatusProducerTimeout   ? "GEMM TMA producer"
                        : v.code == kStatusMmaTimeout      ? "GEMM MMA issuer"
                        : v.code == kStatusEpilogueTimeout ? "GEMM epilogue"
                        : v.code == kStatusAttnTimeout     ? "attention kernel"
                        : v.code == kStatusSelftestTimeout ? "bounded-wait self-test"
                                                           : "unknown";
      std::snprintf(buf, sizeof(buf), "kernel gave up a bounded wait (code 0x%x, %s)%s", v.code,
                    who, sat);
      return fail(TP_ERR_KERNEL, buf);
    }
    if (v.flags & kFlagF16Range) {
      std::snprintf(buf, sizeof(buf),
                    "an fp16 attention intermediate (QKV or dO) exceeded the fp16 range and was "
                    "saturated (flags 0x%x)", v.flags);
      return fail(TP_ERR_KERNEL, buf);
    }
    return TP_OK;
  } catch (...) {
    return fail(TP_ERR_UNSUPPORTED, "internal error");
  }
}

tp_status tp_selftest_bounded_wait(int64_t limit_ns, void* stream) {
  try {
    if (limit_ns < 1000 || limit_ns > static_cast<int64_t>(kWaitLimitNs))
      return fail(TP_ERR_SHAPE, "limit_ns must be in [1e3, 2e9]");
    WaitCtl w = wait_ctl();
    if (w.st == nullptr) return fail(TP_ERR_CUDA, "device status unavailable");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    bounded_wait_selftest_kernel<<<1, 64, 0, s>>>(w, static_cast<unsigned long long>(limit_ns));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "bounded-wait self-test launch");
    return TP_OK;
  } catch (...) {
    return fail(TP_ERR_UNSUPPORTED, "internal error");
  }
}

tp_status tp_profile_enable(int on) {
  try {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    g_prof_on = on != 0;
    if (g_prof_on) g_prof_used = 0;
    return TP_OK;
  } catch (...) {
    return fail(TP_ERR_UNSUPPORTED, "internal error");
  }
}

tp_status tp_profile_read(tp_kernel_kind kind, tp_profile_stats* out) {
  try {
    if (out == nullptr) return fail(TP_ERR_NULL, "out is required");
    if (kind < 0 || kind >= TP_KIND_COUNT) return fail(TP_ERR_SHAPE, "unknown kernel kind");
    std::lock_guard<std::mutex> lock(g_prof_mu);
    tp_profile_stats st{0, 0.0, 0.0, 0.0};
    for (size_t i = 0; i < g_prof_used; ++i) {
      const ProfRecord& r = g_prof[i];
      if (r.kind != kind) continue;
      cudaError_t e = cudaEventSynchronize(r.stop);
      if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
      float ms = 0.0f;
      e = cudaEventElapsedTime(&ms, r.start, r.stop);
      if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
      st.launches += 1;
      st.total_ms += ms;
      st.flops += r.flops;
      st.bytes += r.bytes;
    }
    *out = st;
    return TP_OK;
  } catch (...) {
    return fail(TP_ERR_UNSUPPORTED, "internal error");
  }
}

int64_t tp_launch_count(void) { return g_launches.load(); }

int64_t tp_profile_count(void) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  return static_cast<int64_t>(g_prof_used);
}

tp_status tp_profile_record(int64_t index, tp_launch_record* out) {
  try {
    if (out == nullptr) return fail(TP_ERR_NULL, "out is required");
    std::lock_guard<std::mutex> lock(g_prof_mu);
    if (index < 0 || static_cast<size_t>(index) >= g_prof_used)
      return fail(TP_ERR_SHAPE, "no such launch record");
    const ProfRecord& r = g_prof[static_cast<size_t>(index)];
    cudaError_t e = cudaEventSynchronize(r.stop);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    float ms = 0.0f;
    e = cudaEventElapsedTime(&ms, r.start, r.stop);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
    out->kind = r.kind;
    out->tile = r.tile;
    out->m = r.m;
    out->n = r.n;
    out->k = r.k;
    out->ms = ms;
    out->flops = r.flops;
    out->bytes = r.bytes;
    return TP_OK;
  } catch (...) {
    return fail(TP_ERR_UNSUPPORTED, "internal error");
  }
}

int tp_version(void) { return 100; }

int64_t tp_gemm_plan(int64_t M, int64_t N, int64_t K, int64_t n_shard, int kind, int sms,
                     int tail_scratch, tp_gemm_unit* out, int64_t cap) {
  try {
    const int64_t want = (out != nullptr && cap > 0) ? cap : 0;
    std::vector<tp::GemmPlanUnit> units(static_cast<size_t>(want));
    const int64_t n = tp::gemm_plan_units(M, N, K, n_shard, kind, sms, tail_scratch != 0,
                                          units.data(), want);
    for (int64_t i = 0; i < n && i < want; ++i) {
      const tp::GemmPlanUnit& u = units[static_cast<size_t>(i)];
      out[i] = tp_gemm_unit{u.m0, u.rows, u.n0, u.n_end, u.kb0, u.kb1, u.part, u.tile};
    }
    return n;
  } catch (...) {
    return -1;
  }
}

}  // extern "C"
