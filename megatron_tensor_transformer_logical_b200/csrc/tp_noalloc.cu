// tp_mlp_fwd_noalloc: the partitioned MLP forward for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand libtp a workspace: a host that owns every
// byte of device memory and forbids allocation on the inference path, code
// running where cudaMalloc's implicit device synchronisation is not
// acceptable (a latency-critical serving loop), or a plugin interface that
// passes only inputs and outputs.  For them this entry point keeps the one
// intermediate the MLP forward needs, H = GeLU(X @ A + bA) [M, f], in a
// fixed array compiled into the library, and otherwise runs exactly the
// kernels of tp_mlp_fwd.
//
// The array lives in every GPU's memory from the moment libtp's device code
// is loaded there until the process exits.  Device code could name it
// directly; host code must not (its name in host code is a stand-in, not a
// device address), so its address is looked up with cudaGetSymbolAddress,
// with the device current, on the first call made in each context there
// (a new context, after cudaDeviceReset for instance, loads the device code
// again, possibly at another address, and the lookup is repeated).
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "../../include/libtp.h"
#include "tp_internal.h"

namespace tp {
namespace {

// The limit on H [M, f] (M * f * element size).  The array is 256 bytes
// larger: tp_mlp_fwd's workspace holds H rounded up to 256 bytes plus 256.
constexpr size_t kNoAllocHBytes = size_t(64) << 20;  // 64 MiB
constexpr size_t kNoAllocScratchBytes = kNoAllocHBytes + 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_mlp_fwd_scratch[kNoAllocScratchBytes];

// Device address of the scratch array in the current context (looked up on
// the first call per device and context), or nullptr with the CUDA error in
// *err.
void* scratch_address(cudaError_t* err) {
  static void* addr[kMaxDevices] = {};
  static unsigned long long ctx_ids[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long id = current_context_id();
  if (addr[dev] == nullptr || id == 0 || id != ctx_ids[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_mlp_fwd_scratch);
    if (*err != cudaSuccess) return nullptr;
    addr[dev] = p;
    ctx_ids[dev] = current_context_id();  // the lookup made the context current
  }
  return addr[dev];
}

}  // namespace
}  // namespace tp

extern "C" tp_status tp_mlp_fwd_noalloc(const void* X, const void* A, const void* bA,
                                        const void* B, const void* bB, void* Z, void* Ysave,
                                        int64_t M, int64_t h, int64_t f, int t, tp_dtype dtype,
                                        void* stream) {
  try {
    if (dtype != TP_F32 && dtype != TP_BF16) return tp::fail(TP_ERR_DTYPE, "unknown dtype");
    if (M <= 0 || h <= 0 || f <= 0) return tp::fail(TP_ERR_SHAPE, "M, h and f must be positive");
    const int64_t es = dtype == TP_F32 ? 4 : 2;
    // M * f * es <= 64 MiB, checked without forming a product that could overflow.
    const int64_t max_elems = static_cast<int64_t>(tp::kNoAllocHBytes) / es;
    if (f > max_elems || M > max_elems / f)
      return tp::fail(TP_ERR_SHAPE,
                      "tp_mlp_fwd_noalloc: H [M, f] = [" + std::to_string(M) + ", " +
                          std::to_string(f) + "] does not fit its fixed 64 MiB (67108864-byte) "
                          "array (M * f * element size must be <= 67108864); use tp_mlp_fwd "
                          "with a caller workspace");
    cudaError_t e = cudaSuccess;
    void* scratch = tp::scratch_address(&e);
    if (scratch == nullptr) return tp::cuda_fail(e, "tp_mlp_fwd_noalloc: cudaGetSymbolAddress");
    return tp_mlp_fwd(X, A, bA, B, bB, Z, Ysave, M, h, f, t, dtype, scratch,
                      tp::kNoAllocScratchBytes, stream);
  } catch (...) {
    return tp::fail(TP_ERR_UNSUPPORTED, "internal error");
  }
}
