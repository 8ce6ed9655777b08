// Attention core: placeholder until the kernels land.
#include "tp_internal.h"

namespace tp {

tp_status launch_attn_core_fwd(const AttnShape&, const void*, void*, float*, cudaStream_t) {
  return fail(TP_ERR_UNSUPPORTED, "attention core not built yet");
}

size_t attn_core_bwd_scratch_bytes(const AttnShape& sh) {
  return static_cast<size_t>(sh.b * sh.s) * (sh.h + sh.heads) * 4;
}

tp_status launch_attn_core_bwd(const AttnShape&, const void*, const void*, const float*,
                               const void*, void*, void*, cudaStream_t) {
  return fail(TP_ERR_UNSUPPORTED, "attention core not built yet");
}

}  // namespace tp
