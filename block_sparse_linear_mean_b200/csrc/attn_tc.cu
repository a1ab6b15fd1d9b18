// Tensor-core (tcgen05) block-sparse attention forward: not built yet; the
// SIMT kernel serves every configuration until it is.
#include "internal.h"

namespace sla {

bool attn_tc_supported(const Geom&) { return false; }
size_t attn_tc_scratch_bytes(const Geom&) { return 0; }
cudaError_t launch_attn_tc(const void*, const void*, const void*, const Geom&,
                           const sla_block_lists&, float*, float*, int32_t*,
                           void*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace sla
