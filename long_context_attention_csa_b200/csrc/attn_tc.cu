// Shared-KV MQA on tcgen05 (bf16 operands, fp32 TMEM).
#include "tc.h"

namespace csa {

bool attn_tc_supported(const AttnParams&) { return false; }
size_t attn_tc_scratch(int64_t, int64_t, int, int, int64_t) { return 0; }
cudaError_t launch_attn_tc(const AttnParams&, cudaStream_t, unsigned long long* n) {
  *n = 0;
  return cudaErrorNotSupported;
}

}  // namespace csa
