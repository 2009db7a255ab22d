// Tensor-core (tcgen05) sparse MQA attention — placeholder until the sm_100a kernel lands.
#include "internal.h"

namespace dsv4 {
bool attn_tc_supported(const AttnArgs&, int) { return false; }
cudaError_t launch_attn_tc(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace dsv4
