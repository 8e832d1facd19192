// Block-sparse attention on the 5th-generation tensor cores (tcgen05 + TMEM +
// TMA), bf16, head dim 128, tile 128.
#include "veda_internal.cuh"

namespace veda {

bool attn_tc_supported(const AttnParams&) { return false; }

cudaError_t launch_attn_tc(const AttnParams&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace veda
