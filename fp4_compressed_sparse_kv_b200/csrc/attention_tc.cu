// attention_tc.cu -- step 4 on the tcgen05 tensor cores (not yet enabled).
#include "attention_common.cuh"

namespace csa {

bool attn_tc_supported(int) { return false; }

int attn_units_per_tile(int) { return 4; }

cudaError_t launch_attn_tc(const AttnArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace csa
