// Attention backward, bf16 on the sm_100a tensor cores (not built yet).
#include "params.h"

namespace fa {

cudaError_t launch_bwd_bf16(const AttnParams&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace fa
