// The D = 64 forward: one 128-row query tile and one softmax group per CTA,
// two CTAs per SM (fwd_d64.cu).
#pragma once

#include "params.h"

namespace fa {

cudaError_t launch_fwd_d64(const AttnParams& p, cudaStream_t stream);

}  // namespace fa
