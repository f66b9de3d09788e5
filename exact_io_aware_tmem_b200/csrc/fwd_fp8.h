// Pass 2 of the FP8 (E4M3) forward on the two-tile kernel (fwd_pair.cu).
#pragma once

#include "params.h"

namespace fa {

// D = 128: p.q / p.k hold E4M3 codes [B*N, H or H_kv, 128], ``f`` their
// per-block steps (pass 1's output).
cudaError_t launch_fwd_pair_fp8(const AttnParams& p, const Fp8Args& f, cudaStream_t stream);

}  // namespace fa
