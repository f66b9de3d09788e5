// Balanced decode: the partials kernel with the keys on the TMEM lanes and
// the merge that follows it (decode_t.cu). fa_decode uses it for D = 128 and
// at most 64 query rows per kv head when the caller leaves the split count to
// the library.
#pragma once

#include "params.h"

namespace fa {

// The U = H_kv * sum_b ceil(len_b / 128) units (sequence b, kv head, 128-key
// tile), taken in that order, are cut into ``ctas`` contiguous ranges of
// equal size, one per persistent CTA. A (sequence, kv head) segment cut by a
// range boundary yields one partial per CTA that holds part of it, in slot
// segment + CTA (unique: walking the pieces in order, segment + CTA grows by
// one or two at each step).
struct DecodeTArgs {
  int ctas;          // persistent CTAs (one per SM)
  int* seg_first;    // [B * H_kv] first CTA holding a tile of the segment
  int* seg_last;     // [B * H_kv] last such CTA
  float* o_part;     // [(B * H_kv + ctas) * n_rows, D] fp32 partial O / l
  float* lse_part;   // [(B * H_kv + ctas) * n_rows] fp32 partial LSE
};

// Host: whether the balanced kernel takes a decode of this shape.
inline bool decode_t_eligible(int D, long long n_rows) { return D == 128 && n_rows <= 64; }

// Host: persistent CTAs on the current device (its SM count; 148 when the
// device cannot be queried).
int decode_t_ctas();

// Host: workspace bytes for the balanced decode: o_part, lse_part, seg_first
// and seg_last, each rounded up to 256 bytes.
size_t decode_t_workspace(long long B, int H_kv, long long n_rows, int ctas);

// Host: carve ``workspace`` (at least decode_t_workspace bytes) into ``t``.
void decode_t_carve(DecodeTArgs& t, void* workspace, long long B, int H_kv, long long n_rows);

// The partials kernel and the merge, enqueued on ``stream``.
cudaError_t launch_decode_t(const AttnParams& p, const DecodeArgs& d, const DecodeTArgs& t,
                            cudaStream_t stream);

}  // namespace fa
