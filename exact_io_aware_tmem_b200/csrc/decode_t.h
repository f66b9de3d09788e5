// Balanced decode: the partials kernel with the keys on the TMEM lanes and
// the merge that follows it (decode_t.cu). fa_decode uses it for D = 128 and
// at most 64 query rows per kv head when the caller leaves the split count to
// the library.
#pragma once

#include "params.h"

namespace fa {

// The CTAs form groups of H_kv, one CTA per kv head; CTA c serves kv head
// c % H_kv. The U = sum_b ceil(len_b / 128) units (sequence b, 128-key tile)
// are cut into one contiguous range of equal size per group, so the H_kv
// CTAs of a group read the same token rows of the cache (every head of a
// token lies in one row) at about the same time. A (sequence, kv head)
// segment cut by a range boundary yields one partial per group holding part
// of it, in slot (b + group) * H_kv + kv head (unique: along one head's walk
// b + group grows by one or two at each piece).
struct DecodeTArgs {
  int ctas;          // persistent CTAs: groups * H_kv
  int* seg_first;    // [B * H_kv] first group holding a tile of the segment
  int* seg_last;     // [B * H_kv] last such group
  float* o_part;     // [(B * H_kv + ctas) * n_rows, D] fp32 partial O / l
  float* lse_part;   // [(B * H_kv + ctas) * n_rows] fp32 partial LSE
};

// Host: whether the balanced kernel takes a decode of this shape.
inline bool decode_t_eligible(int D, long long n_rows) { return D == 128 && n_rows <= 64; }

// Host: persistent CTAs on the current device for H_kv kv heads: the most
// whole groups of H_kv that fit its SM count (148 when the device cannot be
// queried), at least one group.
int decode_t_ctas(int H_kv);

// Host: workspace bytes for the balanced decode: o_part, lse_part, seg_first
// and seg_last, each rounded up to 256 bytes.
size_t decode_t_workspace(long long B, int H_kv, long long n_rows, int ctas);

// Host: carve ``workspace`` (at least decode_t_workspace bytes) into ``t``.
void decode_t_carve(DecodeTArgs& t, void* workspace, long long B, int H_kv, long long n_rows);

// The partials kernel and the merge, enqueued on ``stream``.
cudaError_t launch_decode_t(const AttnParams& p, const DecodeArgs& d, const DecodeTArgs& t,
                            cudaStream_t stream);

}  // namespace fa
