// Kernel parameter block and the launchers the C ABI dispatches to.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace fa {

struct AttnParams {
  // Forward inputs / outputs (token-major, see include/fa.h).
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  // Backward inputs / outputs.
  const void* dout;
  void* dq;
  void* dk;
  void* dv;
  float* delta;     // fp32 [H, T]: D_i = dO_i . O_i (backward workspace)
  float* dq_accum;  // fp32 [T, H, D] dQ accumulator of the fused backward, or null
  const int* cu_seqlens;  // null for dense batches
  int B, H, H_kv, N, D;
  int causal;
  int max_seqlen;   // dense: N
  long long total;  // rows of every tensor (dense: B*N)
  float scale;      // multiplies Q K^T
  float scale_log2; // scale * log2(e)
  DevErr err;
  // Debug builds (FA_DEBUG): where one CTA records the clock of its events,
  // or null. [kinds][1024] 64-bit stamps; see FA_STAMP.
  unsigned long long* trace;
  int trace_cta;
};

// Debug builds only: stamp event ``kind`` of step ``idx`` with the SM clock,
// in the traced CTA. The caller picks one thread per event (lane 0 of the
// role's warp). Compiled out otherwise.
#ifdef FA_DEBUG
#define FA_STAMP(p, kind, idx)                                                       \
  do {                                                                               \
    if ((p).trace != nullptr && static_cast<int>(blockIdx.x) == (p).trace_cta &&     \
        (idx) >= 0 && (idx) < 1024)                                                  \
      (p).trace[(kind) * 1024 + (idx)] = static_cast<unsigned long long>(clock64()); \
  } while (0)
// Debug builds only: a failed index check is recorded in the device error
// word (ERR_BOUNDS, ``where``) and the access is skipped by the caller.
#define FA_CHECK(p, cond, where) ((cond) ? true : (fa::record_bounds_dbg((p).err, (where)), false))
#else
#define FA_STAMP(p, kind, idx) \
  do {                         \
  } while (0)
#define FA_CHECK(p, cond, where) true
#endif

__device__ __forceinline__ void record_bounds_dbg(const DevErr& e, unsigned where) {
  atomicOr(e.word, ERR_BOUNDS);
  atomicExch(e.word + 1, where);
}

struct SeqInfo {
  int start;
  int len;
};

__device__ __forceinline__ SeqInfo seq_info(const AttnParams& p, int b) {
  if (p.cu_seqlens != nullptr) {
    const int s = p.cu_seqlens[b];
    return {s, p.cu_seqlens[b + 1] - s};
  }
  return {b * p.N, p.N};
}

// Packed batches: a sequence whose cu_seqlens entries do not fit the sizes the
// host passed is reported (ERR_BOUNDS) and skipped instead of being read.
__device__ __forceinline__ bool seq_ok(const AttnParams& p, const SeqInfo& s) {
  if (p.cu_seqlens == nullptr) return true;
  if (s.start < 0 || s.len < 0 || static_cast<long long>(s.start) + s.len > p.total ||
      s.len > p.max_seqlen) {
    atomicOr(p.err.word, ERR_BOUNDS);
    atomicExch(p.err.word + 1, 0xB0B0u);
    return false;
  }
  return true;
}

// Index of (sequence b, head h, position pos) in the LSE array:
// [B, H, N] for dense batches, [H, T] for packed ones.
__device__ __forceinline__ size_t lse_index(const AttnParams& p, int b, int h, int start,
                                            int pos) {
  if (p.cu_seqlens != nullptr) return static_cast<size_t>(h) * p.total + start + pos;
  return (static_cast<size_t>(b) * p.H + h) * p.N + pos;
}

// Tile order for L2 reuse. The (sequence, head) units are taken in groups of
// ``group`` consecutive units, and every tile of a group is launched before
// the next group's, tile index slowest inside a group: the CTAs running at any
// time then stream the tensors of a few units only, which stay in L2.
// Returns the tile index within its unit and the unit.
struct TileSlot {
  int t;
  int unit;
};

__device__ __forceinline__ TileSlot grouped_slot(unsigned bid, int num_t, int units, int group) {
  const long long per = static_cast<long long>(num_t) * group;
  const int gi = static_cast<int>(bid / per);
  const int gs = min(group, units - gi * group);
  const int local = static_cast<int>(bid - gi * per);
  return {local / gs, gi * group + local % gs};
}

// Host: group size for units that each stream ``bytes_per_unit`` bytes, so that
// a group's streams fit in about 48 MB of the 126 MB L2; ``share`` consecutive
// units stream the same tensors (query heads of one key/value head).
inline int l2_group(long long bytes_per_unit, int share, int units) {
  const long long budget = 48ll << 20;
  long long g = (bytes_per_unit > 0 ? budget / bytes_per_unit : units);
  if (g < 1) g = 1;
  g *= share;
  return static_cast<int>(g < units ? g : units);
}

// Split-KV decode (the forward kernel's decode instantiation). The queries
// are the q_len newest tokens of each of B sequences (``AttnParams::q`` /
// ``o`` are [B*q_len, H, D], ``total`` = B*q_len, ``max_seqlen`` bounds the
// cache lengths); ``k`` / ``v`` point at the caches [cache_rows, H_kv, D].
struct DecodeArgs {
  const int* cache_seqlens;  // [B] keys of each sequence
  const int* block_table;    // [B, max_blocks] page ids, or null: contiguous cache
  int page;                  // paged: rows per page; contiguous: rows per sequence
  int max_blocks;            // block-table row length
  long long cache_rows;      // rows of k / v
  int q_len;                 // query tokens per sequence
  int g;                     // query heads per key/value head
  int n_rows;                // q_len * g rows of one CTA's Q tile (<= 128)
  int n_split;               // key splits per (sequence, kv head)
  int chunk;                 // 128-key tiles per split
  float* o_part;             // [n_split, B*q_len, H, D] fp32 (n_split > 1)
  float* lse_part;           // [n_split, B*q_len, H] fp32 (n_split > 1)
};

// E4M3 forward: per-block steps of the quantised Q and K (pass 1 output),
// [B, H, n_blocks] and [B, H_kv, n_blocks] fp32, n_blocks = ceil(N / 128).
struct Fp8Args {
  const float* q_scale;
  const float* k_scale;
  int n_blocks;
};

// Launchers (return cudaSuccess or the launch error).
cudaError_t launch_fwd_f32(const AttnParams& p, cudaStream_t stream);
cudaError_t launch_bwd_f32(const AttnParams& p, cudaStream_t stream);
// The D = 128 forward, two query tiles per CTA (fwd_pair.cu).
cudaError_t launch_fwd_pair(const AttnParams& p, cudaStream_t stream);
// mask: bit 0 preprocess (D_i, and zeroes dq_accum when it is set), bit 1
// dK/dV kernel, bit 2 dQ kernel (the split backward).
cudaError_t launch_bwd_bf16(const AttnParams& p, cudaStream_t stream, unsigned mask);
// The fused backward (every product once; dQ added into p.dq_accum) and the
// conversion dQ = bf16(scale * dq_accum).
cudaError_t launch_bwd_fused(const AttnParams& p, cudaStream_t stream);
cudaError_t launch_dq_convert(const AttnParams& p, cudaStream_t stream);
cudaError_t launch_wait_selftest(DevErr err, cudaStream_t stream);
cudaError_t launch_exp2_selftest(const float* x, float* y, long long n, cudaStream_t stream);
// E4M3 forward (D = 128) on the same kernel: p.q / p.k hold the codes from
// launch_fp8_quantize, ``f`` their per-block steps.
cudaError_t launch_fwd_pair_fp8(const AttnParams& p, const Fp8Args& f, cudaStream_t stream);
// Pass 1: bf16 x [B*N, Hx, D] -> E4M3 codes x8 and per-block steps [B, Hx, nb].
cudaError_t launch_fp8_quantize(const void* x, void* x8, float* scale, int B, int N, int Hx,
                                int D, cudaStream_t stream);
// Split-KV decode partials (decode_split.cu), and the combine kernel when
// d.n_split > 1.
cudaError_t launch_decode_bf16(const AttnParams& p, const DecodeArgs& d, cudaStream_t stream);

// Host: the argument checks fa_bwd applies to the sizes (status as fa_bwd
// would return it); on success ``rows`` is the row count T of every tensor.
// Declared with the C ABI's status type, which fa_api.cu and noalloc.cu see.
#ifdef EXACT_IO_AWARE_TMEM_FA_H
fa_status check_bwd_sizes(int B, int H, int H_kv, int N, int D, fa_dtype dtype, int causal,
                          const int* cu_seqlens, int max_seqlen, long long total_tokens,
                          long long* rows);
// Host: FA_OK for cudaSuccess; otherwise FA_ERR_CUDA, with ``e`` kept as the
// calling thread's last CUDA error (fa_last_cuda_error_string).
fa_status record_cuda(cudaError_t e);
#endif

// Host: cuTensorMapEncodeTiled through the runtime's driver entry point.
// Encodes a 2-D bf16 view [rows, cols] (row stride ``cols`` elements) with a
// box of box_cols x box_rows and 128-byte swizzle. Returns false on failure.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, unsigned long long rows,
                       unsigned long long cols, unsigned box_cols, unsigned box_rows);

// Host: as make_tmap_bf16_2d for a byte tensor (E4M3 codes), cols in bytes.
bool make_tmap_u8_2d(CUtensorMap* map, const void* base, unsigned long long rows,
                     unsigned long long cols, unsigned box_cols, unsigned box_rows);

// Host: as make_tmap_bf16_2d for an fp32 tensor (box_cols fp32 columns).
bool make_tmap_f32_2d(CUtensorMap* map, const void* base, unsigned long long rows,
                      unsigned long long cols, unsigned box_cols, unsigned box_rows);

// Host: 3-D bf16 view (D, heads, rows) of a token-major [rows, heads, D]
// tensor with a (64, box_heads, box_rows) box and 128-byte swizzle. Column
// blocks at x >= D lie outside the tensor and arrive as zeros.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, long long rows, int heads, int D,
                       unsigned box_heads, unsigned box_rows);

}  // namespace fa
