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
  float* dq_accum;  // fp32 [T, H, D] (bf16 backward)
  float* delta;     // fp32 [H, T]: D_i = dO_i . O_i
  const int* cu_seqlens;  // null for dense batches
  int B, H, H_kv, N, D;
  int causal;
  int max_seqlen;   // dense: N
  long long total;  // rows of every tensor (dense: B*N)
  float scale;      // multiplies Q K^T
  float scale_log2; // scale * log2(e)
  DevErr err;
};

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

// Launchers (return cudaSuccess or the launch error).
cudaError_t launch_fwd_f32(const AttnParams& p, cudaStream_t stream);
cudaError_t launch_bwd_f32(const AttnParams& p, cudaStream_t stream);
cudaError_t launch_fwd_bf16(const AttnParams& p, cudaStream_t stream);
// mask: bit 0 preprocess, bit 1 main kernel, bit 2 dQ conversion.
cudaError_t launch_bwd_bf16(const AttnParams& p, cudaStream_t stream, unsigned mask);
cudaError_t launch_wait_selftest(DevErr err, cudaStream_t stream);

// Host: cuTensorMapEncodeTiled through the runtime's driver entry point.
// Encodes a 2-D bf16 view [rows, cols] (row stride ``cols`` elements) with a
// box of box_cols x box_rows and 128-byte swizzle. Returns false on failure.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, unsigned long long rows,
                       unsigned long long cols, unsigned box_cols, unsigned box_rows);

// Host: 3-D bf16 view (D, heads, rows) of a token-major [rows, heads, D]
// tensor with a (64, 1, box_rows) box and 128-byte swizzle. Column blocks at
// x >= D lie outside the tensor and arrive as zeros.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, long long rows, int heads, int D,
                       unsigned box_rows);

// Host: 3-D fp32 view (D, heads, rows) with a (D, 1, box_rows) box and no
// swizzle, for bulk reduce-adds of [box_rows][D] shared-memory tiles.
bool make_tmap_f32_3d(CUtensorMap* map, const void* base, long long rows, int heads, int D,
                      unsigned box_rows);

}  // namespace fa
