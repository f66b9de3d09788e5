// Pass 1 of the FP8 (E4M3) forward: per-block step and E4M3 codes.
//
// aiqz.cc "Flash Attention V2/V3 optimization" article, section "FP8 low
// precision": the first pass scans each block in high precision for its
// largest |x|, sets the block's step Delta = max|x| / 448 (448 is E4M3's
// largest finite value) and stores round(x / Delta) as E4M3; the second pass
// (fwd_bf16.cu, F8 instantiation) multiplies the codes on the tensor cores
// with an fp32 accumulator.
//
// A block is the 128 consecutive tokens of one head of one sequence - one
// 128-row tile of the forward kernel - so the second pass needs one step per
// tile. Delta and x / Delta are IEEE single-precision divisions, rounding is
// to nearest even onto the E4M3 grid with saturation at +-448
// (cvt.rn.satfinite), and an all-zero block gets Delta = 1.
#include <limits.h>

#include "params.h"

namespace fa {
namespace {

constexpr int QBLOCK = 128;
constexpr int QTHREADS = 512;

// One CTA per (sequence, head, 128-token block). Thread i holds the 8-element
// groups i, i + 512, ... of the block in registers (PER groups at most), so
// the block is read from memory once: loaded, its max |x| reduced over the
// CTA, then converted from the registers and written as codes.
template <int PER>
__global__ void __launch_bounds__(QTHREADS, 2)
    fp8_quantize_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ x8,
                        float* __restrict__ scale, int N, int Hx, int D, int nb) {
  const int t = blockIdx.x % nb;
  const int bh = blockIdx.x / nb;
  const int h = bh % Hx;
  const int b = bh / Hx;
  const int r0 = t * QBLOCK;
  const int rows = min(QBLOCK, N - r0);
  const int per_row = D / 8;
  const int n = rows * per_row;
  auto offset = [&](int i) -> size_t {   // element offset of the i-th group of 8
    const int row = i / per_row;
    return (static_cast<size_t>(b) * N + r0 + row) * Hx * D + static_cast<size_t>(h) * D +
           (i % per_row) * 8;
  };
  uint4 v[PER];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + k * QTHREADS;
    v[k] = (i < n) ? __ldg(reinterpret_cast<const uint4*>(x + offset(i))) : make_uint4(0, 0, 0, 0);
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[e] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[e] & 0xffff0000u)));
    }
  }
  __shared__ float red[QTHREADS / 32];
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int k = 1; k < QTHREADS / 32; ++k) amax = fmaxf(amax, red[k]);
  const float delta = (amax > 0.f) ? __fdiv_rn(amax, 448.f) : 1.f;
  if (threadIdx.x == 0) scale[static_cast<size_t>(bh) * nb + t] = delta;
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + k * QTHREADS;
    if (i < n) {
      const uint32_t lo = pack_e4m3x2(__fdiv_rn(__uint_as_float(v[k].x << 16), delta),
                                      __fdiv_rn(__uint_as_float(v[k].x & 0xffff0000u), delta)) |
                          (static_cast<uint32_t>(pack_e4m3x2(
                               __fdiv_rn(__uint_as_float(v[k].y << 16), delta),
                               __fdiv_rn(__uint_as_float(v[k].y & 0xffff0000u), delta)))
                           << 16);
      const uint32_t hi = pack_e4m3x2(__fdiv_rn(__uint_as_float(v[k].z << 16), delta),
                                      __fdiv_rn(__uint_as_float(v[k].z & 0xffff0000u), delta)) |
                          (static_cast<uint32_t>(pack_e4m3x2(
                               __fdiv_rn(__uint_as_float(v[k].w << 16), delta),
                               __fdiv_rn(__uint_as_float(v[k].w & 0xffff0000u), delta)))
                           << 16);
      *reinterpret_cast<uint2*>(x8 + offset(i)) = make_uint2(lo, hi);
    }
  }
}

}  // namespace

cudaError_t launch_fp8_quantize(const void* x, void* x8, float* scale, int B, int N, int Hx,
                                int D, cudaStream_t stream) {
  const int nb = (N + QBLOCK - 1) / QBLOCK;
  const long long blocks = static_cast<long long>(B) * Hx * nb;
  if (blocks == 0) return cudaSuccess;
  if (blocks > INT_MAX || D % 8 != 0 || D > 256) return cudaErrorInvalidValue;
  // Groups of 8 per thread: ceil(128 rows * D / 8 / 512).
  const int per = (QBLOCK * (D / 8) + QTHREADS - 1) / QTHREADS;
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* q8 = static_cast<uint8_t*>(x8);
  const unsigned g = static_cast<unsigned>(blocks);
  if (per <= 2)
    fp8_quantize_kernel<2><<<g, QTHREADS, 0, stream>>>(xb, q8, scale, N, Hx, D, nb);
  else if (per <= 4)
    fp8_quantize_kernel<4><<<g, QTHREADS, 0, stream>>>(xb, q8, scale, N, Hx, D, nb);
  else
    fp8_quantize_kernel<8><<<g, QTHREADS, 0, stream>>>(xb, q8, scale, N, Hx, D, nb);
  return cudaGetLastError();
}

}  // namespace fa
