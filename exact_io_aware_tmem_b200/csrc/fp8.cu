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
constexpr int QTHREADS = 256;

// One CTA per (sequence, head, 128-token block); 8 elements per step.
__global__ void __launch_bounds__(QTHREADS)
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
  float amax = 0.f;
  for (int i = threadIdx.x; i < n; i += QTHREADS) {
    const uint4 v = *reinterpret_cast<const uint4*>(x + offset(i));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[k] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[k] & 0xffff0000u)));
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
  for (int i = threadIdx.x; i < n; i += QTHREADS) {
    const size_t o = offset(i);
    const uint4 v = *reinterpret_cast<const uint4*>(x + o);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t a = pack_e4m3x2(__fdiv_rn(__uint_as_float(w[2 * k] << 16), delta),
                                     __fdiv_rn(__uint_as_float(w[2 * k] & 0xffff0000u), delta));
      const uint32_t c = pack_e4m3x2(__fdiv_rn(__uint_as_float(w[2 * k + 1] << 16), delta),
                                     __fdiv_rn(__uint_as_float(w[2 * k + 1] & 0xffff0000u), delta));
      packed[k] = a | (c << 16);
    }
    *reinterpret_cast<uint2*>(x8 + o) = make_uint2(packed[0], packed[1]);
  }
}

}  // namespace

cudaError_t launch_fp8_quantize(const void* x, void* x8, float* scale, int B, int N, int Hx,
                                int D, cudaStream_t stream) {
  const int nb = (N + QBLOCK - 1) / QBLOCK;
  const long long blocks = static_cast<long long>(B) * Hx * nb;
  if (blocks == 0) return cudaSuccess;
  if (blocks > INT_MAX || D % 8 != 0) return cudaErrorInvalidValue;
  fp8_quantize_kernel<<<static_cast<unsigned>(blocks), QTHREADS, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<uint8_t*>(x8), scale, N, Hx, D, nb);
  return cudaGetLastError();
}

}  // namespace fa
