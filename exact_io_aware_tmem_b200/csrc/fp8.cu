// Pass 1 of the FP8 (E4M3) forward: per-block step and E4M3 codes.
//
// aiqz.cc "Flash Attention V2/V3 optimization" article, section "FP8 low
// precision": the first pass scans each block in high precision for its
// largest |x|, sets the block's step Delta = max|x| / 448 (448 is E4M3's
// largest finite value) and stores round(x / Delta) as E4M3; the second pass
// (fwd_pair.cu, F8 instantiation) multiplies the codes on the tensor cores
// with an fp32 accumulator.
//
// A block is the 128 consecutive tokens of one head of one sequence - one
// 128-row tile of the forward kernel - so the second pass needs one step per
// tile. Delta and x / Delta are IEEE single-precision divisions (the codes of
// x / Delta reached through products where that provably gives the same
// code, see codes4()), rounding is to nearest even onto the E4M3 grid with
// saturation at +-448 (cvt.rn.satfinite), and an all-zero block gets
// Delta = 1.
#include <limits.h>

#include "params.h"

namespace fa {
namespace {

constexpr int QBLOCK = 128;
constexpr int QTHREADS = 256;

// The E4M3 codes of four elements x (bf16, two words) under the step Delta,
// as RN(x / Delta) gives them, by way of products.
//
// With r = RN(1 / Delta) (Delta normal), RN(x * r) lies within a relative
// 2^-22.4 of RN(x / Delta) (three roundings of 2^-24 each). The products of x
// with r_lo = RN(r (1 - 2^-20)) and r_hi = RN(r (1 + 2^-20)) therefore
// bracket RN(x / Delta), and rounding onto E4M3 is monotonic: where both ends
// take the same code, that code is RN(x / Delta)'s. Where they differ (a
// rounding midpoint of the E4M3 grid within the bracket, about one element in
// 10^5) the caller divides. Returns the four codes of the low end; *same is
// whether the high end agrees.
// Four floats -> four E4M3 codes (round to nearest even, saturating), a in
// byte 0.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 l, h;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 l, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h, %4, %3;\n\t"
      "mov.b32 %0, {l, h};\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

__device__ __forceinline__ uint32_t codes4(uint32_t w0, uint32_t w1, float r_lo, float r_hi,
                                           bool* same) {
  const float x0 = __uint_as_float(w0 << 16), x1 = __uint_as_float(w0 & 0xffff0000u);
  const float x2 = __uint_as_float(w1 << 16), x3 = __uint_as_float(w1 & 0xffff0000u);
  const uint32_t lo = pack_e4m3x4(__fmul_rn(x0, r_lo), __fmul_rn(x1, r_lo), __fmul_rn(x2, r_lo),
                                  __fmul_rn(x3, r_lo));
  const uint32_t hi = pack_e4m3x4(__fmul_rn(x0, r_hi), __fmul_rn(x1, r_hi), __fmul_rn(x2, r_hi),
                                  __fmul_rn(x3, r_hi));
  *same = lo == hi;
  return lo;
}

// Elementwise max of two bf16 pairs.
__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// The same four codes by IEEE division.
__device__ __forceinline__ uint32_t codes4_div(uint32_t w0, uint32_t w1, float delta) {
  const float x0 = __uint_as_float(w0 << 16), x1 = __uint_as_float(w0 & 0xffff0000u);
  const float x2 = __uint_as_float(w1 << 16), x3 = __uint_as_float(w1 & 0xffff0000u);
  return pack_e4m3x4(__fdiv_rn(x0, delta), __fdiv_rn(x1, delta), __fdiv_rn(x2, delta),
                     __fdiv_rn(x3, delta));
}

// One CTA per (sequence, 128-token block, head). The block (at most
// QTHREADS x VPT vectors of 8 bf16) is read once into registers, reduced to
// max |x|, then converted from the registers.
// PER_ROW: D / 8 when fixed at compile time (the addresses then take shifts),
// 0 for any D (a division per address).
template <int VPT, int PER_ROW>
__global__ void __launch_bounds__(QTHREADS, VPT >= 8 ? 32 / VPT : 6)
    fp8_quantize_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ x8,
                        float* __restrict__ scale, int N, int Hx, int D, int nb) {
  static_assert(VPT <= 16, "one bit per four elements");
  // Memory order (heads fastest, then token blocks, then sequences): the
  // CTAs resident at one time read whole token rows (every head's D
  // elements) of a run of consecutive token blocks.
  const int h = blockIdx.x % Hx;
  const int t = (blockIdx.x / Hx) % nb;
  const int b = blockIdx.x / (Hx * nb);
  const int bh = b * Hx + h;
  const int r0 = t * QBLOCK;
  const int rows = min(QBLOCK, N - r0);
  const int per_row = PER_ROW ? PER_ROW : D / 8;
  const int n = rows * per_row;
  // Element offset of this thread's k-th group of 8 (group i = threadIdx.x +
  // k QTHREADS of the block). With a compile-time row width that divides
  // QTHREADS, step k moves the thread down QTHREADS / PER_ROW whole rows: a
  // fixed stride.
  const size_t base = (static_cast<size_t>(b) * N + r0) * Hx * D + static_cast<size_t>(h) * D;
  const size_t row_pitch = static_cast<size_t>(Hx) * D;
  auto offset = [&](int k) -> size_t {
    if constexpr (PER_ROW != 0 && QTHREADS % (PER_ROW ? PER_ROW : 1) == 0) {
      return base + (threadIdx.x / PER_ROW + static_cast<size_t>(k) * (QTHREADS / PER_ROW)) *
                        row_pitch +
             (threadIdx.x % PER_ROW) * 8;
    } else {
      const int i = threadIdx.x + k * QTHREADS;
      return base + static_cast<size_t>(i / per_row) * row_pitch + (i % per_row) * 8;
    }
  };
  uint4 v[VPT];
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int i = threadIdx.x + k * QTHREADS;
    v[k] = i < n ? __ldcs(reinterpret_cast<const uint4*>(x + offset(k))) : make_uint4(0, 0, 0, 0);
  }
  // max |x|: bf16 pairs with their sign bits cleared, two at a time; then
  // the bit patterns of the two non-negative halves order as their values.
  uint32_t m2 = 0;
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    m2 = max_bf16x2(m2, v[k].x & 0x7fff7fffu);
    m2 = max_bf16x2(m2, v[k].y & 0x7fff7fffu);
    m2 = max_bf16x2(m2, v[k].z & 0x7fff7fffu);
    m2 = max_bf16x2(m2, v[k].w & 0x7fff7fffu);
  }
  uint32_t amax_bits = max(m2 << 16, m2 & 0xffff0000u);
  __shared__ uint32_t red[QTHREADS / 32];
#pragma unroll
  for (int s = 16; s > 0; s >>= 1)
    amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, s));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = amax_bits;
  __syncthreads();
  amax_bits = red[0];
#pragma unroll
  for (int k = 1; k < QTHREADS / 32; ++k) amax_bits = max(amax_bits, red[k]);
  const float amax = __uint_as_float(amax_bits);
  const float delta = (amax > 0.f) ? __fdiv_rn(amax, 448.f) : 1.f;
  if (threadIdx.x == 0) scale[static_cast<size_t>(bh) * nb + t] = delta;
  // Delta below the normal range: r would lose precision or overflow, so
  // every element takes the division.
  const bool normal = delta >= 1.17549435e-38f;
  const float r = __frcp_rn(delta);
  const float r_lo = __fmul_rn(r, 1.f - 0x1p-20f);
  const float r_hi = __fmul_rn(r, 1.f + 0x1p-20f);
  uint32_t redo = 0;   // bit 2k + e: word pair e of vector k needs the division
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int i = threadIdx.x + k * QTHREADS;
    if (i < n) {
      bool s0, s1;
      const uint32_t c0 = codes4(v[k].x, v[k].y, r_lo, r_hi, &s0);
      const uint32_t c1 = codes4(v[k].z, v[k].w, r_lo, r_hi, &s1);
      redo |= (s0 && normal ? 0u : 1u << (2 * k)) | (s1 && normal ? 0u : 2u << (2 * k));
      *reinterpret_cast<uint2*>(x8 + offset(k)) = make_uint2(c0, c1);
    }
  }
  // The four-element groups whose bracket holds a rounding midpoint (exact
  // ties among them: x / Delta on a midpoint is common for round inputs)
  // take the division; the later store from this thread replaces the codes
  // above.
  if (redo != 0) {
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (redo & (1u << (2 * k + e))) {
          const size_t o = offset(k) + 4 * e;
          *reinterpret_cast<uint32_t*>(x8 + o) =
              codes4_div(e ? v[k].z : v[k].x, e ? v[k].w : v[k].y, delta);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_fp8_quantize(const void* x, void* x8, float* scale, int B, int N, int Hx,
                                int D, cudaStream_t stream) {
  const int nb = (N + QBLOCK - 1) / QBLOCK;
  const long long blocks = static_cast<long long>(B) * Hx * nb;
  if (blocks == 0) return cudaSuccess;
  if (blocks > INT_MAX || D % 8 != 0) return cudaErrorInvalidValue;
  if (D > 256) return cudaErrorInvalidValue;
  auto xin = static_cast<const __nv_bfloat16*>(x);
  auto out = static_cast<uint8_t*>(x8);
  const unsigned grid = static_cast<unsigned>(blocks);
  if (D == 128)
    fp8_quantize_kernel<8, 16><<<grid, QTHREADS, 0, stream>>>(xin, out, scale, N, Hx, D, nb);
  else if (D == 64)
    fp8_quantize_kernel<4, 8><<<grid, QTHREADS, 0, stream>>>(xin, out, scale, N, Hx, D, nb);
  else if (D <= 128)
    fp8_quantize_kernel<8, 0><<<grid, QTHREADS, 0, stream>>>(xin, out, scale, N, Hx, D, nb);
  else
    fp8_quantize_kernel<16, 0><<<grid, QTHREADS, 0, stream>>>(xin, out, scale, N, Hx, D, nb);
  return cudaGetLastError();
}

}  // namespace fa
