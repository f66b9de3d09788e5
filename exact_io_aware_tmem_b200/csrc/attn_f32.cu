// fp32 attention on CUDA cores (no tensor cores, no bf16 rounding anywhere).
//
// The float32 workload must match the float64 oracle to 1e-5 max-abs, which
// rules out tf32 tensor-core operands; these kernels keep every product and
// sum in fp32 FMAs. Same method as the tensor-core path: the forward visits
// keys in blocks of 32 with the online-softmax recurrence (aiqz.cc "Flash
// Attention V2/V3 optimization", section "V2 algorithm optimisation", steps
// 1-5) and saves LSE; the backward recomputes P from LSE (airsota.com card,
// section 4 item 2) and forms dV, dP, dS, dQ, dK without atomics.
//
// Work split: one warp per query row (forward, dQ) or per key row (dK, dV);
// lane l owns head-dimension entries l, l+32, l+64, l+96; a block of 32 keys
// (or queries) is scored one per lane and broadcast with shuffles.
#include <math.h>

#include "params.h"

namespace fa {
namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int WARPS = 4;
constexpr int DMAX = 128;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(FULL, x, o));
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
  return x;
}

__device__ __forceinline__ float dot_row(const float* a_smem, const float* b, int D) {
  float acc = 0.f;
  for (int d = 0; d < D; ++d) acc = fmaf(a_smem[d], b[d], acc);
  return acc;
}

__global__ void __launch_bounds__(WARPS * 32) fwd_f32_kernel(AttnParams p) {
  __shared__ float qs[WARPS][DMAX];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = blockIdx.z, h = blockIdx.y;
  const SeqInfo s = seq_info(p, b);
  if (!seq_ok(p, s)) return;
  const int qpos = blockIdx.x * WARPS + warp;
  if (qpos >= s.len) return;
  const int D = p.D;
  const int hk = h / (p.H / p.H_kv);
  const float* Q = static_cast<const float*>(p.q);
  const size_t kv_stride = static_cast<size_t>(p.H_kv) * D;
  const float* Kb = static_cast<const float*>(p.k) + (static_cast<size_t>(s.start) * p.H_kv + hk) * D;
  const float* Vb = static_cast<const float*>(p.v) + (static_cast<size_t>(s.start) * p.H_kv + hk) * D;
  const float* qrow = Q + (static_cast<size_t>(s.start + qpos) * p.H + h) * D;
  for (int d = lane; d < D; d += 32) qs[warp][d] = qrow[d];
  __syncwarp();

  const int nvis = p.causal ? min(qpos + 1, s.len) : s.len;
  float m = -INFINITY, l = 0.f;
  float acc[DMAX / 32] = {0.f, 0.f, 0.f, 0.f};
  for (int c0 = 0; c0 < nvis; c0 += 32) {
    const int j = c0 + lane;
    float sc = -INFINITY;
    if (j < nvis) sc = dot_row(qs[warp], Kb + j * kv_stride, D) * p.scale;
    const float m_new = fmaxf(m, warp_max(sc));   // key c0 is visible: finite
    const float alpha = expf(m - m_new);           // 0 on the first block
    const float pj = (j < nvis) ? expf(sc - m_new) : 0.f;
    l = l * alpha + warp_sum(pj);
#pragma unroll
    for (int t = 0; t < DMAX / 32; ++t) acc[t] *= alpha;
    const int cnt = min(32, nvis - c0);
    for (int jj = 0; jj < cnt; ++jj) {
      const float pb = __shfl_sync(FULL, pj, jj);
      const float* vr = Vb + (c0 + jj) * kv_stride;
#pragma unroll
      for (int t = 0; t < DMAX / 32; ++t) {
        const int d = lane + 32 * t;
        if (d < D) acc[t] = fmaf(pb, vr[d], acc[t]);
      }
    }
    m = m_new;
  }
  float* orow = static_cast<float*>(p.o) + (static_cast<size_t>(s.start + qpos) * p.H + h) * D;
  const float inv_l = 1.f / l;
#pragma unroll
  for (int t = 0; t < DMAX / 32; ++t) {
    const int d = lane + 32 * t;
    if (d < D) orow[d] = acc[t] * inv_l;
  }
  if (lane == 0) p.lse[lse_index(p, b, h, s.start, qpos)] = m + logf(l);
}

// D_i = dO_i . O_i, stored [H, T].
__global__ void __launch_bounds__(WARPS * 32) bwd_f32_delta_kernel(AttnParams p) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = blockIdx.z, h = blockIdx.y;
  const SeqInfo s = seq_info(p, b);
  if (!seq_ok(p, s)) return;
  const int qpos = blockIdx.x * WARPS + warp;
  if (qpos >= s.len) return;
  const size_t off = (static_cast<size_t>(s.start + qpos) * p.H + h) * p.D;
  const float* o = static_cast<const float*>(p.o) + off;
  const float* g = static_cast<const float*>(p.dout) + off;
  float acc = 0.f;
  for (int d = lane; d < p.D; d += 32) acc = fmaf(o[d], g[d], acc);
  acc = warp_sum(acc);
  if (lane == 0) p.delta[static_cast<size_t>(h) * p.total + s.start + qpos] = acc;
}

// dQ_i = scale * sum_j dS_ij K_j, one warp per query row.
__global__ void __launch_bounds__(WARPS * 32) bwd_f32_dq_kernel(AttnParams p) {
  __shared__ float qs[WARPS][DMAX];
  __shared__ float gs[WARPS][DMAX];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = blockIdx.z, h = blockIdx.y;
  const SeqInfo s = seq_info(p, b);
  if (!seq_ok(p, s)) return;
  const int qpos = blockIdx.x * WARPS + warp;
  if (qpos >= s.len) return;
  const int D = p.D;
  const int hk = h / (p.H / p.H_kv);
  const size_t kv_stride = static_cast<size_t>(p.H_kv) * D;
  const float* Kb = static_cast<const float*>(p.k) + (static_cast<size_t>(s.start) * p.H_kv + hk) * D;
  const float* Vb = static_cast<const float*>(p.v) + (static_cast<size_t>(s.start) * p.H_kv + hk) * D;
  const size_t off = (static_cast<size_t>(s.start + qpos) * p.H + h) * D;
  for (int d = lane; d < D; d += 32) {
    qs[warp][d] = static_cast<const float*>(p.q)[off + d];
    gs[warp][d] = static_cast<const float*>(p.dout)[off + d];
  }
  __syncwarp();
  const float lse = p.lse[lse_index(p, b, h, s.start, qpos)];
  const float dlt = p.delta[static_cast<size_t>(h) * p.total + s.start + qpos];
  const int nvis = p.causal ? min(qpos + 1, s.len) : s.len;
  float acc[DMAX / 32] = {0.f, 0.f, 0.f, 0.f};
  for (int c0 = 0; c0 < nvis; c0 += 32) {
    const int j = c0 + lane;
    float ds = 0.f;
    if (j < nvis) {
      const float pij = expf(dot_row(qs[warp], Kb + j * kv_stride, D) * p.scale - lse);
      const float dp = dot_row(gs[warp], Vb + j * kv_stride, D);
      ds = pij * (dp - dlt);
    }
    const int cnt = min(32, nvis - c0);
    for (int jj = 0; jj < cnt; ++jj) {
      const float dsb = __shfl_sync(FULL, ds, jj);
      const float* kr = Kb + (c0 + jj) * kv_stride;
#pragma unroll
      for (int t = 0; t < DMAX / 32; ++t) {
        const int d = lane + 32 * t;
        if (d < D) acc[t] = fmaf(dsb, kr[d], acc[t]);
      }
    }
  }
  float* dq = static_cast<float*>(p.dq) + off;
#pragma unroll
  for (int t = 0; t < DMAX / 32; ++t) {
    const int d = lane + 32 * t;
    if (d < D) dq[d] = acc[t] * p.scale;
  }
}

// dV_j = sum_i P_ij dO_i and dK_j = scale * sum_i dS_ij Q_i, one warp per key
// row of one key/value head, summed over the query heads of its group.
__global__ void __launch_bounds__(WARPS * 32) bwd_f32_dkdv_kernel(AttnParams p) {
  __shared__ float ks[WARPS][DMAX];
  __shared__ float vs[WARPS][DMAX];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int b = blockIdx.z, hk = blockIdx.y;
  const SeqInfo s = seq_info(p, b);
  if (!seq_ok(p, s)) return;
  const int kpos = blockIdx.x * WARPS + warp;
  if (kpos >= s.len) return;
  const int D = p.D;
  const int g = p.H / p.H_kv;
  const size_t q_stride = static_cast<size_t>(p.H) * D;
  const size_t koff = (static_cast<size_t>(s.start + kpos) * p.H_kv + hk) * D;
  for (int d = lane; d < D; d += 32) {
    ks[warp][d] = static_cast<const float*>(p.k)[koff + d];
    vs[warp][d] = static_cast<const float*>(p.v)[koff + d];
  }
  __syncwarp();
  float dk[DMAX / 32] = {0.f, 0.f, 0.f, 0.f};
  float dv[DMAX / 32] = {0.f, 0.f, 0.f, 0.f};
  const int i0 = p.causal ? kpos : 0;
  for (int h = hk * g; h < (hk + 1) * g; ++h) {
    const float* Qb = static_cast<const float*>(p.q) + (static_cast<size_t>(s.start) * p.H + h) * D;
    const float* Gb = static_cast<const float*>(p.dout) + (static_cast<size_t>(s.start) * p.H + h) * D;
    for (int c0 = i0; c0 < s.len; c0 += 32) {
      const int i = c0 + lane;
      float pij = 0.f, ds = 0.f;
      if (i < s.len) {
        const float lse = p.lse[lse_index(p, b, h, s.start, i)];
        const float dlt = p.delta[static_cast<size_t>(h) * p.total + s.start + i];
        pij = expf(dot_row(ks[warp], Qb + i * q_stride, D) * p.scale - lse);
        const float dp = dot_row(vs[warp], Gb + i * q_stride, D);
        ds = pij * (dp - dlt);
      }
      const int cnt = min(32, s.len - c0);
      for (int ii = 0; ii < cnt; ++ii) {
        const float pb = __shfl_sync(FULL, pij, ii);
        const float dsb = __shfl_sync(FULL, ds, ii);
        const float* qr = Qb + (c0 + ii) * q_stride;
        const float* gr = Gb + (c0 + ii) * q_stride;
#pragma unroll
        for (int t = 0; t < DMAX / 32; ++t) {
          const int d = lane + 32 * t;
          if (d < D) {
            dv[t] = fmaf(pb, gr[d], dv[t]);
            dk[t] = fmaf(dsb, qr[d], dk[t]);
          }
        }
      }
    }
  }
  float* dkr = static_cast<float*>(p.dk) + koff;
  float* dvr = static_cast<float*>(p.dv) + koff;
#pragma unroll
  for (int t = 0; t < DMAX / 32; ++t) {
    const int d = lane + 32 * t;
    if (d < D) {
      dkr[d] = dk[t] * p.scale;
      dvr[d] = dv[t];
    }
  }
}

}  // namespace

cudaError_t launch_fwd_f32(const AttnParams& p, cudaStream_t stream) {
  const dim3 grid((p.max_seqlen + WARPS - 1) / WARPS, p.H, p.B);
  fwd_f32_kernel<<<grid, WARPS * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_f32(const AttnParams& p, cudaStream_t stream) {
  const int rows = (p.max_seqlen + WARPS - 1) / WARPS;
  bwd_f32_delta_kernel<<<dim3(rows, p.H, p.B), WARPS * 32, 0, stream>>>(p);
  bwd_f32_dq_kernel<<<dim3(rows, p.H, p.B), WARPS * 32, 0, stream>>>(p);
  bwd_f32_dkdv_kernel<<<dim3(rows, p.H_kv, p.B), WARPS * 32, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace fa
