// Attention forward, bf16 in / fp32 accumulate, on the sm_100a tensor cores.
//
// What it computes: for every query row, the online-softmax recurrence of
// aiqz.cc "Flash Attention V2/V3 optimization", section "V2 algorithm
// optimisation" (steps 1-5): over key tiles j,
//     m_new = max(m, rowmax(S_j)),  alpha = e^(m - m_new),
//     l = l * alpha + rowsum(e^(S_j - m_new)),
//     O = O * alpha + e^(S_j - m_new) V_j,
// then O / l once at the end, with S = scale * Q K^T (scale before the max,
// as in the same article's Python demo) and LSE = m + ln l saved for the
// backward pass (airsota.com card, section 4 item 2). Exponentials are taken
// in base 2 on pre-scaled logits (scale * log2 e), which is the same
// recurrence up to rounding.
//
// How, on B200 (one CTA per 128-row Q tile, 192 threads):
//   warp 4      TMA producer: Q tile once, then K_j and V_j tiles through
//               separate multi-stage shared-memory rings (mbarrier full/empty
//               pairs, 128-byte swizzle, no multicast);
//   warp 5      MMA issuer (one thread): S_j = Q K_j^T with tcgen05.mma into
//               one of two TMEM score buffers (Q is the A operand, held in
//               TMEM, so each tile streams only K and V through shared memory
//               and the tensor core is not held back by shared-memory
//               bandwidth), then O += P_{j-1} V_{j-1} with
//               P read straight from TMEM (it overwrites the first half of its
//               score buffer as packed bf16); issuing QK_j before PV_{j-1}
//               lets the softmax of tile j overlap the PV of tile j-1;
//   warps 0-3   softmax, one thread per query row (TMEM lane = row): first
//               copies its Q row from the swizzled shared tile into TMEM; then
//               per tile loads
//               its 128 scores with tcgen05.ld, masks, takes the row max,
//               exponentiates, sums, stores P back to TMEM, rescales its O row
//               in TMEM when the max moved, and finally writes O / l and LSE.
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D), Q [384, 384+D/2).
#include <limits.h>
#include <math.h>

#include "params.h"

namespace fa {
namespace {

constexpr int BM = 128;  // query rows per CTA (= TMEM lanes)
constexpr int BN = 128;  // keys per tile
constexpr int WARP_TMA = 4;
constexpr int WARP_MMA = 5;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S0 = 0;
constexpr uint32_t TM_S1 = 128;
constexpr uint32_t TM_O = 256;
constexpr uint32_t TM_Q = 384;  // Q tile as packed bf16 (D/2 columns), A operand of Q K^T
constexpr uint32_t CHUNK_BYTES = 128 * 128;  // 128 rows x 64 bf16 (one swizzle span)
// The O accumulator is rescaled only when a row max grows by more than this
// many powers of two; P entries are then at most 2^8 before the bf16 cast.
constexpr float RESCALE_LOG2 = 8.f;
constexpr unsigned FULL = 0xffffffffu;

// Codes recorded in the device error word when a wait gives up.
enum : unsigned {
  W_Q = 0x10100, W_KEMPTY = 0x10200, W_VEMPTY = 0x10300, W_KFULL = 0x10400,
  W_VFULL = 0x10500, W_PREADY = 0x10600, W_SFULL = 0x10700, W_ODONE = 0x10800,
  W_QTMEM = 0x10900
};

template <int D>
struct FwdCfg {
  static constexpr int STAGES = (D == 64) ? 4 : 3;
  static constexpr int CHUNKS = D / 64;
  static constexpr uint32_t TILE = BM * D * 2;  // bytes of one 128-row tile
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + TILE;
  static constexpr uint32_t OFF_V = OFF_K + STAGES * TILE;
  static constexpr uint32_t OFF_BAR = OFF_V + STAGES * TILE;
  // q, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], p_ready[2], o_done,
  // q_tmem
  static constexpr int NBAR = 1 + 4 * STAGES + 6;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr uint32_t SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct Bars {
  uint32_t base;
  int stages;
  __device__ uint32_t q() const { return base; }
  __device__ uint32_t k_full(int s) const { return base + 8u * (1 + s); }
  __device__ uint32_t k_empty(int s) const { return base + 8u * (1 + stages + s); }
  __device__ uint32_t v_full(int s) const { return base + 8u * (1 + 2 * stages + s); }
  __device__ uint32_t v_empty(int s) const { return base + 8u * (1 + 3 * stages + s); }
  __device__ uint32_t s_full(int b) const { return base + 8u * (1 + 4 * stages + b); }
  __device__ uint32_t p_ready(int b) const { return base + 8u * (3 + 4 * stages + b); }
  __device__ uint32_t o_done() const { return base + 8u * (5 + 4 * stages); }
  __device__ uint32_t q_tmem() const { return base + 8u * (6 + 4 * stages); }
};

// All 32 lanes wait; the warp proceeds only if every lane saw the phase.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const DevErr& e,
                                          volatile int* abort, unsigned where) {
  const bool ok = mbar_wait(bar, parity, e, abort, where);
  return __all_sync(FULL, ok);
}

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p, int num_m,
                    int group) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);

  // Tile order: groups of heads for L2 reuse of K / V; inside a group the
  // longest causal tiles (largest m_blk) first.
  const TileSlot ts = grouped_slot(blockIdx.x, num_m, p.H * p.B, group);
  const int m_blk = num_m - 1 - ts.t;
  const int rem = ts.unit;
  const int h = rem % p.H;
  const int b = rem / p.H;
  const SeqInfo sq = seq_info(p, b);
  if (!seq_ok(p, sq) || m_blk * BM >= sq.len) return;  // whole CTA, before any shared state
  const int hk = h / (p.H / p.H_kv);
  const int n_kv_all = (sq.len + BN - 1) / BN;
  const int n_kv = p.causal ? min(n_kv_all, m_blk + 1) : n_kv_all;

  const Bars bars{sbase + C::OFF_BAR, C::STAGES};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    *abort = 0;
    mbar_init(bars.q(), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bars.k_full(s), 1);
      mbar_init(bars.k_empty(s), 1);
      mbar_init(bars.v_full(s), 1);
      mbar_init(bars.v_empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars.s_full(i), 1);
      mbar_init(bars.p_ready(i), 128);
    }
    mbar_init(bars.o_done(), 1);
    mbar_init(bars.q_tmem(), 128);
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == WARP_TMA) {
    if (lane == 0) {
      // ---------------------------------------------------- TMA producer ---
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int row_q = sq.start + m_blk * BM;
      mbar_arrive_expect_tx(bars.q(), C::TILE);
#pragma unroll
      for (int c = 0; c < C::CHUNKS; ++c)
        tma_load_2d(sbase + C::OFF_Q + c * CHUNK_BYTES, &tm_q, bars.q(), h * D + c * 64, row_q);
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        const int row_kv = sq.start + j * BN;
        if (!mbar_wait(bars.k_empty(st), ph ^ 1, p.err, abort, W_KEMPTY)) break;
        mbar_arrive_expect_tx(bars.k_full(st), C::TILE);
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_2d(sbase + C::OFF_K + st * C::TILE + c * CHUNK_BYTES, &tm_k, bars.k_full(st),
                      hk * D + c * 64, row_kv);
        if (!mbar_wait(bars.v_empty(st), ph ^ 1, p.err, abort, W_VEMPTY)) break;
        mbar_arrive_expect_tx(bars.v_full(st), C::TILE);
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_2d(sbase + C::OFF_V + st * C::TILE + c * CHUNK_BYTES, &tm_v, bars.v_full(st),
                      hk * D + c * 64, row_kv);
      }
      // Drain: the tensor core's arrivals on the last stages' empty barriers
      // must land before the CTA's shared memory is released.
      for (int j = max(0, n_kv - C::STAGES); j < n_kv && !*abort; ++j) {
        const int st = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        if (!mbar_wait(bars.k_empty(st), ph, p.err, abort, W_KEMPTY)) break;
        if (!mbar_wait(bars.v_empty(st), ph, p.err, abort, W_VEMPTY)) break;
      }
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer ---
      constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, false, true);
      // Shared-memory descriptors, built once and stepped by constant offsets.
      const uint64_t k_desc = sdesc_sw128(sbase + C::OFF_K, 16, 1024);
      const uint64_t v_desc = sdesc_sw128(sbase + C::OFF_V, CHUNK_BYTES, 1024);
      // Q reaches TMEM through the softmax threads.
      if (mbar_wait(bars.q_tmem(), 0, p.err, abort, W_QTMEM)) {
        tc_fence_after();
        for (int j = 0; j <= n_kv; ++j) {
          if (j < n_kv) {
            // S_j = Q K_j^T: M=128, N=128, K=D in steps of 16.
            const int st = j % C::STAGES;
            if (!mbar_wait(bars.k_full(st), (j / C::STAGES) & 1, p.err, abort, W_KFULL)) break;
            tc_fence_after();
            const uint32_t d_s = tmem + ((j & 1) ? TM_S1 : TM_S0);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * CHUNK_BYTES + (kk & 3) * 32;
              mma_ts(d_s, tmem + TM_Q + kk * 8, sdesc_add(k_desc, st * C::TILE + off), IDESC_QK,
                     kk > 0);
            }
            tc_commit(bars.s_full(j & 1));
            tc_commit(bars.k_empty(st));
          }
          if (j >= 1) {
            // O += P_t V_t for t = j - 1: M=128, N=D, K=128 keys in steps of 16.
            const int t = j - 1;
            const int st = t % C::STAGES;
            if (!mbar_wait(bars.p_ready(t & 1), (t >> 1) & 1, p.err, abort, W_PREADY)) break;
            if (!mbar_wait(bars.v_full(st), (t / C::STAGES) & 1, p.err, abort, W_VFULL)) break;
            tc_fence_after();
            const uint32_t a_p = tmem + ((t & 1) ? TM_S1 : TM_S0);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              mma_ts(tmem + TM_O, a_p + kk * 8,
                     sdesc_add(v_desc, st * C::TILE + kk * 2048),
                     IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(bars.v_empty(st));
            tc_commit(bars.o_done());
          }
        }
      }
    }
  } else {
    // ---------------------------------------------------------- softmax ---
    const int row = threadIdx.x;  // 0..127 = TMEM lane
    const int qpos = m_blk * BM + row;
    const int lim = p.causal ? min(qpos, sq.len - 1) : sq.len - 1;  // last visible key
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float c2 = p.scale_log2;
    float m_run = -INFINITY;  // running max of scaled logits, log2 units
    float l_run = 0.f;
    // Copy this row of Q from the swizzled shared tile into TMEM as packed
    // bf16 (even element in the low half): the A operand of S = Q K^T.
    bool ok = warp_wait(bars.q(), 0, p.err, abort, W_Q);
    if (ok) {
#pragma unroll
      for (int c = 0; c < C::CHUNKS; ++c) {
        const uint8_t* rowp = smem + C::OFF_Q + c * CHUNK_BYTES + row * 128;
        uint32_t w[32];
#pragma unroll
        for (int k16 = 0; k16 < 8; ++k16) {
          const uint4 v = *reinterpret_cast<const uint4*>(rowp + ((k16 ^ (row & 7)) << 4));
          w[4 * k16 + 0] = v.x;
          w[4 * k16 + 1] = v.y;
          w[4 * k16 + 2] = v.z;
          w[4 * k16 + 3] = v.w;
        }
        tmem_st32(tmem + lane_off + TM_Q + 32 * c, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bars.q_tmem());
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      const uint32_t s_col = (j & 1) ? TM_S1 : TM_S0;
      if (!warp_wait(bars.s_full(j & 1), (j >> 1) & 1, p.err, abort, W_SFULL)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + s_col + 32 * c, r[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(r[c]);

      const int nvalid = lim - j * BN + 1;  // visible keys in this tile
      if (nvalid < BN) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (32 * c + i >= nvalid) r[c][i] = __float_as_uint(-INFINITY);
      }
      // Row max with 8 independent partial maxima (no 128-long dependency chain).
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], __uint_as_float(r[c][i]));
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      // The reference max only moves when the row max grows by more than
      // RESCALE_LOG2 (log2 units): P = 2^(s c - m_ref) then stays below
      // 2^RESCALE_LOG2, and O / l is the same for any consistent reference.
      const float m_cand = mx * c2;
      const bool grow = m_cand > m_run + RESCALE_LOG2;   // always true on the first tile
      const float m_new = grow ? m_cand : m_run;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = grow ? ex2_approx(m_run - m_use) : 1.f;
      float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      uint32_t pk[2][32];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(r[c][i]), c2, -m_use));
          const float p1 = ex2_approx(fmaf(__uint_as_float(r[c][i + 1]), c2, -m_use));
          sum8[(i >> 1) & 7] += p0 + p1;
          pk[c >> 1][(c & 1) * 16 + i / 2] = pack_bf16x2(p0, p1);
        }
      const float sum = ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) +
                        ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
      // P overwrites the first 64 columns of this score buffer.
      tmem_st32(tmem + lane_off + s_col, pk[0]);
      tmem_st32(tmem + lane_off + s_col + 32, pk[1]);
      tmem_st_wait();
      l_run = l_run * alpha + sum;
      if (j > 0) {
        // O holds PV_{j-1} once o_done completes; rescale it before PV_j.
        if (!warp_wait(bars.o_done(), (j - 1) & 1, p.err, abort, W_ODONE)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(FULL, alpha != 1.f)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + TM_O + 32 * c, o);
            tmem_ld_wait();
            reg_fence(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tmem + lane_off + TM_O + 32 * c, o);
          }
          tmem_st_wait();
        }
      }
      tc_fence_before();
      mbar_arrive(bars.p_ready(j & 1));
      m_run = m_new;
    }
    // ----------------------------------------------------------- epilogue ---
    if (ok && warp_wait(bars.o_done(), (n_kv - 1) & 1, p.err, abort, W_ODONE)) {
      tc_fence_after();
      const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
      const bool store = qpos < sq.len;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.o) +
                            (static_cast<size_t>(sq.start + qpos) * p.H + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + TM_O + 32 * c, o);
        tmem_ld_wait();
        reg_fence(o);
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * v4 + 0]) * inv_l, __uint_as_float(o[8 * v4 + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(o[8 * v4 + 2]) * inv_l, __uint_as_float(o[8 * v4 + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(o[8 * v4 + 4]) * inv_l, __uint_as_float(o[8 * v4 + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(o[8 * v4 + 6]) * inv_l, __uint_as_float(o[8 * v4 + 7]) * inv_l);
            dst[v4] = w;
          }
        }
      }
      if (store) {
        const float lse = (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f
                                        : -INFINITY;
        p.lse[lse_index(p, b, h, sq.start, qpos)] = lse;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int D>
cudaError_t launch_d(const AttnParams& p, cudaStream_t stream) {
  using C = FwdCfg<D>;
  const int num_m = (p.max_seqlen + BM - 1) / BM;
  const long long tiles = static_cast<long long>(num_m) * p.H * p.B;
  if (tiles == 0 || p.total == 0) return cudaSuccess;
  if (tiles > INT_MAX) return cudaErrorInvalidConfiguration;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16_2d(&tq, p.q, p.total, static_cast<unsigned long long>(p.H) * D, 64, BM) ||
      !make_tmap_bf16_2d(&tk, p.k, p.total, static_cast<unsigned long long>(p.H_kv) * D, 64, BN) ||
      !make_tmap_bf16_2d(&tv, p.v, p.total, static_cast<unsigned long long>(p.H_kv) * D, 64, BN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fwd_bf16_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int group = l2_group(4ll * p.max_seqlen * D, p.H / p.H_kv, p.H * p.B);
  fwd_bf16_kernel<D><<<static_cast<unsigned>(tiles), THREADS, C::SMEM, stream>>>(tq, tk, tv, p,
                                                                                 num_m, group);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16(const AttnParams& p, cudaStream_t stream) {
  if (p.D == 64) return launch_d<64>(p, stream);
  if (p.D == 128) return launch_d<128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fa
