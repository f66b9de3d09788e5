// Attention forward at D = 64, bf16 in / fp32 accumulate: one 128-row query
// tile per CTA, one softmax group, two CTAs per SM.
//
// What it computes is the forward of fwd_pair.cu: for every query row the
// online-softmax recurrence of aiqz.cc "Flash Attention V2/V3 optimization",
// section "V2 algorithm optimisation" (steps 1-5), over key tiles j,
//     m_new = max(m, rowmax(S_j)), l = l e^(m - m_new) + rowsum(e^(S_j - m_new)),
//     O = O e^(m - m_new) + e^(S_j - m_new) V_j,
// then O / l and LSE = m + ln l (airsota.com card, section 4 item 2), in
// base 2 on pre-scaled logits, with the reference max moved only when a row
// max exceeds it by more than 2^8 (every P stays below 2^8 before the bf16
// cast; O / l is the same for any consistent reference).
//
// Why a kernel of its own at D = 64: with half the tensor work of D = 128
// per exponential, a key tile costs ~0.84 us of exponentials and a CTA's
// start (Q and first K/V tiles in flight, TMEM, barriers) and end (O out)
// ~6.7 us, which one CTA per SM leaves exposed: at 16 key tiles per CTA a
// third of the time. This kernel takes 256 TMEM columns and ~97 KB of shared
// memory, so two CTAs share an SM and one's start and end overlap the
// other's tiles.
//
// Roles (192 threads):
//   warps 0-3  softmax, one thread per query row (TMEM lane = row): scores,
//              mask, row max, exponentials, P to TMEM, O rescale, epilogue.
//   warp 4     TMA producer: Q once; K through a 3-stage ring and V through
//              a 2-stage ring, K first whenever both have room.
//   warp 5     MMA warp (converged, one elected lane issues): S_j = Q K_j^T
//              (SS: M = N = 128, K = 64) as soon as K_j has landed and the
//              softmax has read S_{j-1}; O += P_j V_j (A = P_j from TMEM) as
//              soon as V_j has landed and P_j is written.
// TMEM: S [0,128), P [128,192) (packed bf16), O [192,256).
#include <limits.h>
#include <math.h>

#include "ex2_fma.cuh"
#include "params.h"

namespace fa {
namespace {
namespace d64 {

constexpr int D = 64;
constexpr int BM = 128;                     // query rows per CTA
constexpr int BN = 128;                     // keys per tile
constexpr int KSTAGES = 3;
constexpr int VSTAGES = 2;
constexpr int THREADS = 192;
constexpr int WARP_TMA = 4;
constexpr int WARP_MMA = 5;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t TM_S = 0;
constexpr uint32_t TM_P = 128;
constexpr uint32_t TM_O = 192;
constexpr uint32_t TILE = BN * D * 2;       // one 128 x 64 bf16 tile: 128-byte rows
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + TILE;
constexpr uint32_t OFF_V = OFF_K + KSTAGES * TILE;
constexpr uint32_t OFF_BAR = OFF_V + VSTAGES * TILE;
// q_full, k_full[K], k_empty[K], v_full[V], v_empty[V], s_full, s_free,
// p_ready, pv_done
constexpr int NBAR = 1 + 2 * KSTAGES + 2 * VSTAGES + 4;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;   // tmem slot, abort
constexpr uint32_t SMEM = OFF_MISC + 16 + 1024;     // + alignment slack
static_assert(2 * (SMEM + 1024) <= 233472, "two CTAs per SM");
constexpr float RESCALE_LOG2 = 8.f;
constexpr unsigned FULL = 0xffffffffu;

struct Bars {
  uint32_t b;
  __device__ uint32_t q_full() const { return b; }
  __device__ uint32_t k_full(int s) const { return b + 8u * (1 + s); }
  __device__ uint32_t k_empty(int s) const { return b + 8u * (1 + KSTAGES + s); }
  __device__ uint32_t v_full(int s) const { return b + 8u * (1 + 2 * KSTAGES + s); }
  __device__ uint32_t v_empty(int s) const { return b + 8u * (1 + 2 * KSTAGES + VSTAGES + s); }
  __device__ uint32_t s_full() const { return b + 8u * (1 + 2 * KSTAGES + 2 * VSTAGES); }
  __device__ uint32_t s_free() const { return b + 8u * (2 + 2 * KSTAGES + 2 * VSTAGES); }
  __device__ uint32_t p_ready() const { return b + 8u * (3 + 2 * KSTAGES + 2 * VSTAGES); }
  __device__ uint32_t pv_done() const { return b + 8u * (4 + 2 * KSTAGES + 2 * VSTAGES); }
};

// Debug builds: event kinds of the traced CTA's stamps (one per key tile j;
// T_W_EPI once, at index 0), and every CTA's SM and global timer (ns) at its
// start and end (kinds 29-31, at index blockIdx.x), whichever CTA is traced.
enum : int {
  T_W_SFULL = 0, T_W_LD = 1, T_W_EXP = 2, T_W_ARR = 3, T_M_S = 4, T_M_PV = 5, T_W_EPI = 6,
  T_CTA_SM = 29, T_CTA_START = 30, T_CTA_END = 31
};

__device__ __forceinline__ void cta_span(const AttnParams& p, int kind) {
#ifdef FA_DEBUG
  if (p.trace != nullptr && blockIdx.x < 1024) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    p.trace[kind * 1024 + blockIdx.x] = t;
    if (kind == T_CTA_START) {
      unsigned sm;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
      p.trace[T_CTA_SM * 1024 + blockIdx.x] = sm + 1ull;
    }
  }
#else
  (void)p;
  (void)kind;
#endif
}

// Codes recorded in the device error word when a wait gives up.
enum : unsigned {
  W_Q = 0x80100, W_KEMPTY = 0x80200, W_VEMPTY = 0x80300, W_KFULL = 0x80400, W_VFULL = 0x80500,
  W_SFULL = 0x80600, W_SFREE = 0x80700, W_PREADY = 0x80800, W_PVDONE = 0x80900
};

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const DevErr& e,
                                          volatile int* abort, unsigned where) {
  const bool ok = mbar_wait(bar, parity, e, abort, where);
  return __all_sync(FULL, ok);
}

// Non-blocking test of a phase, agreed by the whole warp.
__device__ __forceinline__ bool warp_test(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return __all_sync(FULL, done != 0);
}

__global__ void __launch_bounds__(THREADS, 2)
    fwd_d64_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnParams p, int num_m,
                   int group) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);

  // Tile order: groups of heads for L2 reuse of K / V; inside a group the
  // longest causal tiles (largest m_blk) first.
  const TileSlot ts = grouped_slot(blockIdx.x, num_m, p.H * p.B, group);
  const int m_blk = num_m - 1 - ts.t;
  const int h = ts.unit % p.H;
  const int b = ts.unit / p.H;
  const SeqInfo sq = seq_info(p, b);
  if (!seq_ok(p, sq) || m_blk * BM >= sq.len) return;   // whole CTA, before any shared state
  if (threadIdx.x == 0) cta_span(p, T_CTA_START);
  const int hk = h / (p.H / p.H_kv);
  const int n_kv_all = (sq.len + BN - 1) / BN;
  const int n_kv = p.causal ? min(n_kv_all, m_blk + 1) : n_kv_all;

  const Bars bars{sbase + OFF_BAR};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    *abort = 0;
    mbar_init(bars.q_full(), 1);
    for (int s = 0; s < KSTAGES; ++s) {
      mbar_init(bars.k_full(s), 1);
      mbar_init(bars.k_empty(s), 1);
    }
    for (int s = 0; s < VSTAGES; ++s) {
      mbar_init(bars.v_full(s), 1);
      mbar_init(bars.v_empty(s), 1);
    }
    mbar_init(bars.s_full(), 1);
    mbar_init(bars.s_free(), 128);
    mbar_init(bars.p_ready(), 128);
    mbar_init(bars.pv_done(), 1);
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
    // ------------------------------------------------------------ producer ---
    // The whole warp runs the loop; lane 0 issues.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(bars.q_full(), TILE);
      tma_load_2d(sbase + OFF_Q, &tm_q, bars.q_full(), h * D, sq.start + m_blk * BM);
    }
    int jk = 0, jv = 0;
    bool ok = true;
    long long t_last = clock64();
    while (jk < n_kv || jv < n_kv) {
      bool progress = false;
      if (jk < n_kv && warp_test(bars.k_empty(jk % KSTAGES), ((jk / KSTAGES) & 1) ^ 1)) {
        const int st = jk % KSTAGES;
        if (lane == 0) {
          mbar_arrive_expect_tx(bars.k_full(st), TILE);
          tma_load_2d(sbase + OFF_K + st * TILE, &tm_k, bars.k_full(st), hk * D,
                      sq.start + jk * BN);
        }
        ++jk;
        progress = true;
      }
      if (jv < jk && warp_test(bars.v_empty(jv % VSTAGES), ((jv / VSTAGES) & 1) ^ 1)) {
        const int st = jv % VSTAGES;
        if (lane == 0) {
          mbar_arrive_expect_tx(bars.v_full(st), TILE);
          tma_load_2d(sbase + OFF_V + st * TILE, &tm_v, bars.v_full(st), hk * D,
                      sq.start + jv * BN);
        }
        ++jv;
        progress = true;
      }
      if (progress) {
        t_last = clock64();
        continue;
      }
      // Lane 0 decides, so the whole warp leaves the loop together.
      const int stop =
          __shfl_sync(FULL, *abort ? 1 : (clock64() - t_last > p.err.budget ? 2 : 0), 0);
      if (stop == 1) {
        ok = false;
        break;
      }
      if (stop == 2) {
        if (lane == 0) {
          *abort = 1;
          atomicOr(p.err.word, ERR_TIMEOUT);
          atomicExch(p.err.word + 1, jk < n_kv ? W_KEMPTY : W_VEMPTY);
        }
        ok = false;
        break;
      }
    }
    if (ok && lane == 0) {
      // Drain: the tensor core's last arrivals on the empty barriers must
      // land before the CTA's shared memory is released.
      for (int j = max(0, n_kv - KSTAGES); j < n_kv; ++j)
        if (!mbar_wait(bars.k_empty(j % KSTAGES), (j / KSTAGES) & 1, p.err, abort, W_KEMPTY))
          break;
      for (int j = max(0, n_kv - VSTAGES); j < n_kv; ++j)
        if (!mbar_wait(bars.v_empty(j % VSTAGES), (j / VSTAGES) & 1, p.err, abort, W_VEMPTY))
          break;
    }
  } else if (warp == WARP_MMA) {
    // ---------------------------------------------------------- MMA issuer ---
    // The whole warp runs the loop; one elected lane issues and commits. S_j
    // needs K_j, the S columns read by the softmax (S_{j-1}) and, for j = 0,
    // Q; P_j V_j needs V_j and P_j. Each barrier polled completes its next
    // phase only after this warp has acted on the current one.
    const uint32_t leader = elect_one();
    constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, false, false);
    constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, false, true);
    const uint64_t q_desc = sdesc_sw128(sbase + OFF_Q, 16, 1024);   // rows x D, K-major
    const uint64_t k_desc = sdesc_sw128(sbase + OFF_K, 16, 1024);   // keys x D, K-major
    const uint64_t v_desc = sdesc_sw128(sbase + OFF_V, TILE, 1024);  // keys x D, MN-major
    int is = 0, ip = 0;
    long long t_last = clock64();
    while (ip < n_kv) {
      bool progress = false;
      if (is < n_kv && warp_test(bars.k_full(is % KSTAGES), (is / KSTAGES) & 1) &&
          (is == 0 ? warp_test(bars.q_full(), 0)
                   : warp_test(bars.s_free(), (is - 1) & 1))) {
        const int st = is % KSTAGES;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_if(leader, tmem + TM_S, sdesc_add(q_desc, kk * 32),
                    sdesc_add(k_desc, st * TILE + kk * 32), IDESC_QK, kk > 0);
        tc_commit_if(leader, bars.s_full());
        tc_commit_if(leader, bars.k_empty(st));
        if (lane == 0) FA_STAMP(p, T_M_S, is);
        ++is;
        progress = true;
      }
      if (ip < is && warp_test(bars.v_full(ip % VSTAGES), (ip / VSTAGES) & 1) &&
          warp_test(bars.p_ready(), ip & 1)) {
        const int st = ip % VSTAGES;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)   // K = 128 keys in steps of 16
          mma_ts_if(leader, tmem + TM_O, tmem + TM_P + kk * 8,
                    sdesc_add(v_desc, st * TILE + kk * 2048), IDESC_PV,
                    (ip > 0 || kk > 0) ? 1u : 0u);
        tc_commit_if(leader, bars.v_empty(st));
        tc_commit_if(leader, bars.pv_done());
        if (lane == 0) FA_STAMP(p, T_M_PV, ip);
        ++ip;
        progress = true;
      }
      if (progress) {
        t_last = clock64();
        continue;
      }
      const int stop =
          __shfl_sync(FULL, *abort ? 1 : (clock64() - t_last > p.err.budget ? 2 : 0), 0);
      if (stop == 1) break;
      if (stop == 2) {
        if (lane == 0) {
          *abort = 1;
          atomicOr(p.err.word, ERR_TIMEOUT);
          atomicExch(p.err.word + 1, (ip < is) ? W_PREADY : W_KFULL);
        }
        break;
      }
    }
  } else {
    // ------------------------------------------------------------- softmax ---
    const int row = threadIdx.x;   // query row of the tile = TMEM lane
    const int qpos = m_blk * BM + row;
    const bool row_ok = qpos < sq.len;
    const int lim = p.causal ? min(qpos, sq.len - 1) : sq.len - 1;   // last visible key
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float c2 = p.scale_log2;
    const bool stamp = threadIdx.x == 0;   // debug stamps: lane 0 of warp 0
    float m_ref = -INFINITY;   // reference max (log2 units)
    float l = 0.f;             // row sum in that reference
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
      if (!(ok = warp_wait(bars.s_full(), j & 1, p.err, abort, W_SFULL))) break;
      if (stamp) FA_STAMP(p, T_W_SFULL, j);
      tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + TM_S + 32 * c, r[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(r[c]);
      if (stamp) FA_STAMP(p, T_W_LD, j);
      // The scores are in registers: the tensor core may overwrite S.
      tc_fence_before();
      mbar_arrive(bars.s_free());
      const int nvalid = lim - j * BN + 1;   // visible keys in this tile
      if (nvalid < BN) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (32 * c + i >= nvalid) r[c][i] = __float_as_uint(-INFINITY);
      }
      // Row max with 8 independent partial maxima.
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], __uint_as_float(r[c][i]));
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_cand = mx * c2;
      const bool grow = m_cand > m_ref + RESCALE_LOG2;   // always true on the first visible tile
      const float m_prev = m_ref;
      if (grow) m_ref = m_cand;
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      // Arguments and row sums on packed fp32 pairs (0.1188 against 0.1208 ms).
      float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      const float2 c2p = make_float2(c2, c2), nm = make_float2(-m_use, -m_use);
      uint32_t pk[2][32];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 x =
              __ffma2_rn(make_float2(__uint_as_float(r[c][i]), __uint_as_float(r[c][i + 1])), c2p, nm);
          // A quarter of the exponentials (4 of every 16 keys) on the FMA
          // pipe: the two CTAs' softmax warps share each sub-partition's
          // special-function unit (0.1208 against 0.1249 ms on B4 H16 N2048;
          // an eighth 0.1229, three eighths 0.1311).
          const bool fma_pipe = (i % 16) < 4;
          const float p0 = fma_pipe ? ex2_fma(x.x) : ex2_approx(x.x);
          const float p1 = fma_pipe ? ex2_fma(x.y) : ex2_approx(x.y);
          sum2[(i >> 1) & 1] = __fadd2_rn(sum2[(i >> 1) & 1], make_float2(p0, p1));
          pk[c >> 1][(c & 1) * 16 + i / 2] = pack_bf16x2(p0, p1);
        }
      const float sum = (sum2[0].x + sum2[1].x) + (sum2[0].y + sum2[1].y);
      if (stamp) FA_STAMP(p, T_W_EXP, j);
      const float alpha = (grow && m_prev != -INFINITY) ? ex2_approx(m_prev - m_use) : 1.f;
      l = grow ? l * alpha + sum : l + sum;
      // P_{j-1} V_{j-1} has read P and added into O.
      if (j > 0 && !(ok = warp_wait(bars.pv_done(), (j - 1) & 1, p.err, abort, W_PVDONE)))
        break;
      tc_fence_after();
      tmem_st32(tmem + lane_off + TM_P, pk[0]);
      tmem_st32(tmem + lane_off + TM_P + 32, pk[1]);
      if (j > 0 && __any_sync(FULL, alpha != 1.f)) {
        // O row moves to the new reference.
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
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bars.p_ready());
      if (stamp) FA_STAMP(p, T_W_ARR, j);
    }
    // ----------------------------------------------------------- epilogue ---
    const int last = n_kv - 1;
    if (ok && warp_wait(bars.pv_done(), last & 1, p.err, abort, W_PVDONE)) {
      tc_fence_after();
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      const float lse = (l > 0.f) ? (m_ref + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      const size_t out_row = static_cast<size_t>(sq.start + qpos) * p.H + h;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + TM_O + 32 * c, o);
        tmem_ld_wait();
        reg_fence(o);
        if (row_ok) {
          uint4* dst =
              reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + out_row * D + 32 * c);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 wv;
            wv.x = pack_bf16x2(__uint_as_float(o[8 * v4 + 0]) * inv_l,
                               __uint_as_float(o[8 * v4 + 1]) * inv_l);
            wv.y = pack_bf16x2(__uint_as_float(o[8 * v4 + 2]) * inv_l,
                               __uint_as_float(o[8 * v4 + 3]) * inv_l);
            wv.z = pack_bf16x2(__uint_as_float(o[8 * v4 + 4]) * inv_l,
                               __uint_as_float(o[8 * v4 + 5]) * inv_l);
            wv.w = pack_bf16x2(__uint_as_float(o[8 * v4 + 6]) * inv_l,
                               __uint_as_float(o[8 * v4 + 7]) * inv_l);
            dst[v4] = wv;
          }
        }
      }
      if (row_ok) p.lse[lse_index(p, b, h, sq.start, qpos)] = lse;
      if (stamp) FA_STAMP(p, T_W_EPI, 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  if (threadIdx.x == 0) cta_span(p, T_CTA_END);
}

}  // namespace d64
}  // namespace

// The D = 64 forward (fa_fwd uses it).
cudaError_t launch_fwd_d64(const AttnParams& p, cudaStream_t stream) {
  using namespace d64;
  if (p.D != D) return cudaErrorInvalidValue;
  const int num_m = (p.max_seqlen + BM - 1) / BM;
  const long long tiles = static_cast<long long>(num_m) * p.H * p.B;
  if (tiles == 0 || p.total == 0) return cudaSuccess;
  if (tiles > INT_MAX) return cudaErrorInvalidConfiguration;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16_2d(&tq, p.q, p.total, static_cast<unsigned long long>(p.H) * D, 64, BM) ||
      !make_tmap_bf16_2d(&tk, p.k, p.total, static_cast<unsigned long long>(p.H_kv) * D, 64, BN) ||
      !make_tmap_bf16_2d(&tv, p.v, p.total, static_cast<unsigned long long>(p.H_kv) * D, 64, BN))
    return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(fwd_d64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  const int group = l2_group(4ll * p.max_seqlen * D, p.H / p.H_kv, p.H * p.B);
  fwd_d64_kernel<<<static_cast<unsigned>(tiles), THREADS, SMEM, stream>>>(tq, tk, tv, p, num_m,
                                                                          group);
  return cudaGetLastError();
}

}  // namespace fa
