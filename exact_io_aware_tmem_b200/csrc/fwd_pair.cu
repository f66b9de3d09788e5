// Attention forward, two 128-row query tiles per CTA, bf16 in / fp32
// accumulate, on the sm_100a tensor cores (D = 128).
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
// in base 2 on pre-scaled logits (scale * log2 e). The reference max m only
// moves when a row max exceeds it by more than 2^8 (P <= 2^8 before the bf16
// cast); O / l is the same for any reference, so the recurrence is unchanged
// up to rounding and the O rescale is rare.
//
// How, on B200. One CTA per pair of 128-row query tiles (Q_0, Q_1) of one
// (sequence, head); each K_j, V_j tile brought into shared memory serves both.
//   warps 0-3   softmax group 0, rows of Q_0 (thread = row = TMEM lane);
//   warps 4-7   softmax group 1, rows of Q_1;
//   warp 8      TMA producer: Q_0 and Q_1 once, then K_j and V_j through
//               their own rings (K ahead of V whenever both have room);
//   warp 9      MMA warp, converged, one elect.sync lane issuing. Per key
//               tile j: P_0 V_j, S_0 = Q_0 K_{j+1}^T, P_1 V_j,
//               S_1 = Q_1 K_{j+1}^T, so each group exponentiates tile j+1
//               while the tensor core works for the other group.
// The two groups share nothing but the K / V tiles: each owns its S, P and O
// in TMEM (S_g [128 g, 128 g + 128), O_g [256 + D g, ...), P_g as bf16 over
// the first 64 columns of S_g once the scores are in registers). S_g of tile
// j+1 completing implies P_g V_j has completed (the tensor core runs one
// thread's MMAs in order and a commit covers all earlier ones), so a group
// can rescale its O between the two without any other signal.
// F8 (D = 128): pass 2 of the FP8 forward (aiqz.cc article, section "FP8 low
// precision"). Q and K arrive as E4M3 codes, one 128-byte row per token, with
// one fp32 step per 128-token block (pass 1, fp8.cu); S = Q_hat K_hat^T runs
// as a kind::f8f6f4 MMA with fp32 accumulation and is scaled by the two
// blocks' Delta_Q Delta_K with the logit scale. P V stays bf16. The smaller Q
// and K tiles leave room for four K and four V stages.
#include <limits.h>
#include <math.h>

#include "params.h"

namespace fa {
namespace {

namespace pair {

constexpr int BM = 128;            // rows per query tile
constexpr int BN = 128;            // keys per tile
constexpr int THREADS = 320;
constexpr int WARP_TMA = 8;
constexpr int WARP_MMA = 9;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S = 0;       // S_g at TM_S + 128 g
constexpr uint32_t TM_O = 256;     // O_g at TM_O + D g
constexpr uint32_t SPAN = 128 * 128;          // 128 rows x 128 bytes (one swizzle column block)
constexpr int KS_MAX = 4;
constexpr int VS_MAX = 4;

template <int D, bool F8>
struct Cfg {
  static_assert(D == 128, "head dim (D = 64 has its own kernel, fwd_d64.cu)");
  static_assert(!F8 || D == 128, "E4M3 rows of 128 bytes");
  static constexpr uint32_t TILE = BM * D * 2;       // bf16 tile, 32 KB at D = 128
  static constexpr uint32_t QK_TILE = F8 ? BM * D : TILE;   // Q or K tile
  static constexpr int QK_CHUNKS = F8 ? 1 : D / 64;  // 128-byte column blocks of a Q / K row
  static constexpr int KS = F8 ? 4 : (D == 128 ? 3 : 4);   // K stages
  static constexpr int VS = F8 ? 4 : (D == 128 ? 2 : 4);   // V stages
  static constexpr uint32_t OFF_Q = 0;               // Q_0, Q_1
  static constexpr uint32_t OFF_K = OFF_Q + 2 * QK_TILE;
  static constexpr uint32_t OFF_V = OFF_K + KS * QK_TILE;
  static constexpr uint32_t OFF_BAR = OFF_V + VS * TILE;
  // q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[2],
  // p_ready[2], o_full (laid out for the largest ring depths)
  static constexpr int NBAR = 1 + 2 * KS_MAX + 2 * VS_MAX + 5;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  // No alignment slack: the dynamic shared memory must start on a 1024-byte
  // boundary (128-byte swizzle atoms); the kernel checks and reports.
  static constexpr uint32_t SMEM = OFF_MISC + 16;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(KS <= KS_MAX && VS <= VS_MAX, "ring depths");
};
constexpr float RESCALE_LOG2 = 8.f;
constexpr unsigned FULL = 0xffffffffu;

struct Bars {
  uint32_t b;
  __device__ uint32_t q_full() const { return b; }
  __device__ uint32_t k_full(int s) const { return b + 8u * (1 + s); }
  __device__ uint32_t k_empty(int s) const { return b + 8u * (1 + KS_MAX + s); }
  __device__ uint32_t v_full(int s) const { return b + 8u * (1 + 2 * KS_MAX + s); }
  __device__ uint32_t v_empty(int s) const { return b + 8u * (1 + 2 * KS_MAX + VS_MAX + s); }
  __device__ uint32_t s_full(int g) const { return b + 8u * (1 + 2 * KS_MAX + 2 * VS_MAX + g); }
  __device__ uint32_t p_ready(int g) const { return b + 8u * (3 + 2 * KS_MAX + 2 * VS_MAX + g); }
  __device__ uint32_t o_full() const { return b + 8u * (5 + 2 * KS_MAX + 2 * VS_MAX); }
};

// Event kinds of the debug build's stamps (one per key tile j unless noted);
// group g's softmax kinds are T_W_SFULL + 4 g, ...
enum : int {
  T_P_K = 0, T_P_V = 1, T_M_VFULL = 2, T_M_PV0 = 3, T_M_S0 = 4 /* S_0 of tile j+1, index j+1 */,
  T_M_PV1 = 5, T_M_S1 = 6 /* index j+1 */, T_W_SFULL = 7, T_W_LD = 8, T_W_EXP = 9, T_W_ARR = 10,
  T_M_PREADY0 = 15, T_M_PREADY1 = 16
};

enum : unsigned {
  W_Q = 0x50100, W_KEMPTY = 0x50200, W_VEMPTY = 0x50300, W_KFULL = 0x50400, W_VFULL = 0x50500,
  W_SFULL = 0x50600, W_PREADY = 0x50700, W_OFULL = 0x50800, BAD_ALIGN = 0x50900
};

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const DevErr& e,
                                          volatile int* abort, unsigned where) {
  const bool ok = mbar_wait(bar, parity, e, abort, where);
  return __all_sync(FULL, ok);
}

// 320 threads: ten warps, three on two of the four SM sub-partitions, whose
// 16K registers then allow 168 per thread.
template <int D, bool F8>
__global__ void __launch_bounds__(THREADS, 1)
    fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p, int num_m2,
                    int group, const Fp8Args f8) {
  using C = Cfg<D, F8>;
  constexpr int KS = C::KS, VS = C::VS;
  constexpr uint32_t TILE = C::TILE, QK_TILE = C::QK_TILE;
  constexpr uint32_t OFF_Q = C::OFF_Q, OFF_K = C::OFF_K, OFF_V = C::OFF_V;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if ((sbase & 1023u) != 0) {
    if (threadIdx.x == 0) {
      atomicOr(p.err.word, ERR_BOUNDS);
      atomicExch(p.err.word + 1, BAD_ALIGN);
    }
    return;
  }
  // Tile order: groups of heads for L2 reuse of K / V; inside a group the
  // longest causal pairs (largest m2) first.
  const TileSlot ts = grouped_slot(blockIdx.x, num_m2, p.H * p.B, group);
  const int m2 = num_m2 - 1 - ts.t;
  const int h = ts.unit % p.H;
  const int b = ts.unit / p.H;
  const SeqInfo sq = seq_info(p, b);
  if (!seq_ok(p, sq) || m2 * 2 * BM >= sq.len) return;  // whole CTA, before any shared state
  const int hk = h / (p.H / p.H_kv);
  const int n_all = (sq.len + BN - 1) / BN;
  // Key tiles of each query tile (0: tile 2 m2, 1: tile 2 m2 + 1; none when
  // the second tile starts past the end of the sequence).
  const int n_0 = p.causal ? min(n_all, 2 * m2 + 1) : n_all;
  const int n_1 = ((2 * m2 + 1) * BM >= sq.len) ? 0 : (p.causal ? min(n_all, 2 * m2 + 2) : n_all);
  const int n_kv = max(n_0, n_1);

  const Bars bars{sbase + C::OFF_BAR};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    *abort = 0;
    mbar_init(bars.q_full(), 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(bars.k_full(s), 1);
      mbar_init(bars.k_empty(s), 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(bars.v_full(s), 1);
      mbar_init(bars.v_empty(s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bars.s_full(g), 1);
      mbar_init(bars.p_ready(g), 128);
    }
    mbar_init(bars.o_full(), 1);
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
    // The whole warp runs the loop; lane 0 issues the copies.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      // Both query tiles; rows past the tensor arrive as zeros (and are
      // never written out).
      mbar_arrive_expect_tx(bars.q_full(), 2 * QK_TILE);
      for (int g = 0; g < 2; ++g)
        for (int c = 0; c < C::QK_CHUNKS; ++c)
          tma_load_2d(sbase + OFF_Q + g * QK_TILE + c * SPAN, &tm_q, bars.q_full(),
                      h * D + c * 64, sq.start + (2 * m2 + g) * BM);
    }
    int jk = 0, jv = 0;
    long long t_last = clock64();
    while (jk < n_kv || jv < n_kv) {
      bool progress = false;
      if (jk < n_kv &&
          __all_sync(FULL, mbar_try_wait(bars.k_empty(jk % KS), ((jk / KS) & 1) ^ 1))) {
        const int st = jk % KS;
        if (lane == 0) {
          mbar_arrive_expect_tx(bars.k_full(st), QK_TILE);
          for (int c = 0; c < C::QK_CHUNKS; ++c)
            tma_load_2d(sbase + OFF_K + st * QK_TILE + c * SPAN, &tm_k, bars.k_full(st),
                        hk * D + c * 64, sq.start + jk * BN);
          FA_STAMP(p, T_P_K, jk);
        }
        __syncwarp();
        ++jk;
        progress = true;
      }
      if (jv < jk &&
          __all_sync(FULL, mbar_try_wait(bars.v_empty(jv % VS), ((jv / VS) & 1) ^ 1))) {
        const int st = jv % VS;
        if (lane == 0) {
          mbar_arrive_expect_tx(bars.v_full(st), TILE);
          for (int c = 0; c < D / 64; ++c)
            tma_load_2d(sbase + OFF_V + st * TILE + c * SPAN, &tm_v, bars.v_full(st),
                        hk * D + c * 64, sq.start + jv * BN);
          FA_STAMP(p, T_P_V, jv);
        }
        __syncwarp();
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
      if (stop == 1) break;
      if (stop == 2) {
        if (lane == 0) {
          *abort = 1;
          atomicOr(p.err.word, ERR_TIMEOUT);
          atomicExch(p.err.word + 1, jk < n_kv ? W_KEMPTY : W_VEMPTY);
        }
        break;
      }
    }
    if (lane == 0) {
      // Drain: the tensor core's arrivals on the last stages' empty barriers
      // must land before the CTA's shared memory is released.
      for (int j = max(0, n_kv - KS); j < n_kv && !*abort; ++j)
        if (!mbar_wait(bars.k_empty(j % KS), (j / KS) & 1, p.err, abort, W_KEMPTY)) break;
      for (int j = max(0, n_kv - VS); j < n_kv && !*abort; ++j)
        if (!mbar_wait(bars.v_empty(j % VS), (j / VS) & 1, p.err, abort, W_VEMPTY)) break;
    }
  } else if (warp == WARP_MMA) {
    // ---------------------------------------------------------- MMA issuer ---
    // The whole warp runs the loop (waits and operands stay warp-uniform);
    // one elected lane issues the tensor-core instructions and commits.
    const uint32_t leader = elect_one();
    constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, false, false);
    constexpr uint32_t IDESC_QK8 = idesc_e4m3(BM, BN);
    constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, false, true);
    const uint64_t q_desc = sdesc_sw128(sbase + OFF_Q, 16, 1024);
    const uint64_t k_desc = sdesc_sw128(sbase + OFF_K, 16, 1024);
    const uint64_t v_desc = sdesc_sw128(sbase + OFF_V, SPAN, 1024);
    // S_g = Q_g K_j^T (M = 128 rows, N = 128 keys, K = D in steps of 16
    // bf16 or 32 E4M3 codes: 32 bytes of a row either way).
    auto issue_s = [&](int g, int j) {
      const int st = j % KS;
      if constexpr (F8) {
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_ss_e4m3_if(leader, tmem + TM_S + g * BN, sdesc_add(q_desc, g * QK_TILE + kk * 32),
                         sdesc_add(k_desc, st * QK_TILE + kk * 32), IDESC_QK8, kk > 0);
      } else {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o = (kk >> 2) * SPAN + (kk & 3) * 32;
          mma_ss_if(leader, tmem + TM_S + g * BN, sdesc_add(q_desc, g * TILE + o),
                    sdesc_add(k_desc, st * TILE + o), IDESC_QK, kk > 0);
        }
      }
      tc_commit_if(leader, bars.s_full(g));
    };
    // O_g += P_g V_j (M = 128 rows, N = D, K = 128 keys in steps of 16; P_g
    // packed two keys per TMEM column over the first 64 columns of S_g).
    auto issue_pv = [&](int g, int j) {
      const int st = j % VS;
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk)
        mma_ts_if(leader, tmem + TM_O + g * D, tmem + TM_S + g * BN + kk * 8,
                  sdesc_add(v_desc, st * TILE + kk * 2048), IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
    };
    bool ok = warp_wait(bars.q_full(), 0, p.err, abort, W_Q) &&
              warp_wait(bars.k_full(0), 0, p.err, abort, W_KFULL);
    if (ok) {
      tc_fence_after();
      if (n_0 > 0) issue_s(0, 0);
      if (n_1 > 0) issue_s(1, 0);
      tc_commit_if(leader, bars.k_empty(0));
    }
    for (int j = 0; ok && j < n_kv; ++j) {
      if (!(ok = warp_wait(bars.v_full(j % VS), (j / VS) & 1, p.err, abort, W_VFULL))) break;
      if (lane == 0) FA_STAMP(p, T_M_VFULL, j);
      const bool next = j + 1 < n_kv;
      bool k_next = false;   // K_{j+1} seen in shared memory
#pragma unroll
      for (int g = 0; g < 2 && ok; ++g) {
        const int n_g = g ? n_1 : n_0;
        if (j < n_g) {
          if (!(ok = warp_wait(bars.p_ready(g), j & 1, p.err, abort, W_PREADY))) break;
          if (lane == 0) FA_STAMP(p, g ? T_M_PREADY1 : T_M_PREADY0, j);
          tc_fence_after();
          issue_pv(g, j);
          if (lane == 0) FA_STAMP(p, g ? T_M_PV1 : T_M_PV0, j);
        }
        // S_g of the next tile overwrites P_g: it follows P_g V_j.
        if (j + 1 < n_g) {
          if (!k_next) {
            if (!(ok = warp_wait(bars.k_full((j + 1) % KS), ((j + 1) / KS) & 1, p.err, abort,
                                 W_KFULL)))
              break;
            tc_fence_after();
            k_next = true;
          }
          issue_s(g, j + 1);
          if (lane == 0) FA_STAMP(p, g ? T_M_S1 : T_M_S0, j + 1);
        }
      }
      if (!ok) break;
      tc_commit_if(leader, bars.v_empty(j % VS));
      if (next) tc_commit_if(leader, bars.k_empty((j + 1) % KS));
    }
    tc_commit_if(leader, bars.o_full());
  } else {
    // ------------------------------------------------------------- softmax ---
    const int g = warp >> 2;          // query tile of this group
    const int quarter = warp & 3;     // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    const int qpos = (2 * m2 + g) * BM + row;
    const bool row_ok = qpos < sq.len;
    const int lim = p.causal ? min(qpos, sq.len - 1) : sq.len - 1;   // last visible key
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_col = tmem + lane_off + TM_S + g * BN;
    const uint32_t o_col = tmem + lane_off + TM_O + g * D;
    const int n = g ? n_1 : n_0;
    // Logit scale in log2 units per raw score; E4M3 scores are in units of
    // Delta_Q Delta_K of their two blocks (Delta_K per key tile below).
    float c2 = p.scale_log2;
    const float* kscale_row = nullptr;
    if constexpr (F8) {
      if (n > 0) c2 *= __ldg(f8.q_scale + (static_cast<size_t>(b) * p.H + h) * f8.n_blocks +
                             2 * m2 + g);
      kscale_row = f8.k_scale + (static_cast<size_t>(b) * p.H_kv + hk) * f8.n_blocks;
    }
    const bool stamp = quarter == 0 && lane == 0;   // debug stamps: first warp of each group
    [[maybe_unused]] const int tk = 4 * g;
    float m_ref = -INFINITY;  // reference max (log2 units)
    float l = 0.f;            // row sum in that reference
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) {
      const float c2t = F8 ? c2 * __ldg(kscale_row + j) : c2;   // log2 units per raw score
      if (!(ok = warp_wait(bars.s_full(g), j & 1, p.err, abort, W_SFULL))) break;
      if (stamp) FA_STAMP(p, T_W_SFULL + tk, j);
      tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_col + 32 * c, r[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(r[c]);
      if (stamp) FA_STAMP(p, T_W_LD + tk, j);
      const int nvalid = lim - j * BN + 1;   // visible keys in this tile
      if (nvalid < BN) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (32 * c + i >= nvalid) r[c][i] = __float_as_uint(-INFINITY);
      }
      // Row max with 4 independent partial maxima.
      float mx4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) mx4[i] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; ++i) mx4[i & 3] = fmaxf(mx4[i & 3], __uint_as_float(r[c][i]));
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      const float m_cand = mx * c2t;
      const bool grow = m_cand > m_ref + RESCALE_LOG2;   // always true on the first visible tile
      const float m_new = grow ? m_cand : m_ref;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      // Arguments and row sums on packed fp32 pairs. Besides halving those
      // instructions this spills less at the 168-register cap than the
      // scalar form (0.483 against 0.499 ms on causal N8192); packing the
      // arguments alone spilled more and was slower (0.516).
      float2 sum2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      const float2 c2p = make_float2(c2t, c2t), nm = make_float2(-m_use, -m_use);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 x =
              __ffma2_rn(make_float2(__uint_as_float(r[c][i]), __uint_as_float(r[c][i + 1])), c2p, nm);
          const float p0 = ex2_approx(x.x);
          const float p1 = ex2_approx(x.y);
          sum2[(i >> 1) & 1] = __fadd2_rn(sum2[(i >> 1) & 1], make_float2(p0, p1));
          pk[i >> 1] = pack_bf16x2(p0, p1);
        }
        // P over the first 64 columns of S_g: keys 32 c .. 32 c + 31 in
        // columns 16 c .. 16 c + 15 (this thread's scores are in registers).
        tmem_st16(s_col + 16 * c, pk);
      }
      const float sum = (sum2[0].x + sum2[1].x) + (sum2[0].y + sum2[1].y);
      if (stamp) FA_STAMP(p, T_W_EXP + tk, j);
      // The reference moved: rescale the row sum and (from the second tile
      // on) the O row, which holds P V of the earlier tiles only: S_g of this
      // tile completing means P_g V of the previous tile has completed.
      const float alpha = (grow && m_ref != -INFINITY) ? ex2_approx(m_ref - m_use) : 1.f;
      l = l * alpha + sum;
      if (j > 0 && __any_sync(FULL, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(o_col + 32 * c, o);
          tmem_ld_wait();
          reg_fence(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(o_col + 32 * c, o);
        }
      }
      m_ref = m_new;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bars.p_ready(g));
      if (stamp) FA_STAMP(p, T_W_ARR + tk, j);
    }
    // ------------------------------------------------------------ epilogue ---
    if (ok && n > 0 && warp_wait(bars.o_full(), 0, p.err, abort, W_OFULL)) {
      tc_fence_after();
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      const size_t out_row = static_cast<size_t>(sq.start + qpos) * p.H + h;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(o_col + 32 * c, o);
        tmem_ld_wait();
        reg_fence(o);
        if (row_ok && FA_CHECK(p, out_row < static_cast<size_t>(p.total) * p.H, 0xDB0501u)) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + out_row * D +
                                                32 * c);
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
      if (row_ok)
        p.lse[lse_index(p, b, h, sq.start, qpos)] =
            (l > 0.f) ? (m_ref + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace pair

}  // namespace

namespace {

template <int D>
cudaError_t launch_pair_d(const AttnParams& p, cudaStream_t stream) {
  using namespace pair;
  using C = Cfg<D, false>;
  const int num_m2 = (p.max_seqlen + 2 * BM - 1) / (2 * BM);
  const long long tiles = static_cast<long long>(num_m2) * p.H * p.B;
  if (tiles == 0 || p.total == 0) return cudaSuccess;
  if (tiles > INT_MAX) return cudaErrorInvalidConfiguration;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16_2d(&tq, p.q, p.total, static_cast<unsigned long long>(p.H) * D, 64, BM) ||
      !make_tmap_bf16_2d(&tk, p.k, p.total, static_cast<unsigned long long>(p.H_kv) * D, 64, BN) ||
      !make_tmap_bf16_2d(&tv, p.v, p.total, static_cast<unsigned long long>(p.H_kv) * D, 64, BN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fwd_pair_kernel<D, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int group = l2_group(4ll * p.max_seqlen * D, p.H / p.H_kv, p.H * p.B);
  fwd_pair_kernel<D, false><<<static_cast<unsigned>(tiles), THREADS, C::SMEM, stream>>>(
      tq, tk, tv, p, num_m2, group, Fp8Args{});
  return cudaGetLastError();
}

}  // namespace

// Pass 2 of the FP8 forward at D = 128: p.q / p.k hold the E4M3 codes, ``f``
// their per-block steps (fa_fwd_fp8 uses it).
cudaError_t launch_fwd_pair_fp8(const AttnParams& p, const Fp8Args& f, cudaStream_t stream) {
  using namespace pair;
  constexpr int D = 128;
  using C = Cfg<D, true>;
  if (p.D != D) return cudaErrorInvalidValue;
  const int num_m2 = (p.max_seqlen + 2 * BM - 1) / (2 * BM);
  const long long tiles = static_cast<long long>(num_m2) * p.H * p.B;
  if (tiles == 0 || p.total == 0) return cudaSuccess;
  if (tiles > INT_MAX) return cudaErrorInvalidConfiguration;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_u8_2d(&tq, p.q, p.total, static_cast<unsigned long long>(p.H) * D, 128, BM) ||
      !make_tmap_u8_2d(&tk, p.k, p.total, static_cast<unsigned long long>(p.H_kv) * D, 128, BN) ||
      !make_tmap_bf16_2d(&tv, p.v, p.total, static_cast<unsigned long long>(p.H_kv) * D, 64, BN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fwd_pair_kernel<D, true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int group = l2_group(3ll * p.max_seqlen * D, p.H / p.H_kv, p.H * p.B);
  fwd_pair_kernel<D, true><<<static_cast<unsigned>(tiles), THREADS, C::SMEM, stream>>>(
      tq, tk, tv, p, num_m2, group, f);
  return cudaGetLastError();
}

cudaError_t launch_fwd_pair(const AttnParams& p, cudaStream_t stream) {
  if (p.D == 128) return launch_pair_d<128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fa
