// Attention backward in one pass over the (query tile, key tile) pairs: every
// product of the method once, bf16 in / fp32 accumulate, on the sm_100a
// tensor cores.
//
// What it computes, for the loss sum(O * dO): the scores and probabilities are
// rebuilt from Q, K and the saved LSE instead of being stored (agentalpha.top
// "flash attention" answer, section 2; airsota.com card, section 4 item 2), and
// the gradient relations the "Flash Attention self-test" (book.bogosort.top,
// section D) asks for are applied tile by tile:
//     P = exp(scale Q K^T - LSE),   dV = P^T dO,   dP = dO V^T,
//     D_i = dO_i . O_i,   dS = P * (dP - D),   dQ = scale dS K,   dK = scale dS^T Q.
//
// One CTA per (sequence, key/value head, 128-key tile j). K_j and V_j stay in
// shared memory while the CTA walks the 128-row query tiles of every query
// head of its GQA group (step t = one query tile of one head). Keys sit on the
// TMEM lanes for the key-side products; per step, five products, each once:
//     S^T  = K Q_t^T            (A, B in shared memory)          -> TMEM S
//     dP^T = V dO_t^T           (A, B in shared memory)          -> TMEM dP
//     dV  += P^T dO_t           (A = P^T, bf16 in TMEM over S)   -> TMEM dV
//     dQ_t = dS K               (A = dS, read MN-major from a swizzled dS^T
//                                tile the dS warps write to shared memory;
//                                queries on the TMEM lanes)      -> TMEM dQ
//     dK  += dS^T Q_t           (A = dS^T, the same tile read K-major)
//                                                                -> TMEM dK
// and the fp32 dQ_t partial is added into the caller's fp32 accumulator
// dQacc [T, H, D] (zeroed by the preprocess kernel; a convert kernel writes
// dQ = bf16(scale dQacc) afterwards): four dQ warps read it out of TMEM in
// one go, stage it in 32 x 32 boxes in shared memory, and one lane of each
// adds its boxes with TMA tensor reductions, which run on their own. The accumulation order over
// key tiles is not fixed, so dQ is reproducible only to rounding; dK and dV
// are summed in a fixed order inside one CTA.
//
// TMEM columns: S [0,128), dP [128,256), dV, dK after them. At D = 128 the
// 512 columns are full, so dQ_t is formed over dP (the dS warps have read dP_t
// before they signal dS_t), and dP_{t+1} waits until dQ_t has been read out.
// At D = 64 dQ_t has columns of its own.
//
// Roles (512 threads, four warpgroups):
//   warps 0-7   dS warps (warpgroups 0, 1; 136 registers). Thread = key row
//               (TMEM lane) for S^T / dP^T, warps w and w+4 taking query
//               columns [64 hf, 64 hf + 64). Per step: exponentials of S^T_t
//               -> P^T_t into TMEM, then dS^T_t into the shared dS tile.
//   warps 8-11  dQ warps (warpgroup 2; 160 registers, enough to hold a whole
//               row block of dQ_t). Thread = query row of dQ_t (TMEM lane):
//               the read-out in one go, dq_free, then the staging and the
//               reductions, off the dS warps' path. With the read-out this
//               short, dP_{t+1} follows dQ_t closely and the staging runs
//               during the exponentials of step t+1 rather than during its
//               dS phase, whose shared-memory stores it would compete with.
//   warp 12     TMA producer (warpgroup 3; 80 registers): K, V once; Q_t (with
//               the step's LSE and D_i staged beside it) through a two-stage
//               ring, dO_t through one stage (dV_t, its last reader, runs long
//               before dP_{t+1}).
//   warp 13     MMA warp (warpgroup 3), converged, one elect.sync lane
//               issuing. Order per step: dP_t, dV_t, S_{t+1}, dQ_t, dK_t. dQ_t
//               goes right after dS_t because its read-out gates dP_{t+1}; the
//               exponentials of step t+1 overlap dQ_t and dK_t, and the dS
//               phase of step t overlaps dV_t and S_{t+1}.
//   warps 14-15 no role (they complete warpgroup 3 for its register count).
#include <limits.h>
#include <math.h>

#include <algorithm>

#include "ex2_fma.cuh"
#include "params.h"

namespace fa {
namespace {

namespace fused {

constexpr int BT = 128;        // keys per CTA = query rows per step = TMEM lanes
constexpr int THREADS = 512;
constexpr int N_DS = 256;      // dS warps' threads (warpgroups 0 and 1)
constexpr int WARP_DQ0 = 8;    // dQ warps 8-11 (warpgroup 2): TMEM lane quarters 0-3
constexpr int N_DQ = 128;      // dQ warps' threads
constexpr int WARP_TMA = 12;   // warpgroup 3: producer, MMA warp, two idle warps
constexpr int WARP_MMA = 13;
// Registers per thread (setmaxnreg): the block launches at 128 (16 warps,
// four per SM sub-partition, 16K registers each). Warpgroup 3 gives back 48
// of them per thread; the dQ warps take 32 (160: a whole dQ_t row block in
// registers) and each dS warpgroup 8 (136: nothing spills, where at 128 the
// dS warps' packed arithmetic did; -2.5 % on causal N8192).
// 2 x 136 + 160 + 80 = 4 x 128 on every sub-partition and for the block.
constexpr uint32_t REG_DS = 136;
constexpr uint32_t REG_DQ = 160;
constexpr uint32_t REG_CTRL = 80;
static_assert(2 * REG_DS + REG_DQ + REG_CTRL == 4 * 128, "register split of the block");
constexpr uint32_t TMEM_COLS = 512;
constexpr unsigned FULL = 0xffffffffu;
constexpr uint32_t SPAN = BT * 128;   // 128 rows x 128 bytes: one 128-byte swizzle column block
constexpr float LOG2E = 1.4426950408889634f;

template <int D>
struct Cfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr uint32_t TILE = BT * D * 2;       // one 128-row bf16 tile of Q, K, V or dO
  static constexpr int QS = 2;                       // Q stages (with LSE, D_i)
  static constexpr int GS = 1;                       // dO stages (dO_{t+1} is read after dV_t)
  static constexpr bool ALIAS = D == 128;            // dQ_t formed over dP
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 256 + D;
  static constexpr uint32_t TM_DQ = ALIAS ? TM_DP : 256 + 2 * D;
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = OFF_K + TILE;
  static constexpr uint32_t OFF_Q = OFF_V + TILE;
  static constexpr uint32_t OFF_DO = OFF_Q + QS * TILE;
  static constexpr uint32_t OFF_DS = OFF_DO + GS * TILE;       // dS^T: 128 keys x 128 queries bf16
  static constexpr uint32_t OFF_STG = OFF_DS + 2 * SPAN;       // dQ staging: 8 KB per dQ warp
  static constexpr uint32_t OFF_LSE = OFF_STG + 8 * 4096;      // float [QS][BT]: -LSE * log2(e)
  static constexpr uint32_t OFF_DLT = OFF_LSE + QS * BT * 4;   // float [QS][BT]: -D_i
  static constexpr uint32_t OFF_BAR = OFF_DLT + QS * BT * 4;
  // kv_full, q_full[QS], q_empty[QS], do_full[GS], do_empty[GS], s_full,
  // dp_full, p_ready, ds_ready, dq_full, dq_free, dkv_done
  static constexpr int NBAR = 1 + 2 * QS + 2 * GS + 7;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  // No alignment slack: the dynamic shared memory must start on a 1024-byte
  // boundary (128-byte swizzle atoms); the kernel checks and reports.
  static constexpr uint32_t SMEM = OFF_MISC + 16;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(TM_DQ + D <= TMEM_COLS, "TMEM budget");
};

template <int D>
struct Bars {
  using C = Cfg<D>;
  uint32_t b;
  __device__ uint32_t kv_full() const { return b; }
  __device__ uint32_t q_full(int s) const { return b + 8u * (1 + s); }
  __device__ uint32_t q_empty(int s) const { return b + 8u * (1 + C::QS + s); }
  __device__ uint32_t do_full(int s) const { return b + 8u * (1 + 2 * C::QS + s); }
  __device__ uint32_t do_empty(int s) const { return b + 8u * (1 + 2 * C::QS + C::GS + s); }
  __device__ uint32_t s_full() const { return b + 8u * (1 + 2 * C::QS + 2 * C::GS); }
  __device__ uint32_t dp_full() const { return b + 8u * (2 + 2 * C::QS + 2 * C::GS); }
  __device__ uint32_t p_ready() const { return b + 8u * (3 + 2 * C::QS + 2 * C::GS); }
  __device__ uint32_t ds_ready() const { return b + 8u * (4 + 2 * C::QS + 2 * C::GS); }
  __device__ uint32_t dq_full() const { return b + 8u * (5 + 2 * C::QS + 2 * C::GS); }
  __device__ uint32_t dq_free() const { return b + 8u * (6 + 2 * C::QS + 2 * C::GS); }
  __device__ uint32_t dkv_done() const { return b + 8u * (7 + 2 * C::QS + 2 * C::GS); }
};

// Event kinds of the debug build's stamps (one per step t unless noted):
// P_ producer, M_ MMA warp, S_ dS warps, Q_ dQ warps.
enum : int {
  T_P_Q = 0, T_P_DO = 1, T_M_PREADY = 2, T_M_SNEXT = 3 /* S_{t+1}, index t+1 */,
  T_M_DSREADY = 4, T_M_DQ = 5, T_M_DQFREE = 6, T_M_DP = 7 /* dP_{t+1}, index t+1 */,
  T_S_SFULL = 8, T_S_PREADY = 9, T_Q_DQFULL = 10, T_Q_DQFREE = 11, T_Q_STAGED = 12,
  T_S_DPFULL = 13, T_S_DSREADY = 14, T_M_DV = 15, T_S_SLD = 16 /* scores in registers */,
  T_S_EXPD = 17 /* exponentials done */, T_S_DPLD = 18 /* dP in registers */,
  T_S_DSC = 19 /* dS formed */, T_S_DSST = 20 /* dS stored to shared memory */
};

enum : unsigned {
  W_KV = 0x40100, W_QEMPTY = 0x40200, W_QFULL = 0x40300, W_SFULL = 0x40400, W_PREADY = 0x40500,
  W_DPFULL = 0x40600, W_DSREADY = 0x40700, W_DKV = 0x40800, W_DOFULL = 0x40900,
  W_DOEMPTY = 0x40A00, W_DQFULL = 0x40B00, W_DQFREE = 0x40C00, BAD_ALIGN = 0x40D00
};

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const DevErr& e,
                                          volatile int* abort, unsigned where) {
  const bool ok = mbar_wait(bar, parity, e, abort, where);
  return __all_sync(FULL, ok);
}

template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// One 128-row tile of a token-major tensor (its D / 64 column blocks).
template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                          int head, int row) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) tma_load_3d(dst + c * SPAN, map, bar, 64 * c, head, row);
}

// Packed-bf16 TMEM column of k-step kk (16 elements) when each 64-wide half
// of a 128-wide operand was written by its own thread into the first 32 of
// its 64 columns: halves start 64 columns apart.
__device__ __forceinline__ uint32_t packed_col(int kk) { return (kk >> 2) * 64 + (kk & 3) * 8; }

__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const uint32_t (&a)[32],
                                               float scale) {
#pragma unroll
  for (int v4 = 0; v4 < 4; ++v4) {
    uint4 w;
    w.x = pack_bf16x2(__uint_as_float(a[8 * v4 + 0]) * scale, __uint_as_float(a[8 * v4 + 1]) * scale);
    w.y = pack_bf16x2(__uint_as_float(a[8 * v4 + 2]) * scale, __uint_as_float(a[8 * v4 + 3]) * scale);
    w.z = pack_bf16x2(__uint_as_float(a[8 * v4 + 4]) * scale, __uint_as_float(a[8 * v4 + 5]) * scale);
    w.w = pack_bf16x2(__uint_as_float(a[8 * v4 + 6]) * scale, __uint_as_float(a[8 * v4 + 7]) * scale);
    reinterpret_cast<uint4*>(dst)[v4] = w;
  }
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// Global [y .. y + 31, x .. x + 31] (fp32) += the 32 x 32 box at ``src``
// (128-byte swizzled), by the tensor-memory accelerator; completion is
// tracked per issuing thread in bulk groups.
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, uint32_t src, int x,
                                                  int y) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];" ::
          "l"(reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(src)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// This thread's bulk groups have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// This thread's bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
    bwd_fused_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_dqa, const AttnParams p, int num_j,
                     int group) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if ((sbase & 1023u) != 0) {
    if (threadIdx.x == 0) {
      atomicOr(p.err.word, ERR_BOUNDS);
      atomicExch(p.err.word + 1, BAD_ALIGN);
    }
    return;
  }

  // Tile order: groups of key/value heads for L2 reuse of Q, dO and the dQ
  // accumulator; inside a group the causal CTAs with the most query tiles
  // (small key tile j) first.
  const TileSlot ts = grouped_slot(blockIdx.x, num_j, p.H_kv * p.B, group);
  const int j = ts.t;
  const int hk = ts.unit % p.H_kv;
  const int b = ts.unit / p.H_kv;
  const SeqInfo sq = seq_info(p, b);
  if (!seq_ok(p, sq) || j * BT >= sq.len) return;
  const int g = p.H / p.H_kv;
  const int n_q = (sq.len + BT - 1) / BT;
  const int i0 = p.causal ? j : 0;   // first query tile with a visible key
  const int n_qt = n_q - i0;         // query tiles per head
  const int n_steps = g * n_qt;

  const Bars<D> bars{sbase + C::OFF_BAR};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    *abort = 0;
    mbar_init(bars.kv_full(), 1);
    for (int s = 0; s < C::QS; ++s) {
      mbar_init(bars.q_full(s), 2);  // Q bytes + the staged LSE / D_i
      mbar_init(bars.q_empty(s), 1);
    }
    for (int s = 0; s < C::GS; ++s) {
      mbar_init(bars.do_full(s), 1);
      mbar_init(bars.do_empty(s), 1);
    }
    mbar_init(bars.s_full(), 1);
    mbar_init(bars.dp_full(), 1);
    mbar_init(bars.p_ready(), N_DS);
    mbar_init(bars.ds_ready(), N_DS);
    mbar_init(bars.dq_full(), 1);
    mbar_init(bars.dq_free(), N_DQ);
    mbar_init(bars.dkv_done(), 1);
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

  // Each warpgroup sets its register count at the head of its own branch,
  // so the compiler fits each branch's code to it.
  if (warp / 4 == WARP_TMA / 4) {
  regs_dec<REG_CTRL>();
  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ producer ---
    float* s_lse = reinterpret_cast<float*>(smem + C::OFF_LSE);
    float* s_dlt = reinterpret_cast<float*>(smem + C::OFF_DLT);
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const int row_kv = sq.start + j * BT;
      mbar_arrive_expect_tx(bars.kv_full(), 2 * C::TILE);
      load_tile<D>(sbase + C::OFF_K, &tm_k, bars.kv_full(), hk, row_kv);
      load_tile<D>(sbase + C::OFF_V, &tm_v, bars.kv_full(), hk, row_kv);
    }
    // LSE and D_i of step t (four query rows per lane), fetched one step
    // ahead into registers so the global loads overlap the wait for a stage.
    float pl[BT / 32], pd[BT / 32];
    auto fetch = [&](int t) {
      const int h = hk * g + t / n_qt;
      const int qbase = (i0 + t % n_qt) * BT;
#pragma unroll
      for (int k = 0; k < BT / 32; ++k) {
        const int qpos = qbase + lane + 32 * k;
        const bool qv = qpos < sq.len;
        pl[k] = qv ? __ldg(p.lse + lse_index(p, b, h, sq.start, qpos)) : 0.f;
        pd[k] = qv ? __ldg(p.delta + static_cast<size_t>(h) * p.total + sq.start + qpos) : 0.f;
      }
    };
    if (n_steps > 0) fetch(0);
    for (int t = 0; t < n_steps; ++t) {
      const int st = t % C::QS;
      const int gt = t % C::GS;
      const int h = hk * g + t / n_qt;
      const int row_q = sq.start + (i0 + t % n_qt) * BT;
      if (!warp_wait(bars.q_empty(st), ((t / C::QS) & 1) ^ 1, p.err, abort, W_QEMPTY)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(bars.q_full(st), C::TILE);
        load_tile<D>(sbase + C::OFF_Q + st * C::TILE, &tm_q, bars.q_full(st), h, row_q);
        FA_STAMP(p, T_P_Q, t);
      }
#pragma unroll
      for (int k = 0; k < BT / 32; ++k) {
        // Negated, so the dS warps add them in packed fp32 pairs.
        s_lse[st * BT + lane + 32 * k] = -(pl[k] * LOG2E);
        s_dlt[st * BT + lane + 32 * k] = -pd[k];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.q_full(st));
      if (!warp_wait(bars.do_empty(gt), ((t / C::GS) & 1) ^ 1, p.err, abort, W_DOEMPTY)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(bars.do_full(gt), C::TILE);
        load_tile<D>(sbase + C::OFF_DO + gt * C::TILE, &tm_do, bars.do_full(gt), h, row_q);
        FA_STAMP(p, T_P_DO, t);
      }
      if (t + 1 < n_steps) fetch(t + 1);
    }
    // Drain: the tensor core's last arrivals on the empty barriers land
    // before the CTA's shared memory is released.
    for (int t = max(0, n_steps - C::QS); t < n_steps && !*abort; ++t)
      if (!warp_wait(bars.q_empty(t % C::QS), (t / C::QS) & 1, p.err, abort, W_QEMPTY)) break;
    for (int t = max(0, n_steps - C::GS); t < n_steps && !*abort; ++t)
      if (!warp_wait(bars.do_empty(t % C::GS), (t / C::GS) & 1, p.err, abort, W_DOEMPTY)) break;
  } else if (warp == WARP_MMA) {
    // ---------------------------------------------------------- MMA issuer ---
    // The whole warp runs the loop (waits and operands stay warp-uniform);
    // one elected lane issues the tensor-core instructions and commits.
    const uint32_t leader = elect_one();
    constexpr uint32_t ID_SDP = idesc_bf16(BT, BT, false, false);  // S^T, dP^T
    constexpr uint32_t ID_KV = idesc_bf16(BT, D, false, true);     // dV, dK (A from TMEM)
    constexpr uint32_t ID_DQ = idesc_bf16(BT, D, true, true);      // dQ_t = dS K
    const uint64_t k_kmaj = sdesc_sw128(sbase + C::OFF_K, 16, 1024);
    const uint64_t v_kmaj = sdesc_sw128(sbase + C::OFF_V, 16, 1024);
    const uint64_t q_kmaj = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);
    const uint64_t g_kmaj = sdesc_sw128(sbase + C::OFF_DO, 16, 1024);
    const uint64_t q_mn = sdesc_sw128(sbase + C::OFF_Q, SPAN, 1024);
    const uint64_t g_mn = sdesc_sw128(sbase + C::OFF_DO, SPAN, 1024);
    const uint64_t k_mn = sdesc_sw128(sbase + C::OFF_K, SPAN, 1024);
    // dS as the A operand of dQ_t: queries (M) run along the rows of the dS^T
    // tile, in two 64-query column blocks one span apart; keys (K) down them.
    const uint64_t ds_mn = sdesc_sw128(sbase + C::OFF_DS, SPAN, 1024);
    // dS^T as the A operand of dK: keys (M) down the rows, queries (K) along
    // them, K-major like the Q and K tiles.
    const uint64_t ds_kmaj = sdesc_sw128(sbase + C::OFF_DS, 16, 1024);
    auto issue_s = [&](int st) {     // S^T = K Q^T, K-dim = D
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t o = (kk >> 2) * SPAN + (kk & 3) * 32;
        mma_ss_if(leader, tmem + C::TM_S, sdesc_add(k_kmaj, o),
                  sdesc_add(q_kmaj, st * C::TILE + o), ID_SDP, kk > 0);
      }
      tc_commit_if(leader, bars.s_full());
    };
    auto issue_dp = [&](int gt) {    // dP^T = V dO^T, K-dim = D
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t o = (kk >> 2) * SPAN + (kk & 3) * 32;
        mma_ss_if(leader, tmem + C::TM_DP, sdesc_add(v_kmaj, o),
                  sdesc_add(g_kmaj, gt * C::TILE + o), ID_SDP, kk > 0);
      }
      tc_commit_if(leader, bars.dp_full());
    };
    bool ok = warp_wait(bars.kv_full(), 0, p.err, abort, W_KV);
    if (ok && n_steps > 0) {
      ok = warp_wait(bars.q_full(0), 0, p.err, abort, W_QFULL);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      ok = ok && warp_wait(bars.do_full(0), 0, p.err, abort, W_DOFULL);
      if (ok) {
        tc_fence_after();
        issue_dp(0);
      }
    }
    for (int t = 0; ok && t < n_steps; ++t) {
      const int st = t % C::QS;
      const int gt = t % C::GS;
      const bool more = t + 1 < n_steps;
      // dV += P^T_t dO_t (K-dim = 128 queries of the step).
      if (!(ok = warp_wait(bars.p_ready(), t & 1, p.err, abort, W_PREADY))) break;
      if (lane == 0) FA_STAMP(p, T_M_PREADY, t);
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BT / 16; ++kk)
        mma_ts_if(leader, tmem + C::TM_DV, tmem + C::TM_S + packed_col(kk),
                  sdesc_add(g_mn, gt * C::TILE + kk * 2048), ID_KV, (t > 0 || kk > 0) ? 1u : 0u);
      tc_commit_if(leader, bars.do_empty(gt));
      if (lane == 0) FA_STAMP(p, T_M_DV, t);
      // S^T_{t+1}: overwrites P^T_t, so it follows dV_t in the tensor pipe.
      if (more) {
        if (!(ok = warp_wait(bars.q_full((t + 1) % C::QS), ((t + 1) / C::QS) & 1, p.err, abort,
                             W_QFULL)))
          break;
        tc_fence_after();
        issue_s((t + 1) % C::QS);
        if (lane == 0) FA_STAMP(p, T_M_SNEXT, t + 1);
      }
      // dQ_t = dS_t K (K-dim = 128 keys), then dK += dS^T_t Q_t (K-dim = 128
      // queries). Both read dS from the shared dS^T tile (MN-major for dQ,
      // K-major for dK), so dQ_t - whose read-out gates dP_{t+1} - goes first.
      if (!(ok = warp_wait(bars.ds_ready(), t & 1, p.err, abort, W_DSREADY))) break;
      if (lane == 0) FA_STAMP(p, T_M_DSREADY, t);
      tc_fence_after();
      if (!C::ALIAS && t > 0) {
        // dQ_{t-1} must have been read out of its columns.
        if (!(ok = warp_wait(bars.dq_free(), (t - 1) & 1, p.err, abort, W_DQFREE))) break;
        tc_fence_after();
      }
#pragma unroll
      for (int kk = 0; kk < BT / 16; ++kk)   // K-dim = 128 keys in steps of 16
        mma_ss_if(leader, tmem + C::TM_DQ, sdesc_add(ds_mn, kk * 2048), sdesc_add(k_mn, kk * 2048),
                  ID_DQ, kk > 0);
      tc_commit_if(leader, bars.dq_full());
      if (lane == 0) FA_STAMP(p, T_M_DQ, t);
#pragma unroll
      for (int kk = 0; kk < BT / 16; ++kk) {
        const uint32_t o = (kk >> 2) * SPAN + (kk & 3) * 32;   // queries 16 kk .. 16 kk + 15
        mma_ss_if(leader, tmem + C::TM_DK, sdesc_add(ds_kmaj, o),
                  sdesc_add(q_mn, st * C::TILE + kk * 2048), ID_KV, (t > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit_if(leader, bars.q_empty(st));
      if (more) {
        if (C::ALIAS) {
          // dP_{t+1} overwrites dQ_t: wait until it has been read out.
          if (!(ok = warp_wait(bars.dq_free(), t & 1, p.err, abort, W_DQFREE))) break;
          if (lane == 0) FA_STAMP(p, T_M_DQFREE, t);
        }
        if (!(ok = warp_wait(bars.do_full((t + 1) % C::GS), ((t + 1) / C::GS) & 1, p.err, abort,
                             W_DOFULL)))
          break;
        tc_fence_after();
        issue_dp((t + 1) % C::GS);
        if (lane == 0) FA_STAMP(p, T_M_DP, t + 1);
      }
    }
    tc_commit_if(leader, bars.dkv_done());
  }   // warps 14 and 15: no role
  } else if (warp / 4 == WARP_DQ0 / 4) {
    regs_inc<REG_DQ>();
    // ------------------------------------------------------------ dQ warps ---
    // Thread = query row (warp & 3) * 32 + lane of the step's tile. The
    // whole row block of dQ_t (D / 32 boxes of 32 x 32 fp32) comes out of
    // TMEM at once and dq_free goes out; then, two boxes a round, the boxes
    // are staged 128-byte swizzled in this warp's 8 KB of the staging area
    // and one lane adds them into dQacc with TMA tensor reductions, which run
    // on their own.
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t stg = sbase + C::OFF_STG + (warp - WARP_DQ0) * 8192u;
    const bool stamp = warp == WARP_DQ0 && lane == 0;   // debug stamps
    for (int t = 0; t < n_steps; ++t) {
      if (!warp_wait(bars.dq_full(), t & 1, p.err, abort, W_DQFULL)) break;
      if (stamp) FA_STAMP(p, T_Q_DQFULL, t);
      tc_fence_after();
      uint32_t a[D / 32][32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(tmem + lane_off + C::TM_DQ + 32 * c, a[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) reg_fence(a[c]);
      tc_fence_before();
      mbar_arrive(bars.dq_free());
      if (stamp) FA_STAMP(p, T_Q_DQFREE, t);
      const int h = hk * g + t / n_qt;
      const int row0 = sq.start + (i0 + t % n_qt) * BT + (warp & 3) * 32;
      // Rows past the sequence's end hold exact zeros (their dS rows are
      // zero), so adding them to the next sequence's rows changes nothing;
      // rows past the tensor are clipped by the copy. A box wholly past the
      // sequence is not added at all.
      const bool add = row0 < sq.start + sq.len;
#pragma unroll
      for (int rd = 0; rd < D / 64; ++rd) {
        // The slots' previous boxes must have been read.
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int m = 0; m < 8; ++m)
            st_shared_v4(stg + c * 4096u + lane * 128 + ((m ^ (lane & 7)) << 4),
                         a[2 * rd + c][4 * m], a[2 * rd + c][4 * m + 1], a[2 * rd + c][4 * m + 2],
                         a[2 * rd + c][4 * m + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && add &&
            FA_CHECK(p, row0 >= 0 && row0 < p.total && h < p.H, 0xDB0402u)) {
          tma_reduce_add_2d(&tm_dqa, stg, h * D + 64 * rd, row0);
          tma_reduce_add_2d(&tm_dqa, stg + 4096u, h * D + 64 * rd + 32, row0);
        }
        if (lane == 0) bulk_commit();
      }
      if (stamp) FA_STAMP(p, T_Q_STAGED, t);
    }
    // The reductions read this CTA's shared memory: all must be done before exit.
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else {
    regs_inc<REG_DS>();
    // ------------------------------------------------------------ dS warps ---
    // Key-side work: thread = key row r (TMEM lane); warps w and w+4 take the
    // query columns [64 hf, 64 hf + 64) of the step.
    const int r = threadIdx.x & (BT - 1);
    const int hf = threadIdx.x >> 7;
    const int kpos = j * BT + r;
    const bool key_ok = kpos < sq.len;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float* s_lse = reinterpret_cast<const float*>(smem + C::OFF_LSE);
    const float* s_dlt = reinterpret_cast<const float*>(smem + C::OFF_DLT);
    const float c2 = p.scale_log2;
    // Visible queries of this key row: qpos in [qlo, qhi).
    const int qlo = p.causal ? kpos : 0;
    const int qhi = key_ok ? sq.len : 0;
    // This thread's 128-byte row block of the dS^T tile (keys = rows, 64
    // queries per 128-byte block, 16-byte chunks XOR-swizzled by row & 7).
    uint8_t* ds_row = smem + C::OFF_DS + hf * SPAN + r * 128;

    const bool stamp = threadIdx.x == 0;   // debug stamps: lane 0 of warp 0
    bool ok = true;
    for (int t = 0; t < n_steps && ok; ++t) {
      const int st = t % C::QS;
      const int qbase = (i0 + t % n_qt) * BT + 64 * hf;   // first query of this half
      const float* lse_t = s_lse + st * BT + 64 * hf;
      const float* dlt_t = s_dlt + st * BT + 64 * hf;
      if (!(ok = warp_wait(bars.q_full(st), (t / C::QS) & 1, p.err, abort, W_QFULL))) break;
      if (!(ok = warp_wait(bars.s_full(), t & 1, p.err, abort, W_SFULL))) break;
      if (stamp) FA_STAMP(p, T_S_SFULL, t);
      tc_fence_after();
      const bool full = qbase >= qlo && qbase + 64 <= qhi;
      uint32_t pk[32];   // P^T as packed bf16, the value dS is formed from
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t sr[32];
        tmem_ld32(tmem + lane_off + C::TM_S + 64 * hf + 32 * c, sr);
        tmem_ld_wait();
        reg_fence(sr);
        if (stamp && c == 0) FA_STAMP(p, T_S_SLD, t);
        // LSE read four at a time (one broadcast load per four columns).
        const float4* lse4 = reinterpret_cast<const float4*>(lse_t + 32 * c);
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
          const float4 l4 = lse4[q >> 2];
          const float la = (q & 2) ? l4.z : l4.x;
          const float lb = (q & 2) ? l4.w : l4.y;
          // An eighth of the exponentials (2 of every 16 queries) on the
          // FMA pipe: warps w and w + 4 share each sub-partition's
          // special-function unit (-1.5 to -4 % on the backward).
          // Pairs of scores on the packed fp32 FMA path (la, lb hold -LSE log2 e).
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[q]), __uint_as_float(sr[q + 1])),
                                      make_float2(c2, c2), make_float2(la, lb));
          const float x0 = x.x, x1 = x.y;
          const bool fma_pipe = (q % 16) == 0;
          float p0 = fma_pipe ? ex2_fma(x0) : ex2_approx(x0);
          float p1 = fma_pipe ? ex2_fma(x1) : ex2_approx(x1);
          if (!full) {
            const int qp = qbase + 32 * c + q;
            p0 = (qp >= qlo && qp < qhi) ? p0 : 0.f;
            p1 = (qp + 1 >= qlo && qp + 1 < qhi) ? p1 : 0.f;
          }
          pk[16 * c + (q >> 1)] = pack_bf16x2(p0, p1);
        }
      }
      if (stamp) FA_STAMP(p, T_S_EXPD, t);
      // P^T over the first 32 of this half's own 64 S^T columns.
      tmem_st32(tmem + lane_off + C::TM_S + 64 * hf, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bars.p_ready());
      if (stamp) FA_STAMP(p, T_S_PREADY, t);


      if (!(ok = warp_wait(bars.dp_full(), t & 1, p.err, abort, W_DPFULL))) break;
      if (stamp) FA_STAMP(p, T_S_DPFULL, t);
      tc_fence_after();
      uint32_t dsk[32];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t dr[32];
        tmem_ld32(tmem + lane_off + C::TM_DP + 64 * hf + 32 * c, dr);
        tmem_ld_wait();
        reg_fence(dr);
        if (stamp && c == 0) FA_STAMP(p, T_S_DPLD, t);
        const float4* dlt4 = reinterpret_cast<const float4*>(dlt_t + 32 * c);
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
          const float4 d4 = dlt4[q >> 2];
          const float da = (q & 2) ? d4.z : d4.x;
          const float db = (q & 2) ? d4.w : d4.y;
          // bf16 -> fp32 is exact: the 16 bits become the high half.
          const uint32_t w = pk[16 * c + (q >> 1)];
          const float p0 = __uint_as_float(w << 16);
          const float p1 = __uint_as_float(w & 0xffff0000u);
          // dS = P (dP - D) on packed pairs (da, db hold -D).
          const float2 v = __fmul2_rn(
              make_float2(p0, p1),
              __fadd2_rn(make_float2(__uint_as_float(dr[q]), __uint_as_float(dr[q + 1])),
                         make_float2(da, db)));
          dsk[16 * c + (q >> 1)] = pack_bf16x2(v.x, v.y);
        }
      }
      // dS^T into the shared dS^T tile: the A operand of dQ (read MN-major)
      // and of dK (read K-major). dP_t completing means dQ_{t-1} and dK_{t-1}
      // (issued before it) have read the tile.
      if (stamp) FA_STAMP(p, T_S_DSC, t);
#pragma unroll
      for (int m = 0; m < 8; ++m)
        *reinterpret_cast<uint4*>(ds_row + ((m ^ (r & 7)) << 4)) =
            make_uint4(dsk[4 * m + 0], dsk[4 * m + 1], dsk[4 * m + 2], dsk[4 * m + 3]);
      if (stamp) FA_STAMP(p, T_S_DSST, t);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bars.ds_ready());
      if (stamp) FA_STAMP(p, T_S_DSREADY, t);
    }
    // --------------------------------------------------- dK / dV epilogue ---
    if (ok && warp_wait(bars.dkv_done(), 0, p.err, abort, W_DKV)) {
      tc_fence_after();
      const size_t off = (static_cast<size_t>(sq.start + kpos) * p.H_kv + hk) * D;
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        const int c = (D / 64) * hf + cc;   // 32-column block of the head dim
        uint32_t a[32], v[32];
        tmem_ld32(tmem + lane_off + C::TM_DK + 32 * c, a);
        tmem_ld32(tmem + lane_off + C::TM_DV + 32 * c, v);
        tmem_ld_wait();
        reg_fence(a);
        reg_fence(v);
        if (key_ok && FA_CHECK(p, sq.start + kpos < p.total && hk < p.H_kv, 0xDB0401u)) {
          store_row_bf16(static_cast<__nv_bfloat16*>(p.dk) + off + 32 * c, a, p.scale);
          store_row_bf16(static_cast<__nv_bfloat16*>(p.dv) + off + 32 * c, v, 1.f);
        }
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

}  // namespace fused

// dQ = bf16(scale * dQacc), eight elements per thread.
__global__ void __launch_bounds__(256) dq_convert_kernel(const float* __restrict__ acc,
                                                         __nv_bfloat16* __restrict__ dq,
                                                         long long n8, float scale) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += stride) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 c = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    uint4 w;
    w.x = pack_bf16x2(a.x * scale, a.y * scale);
    w.y = pack_bf16x2(a.z * scale, a.w * scale);
    w.z = pack_bf16x2(c.x * scale, c.y * scale);
    w.w = pack_bf16x2(c.z * scale, c.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = w;
  }
}

template <int D>
cudaError_t launch_fused_d(const AttnParams& p, cudaStream_t stream) {
  using C = fused::Cfg<D>;
  const int num_t = (p.max_seqlen + fused::BT - 1) / fused::BT;
  const long long tiles = static_cast<long long>(num_t) * p.H_kv * p.B;
  if (tiles > INT_MAX) return cudaErrorInvalidConfiguration;
  if (tiles == 0) return cudaSuccess;
  CUtensorMap tq, tk, tv, tg;
  if (!make_tmap_bf16_3d(&tq, p.q, p.total, p.H, D, 1, fused::BT) ||
      !make_tmap_bf16_3d(&tk, p.k, p.total, p.H_kv, D, 1, fused::BT) ||
      !make_tmap_bf16_3d(&tv, p.v, p.total, p.H_kv, D, 1, fused::BT) ||
      !make_tmap_bf16_3d(&tg, p.dout, p.total, p.H, D, 1, fused::BT))
    return cudaErrorInvalidValue;
  CUtensorMap ta;
  if (!make_tmap_f32_2d(&ta, p.dq_accum, p.total, static_cast<unsigned long long>(p.H) * D, 32, 32))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(fused::bwd_fused_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  // A group's streams: Q and dO (bf16) plus the dQ accumulator (fp32) of its
  // g query heads.
  const int group = l2_group(8ll * p.max_seqlen * D * (p.H / p.H_kv), 1, p.H_kv * p.B);
  fused::bwd_fused_kernel<D><<<static_cast<unsigned>(tiles), fused::THREADS, C::SMEM, stream>>>(
      tq, tk, tv, tg, ta, p, num_t, group);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_fused(const AttnParams& p, cudaStream_t stream) {
  if (p.total == 0) return cudaSuccess;
  if (p.D == 64) return launch_fused_d<64>(p, stream);
  if (p.D == 128) return launch_fused_d<128>(p, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_dq_convert(const AttnParams& p, cudaStream_t stream) {
  const long long n8 = p.total * p.H * p.D / 8;
  if (n8 == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<long long>((n8 + 255) / 256, 148LL * 8));
  dq_convert_kernel<<<blocks, 256, 0, stream>>>(p.dq_accum, static_cast<__nv_bfloat16*>(p.dq),
                                                n8, p.scale);
  return cudaGetLastError();
}

}  // namespace fa
