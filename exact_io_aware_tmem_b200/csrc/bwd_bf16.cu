// Attention backward, bf16 in / fp32 accumulate, on the sm_100a tensor cores.
//
// What it computes, for the loss sum(O * dO): the backward pass rebuilds the
// scores and probabilities from Q, K and the saved LSE instead of storing the
// N x N matrix (agentalpha.top "flash attention" answer, section 2; airsota.com
// card, section 4 item 2), then applies the gradient relations the "Flash
// Attention self-test" (book.bogosort.top, section D) asks for:
//     P = exp(scale Q K^T - LSE),   dV = P^T dO,   dP = dO V^T,
//     D_i = dO_i . O_i,   dS = P * (dP - D),   dQ = scale dS K,   dK = scale dS^T Q.
//
// Three kernels, in stream order:
//   bwd_preprocess   D_i = dO_i . O_i (fp32, [H, T]); HBM-bound.
//   bwd_dkdv         one CTA per (sequence, key/value head, 128-key tile); K
//                    and V stay in shared memory while the CTA walks the
//                    128-row query tiles of every query head of its group
//                    (GQA dK/dV accumulate in TMEM). Keys on the TMEM lanes:
//                      S^T  = K Q_i^T,   dP^T = V dO_i^T          (TMEM)
//                      P^T  = exp2(S^T c - LSE log2 e)  -> bf16 over S^T
//                      dS^T = P^T * (dP^T - D)          -> bf16 over dP^T
//                      dV  += P^T dO_i,  dK += dS^T Q_i (A operands from TMEM)
//   bwd_dq           one CTA per (sequence, query head, 128-row query tile);
//                    Q and dO stay in shared memory while K_j, V_j stream
//                    through their own rings. Queries on the TMEM lanes:
//                      S = Q K_j^T (one buffer, handed back as soon as its
//                      softmax group has loaded it), dP = dO V_j^T (one
//                      buffer per group)
//                      dS = P * (dP - D) -> bf16 over dP,  dQ += dS K_j
//                    then dQ = bf16(scale dQ), each row written once.
// Recomputing S and dP in bwd_dq costs two extra products per tile pair, and
// buys what the single fused kernel could not have at once on this part: only
// 128-wide tensor-core instructions (64-wide ones with both operands in shared
// memory are bound by shared-memory bandwidth), P and dS as TMEM operands (no
// dS round trip through shared memory), no atomic dQ accumulation and no fp32
// dQ workspace.
//
// Roles in both kernels (320 threads): warps 0-7 softmax / dS (thread = TMEM
// lane row; dK/dV: warps w and w+4 share a lane quarter and split the 128
// columns in halves; dQ: two groups of four warps on alternate key tiles),
// warp 8 TMA producer, warp 9 MMA warp (converged, one elect.sync lane
// issuing the tensor-core instructions).
// D = 64 runs the D = 128 code: the tensor maps are 3-D (D, heads, tokens), so
// the second 64-wide column block is out of bounds and arrives as zeros.
#include <limits.h>
#include <math.h>

#include <algorithm>

#include "params.h"

namespace fa {
namespace {

constexpr int BT = 128;      // rows per tile (keys in dkdv, queries in dq) = TMEM lanes
constexpr int DP = 128;      // padded head dim
constexpr int THREADS = 320;
constexpr int N_SOFTMAX = 256;
constexpr int WARP_TMA = 8;
constexpr int WARP_MMA = 9;
constexpr uint32_t TMEM_COLS = 512;
constexpr unsigned FULL = 0xffffffffu;
constexpr uint32_t CHUNK = BT * 128;       // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr uint32_t TILE = BT * DP * 2;     // 32 KB: one 128-row tile of Q, K, V or dO
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const DevErr& e,
                                          volatile int* abort, unsigned where) {
  const bool ok = mbar_wait(bar, parity, e, abort, where);
  return __all_sync(FULL, ok);
}

// One 128-row tile (both 64-column halves of the padded head dim).
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                          int head, int row) {
  tma_load_3d(dst, map, bar, 0, head, row);
  tma_load_3d(dst + CHUNK, map, bar, 64, head, row);
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

// ------------------------------------------------------------ preprocess ---

// One warp per (token, head) row: D_i = dO_i . O_i into delta [H, T], and,
// for the fused backward, the row's dQ accumulator set to zero.
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const AttnParams p) {
  const long long rows = p.total * p.H;
  const int lane = threadIdx.x % 32;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  for (long long r = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; r < rows; r += warps) {
    const long long tok = r / p.H;
    const int h = static_cast<int>(r % p.H);
    const size_t off = static_cast<size_t>(r) * p.D;
    const __nv_bfloat16* o = static_cast<const __nv_bfloat16*>(p.o) + off;
    const __nv_bfloat16* g = static_cast<const __nv_bfloat16*>(p.dout) + off;
    float acc = 0.f;
    for (int d = 2 * lane; d < p.D; d += 64) {
      const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o + d));
      const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(g + d));
      acc = fmaf(of.x, gf.x, acc);
      acc = fmaf(of.y, gf.y, acc);
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(FULL, acc, s);
    if (lane == 0) p.delta[static_cast<size_t>(h) * p.total + tok] = acc;
    if (p.dq_accum != nullptr)
      for (int d = 4 * lane; d < p.D; d += 128)
        *reinterpret_cast<float4*>(p.dq_accum + off + d) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ------------------------------------------------------------------ dK/dV ---

namespace dkdv {

constexpr int QS = 2;  // Q / dO stages
constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 384;
constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = OFF_K + TILE;
constexpr uint32_t OFF_Q = OFF_V + TILE;
constexpr uint32_t OFF_DO = OFF_Q + QS * TILE;
constexpr uint32_t OFF_LSE = OFF_DO + QS * TILE;   // float [QS][BT]: LSE * log2(e)
constexpr uint32_t OFF_DLT = OFF_LSE + QS * BT * 4;  // float [QS][BT]: D_i
constexpr uint32_t OFF_BAR = OFF_DLT + QS * BT * 4;
// kv_full, q_full[QS], q_empty[QS], s_full, dp_full, p_ready, ds_ready,
// dkv_done, do_full[QS]. A stage's Q (with its LSE and D_i) and its dO land
// on separate barriers, so S^T_t needs only Q_t.
constexpr int NBAR = 1 + 3 * QS + 5;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
static_assert(SMEM <= 232448, "shared memory budget");

enum : unsigned {
  W_KV = 0x20100, W_QEMPTY = 0x20200, W_QFULL = 0x20300, W_SFULL = 0x20400, W_PREADY = 0x20500,
  W_DPFULL = 0x20600, W_DSREADY = 0x20700, W_DKV = 0x20800, W_DOFULL = 0x20900
};

struct Bars {
  uint32_t b;
  __device__ uint32_t kv_full() const { return b; }
  __device__ uint32_t q_full(int s) const { return b + 8u * (1 + s); }
  __device__ uint32_t q_empty(int s) const { return b + 8u * (1 + QS + s); }
  __device__ uint32_t s_full() const { return b + 8u * (1 + 2 * QS); }
  __device__ uint32_t dp_full() const { return b + 8u * (2 + 2 * QS); }
  __device__ uint32_t p_ready() const { return b + 8u * (3 + 2 * QS); }
  __device__ uint32_t ds_ready() const { return b + 8u * (4 + 2 * QS); }
  __device__ uint32_t dkv_done() const { return b + 8u * (5 + 2 * QS); }
  __device__ uint32_t do_full(int s) const { return b + 8u * (6 + 2 * QS + s); }
};

__global__ void __launch_bounds__(THREADS, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do, const AttnParams p, int num_j,
                    int group) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);

  // Tile order: groups of key/value heads for L2 reuse of Q / dO; inside a
  // group the causal CTAs with the most query tiles (small key tile j) first.
  const TileSlot ts = grouped_slot(blockIdx.x, num_j, p.H_kv * p.B, group);
  const int j = ts.t;
  const int rem = ts.unit;
  const int hk = rem % p.H_kv;
  const int b = rem / p.H_kv;
  const SeqInfo sq = seq_info(p, b);
  if (!seq_ok(p, sq) || j * BT >= sq.len) return;
  const int g = p.H / p.H_kv;
  const int n_q = (sq.len + BT - 1) / BT;
  const int i0 = p.causal ? j : 0;   // first query tile with a visible key
  const int n_qt = n_q - i0;         // query tiles per head
  const int n_steps = g * n_qt;

  const Bars bars{sbase + OFF_BAR};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    *abort = 0;
    mbar_init(bars.kv_full(), 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(bars.q_full(s), 2);  // Q bytes + staged LSE / D_i
      mbar_init(bars.q_empty(s), 1);
      mbar_init(bars.do_full(s), 1);  // dO bytes
    }
    mbar_init(bars.s_full(), 1);
    mbar_init(bars.dp_full(), 1);
    mbar_init(bars.p_ready(), N_SOFTMAX);
    mbar_init(bars.ds_ready(), N_SOFTMAX);
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

  if (warp == WARP_TMA) {
    // ---------------------------------------------------------- producer ---
    float* s_lse = reinterpret_cast<float*>(smem + OFF_LSE);
    float* s_dlt = reinterpret_cast<float*>(smem + OFF_DLT);
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const int row_kv = sq.start + j * BT;
      mbar_arrive_expect_tx(bars.kv_full(), 2 * TILE);
      load_tile(sbase + OFF_K, &tm_k, bars.kv_full(), hk, row_kv);
      load_tile(sbase + OFF_V, &tm_v, bars.kv_full(), hk, row_kv);
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
      const int st = t % QS;
      const int h = hk * g + t / n_qt;
      const int qbase = (i0 + t % n_qt) * BT;
      if (!warp_wait(bars.q_empty(st), ((t / QS) & 1) ^ 1, p.err, abort, W_QEMPTY)) break;
      if (lane == 0) {
        const int row_q = sq.start + qbase;
        mbar_arrive_expect_tx(bars.q_full(st), TILE);
        load_tile(sbase + OFF_Q + st * TILE, &tm_q, bars.q_full(st), h, row_q);
        mbar_arrive_expect_tx(bars.do_full(st), TILE);
        load_tile(sbase + OFF_DO + st * TILE, &tm_do, bars.do_full(st), h, row_q);
      }
#pragma unroll
      for (int k = 0; k < BT / 32; ++k) {
        s_lse[st * BT + lane + 32 * k] = pl[k] * LOG2E;
        s_dlt[st * BT + lane + 32 * k] = pd[k];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.q_full(st));
      if (t + 1 < n_steps) fetch(t + 1);
    }
    // Drain: the tensor core's last arrivals on q_empty land before exit.
    for (int t = max(0, n_steps - QS); t < n_steps && !*abort; ++t)
      if (!warp_wait(bars.q_empty(t % QS), (t / QS) & 1, p.err, abort, W_QEMPTY)) break;
  } else if (warp == WARP_MMA) {
    {
      // -------------------------------------------------------- MMA issuer ---
      // The whole warp runs the loop (waits and operands stay warp-uniform);
      // one elected lane issues the tensor-core instructions and commits.
      const uint32_t leader = elect_one();
      constexpr uint32_t ID_SDP = idesc_bf16(BT, BT, false, false);  // S^T, dP^T
      constexpr uint32_t ID_DVK = idesc_bf16(BT, DP, false, true);   // dV, dK
      const uint64_t k_kmaj = sdesc_sw128(sbase + OFF_K, 16, 1024);
      const uint64_t v_kmaj = sdesc_sw128(sbase + OFF_V, 16, 1024);
      const uint64_t q_kmaj = sdesc_sw128(sbase + OFF_Q, 16, 1024);
      const uint64_t g_kmaj = sdesc_sw128(sbase + OFF_DO, 16, 1024);
      const uint64_t q_mn = sdesc_sw128(sbase + OFF_Q, CHUNK, 1024);
      const uint64_t g_mn = sdesc_sw128(sbase + OFF_DO, CHUNK, 1024);
      // S^T_t = K Q_t^T and dP^T_t = V dO_t^T for stage st.
      auto issue_s = [&](int st) {
#pragma unroll
        for (int kk = 0; kk < DP / 16; ++kk) {
          const uint32_t o = (kk >> 2) * CHUNK + (kk & 3) * 32;
          mma_ss_if(leader, tmem + TM_S, sdesc_add(k_kmaj, o), sdesc_add(q_kmaj, st * TILE + o),
                    ID_SDP, kk > 0);
        }
        tc_commit_if(leader, bars.s_full());
      };
      auto issue_dp = [&](int st) {
#pragma unroll
        for (int kk = 0; kk < DP / 16; ++kk) {
          const uint32_t o = (kk >> 2) * CHUNK + (kk & 3) * 32;
          mma_ss_if(leader, tmem + TM_DP, sdesc_add(v_kmaj, o), sdesc_add(g_kmaj, st * TILE + o),
                    ID_SDP, kk > 0);
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
      // Per step t: dV_t (after P_t), then S_{t+1} (it overwrites P_t, so it
      // follows dV_t in the tensor pipe), then dK_t (after dS_t) and dP_{t+1}
      // (it overwrites dS_t). The exp phase of step t+1 thus overlaps dK_t and
      // dP_{t+1}, and the dS phase of step t overlaps dV_t and S_{t+1}.
      for (int t = 0; ok && t < n_steps; ++t) {
        const int st = t % QS;
        if (!(ok = warp_wait(bars.p_ready(), t & 1, p.err, abort, W_PREADY))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk)
          mma_ts_if(leader, tmem + TM_DV, tmem + TM_S + packed_col(kk),
                 sdesc_add(g_mn, st * TILE + kk * 2048), ID_DVK, (t > 0 || kk > 0) ? 1u : 0u);
        const bool more = t + 1 < n_steps;
        const int sn = (t + 1) % QS;
        if (more) {
          if (!(ok = warp_wait(bars.q_full(sn), ((t + 1) / QS) & 1, p.err, abort, W_QFULL)))
            break;
          tc_fence_after();
          issue_s(sn);
        }
        if (!(ok = warp_wait(bars.ds_ready(), t & 1, p.err, abort, W_DSREADY))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk)
          mma_ts_if(leader, tmem + TM_DK, tmem + TM_DP + packed_col(kk),
                 sdesc_add(q_mn, st * TILE + kk * 2048), ID_DVK, (t > 0 || kk > 0) ? 1u : 0u);
        if (more) {
          if (!(ok = warp_wait(bars.do_full(sn), ((t + 1) / QS) & 1, p.err, abort, W_DOFULL)))
            break;
          tc_fence_after();
          issue_dp(sn);
        }
        tc_commit_if(leader, bars.q_empty(st));
      }
      tc_commit_if(leader, bars.dkv_done());
    }
  } else {
    // ------------------------------------------------- softmax / dS warps ---
    // Thread = key row r (TMEM lane); warps w and w+4 take query columns
    // [64 hf, 64 hf + 64) of the 128-wide step.
    const int r = threadIdx.x & (BT - 1);
    const int hf = threadIdx.x >> 7;
    const int kpos = j * BT + r;
    const bool key_ok = kpos < sq.len;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float* s_lse = reinterpret_cast<const float*>(smem + OFF_LSE);
    const float* s_dlt = reinterpret_cast<const float*>(smem + OFF_DLT);
    const float c2 = p.scale_log2;
    // Visible queries of this key row: qpos in [qlo, qhi).
    const int qlo = p.causal ? kpos : 0;
    const int qhi = key_ok ? sq.len : 0;
    bool ok = true;
    for (int t = 0; t < n_steps && ok; ++t) {
      const int st = t % QS;
      const int qbase = (i0 + t % n_qt) * BT + 64 * hf;   // first query of this half
      const float* lse_t = s_lse + st * BT + 64 * hf;
      const float* dlt_t = s_dlt + st * BT + 64 * hf;
      if (!(ok = warp_wait(bars.q_full(st), (t / QS) & 1, p.err, abort, W_QFULL))) break;
      if (!(ok = warp_wait(bars.s_full(), t & 1, p.err, abort, W_SFULL))) break;
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(tmem + lane_off + TM_S + 64 * hf, sr[0]);
      tmem_ld32(tmem + lane_off + TM_S + 64 * hf + 32, sr[1]);
      tmem_ld_wait();
      reg_fence(sr[0]);
      reg_fence(sr[1]);
      const bool full = qbase >= qlo && qbase + 64 <= qhi;
      float pr[64];
      uint32_t pk[32];
      // LSE and D_i are read four at a time (one broadcast load per four
      // columns): per-element loads would crowd the shared-memory pipe the
      // tensor core's operand reads and the mbarrier polls also use.
      const float4* lse4 = reinterpret_cast<const float4*>(lse_t);
#pragma unroll
      for (int q = 0; q < 64; q += 2) {
        const float4 l4 = lse4[q >> 2];
        const float la = (q & 2) ? l4.z : l4.x;
        const float lb = (q & 2) ? l4.w : l4.y;
        float p0 = ex2_approx(fmaf(__uint_as_float(sr[q >> 5][q & 31]), c2, -la));
        float p1 = ex2_approx(fmaf(__uint_as_float(sr[q >> 5][(q + 1) & 31]), c2, -lb));
        if (!full) {
          const int qp = qbase + q;
          p0 = (qp >= qlo && qp < qhi) ? p0 : 0.f;
          p1 = (qp + 1 >= qlo && qp + 1 < qhi) ? p1 : 0.f;
        }
        pr[q] = p0;
        pr[q + 1] = p1;
        pk[q >> 1] = pack_bf16x2(p0, p1);
      }
      // P^T over the first 32 of this half's own 64 S^T columns.
      tmem_st32(tmem + lane_off + TM_S + 64 * hf, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bars.p_ready());

      if (!(ok = warp_wait(bars.dp_full(), t & 1, p.err, abort, W_DPFULL))) break;
      tc_fence_after();
      uint32_t dr[2][32];
      tmem_ld32(tmem + lane_off + TM_DP + 64 * hf, dr[0]);
      tmem_ld32(tmem + lane_off + TM_DP + 64 * hf + 32, dr[1]);
      tmem_ld_wait();
      reg_fence(dr[0]);
      reg_fence(dr[1]);
      uint32_t dk[32];
      const float4* dlt4 = reinterpret_cast<const float4*>(dlt_t);
#pragma unroll
      for (int q = 0; q < 64; q += 2) {
        const float4 d4 = dlt4[q >> 2];
        const float da = (q & 2) ? d4.z : d4.x;
        const float db = (q & 2) ? d4.w : d4.y;
        const float d0 = pr[q] * (__uint_as_float(dr[q >> 5][q & 31]) - da);
        const float d1 = pr[q + 1] * (__uint_as_float(dr[q >> 5][(q + 1) & 31]) - db);
        dk[q >> 1] = pack_bf16x2(d0, d1);
      }
      // dS^T over the first 32 of this half's own 64 dP^T columns.
      tmem_st32(tmem + lane_off + TM_DP + 64 * hf, dk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bars.ds_ready());
    }
    // ---------------------------------------------------- dK / dV epilogue ---
    if (ok && warp_wait(bars.dkv_done(), 0, p.err, abort, W_DKV)) {
      tc_fence_after();
      const size_t off = (static_cast<size_t>(sq.start + kpos) * p.H_kv + hk) * p.D;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * hf + cc;   // 32-column block of the head dim
        uint32_t a[32], v[32];
        tmem_ld32(tmem + lane_off + TM_DK + 32 * c, a);
        tmem_ld32(tmem + lane_off + TM_DV + 32 * c, v);
        tmem_ld_wait();
        reg_fence(a);
        reg_fence(v);
        if (key_ok && 32 * c < p.D) {
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

}  // namespace dkdv

// --------------------------------------------------------------------- dQ ---

namespace dq {

constexpr int KS = 3;  // K stages (K_j is read until dQ_j, late in tile j)
constexpr int VS = 2;  // V stages (V_j is free once dP_j has been computed)
// TMEM: S [0,128) (one buffer, handed back as soon as its group has loaded
// it), dP / dS of group 0 [128,256) and group 1 [256,384), dQ [384,512).
constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DQ = 384;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_DO = OFF_Q + TILE;
constexpr uint32_t OFF_K = OFF_DO + TILE;
constexpr uint32_t OFF_V = OFF_K + KS * TILE;
constexpr uint32_t OFF_BAR = OFF_V + VS * TILE;
// q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[2],
// s_free, dp_full[2], ds_ready[2], dq_done. Tile j belongs to softmax group
// j & 1, and its S, dP and dS signals use that group's own barrier, so every
// waiter sees the phases of a barrier in order.
constexpr int NBAR = 1 + 2 * KS + 2 * VS + 8;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
// No alignment slack: the layout only fits if the dynamic shared memory
// starts on a 1024-byte boundary (the 128-byte swizzle atoms need it); the
// kernel checks this and reports instead of running misaligned.
constexpr uint32_t SMEM = OFF_MISC + 16;
static_assert(SMEM <= 232448, "shared memory budget");

enum : unsigned {
  W_Q = 0x30100, W_KEMPTY = 0x30200, W_KFULL = 0x30300, W_SFULL = 0x30400, W_DPFULL = 0x30500,
  W_DSREADY = 0x30600, W_DQ = 0x30700, W_SFREE = 0x30800, W_VEMPTY = 0x30900, W_VFULL = 0x30a00
};

struct Bars {
  uint32_t b;
  __device__ uint32_t q_full() const { return b; }
  __device__ uint32_t k_full(int s) const { return b + 8u * (1 + s); }
  __device__ uint32_t k_empty(int s) const { return b + 8u * (1 + KS + s); }
  __device__ uint32_t v_full(int s) const { return b + 8u * (1 + 2 * KS + s); }
  __device__ uint32_t v_empty(int s) const { return b + 8u * (1 + 2 * KS + VS + s); }
  __device__ uint32_t s_full(int i) const { return b + 8u * (1 + 2 * KS + 2 * VS + i); }
  __device__ uint32_t s_free() const { return b + 8u * (3 + 2 * KS + 2 * VS); }
  __device__ uint32_t dp_full(int i) const { return b + 8u * (4 + 2 * KS + 2 * VS + i); }
  __device__ uint32_t ds_ready(int i) const { return b + 8u * (6 + 2 * KS + 2 * VS + i); }
  __device__ uint32_t dq_done() const { return b + 8u * (8 + 2 * KS + 2 * VS); }
};

__global__ void __launch_bounds__(THREADS, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_do, const AttnParams p, int num_i,
                  int group) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if ((sbase & 1023u) != 0) {
    if (threadIdx.x == 0) {
      atomicOr(p.err.word, ERR_BOUNDS);
      atomicExch(p.err.word + 1, 0x30A11Bu);
    }
    return;
  }

  // Tile order: groups of query heads for L2 reuse of K / V; inside a group
  // the causal CTAs with the most key tiles (large query tile i) first.
  const TileSlot ts = grouped_slot(blockIdx.x, num_i, p.H * p.B, group);
  const int i = num_i - 1 - ts.t;
  const int rem = ts.unit;
  const int h = rem % p.H;
  const int b = rem / p.H;
  const SeqInfo sq = seq_info(p, b);
  if (!seq_ok(p, sq) || i * BT >= sq.len) return;
  const int hk = h / (p.H / p.H_kv);
  const int n_kv_all = (sq.len + BT - 1) / BT;
  const int n_kv = p.causal ? min(n_kv_all, i + 1) : n_kv_all;

  const Bars bars{sbase + OFF_BAR};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
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
    for (int k = 0; k < 2; ++k) {
      mbar_init(bars.s_full(k), 1);
      mbar_init(bars.dp_full(k), 1);
      mbar_init(bars.ds_ready(k), N_SOFTMAX / 2);  // one softmax group per tile
    }
    mbar_init(bars.s_free(), N_SOFTMAX / 2);
    mbar_init(bars.dq_done(), 1);
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
      // ---------------------------------------------------------- producer ---
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      const int row_q = sq.start + i * BT;
      mbar_arrive_expect_tx(bars.q_full(), 2 * TILE);
      load_tile(sbase + OFF_Q, &tm_q, bars.q_full(), h, row_q);
      load_tile(sbase + OFF_DO, &tm_do, bars.q_full(), h, row_q);
      // K and V run through rings of different depth and are loaded
      // independently (K first when both have a free slot), so a K load
      // never waits behind a V slot.
      int jk = 0, jv = 0;
      long long t_last = clock64();
      while (jk < n_kv || jv < n_kv) {
        bool progress = false;
        if (jk < n_kv && mbar_try_wait(bars.k_empty(jk % KS), ((jk / KS) & 1) ^ 1)) {
          mbar_arrive_expect_tx(bars.k_full(jk % KS), TILE);
          load_tile(sbase + OFF_K + (jk % KS) * TILE, &tm_k, bars.k_full(jk % KS), hk,
                    sq.start + jk * BT);
          ++jk;
          progress = true;
        }
        if (jv < n_kv && jv < jk && mbar_try_wait(bars.v_empty(jv % VS), ((jv / VS) & 1) ^ 1)) {
          mbar_arrive_expect_tx(bars.v_full(jv % VS), TILE);
          load_tile(sbase + OFF_V + (jv % VS) * TILE, &tm_v, bars.v_full(jv % VS), hk,
                    sq.start + jv * BT);
          ++jv;
          progress = true;
        }
        if (progress) {
          t_last = clock64();
        } else if (*abort) {
          break;
        } else if (clock64() - t_last > p.err.budget) {
          *abort = 1;
          atomicOr(p.err.word, ERR_TIMEOUT);
          atomicExch(p.err.word + 1, jk < n_kv ? W_KEMPTY : W_VEMPTY);
          break;
        }
      }
      // Drain: the tensor core's last arrivals on the empty barriers land
      // before exit.
      for (int jj = max(0, n_kv - KS); jj < n_kv && !*abort; ++jj)
        if (!mbar_wait(bars.k_empty(jj % KS), (jj / KS) & 1, p.err, abort, W_KEMPTY)) break;
      for (int jj = max(0, n_kv - VS); jj < n_kv && !*abort; ++jj)
        if (!mbar_wait(bars.v_empty(jj % VS), (jj / VS) & 1, p.err, abort, W_VEMPTY)) break;
    }
  } else if (warp == WARP_MMA) {
    {
      // -------------------------------------------------------- MMA issuer ---
      // The whole warp runs the loop (waits and operands stay warp-uniform);
      // one elected lane issues the tensor-core instructions and commits.
      const uint32_t leader = elect_one();
      constexpr uint32_t ID_SDP = idesc_bf16(BT, BT, false, false);  // S, dP
      constexpr uint32_t ID_DQ = idesc_bf16(BT, DP, false, true);    // dQ += dS K
      const uint64_t q_kmaj = sdesc_sw128(sbase + OFF_Q, 16, 1024);
      const uint64_t g_kmaj = sdesc_sw128(sbase + OFF_DO, 16, 1024);
      const uint64_t k_kmaj = sdesc_sw128(sbase + OFF_K, 16, 1024);
      const uint64_t v_kmaj = sdesc_sw128(sbase + OFF_V, 16, 1024);
      const uint64_t k_mn = sdesc_sw128(sbase + OFF_K, CHUNK, 1024);
      auto issue_s = [&](int jj) {   // S_jj = Q K_jj^T
        const int st = jj % KS;
#pragma unroll
        for (int kk = 0; kk < DP / 16; ++kk) {
          const uint32_t o = (kk >> 2) * CHUNK + (kk & 3) * 32;
          mma_ss_if(leader, tmem + TM_S, sdesc_add(q_kmaj, o), sdesc_add(k_kmaj, st * TILE + o), ID_SDP,
                 kk > 0);
        }
        tc_commit_if(leader, bars.s_full(jj & 1));
      };
      auto issue_dp = [&](int jj) {  // dP_jj = dO V_jj^T; V_jj is free afterwards
        const int st = jj % VS;
#pragma unroll
        for (int kk = 0; kk < DP / 16; ++kk) {
          const uint32_t o = (kk >> 2) * CHUNK + (kk & 3) * 32;
          mma_ss_if(leader, tmem + TM_DP + (jj & 1) * BT, sdesc_add(g_kmaj, o),
                 sdesc_add(v_kmaj, st * TILE + o), ID_SDP, kk > 0);
        }
        tc_commit_if(leader, bars.dp_full(jj & 1));
        tc_commit_if(leader, bars.v_empty(st));
      };
      bool ok = warp_wait(bars.q_full(), 0, p.err, abort, W_Q) &&
                warp_wait(bars.k_full(0), 0, p.err, abort, W_KFULL) &&
                warp_wait(bars.v_full(0), 0, p.err, abort, W_VFULL);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      // Per tile jj: S_{jj+1} and dP_{jj+1} as soon as the group of tile jj
      // has loaded S_jj (dP_{jj+1} goes to the other group's buffer, whose
      // previous dS was consumed by dQ_{jj-1}), then dQ += dS_jj K_jj once
      // dS_jj is in TMEM. The two groups' exp and dS phases then overlap each
      // other and the tensor core.
      for (int jj = 0; ok && jj < n_kv; ++jj) {
        const int st = jj % KS;
        if (jj + 1 < n_kv) {
          if (!(ok = warp_wait(bars.k_full((jj + 1) % KS), ((jj + 1) / KS) & 1, p.err, abort,
                               W_KFULL)))
            break;
          if (!(ok = warp_wait(bars.s_free(), jj & 1, p.err, abort, W_SFREE))) break;
          tc_fence_after();
          issue_s(jj + 1);
          if (!(ok = warp_wait(bars.v_full((jj + 1) % VS), ((jj + 1) / VS) & 1, p.err, abort,
                               W_VFULL)))
            break;
          tc_fence_after();
          issue_dp(jj + 1);
        }
        if (!(ok = warp_wait(bars.ds_ready(jj & 1), (jj >> 1) & 1, p.err, abort, W_DSREADY)))
          break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk)
          mma_ts_if(leader, tmem + TM_DQ, tmem + TM_DP + (jj & 1) * BT + kk * 8,
                 sdesc_add(k_mn, st * TILE + kk * 2048), ID_DQ, (jj > 0 || kk > 0) ? 1u : 0u);
        tc_commit_if(leader, bars.k_empty(st));
      }
      tc_commit_if(leader, bars.dq_done());
    }
  } else {
    // ------------------------------------------------- softmax / dS warps ---
    // Thread = query row r (TMEM lane). Warps 0-3 (group 0) take the even key
    // tiles and warps 4-7 (group 1) the odd ones, each thread a whole
    // 128-key row, so one group's exp phase overlaps the other's dS phase.
    const int r = threadIdx.x & (BT - 1);
    const int grp = threadIdx.x >> 7;
    const int qpos = i * BT + r;
    const bool row_ok = qpos < sq.len;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float c2 = p.scale_log2;
    const float lse2 = row_ok ? p.lse[lse_index(p, b, h, sq.start, qpos)] * LOG2E : 0.f;
    const float dlt = row_ok ? p.delta[static_cast<size_t>(h) * p.total + sq.start + qpos] : 0.f;
    // Visible keys of this query row: kpos <= lim (none when the row is past the end).
    const int lim = row_ok ? (p.causal ? qpos : sq.len - 1) : -1;
    bool ok = true;
    for (int jj = grp; jj < n_kv && ok; jj += 2) {
      const int kbase = jj * BT;
      if (!(ok = warp_wait(bars.s_full(grp), (jj >> 1) & 1, p.err, abort, W_SFULL))) break;
      tc_fence_after();
      const bool full = kbase + BT - 1 <= lim;
      uint32_t pk[64];   // P as packed bf16, the value dS is formed from
#pragma unroll
      for (int c = 0; c < 4; ++c) {   // four 32-key blocks
        uint32_t sr[32];
        tmem_ld32(tmem + lane_off + TM_S + 32 * c, sr);
        tmem_ld_wait();
        reg_fence(sr);
        if (c == 3) {
          tc_fence_before();
          mbar_arrive(bars.s_free());   // S may be overwritten by S_{jj+1} now
        }
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          const int kc = 32 * c + k;
          float p0 = ex2_approx(fmaf(__uint_as_float(sr[k]), c2, -lse2));
          float p1 = ex2_approx(fmaf(__uint_as_float(sr[k + 1]), c2, -lse2));
          if (!full) {
            p0 = (kbase + kc <= lim) ? p0 : 0.f;
            p1 = (kbase + kc + 1 <= lim) ? p1 : 0.f;
          }
          pk[kc / 2] = pack_bf16x2(p0, p1);
        }
      }
      const uint32_t dp_col = TM_DP + (jj & 1) * BT;
      if (!(ok = warp_wait(bars.dp_full(jj & 1), (jj >> 1) & 1, p.err, abort, W_DPFULL))) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t dr[32];
        tmem_ld32(tmem + lane_off + dp_col + 32 * c, dr);
        tmem_ld_wait();
        reg_fence(dr);
        uint32_t dk[16];
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          // bf16 -> fp32 is exact: the 16 bits become the high half.
          const uint32_t w = pk[16 * c + k / 2];
          const float p0 = __uint_as_float(w << 16);
          const float p1 = __uint_as_float(w & 0xffff0000u);
          dk[k / 2] = pack_bf16x2(p0 * (__uint_as_float(dr[k]) - dlt),
                                  p1 * (__uint_as_float(dr[k + 1]) - dlt));
        }
        // dS into columns [16 c, 16 c + 16) of this group's dP buffer, which
        // this thread has already read (columns [0, 32 c + 32)).
        tmem_st16(tmem + lane_off + dp_col + 16 * c, dk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bars.ds_ready(grp));
    }
    // ------------------------------------------------------------ epilogue ---
    if (ok && warp_wait(bars.dq_done(), 0, p.err, abort, W_DQ)) {
      tc_fence_after();
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.dq) +
                           (static_cast<size_t>(sq.start + qpos) * p.H + h) * p.D;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * grp + cc;
        uint32_t a[32];
        tmem_ld32(tmem + lane_off + TM_DQ + 32 * c, a);
        tmem_ld_wait();
        reg_fence(a);
        if (row_ok && 32 * c < p.D) store_row_bf16(dst + 32 * c, a, p.scale);
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

}  // namespace dq

}  // namespace

cudaError_t launch_bwd_bf16(const AttnParams& p, cudaStream_t stream, unsigned mask) {
  if (p.D != 64 && p.D != 128) return cudaErrorInvalidValue;
  if (p.total == 0) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  if (mask & 1u) {
    const long long rows = p.total * p.H;
    const int blocks = static_cast<int>(std::min<long long>((rows + 7) / 8, 148LL * 16));
    bwd_preprocess_kernel<<<blocks, 256, 0, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (!(mask & 6u)) return cudaSuccess;
  const int num_t = (p.max_seqlen + BT - 1) / BT;
  CUtensorMap tq, tk, tv, tg;
  if (!make_tmap_bf16_3d(&tq, p.q, p.total, p.H, p.D, 1, BT) ||
      !make_tmap_bf16_3d(&tk, p.k, p.total, p.H_kv, p.D, 1, BT) ||
      !make_tmap_bf16_3d(&tv, p.v, p.total, p.H_kv, p.D, 1, BT) ||
      !make_tmap_bf16_3d(&tg, p.dout, p.total, p.H, p.D, 1, BT))
    return cudaErrorInvalidValue;
  if (mask & 2u) {
    const long long tiles = static_cast<long long>(num_t) * p.H_kv * p.B;
    if (tiles > INT_MAX) return cudaErrorInvalidConfiguration;
    if (tiles > 0) {
      e = cudaFuncSetAttribute(dkdv::bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               dkdv::SMEM);
      if (e != cudaSuccess) return e;
      dkdv::bwd_dkdv_kernel<<<static_cast<unsigned>(tiles), THREADS, dkdv::SMEM, stream>>>(
          tq, tk, tv, tg, p, num_t,
          l2_group(4ll * p.max_seqlen * DP * (p.H / p.H_kv), 1, p.H_kv * p.B));
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  if (mask & 4u) {
    const long long tiles = static_cast<long long>(num_t) * p.H * p.B;
    if (tiles > INT_MAX) return cudaErrorInvalidConfiguration;
    if (tiles > 0) {
      e = cudaFuncSetAttribute(dq::bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               dq::SMEM);
      if (e != cudaSuccess) return e;
      dq::bwd_dq_kernel<<<static_cast<unsigned>(tiles), THREADS, dq::SMEM, stream>>>(
          tq, tk, tv, tg, p, num_t, l2_group(4ll * p.max_seqlen * DP, p.H / p.H_kv, p.H * p.B));
      e = cudaGetLastError();
    }
  }
  return e;
}

}  // namespace fa
