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
//   bwd_preprocess   D_i = dO_i . O_i (fp32, [H, T]) and zeroes the fp32 dQ
//                    accumulator [T, H, D]; HBM-bound.
//   bwd_main         one CTA per (sequence, key/value head, 128-key tile j);
//                    K_j and V_j stay in shared memory while the CTA walks
//                    every 64-row query tile i of every query head of the
//                    group (GQA dK/dV accumulate in TMEM, no extra reduction).
//                    Per step, in TMEM (keys on the 128 lanes):
//                      S^T  = K_j Q_i^T              (M=128 keys, N=64, K=D)
//                      P^T  = exp2(S^T c - LSE_i log2 e), masked, bf16 over S^T
//                      dV  += P^T dO_i               (A = P^T from TMEM)
//                      dP^T = V_j dO_i^T
//                      dS^T = P^T * (dP^T - D_i)  -> bf16 in shared memory
//                      dK  += dS^T Q_i
//                      dQ_i^T = K_j^T dS^T           (M=128 = D lanes, N=64)
//                    and the dQ^T tile is staged in shared memory and added
//                    into the fp32 accumulator with one TMA bulk reduce-add
//                    per step (the separate dQ-accumulation path); dK, dV
//                    are scaled and stored at the end.
//   bwd_dq_convert   dQ = bf16(scale * accumulator).
//
// Roles in bwd_main (448 threads): warps 0-7 softmax / dS and the dK/dV
// epilogue (thread = key row = TMEM lane, warps w and w+4 split the 64 query
// columns); warps 8-11 dQ drain (thread = head-dim row of dQ^T); warp 12 TMA
// producer; warp 13 MMA issuer.
// TMEM columns: dV [0,128) dK [128,256) S/P [256,320) dP [320,384)
//               dQ^T x2 [384,512).
// D = 64 runs the same kernel: the tensor maps are 3-D (D, heads, tokens), so
// the second 64-wide column block is out of bounds and arrives as zeros.
#include <limits.h>
#include <math.h>

#include <algorithm>

#include "params.h"

namespace fa {
namespace {

constexpr int BN = 128;  // keys per CTA (TMEM lanes)
constexpr int BM = 64;   // query rows per step
constexpr int DP = 128;  // padded head dim
constexpr int QS = 3;    // Q / dO pipeline stages
constexpr int THREADS = 448;
constexpr int WARP_DQ0 = 8;    // first of the four dQ drain warps
constexpr int WARP_TMA = 12;
constexpr int WARP_MMA = 13;
constexpr int N_SOFTMAX = 256; // threads in warps 0-7
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_DV = 0, TM_DK = 128, TM_S = 256, TM_DP = 320, TM_DQ = 384;
constexpr unsigned FULL = 0xffffffffu;

constexpr uint32_t KV_CHUNK = BN * 128;      // 128 rows x 64 bf16
constexpr uint32_t KV_TILE = BN * DP * 2;    // 32 KB
constexpr uint32_t Q_CHUNK = BM * 128;       // 64 rows x 64 bf16
constexpr uint32_t Q_TILE = BM * DP * 2;     // 16 KB
constexpr uint32_t DS_TILE = BN * BM * 2;    // 16 KB, 128 rows x 128 B
constexpr uint32_t DQ_STAGE = BM * DP * 4;   // 32 KB, fp32 [64 queries][D]

constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = OFF_K + KV_TILE;
constexpr uint32_t OFF_Q = OFF_V + KV_TILE;
constexpr uint32_t OFF_DO = OFF_Q + QS * Q_TILE;
constexpr uint32_t OFF_DS = OFF_DO + QS * Q_TILE;
constexpr uint32_t OFF_DQS = OFF_DS + 2 * DS_TILE;  // dQ tile staged for the bulk reduce
constexpr uint32_t OFF_LSE = OFF_DQS + DQ_STAGE;     // float [QS][BM]: LSE * log2(e)
constexpr uint32_t OFF_DLT = OFF_LSE + QS * BM * 4;  // float [QS][BM]: D_i
constexpr uint32_t OFF_BAR = OFF_DLT + QS * BM * 4;
// kv_full, q_full[QS], q_empty[QS], s_full, p_ready, dp_full, ds_ready,
// ds_empty[2], dq_full[2], dq_empty[2], dkv_done, dq_staged, dq_sfree
constexpr int NBAR = 1 + 2 * QS + 4 + 2 + 2 + 2 + 1 + 2;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
// No alignment slack: the layout only fits if the dynamic shared memory
// starts on a 1024-byte boundary (the 128-byte swizzle atoms need it). The
// kernel checks this at run time and reports instead of running misaligned.
constexpr uint32_t SMEM = OFF_MISC + 16;
static_assert(SMEM <= 232448, "shared memory budget");

enum : unsigned {
  W_KV = 0x20100, W_QEMPTY = 0x20200, W_QFULL = 0x20300, W_SFULL = 0x20400, W_PREADY = 0x20500,
  W_DPFULL = 0x20600, W_DSREADY = 0x20700, W_DSEMPTY = 0x20800, W_DQFULL = 0x20900,
  W_DQEMPTY = 0x20a00, W_DKV = 0x20b00, W_DQSTAGED = 0x20c00, W_DQSFREE = 0x20d00
};

struct Bars {
  uint32_t b;
  __device__ uint32_t kv_full() const { return b; }
  __device__ uint32_t q_full(int s) const { return b + 8u * (1 + s); }
  __device__ uint32_t q_empty(int s) const { return b + 8u * (1 + QS + s); }
  __device__ uint32_t s_full() const { return b + 8u * (1 + 2 * QS); }
  __device__ uint32_t p_ready() const { return b + 8u * (2 + 2 * QS); }
  __device__ uint32_t dp_full() const { return b + 8u * (3 + 2 * QS); }
  __device__ uint32_t ds_ready() const { return b + 8u * (4 + 2 * QS); }
  __device__ uint32_t ds_empty(int i) const { return b + 8u * (5 + 2 * QS + i); }
  __device__ uint32_t dq_full(int i) const { return b + 8u * (7 + 2 * QS + i); }
  __device__ uint32_t dq_empty(int i) const { return b + 8u * (9 + 2 * QS + i); }
  __device__ uint32_t dkv_done() const { return b + 8u * (11 + 2 * QS); }
  __device__ uint32_t dq_staged() const { return b + 8u * (12 + 2 * QS); }
  __device__ uint32_t dq_sfree() const { return b + 8u * (13 + 2 * QS); }
};

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const DevErr& e,
                                          volatile int* abort, unsigned where) {
  const bool ok = mbar_wait(bar, parity, e, abort, where);
  return __all_sync(FULL, ok);
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Element-wise add of a shared-memory tile into global memory by the TMA
// unit (no multicast), tracked as a bulk async-group of this thread.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, uint32_t src, int x,
                                                  int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group"
      " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(x), "r"(y), "r"(z)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until this thread's bulk groups have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Wait until this thread's bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ------------------------------------------------------------ preprocess ---

// One warp per (token, head) row: D_i = dO_i . O_i into delta [H, T], and the
// row of the fp32 dQ accumulator set to zero.
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
    float4* dq = reinterpret_cast<float4*>(p.dq_accum + off);
    for (int d4 = lane; d4 < p.D / 4; d4 += 32) dq[d4] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// dQ = bf16(scale * accumulator), 8 elements per thread per iteration.
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const AttnParams p) {
  const long long n8 = p.total * p.H * p.D / 8;
  const float4* src = reinterpret_cast<const float4*>(p.dq_accum);
  uint4* dst = static_cast<uint4*>(p.dq);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = src[2 * i];
    const float4 b = src[2 * i + 1];
    uint4 w;
    w.x = pack_bf16x2(a.x * p.scale, a.y * p.scale);
    w.y = pack_bf16x2(a.z * p.scale, a.w * p.scale);
    w.z = pack_bf16x2(b.x * p.scale, b.y * p.scale);
    w.w = pack_bf16x2(b.z * p.scale, b.w * p.scale);
    dst[i] = w;
  }
}

// ------------------------------------------------------------------ main ---

__global__ void __launch_bounds__(THREADS, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const AttnParams p, int num_j) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  if ((sbase & 1023u) != 0) {
    if (threadIdx.x == 0) {
      atomicOr(p.err.word, ERR_BOUNDS);
      atomicExch(p.err.word + 1, 0x20A11Bu);
    }
    return;
  }

  // Tile order: causal CTAs with the most query tiles (small j) first.
  const int HB = p.H_kv * p.B;
  const int j = static_cast<int>(blockIdx.x / HB);
  const int rem = static_cast<int>(blockIdx.x % HB);
  const int hk = rem % p.H_kv;
  const int b = rem / p.H_kv;
  (void)num_j;
  const SeqInfo sq = seq_info(p, b);
  if (!seq_ok(p, sq) || j * BN >= sq.len) return;
  const int g = p.H / p.H_kv;
  const int n_q = (sq.len + BM - 1) / BM;
  const int i0 = p.causal ? (j * BN) / BM : 0;
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
      mbar_init(bars.q_full(s), 2);  // TMA bytes + staged LSE / D_i
      mbar_init(bars.q_empty(s), 1);
    }
    mbar_init(bars.s_full(), 1);
    mbar_init(bars.p_ready(), N_SOFTMAX);
    mbar_init(bars.dp_full(), 1);
    mbar_init(bars.ds_ready(), N_SOFTMAX);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars.ds_empty(i), 1);
      mbar_init(bars.dq_full(i), 1);
      mbar_init(bars.dq_empty(i), 128);
    }
    mbar_init(bars.dkv_done(), 1);
    mbar_init(bars.dq_staged(), 128);
    mbar_init(bars.dq_sfree(), 1);
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
    // Lane 0 issues the TMA copies; all 32 lanes stage the step's LSE and D_i
    // values next to its Q / dO tiles, published by the same q_full barrier.
    float* s_lse = reinterpret_cast<float*>(smem + OFF_LSE);
    float* s_dlt = reinterpret_cast<float*>(smem + OFF_DLT);
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_dq);
      const int row_kv = sq.start + j * BN;
      mbar_arrive_expect_tx(bars.kv_full(), 2 * KV_TILE);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        tma_load_3d(sbase + OFF_K + c * KV_CHUNK, &tm_k, bars.kv_full(), c * 64, hk, row_kv);
        tma_load_3d(sbase + OFF_V + c * KV_CHUNK, &tm_v, bars.kv_full(), c * 64, hk, row_kv);
      }
    }
    for (int t = 0; t < n_steps; ++t) {
      const int st = t % QS;
      const int h = hk * g + t / n_qt;
      const int qbase = (i0 + t % n_qt) * BM;
      if (!warp_wait(bars.q_empty(st), ((t / QS) & 1) ^ 1, p.err, abort, W_QEMPTY)) break;
      if (lane == 0) {
        // Tiles first, so the copies overlap the LSE / D_i loads below.
        const int row_q = sq.start + qbase;
        mbar_arrive_expect_tx(bars.q_full(st), 2 * Q_TILE);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(sbase + OFF_Q + st * Q_TILE + c * Q_CHUNK, &tm_q, bars.q_full(st), c * 64, h,
                      row_q);
          tma_load_3d(sbase + OFF_DO + st * Q_TILE + c * Q_CHUNK, &tm_do, bars.q_full(st), c * 64,
                      h, row_q);
        }
      }
      for (int q = lane; q < BM; q += 32) {
        const int qpos = qbase + q;
        const bool qv = qpos < sq.len;
        s_lse[st * BM + q] =
            qv ? p.lse[lse_index(p, b, h, sq.start, qpos)] * 1.4426950408889634f : 0.f;
        s_dlt[st * BM + q] = qv ? p.delta[static_cast<size_t>(h) * p.total + sq.start + qpos] : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.q_full(st));
    }
    for (int t = max(0, n_steps - QS); t < n_steps && !*abort; ++t)
      if (!warp_wait(bars.q_empty(t % QS), (t / QS) & 1, p.err, abort, W_QEMPTY)) break;
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      // -------------------------------------------------------- MMA issuer ---
      constexpr uint32_t ID_SDP = idesc_bf16(BN, BM, false, false);   // S^T, dP^T
      constexpr uint32_t ID_DVK = idesc_bf16(BN, DP, false, true);    // dV, dK
      constexpr uint32_t ID_DQ = idesc_bf16(DP, BM, true, true);      // dQ^T
      // Shared-memory descriptors, built once and stepped by constant offsets.
      const uint64_t k_kmaj = sdesc_sw128(sbase + OFF_K, 16, 1024);         // K as A (S^T)
      const uint64_t v_kmaj = sdesc_sw128(sbase + OFF_V, 16, 1024);         // V as A (dP^T)
      const uint64_t k_mnmaj = sdesc_sw128(sbase + OFF_K, KV_CHUNK, 1024);  // K^T as A (dQ^T)
      const uint64_t q_kmaj = sdesc_sw128(sbase + OFF_Q, 16, 1024);         // Q as B (S^T)
      const uint64_t g_kmaj = sdesc_sw128(sbase + OFF_DO, 16, 1024);        // dO as B (dP^T)
      const uint64_t q_mnmaj = sdesc_sw128(sbase + OFF_Q, Q_CHUNK, 1024);   // Q as B (dK)
      const uint64_t g_mnmaj = sdesc_sw128(sbase + OFF_DO, Q_CHUNK, 1024);  // dO as B (dV)
      const uint64_t ds_kmaj = sdesc_sw128(sbase + OFF_DS, 16, 1024);       // dS^T as A (dK)
      const uint64_t ds_mnmaj = sdesc_sw128(sbase + OFF_DS, KV_CHUNK, 1024);  // dS^T as B (dQ^T)
      bool ok = mbar_wait(bars.kv_full(), 0, p.err, abort, W_KV);
      for (int t = 0; ok && t <= n_steps; ++t) {
        if (t < n_steps) {
          const int st = t % QS;
          if (!(ok = mbar_wait(bars.q_full(st), (t / QS) & 1, p.err, abort, W_QFULL))) break;
          tc_fence_after();
          // S^T = K Q^T
#pragma unroll
          for (int kk = 0; kk < DP / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * KV_CHUNK + (kk & 3) * 32;
            const uint32_t qo = (kk >> 2) * Q_CHUNK + (kk & 3) * 32;
            mma_ss(tmem + TM_S, sdesc_add(k_kmaj, ko), sdesc_add(q_kmaj, st * Q_TILE + qo), ID_SDP,
                   kk > 0);
          }
          tc_commit(bars.s_full());
          // dP^T = V dO^T, once the softmax warps are done with dP^T of t-1.
          if (t >= 1 && !(ok = mbar_wait(bars.ds_ready(), (t - 1) & 1, p.err, abort, W_DSREADY)))
            break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < DP / 16; ++kk) {
            const uint32_t vo = (kk >> 2) * KV_CHUNK + (kk & 3) * 32;
            const uint32_t go = (kk >> 2) * Q_CHUNK + (kk & 3) * 32;
            mma_ss(tmem + TM_DP, sdesc_add(v_kmaj, vo), sdesc_add(g_kmaj, st * Q_TILE + go), ID_SDP,
                   kk > 0);
          }
          tc_commit(bars.dp_full());
        }
        if (t >= 1) {
          const int u = t - 1;
          const int su = u % QS;
          const uint32_t ds_off = (u & 1) * DS_TILE;
          if (t == n_steps &&
              !(ok = mbar_wait(bars.ds_ready(), u & 1, p.err, abort, W_DSREADY)))
            break;
          tc_fence_after();
          // dK += dS^T Q   (A: dS^T K-major in smem; B: Q MN-major)
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            mma_ss(tmem + TM_DK, sdesc_add(ds_kmaj, ds_off + kk * 32),
                   sdesc_add(q_mnmaj, su * Q_TILE + kk * 2048), ID_DVK,
                   (u > 0 || kk > 0) ? 1u : 0u);
          // dQ^T = K^T dS^T  (A: K MN-major; B: dS^T MN-major), into dQ buffer u&1
          if (!(ok = mbar_wait(bars.dq_empty(u & 1), ((u >> 1) & 1) ^ 1, p.err, abort,
                               W_DQEMPTY)))
            break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_ss(tmem + TM_DQ + (u & 1) * BM, sdesc_add(k_mnmaj, kk * 2048),
                   sdesc_add(ds_mnmaj, ds_off + kk * 2048), ID_DQ, kk > 0);
          tc_commit(bars.dq_full(u & 1));
          tc_commit(bars.ds_empty(u & 1));
          tc_commit(bars.q_empty(su));
        }
        if (t < n_steps) {
          const int st = t % QS;
          if (!(ok = mbar_wait(bars.p_ready(), t & 1, p.err, abort, W_PREADY))) break;
          tc_fence_after();
          // dV += P^T dO  (A: P^T from TMEM, queries 0-31 in packed columns
          // 0-15 and 32-63 in columns 32-47; B: dO MN-major)
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            mma_ts(tmem + TM_DV, tmem + TM_S + kk * 8 + (kk >= 2 ? 16 : 0),
                   sdesc_add(g_mnmaj, st * Q_TILE + kk * 2048), ID_DVK,
                   (t > 0 || kk > 0) ? 1u : 0u);
        }
      }
      tc_commit(bars.dkv_done());
    }
  } else if (warp < WARP_DQ0) {
    // ------------------------------------------------- softmax / dS warps ---
    // Thread = key row r (TMEM lane); warps w and w+4 share a lane quarter and
    // take query columns [32 hf, 32 hf + 32) of the 64-wide step.
    const int r = threadIdx.x & (BN - 1);
    const int hf = threadIdx.x >> 7;
    const int kpos = j * BN + r;          // key position in the sequence
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
      const int qbase = (i0 + t % n_qt) * BM + 32 * hf;   // first query of this half
      const int st = t % QS;
      const float* lse_t = s_lse + st * BM + 32 * hf;
      const float* dlt_t = s_dlt + st * BM + 32 * hf;
      // The stage's LSE / D_i values (and Q, dO) have landed.
      if (!(ok = warp_wait(bars.q_full(st), (t / QS) & 1, p.err, abort, W_QFULL))) break;
      if (!(ok = warp_wait(bars.s_full(), t & 1, p.err, abort, W_SFULL))) break;
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(tmem + lane_off + TM_S + 32 * hf, sr);
      tmem_ld_wait();
      reg_fence(sr);
      // Whole half visible (no causal edge, no sequence end inside it)?
      const bool full = qbase >= qlo && qbase + 32 <= qhi;
      float pr[32];
      uint32_t pk[16];
#pragma unroll
      for (int q = 0; q < 32; q += 2) {
        float p0 = ex2_approx(fmaf(__uint_as_float(sr[q]), c2, -lse_t[q]));
        float p1 = ex2_approx(fmaf(__uint_as_float(sr[q + 1]), c2, -lse_t[q + 1]));
        if (!full) {
          const int qp = qbase + q;
          p0 = (qp >= qlo && qp < qhi) ? p0 : 0.f;
          p1 = (qp + 1 >= qlo && qp + 1 < qhi) ? p1 : 0.f;
        }
        pr[q] = p0;
        pr[q + 1] = p1;
        pk[q >> 1] = pack_bf16x2(p0, p1);
      }
      // P^T (bf16, 16 packed columns) over the first half of this half's own
      // S^T columns, which only this thread has read.
      tmem_st16(tmem + lane_off + TM_S + 32 * hf, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bars.p_ready());

      if (!(ok = warp_wait(bars.dp_full(), t & 1, p.err, abort, W_DPFULL))) break;
      tc_fence_after();
      uint32_t dr[32];
      tmem_ld32(tmem + lane_off + TM_DP + 32 * hf, dr);
      tmem_ld_wait();
      reg_fence(dr);
      // dS^T row half into the shared buffer t&1 once the MMAs of step t-2
      // are done with it.
      if (!(ok = warp_wait(bars.ds_empty(t & 1), ((t >> 1) & 1) ^ 1, p.err, abort, W_DSEMPTY)))
        break;
      uint8_t* ds_row = smem + OFF_DS + (t & 1) * DS_TILE + r * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {   // 16-byte chunk 4hf+c holds queries 8c..8c+7 of the half
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = 8 * c + 2 * e;
          const float d0 = pr[q] * (__uint_as_float(dr[q]) - dlt_t[q]);
          const float d1 = pr[q + 1] * (__uint_as_float(dr[q + 1]) - dlt_t[q + 1]);
          w[e] = pack_bf16x2(d0, d1);
        }
        const int chunk = 4 * hf + c;
        *reinterpret_cast<uint4*>(ds_row + ((chunk ^ (r & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bars.ds_ready());
    }
    // ---------------------------------------------------- dK / dV epilogue ---
    if (ok && warp_wait(bars.dkv_done(), 0, p.err, abort, W_DKV)) {
      tc_fence_after();
      const bool store = key_ok;
      const size_t off = (static_cast<size_t>(sq.start + kpos) * p.H_kv + hk) * p.D;
      __nv_bfloat16* dk = static_cast<__nv_bfloat16*>(p.dk) + off;
      __nv_bfloat16* dv = static_cast<__nv_bfloat16*>(p.dv) + off;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * hf + cc;   // 32-column block of the head dim
        uint32_t a[32], v[32];
        tmem_ld32(tmem + lane_off + TM_DK + 32 * c, a);
        tmem_ld32(tmem + lane_off + TM_DV + 32 * c, v);
        tmem_ld_wait();
        reg_fence(a);
        reg_fence(v);
        if (store && 32 * c < p.D) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 wk, wv;
            uint32_t* pk4 = &wk.x;
            uint32_t* pv4 = &wv.x;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 8 * v4 + 2 * e;
              pk4[e] = pack_bf16x2(__uint_as_float(a[i]) * p.scale,
                                   __uint_as_float(a[i + 1]) * p.scale);
              pv4[e] = pack_bf16x2(__uint_as_float(v[i]), __uint_as_float(v[i + 1]));
            }
            reinterpret_cast<uint4*>(dk + 32 * c)[v4] = wk;
            reinterpret_cast<uint4*>(dv + 32 * c)[v4] = wv;
          }
        }
      }
    }
  } else if (warp < WARP_TMA) {
    // ------------------------------------------------------ dQ drain warps ---
    // Thread = head-dim row d of dQ^T (TMEM lane). Each step's 64 x D tile is
    // written to shared memory as fp32 [query][d] and added into the global
    // accumulator by one TMA bulk reduce issued by thread d = 0.
    const int d = (warp - WARP_DQ0) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp - WARP_DQ0) * 32) << 16;
    float* stage = reinterpret_cast<float*>(smem + OFF_DQS);
    for (int u = 0; u < n_steps; ++u) {
      if (!warp_wait(bars.dq_full(u & 1), (u >> 1) & 1, p.err, abort, W_DQFULL)) break;
      tc_fence_after();
      uint32_t qr[2][32];
      tmem_ld32(tmem + lane_off + TM_DQ + (u & 1) * BM, qr[0]);
      tmem_ld32(tmem + lane_off + TM_DQ + (u & 1) * BM + 32, qr[1]);
      tmem_ld_wait();
      reg_fence(qr[0]);
      reg_fence(qr[1]);
      tc_fence_before();
      mbar_arrive(bars.dq_empty(u & 1));
      // The previous step's reduce has finished reading the staging tile.
      if (!warp_wait(bars.dq_sfree(), (u & 1) ^ 1, p.err, abort, W_DQSFREE)) break;
      if (d < p.D) {
#pragma unroll
        for (int q = 0; q < BM; ++q) stage[q * p.D + d] = __uint_as_float(qr[q >> 5][q & 31]);
      }
      fence_async_smem();
      mbar_arrive(bars.dq_staged());
      if (d == 0) {
        // Never leaves the loop on its own (its warp-mates would wait for it
        // in the next warp_wait); after a failed wait it only skips the add.
        if (mbar_wait(bars.dq_staged(), u & 1, p.err, abort, W_DQSTAGED)) {
          const int h = hk * g + u / n_qt;
          const int row_q = sq.start + (i0 + u % n_qt) * BM;
          // Rows past the sequence end hold zeros (their dS was masked to 0).
          tma_reduce_add_3d(&tm_dq, smem_u32(stage), 0, h, row_q);
          bulk_wait_read();
        }
        mbar_arrive(bars.dq_sfree());
      }
    }
    if (d == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_bwd_bf16(const AttnParams& p, cudaStream_t stream, unsigned mask) {
  if (p.D != 64 && p.D != 128) return cudaErrorInvalidValue;
  if (p.total == 0) return cudaSuccess;
  const long long rows = p.total * p.H;
  cudaError_t e = cudaSuccess;
  if (mask & 1u) {
    const int pre_blocks = static_cast<int>(std::min<long long>((rows + 7) / 8, 148LL * 16));
    bwd_preprocess_kernel<<<pre_blocks, 256, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (!(mask & 2u)) goto convert;
  {

  const int num_j = (p.max_seqlen + BN - 1) / BN;
  const long long tiles = static_cast<long long>(num_j) * p.H_kv * p.B;
  if (tiles > INT_MAX) return cudaErrorInvalidConfiguration;
  if (tiles > 0) {
    CUtensorMap tq, tk, tv, tg, tdq;
    if (!make_tmap_bf16_3d(&tq, p.q, p.total, p.H, p.D, BM) ||
        !make_tmap_bf16_3d(&tk, p.k, p.total, p.H_kv, p.D, BN) ||
        !make_tmap_bf16_3d(&tv, p.v, p.total, p.H_kv, p.D, BN) ||
        !make_tmap_bf16_3d(&tg, p.dout, p.total, p.H, p.D, BM) ||
        !make_tmap_f32_3d(&tdq, p.dq_accum, p.total, p.H, p.D, BM))
      return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(bwd_main_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    bwd_main_kernel<<<static_cast<unsigned>(tiles), THREADS, SMEM, stream>>>(tq, tk, tv, tg, tdq,
                                                                           p, num_j);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  }
convert:
  if (mask & 4u) {
    const long long n8 = rows * p.D / 8;
    const int cv_blocks = static_cast<int>(std::min<long long>((n8 + 255) / 256, 148LL * 16));
    bwd_dq_convert_kernel<<<cv_blocks, 256, 0, stream>>>(p);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace fa
