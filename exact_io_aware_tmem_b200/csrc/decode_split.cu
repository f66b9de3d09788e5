// Split-KV decode over a contiguous or paged bf16 KV cache, on the sm_100a
// tensor cores: the form fa_decode takes when the caller fixes the number of
// key splits, or when the balanced kernel (decode_t.cu) does not take the
// shape (D = 64, or more than 64 query rows per kv head).
//
// What it computes: the q_len newest tokens of each sequence attend to its
// cached keys (agentalpha.top "flash attention" answer, follow-up 2: the key
// range is cut into splits, each split runs the online-softmax recurrence of
// aiqz.cc "Flash Attention V2/V3 optimization", section "V2 algorithm
// optimisation" (steps 1-5) over its key tiles j,
//     m_new = max(m, rowmax(S_j)),  alpha = e^(m - m_new),
//     l = l * alpha + rowsum(e^(S_j - m_new)),
//     O = O * alpha + e^(S_j - m_new) V_j,
// and the splits' (O / l, LSE) pairs are merged with the same update). S =
// scale * Q K^T, exponentials in base 2 on pre-scaled logits.
//
// How, on B200 (one CTA per (sequence, kv head, split); 352 threads at
// D = 128, 320 at D = 64). The CTA's 128 TMEM lanes hold the q_len x g query
// rows of one kv head (row r = token r / g of head hk * g + r % g):
//   warp 8      TMA producer (the whole warp runs its loop, lane 0 issues):
//               the Q block once, then K_j and V_j tiles through separate
//               multi-stage shared-memory rings (mbarrier full/empty pairs,
//               128-byte swizzle, no multicast), K loaded ahead of V whenever
//               both rings have room; one box per page of a paged cache;
//   warp 9      MMA warp, converged, one elect.sync lane issuing: S_j =
//               Q K_j^T with tcgen05.mma into TMEM score buffer j mod 2 (Q is
//               the A operand, held in TMEM) as soon as the softmax has
//               loaded S_{j-2};
//   warp 10     (D = 128) the same for O += P_j V_j, with P read straight
//               from its own TMEM columns as packed bf16. At D = 64 warp 9
//               issues these too, QK_{j+2} ahead of each PV_j;
//   warps 0-7   softmax, two groups of four warps; group g takes the key
//               tiles j = g, g+2, g+4, ... One thread per query row (TMEM
//               lane = row): it loads its 128 scores with tcgen05.ld,
//               releases the score buffer, masks, takes the row max,
//               exponentiates, sums, stores P to TMEM and rescales its O row
//               in TMEM when the reference max moved. Group 0 first copies Q
//               from the swizzled shared tile into TMEM. At the end both
//               groups merge their row sums and each writes half of O / l
//               (fp32 partials for the merge kernel when there are several
//               splits, else the final bf16 O and LSE).
// The two groups run the same recurrence with one shared reference max per
// row: the group on tile j takes the reference of tile j-1 from the other
// group (a shared-memory word per row, published by an mbarrier arrive as
// soon as that tile's row max is known, long before its exponentials are
// done), so the exponential work of neighbouring tiles overlaps instead of
// running back to back. Each group keeps its own partial row sum l_g, in the
// reference of its own last tile; O has a single accumulator whose reference
// is always the latest one, which is what lets P_j V_j add into it directly.
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D), Q [384, 384+D/2),
// P [448, 512).
#include <limits.h>
#include <math.h>

#include "params.h"

namespace fa {
namespace {

constexpr int BM = 128;  // query rows per CTA (= TMEM lanes)
constexpr int BN = 128;  // keys per tile
constexpr int WARP_TMA = 8;
constexpr int WARP_MMA = 9;   // MMA issuer (and the TMEM allocation)
constexpr int WARP_PV = 10;   // P V issuer when the MMAs are split over two warps
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S0 = 0;
constexpr uint32_t TM_O = 256;
constexpr uint32_t TM_Q = 384;  // Q tile as packed bf16 (D/2 columns), A operand of Q K^T
constexpr uint32_t TM_P = 448;  // P tile as packed bf16 (64 columns), A operand of P V
constexpr uint32_t CHUNK_BYTES = 128 * 128;  // 128 rows x 64 bf16 (one swizzle span)
// The reference max only moves when a row max exceeds it by more than this
// many powers of two; P entries are then at most 2^8 before the bf16 cast.
constexpr float RESCALE_LOG2 = 8.f;
constexpr unsigned FULL = 0xffffffffu;

// Codes recorded in the device error word when a wait gives up.
enum : unsigned {
  W_Q = 0x10100, W_KEMPTY = 0x10200, W_VEMPTY = 0x10300, W_KFULL = 0x10400,
  W_VFULL = 0x10500, W_PREADY = 0x10600, W_SFULL = 0x10700, W_PVDONE = 0x10800,
  W_QTMEM = 0x10900, W_SFREE = 0x10A00, W_MREF = 0x10B00, W_FIN = 0x10C00, W_VFIX = 0x10D00,
  W_VTAIL = 0x10E00, BAD_CACHE_LEN = 0x10F01, BAD_PAGE = 0x10F02
};

template <int D>
struct Cfg {
  static constexpr int STAGES = (D == 64) ? 4 : 3;
  // D = 128: one warp issues the score MMAs and another the P V MMAs, so a
  // score MMA never waits behind the P V product of the tile before it.
  // D = 64 (half the MMA work per exponential): one warp issues both in a
  // fixed interleave, measured faster there.
  static constexpr bool SPLIT_MMA = D == 128;
  static constexpr int THREADS = SPLIT_MMA ? 352 : 320;
  static constexpr int CHUNKS = D / 64;            // 128-byte blocks of a bf16 row
  static constexpr uint32_t TILE = BM * D * 2;     // bytes of one bf16 128-row tile
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + TILE;
  static constexpr uint32_t OFF_V = OFF_K + STAGES * TILE;
  // Per-row exchange words: reference max per group [2][128], then final
  // (m, l) per group [2][2][128], kept in the Q tile once Q is in TMEM.
  static constexpr uint32_t XCHG = 6 * BM * 4;
  static constexpr uint32_t OFF_X = OFF_Q;
  static constexpr uint32_t OFF_BAR = OFF_V + STAGES * TILE;
  // q, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[2], s_free[2],
  // mref[2], pv_done[2], p_ready, q_tmem, fin, v_fix
  static constexpr int NBAR = 1 + 4 * STAGES + 12;
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr uint32_t SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  static constexpr uint32_t OFF_MREF = OFF_X;
  static constexpr uint32_t OFF_FIN = OFF_X + 2 * BM * 4;
  static_assert(XCHG <= TILE, "exchange words fit in the Q tile");
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
  __device__ uint32_t s_free(int b) const { return base + 8u * (3 + 4 * stages + b); }
  __device__ uint32_t mref(int g) const { return base + 8u * (5 + 4 * stages + g); }
  __device__ uint32_t pv_done(int g) const { return base + 8u * (7 + 4 * stages + g); }
  __device__ uint32_t p_ready() const { return base + 8u * (9 + 4 * stages); }
  __device__ uint32_t q_tmem() const { return base + 8u * (10 + 4 * stages); }
  __device__ uint32_t fin() const { return base + 8u * (11 + 4 * stages); }
  __device__ uint32_t v_fix() const { return base + 8u * (12 + 4 * stages); }
};

__device__ __forceinline__ void record_bounds(const DevErr& e, unsigned where) {
  atomicOr(e.word, ERR_BOUNDS);
  atomicExch(e.word + 1, where);
}

// All 32 lanes wait; the warp proceeds only if every lane saw the phase.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const DevErr& e,
                                          volatile int* abort, unsigned where) {
  const bool ok = mbar_wait(bar, parity, e, abort, where);
  return __all_sync(FULL, ok);
}

// One CTA per (sequence, kv head, key split); its Q tile is the q_len newest
// tokens x the g query heads of the kv head (rows r = token * g + head), and
// it writes that split's partial O / l and LSE (or the final O and LSE when
// there is one split).
template <int D>
__global__ void __launch_bounds__(Cfg<D>::THREADS, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const AttnParams p,
                        const DecodeArgs dec) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);

  const int split = blockIdx.x % dec.n_split;
  const int rem = blockIdx.x / dec.n_split;
  const int hk = rem % p.H_kv;
  const int b = rem / p.H_kv;
  const int len = __ldg(dec.cache_seqlens + b);   // keys in the cache
  if (len < 0 || len > p.max_seqlen) {
    if (threadIdx.x == 0) record_bounds(p.err, BAD_CACHE_LEN);
    return;
  }
  const int j0 = split * dec.chunk;                          // first key tile of this CTA
  const int n_kv = min((len + BN - 1) / BN - j0, dec.chunk);  // key tiles of this CTA
  if (n_kv <= 0) {
    // No key in this split: LSE -inf and O 0, so the merge gives it no
    // weight (the whole output when the sequence is empty).
    const int r = threadIdx.x;
    if (r < dec.n_rows) {
      const int tok = b * dec.q_len + r / dec.g;
      const int hq = hk * dec.g + r % dec.g;
      const size_t row = static_cast<size_t>(tok) * p.H + hq;
      if (dec.n_split == 1) {
        p.lse[row] = -INFINITY;
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + row * D);
        for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
      } else {
        const size_t prow = static_cast<size_t>(split) * p.total * p.H + row;
        dec.lse_part[prow] = -INFINITY;
        float4* dst = reinterpret_cast<float4*>(dec.o_part + prow * D);
        for (int i = 0; i < D / 4; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    return;
  }
  // The split holding the sequence's last, partly filled key tile zeroes
  // that tile's V rows past the end (the cache may hold anything there, and
  // 0 * NaN in P V would not be 0) before PV reads it.
  const bool v_tail = j0 + n_kv == (len + BN - 1) / BN && (len % BN) != 0;

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
      mbar_init(bars.s_free(i), 128);
      mbar_init(bars.mref(i), 128);
      mbar_init(bars.pv_done(i), 1);
    }
    mbar_init(bars.p_ready(), 128);
    mbar_init(bars.q_tmem(), 128);
    mbar_init(bars.fin(), 256);
    mbar_init(bars.v_fix(), 1);
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
    // ------------------------------------------------------ TMA producer ---
    // The whole warp runs the producer loop; lane 0 issues the copies.
    //
    // Paged cache: the page ids a stream (K or V) needs are read 32 at a
    // time, one coalesced load per batch, lane L holding page base + L, with
    // the next batch already in flight; a tile's ids then come by shuffle.
    // Looking each id up on its own put an L2 round trip in front of every
    // TMA issue. -1: a page past the sequence's end (or past the table row).
    const int n_pages = (len + dec.page - 1) / max(dec.page, 1);
    auto page_id = [&](int pg) -> int {
      return (pg < n_pages && pg < dec.max_blocks)
                 ? __ldg(dec.block_table + static_cast<size_t>(b) * dec.max_blocks + pg)
                 : -1;
    };
    struct PageBatch {
      int base, cur, nxt;
    };
    auto batch_init = [&](PageBatch& pb, int first) {
      pb.base = first;
      pb.cur = page_id(first + lane);
      pb.nxt = page_id(first + 32 + lane);
    };
    // Page id of page pg0 + min(lane, n - 1): the n (<= 8) pages of one tile,
    // one per lane. pg0 is warp-uniform and never decreases. A tile's pages
    // never straddle two batches (pg0 is a multiple of n, and n divides 32),
    // so only the current batch is read; the next one is used only when the
    // batch advances, long after its load was issued.
    auto batch_get = [&](PageBatch& pb, int pg0, int n) -> int {
      while (pg0 >= pb.base + 32) {
        pb.base += 32;
        pb.cur = pb.nxt;
        pb.nxt = page_id(pb.base + 32 + lane);
      }
      const int off = pg0 + min(lane, n - 1) - pb.base;   // < 32
      return __shfl_sync(FULL, pb.cur, off & 31);
    };
    const bool paged = dec.block_table != nullptr;
    const int box = paged ? min(dec.page, BN) : BN;   // rows per TMA box
    // K / V tile jt (absolute key tile) into shared memory at ``dst``. The
    // caller has posted the tile's expected bytes on ``bar``.
    auto load_kv = [&](uint32_t dst, const CUtensorMap* map, uint32_t bar, int jt, PageBatch& pb) {
      if (!paged) {
        if (lane == 0) {
          const int row = b * dec.page + jt * BN;
#pragma unroll
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_2d(dst + c * CHUNK_BYTES, map, bar, hk * D + c * 64, row);
        }
      } else {
        // One box per page (or one 128-row box inside a larger page), lane u
        // issuing page u's box so small pages do not serialise on one
        // thread. Pages past the sequence's end load from beyond the cache:
        // zeros.
        const int n = BN / box;
        const int blk = batch_get(pb, jt * BN / dec.page, n);
        if (lane < n) {
          const int key = jt * BN + lane * box;
          int row = static_cast<int>(dec.cache_rows);
          if (key < len) {
            if (blk >= 0 && static_cast<long long>(blk + 1) * dec.page <= dec.cache_rows)
              row = blk * dec.page + key % dec.page;
            else
              record_bounds(p.err, BAD_PAGE);
          }
#pragma unroll
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_2d(dst + c * CHUNK_BYTES + lane * box * 128, map, bar, hk * D + c * 64, row);
        }
      }
    };
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      // q_len tokens x g heads: one (64, g, q_len) box per column block.
      mbar_arrive_expect_tx(bars.q(), dec.n_rows * 128 * C::CHUNKS);
#pragma unroll
      for (int c = 0; c < C::CHUNKS; ++c)
        tma_load_3d(sbase + C::OFF_Q + c * CHUNK_BYTES, &tm_q, bars.q(), c * 64, hk * dec.g,
                    b * dec.q_len);
    }
    // K and V run through separate rings and are loaded independently, K
    // first whenever both have a free slot: K_j is consumed early (QK_j runs
    // two tiles ahead of PV_j), and a K load that waited behind a V slot
    // would stall the score MMAs on the slowest event of the loop.
    PageBatch kpb{0, -1, -1}, vpb{0, -1, -1};
    if (paged) {
      batch_init(kpb, j0 * BN / dec.page);
      batch_init(vpb, j0 * BN / dec.page);
    }
    int jk = 0, jv = 0;
    long long t_last = clock64();
    while (jk < n_kv || jv < n_kv) {
      bool progress = false;
      if (jk < n_kv &&
          __all_sync(FULL, mbar_try_wait(bars.k_empty(jk % C::STAGES),
                                         ((jk / C::STAGES) & 1) ^ 1))) {
        const int st = jk % C::STAGES;
        if (lane == 0) mbar_arrive_expect_tx(bars.k_full(st), C::TILE);
        __syncwarp();
        load_kv(sbase + C::OFF_K + st * C::TILE, &tm_k, bars.k_full(st), j0 + jk, kpb);
        ++jk;
        progress = true;
      }
      if (jv < jk &&
          __all_sync(FULL, mbar_try_wait(bars.v_empty(jv % C::STAGES),
                                         ((jv / C::STAGES) & 1) ^ 1))) {
        const int st = jv % C::STAGES;
        if (lane == 0) mbar_arrive_expect_tx(bars.v_full(st), C::TILE);
        __syncwarp();
        load_kv(sbase + C::OFF_V + st * C::TILE, &tm_v, bars.v_full(st), j0 + jv, vpb);
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
    if (v_tail) {
      // Zero the rows past the sequence's end of the last V tile once it has
      // landed, then publish them to the tensor core (v_fix).
      const int t = n_kv - 1;
      const int st = t % C::STAGES;
      if (warp_wait(bars.v_full(st), (t / C::STAGES) & 1, p.err, abort, W_VTAIL)) {
        const int first = len - (j0 + t) * BN;   // rows [first, 128) are past the end
        uint8_t* tile = smem + C::OFF_V + st * C::TILE;
        for (int i = lane; i < (BN - first) * 8 * C::CHUNKS; i += 32) {
          const int c = i / ((BN - first) * 8);
          const int rr = first + (i / 8) % (BN - first);
          *reinterpret_cast<uint4*>(tile + c * CHUNK_BYTES + rr * 128 + (i % 8) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.v_fix());
      }
    }
    if (lane == 0) {
      // Drain: the tensor core's arrivals on the last stages' empty barriers
      // must land before the CTA's shared memory is released.
      for (int j = max(0, n_kv - C::STAGES); j < n_kv && !*abort; ++j) {
        const int st = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        if (!mbar_wait(bars.k_empty(st), ph, p.err, abort, W_KEMPTY)) break;
        if (!mbar_wait(bars.v_empty(st), ph, p.err, abort, W_VEMPTY)) break;
      }
    }
  } else if (warp == WARP_MMA || (C::SPLIT_MMA && warp == WARP_PV)) {
    // -------------------------------------------------------- MMA issuers ---
    // The whole warp runs the loop (waits and operands stay warp-uniform);
    // one elected lane issues the tensor-core instructions and commits. A
    // commit tracks the tcgen05 operations its own thread issued.
    //   S_j = Q K_j^T into score buffer j mod 2 (M=128, N=128, K=D in steps
    //   of 16) once K_j has landed and the buffer's group has loaded S_{j-2};
    //   O += P_j V_j (M=128, N=D, K=128 keys in steps of 16) once V_j has
    //   landed and P_j is in TMEM. One thread issues every P V product, so
    //   they run in key order on the single O accumulator.
    // Split (two warps): the score warp runs up to two tiles ahead on its
    // own. Single warp: QK_0 and QK_1 first, then QK_{j+2} ahead of each PV_j.
    const bool do_qk = warp == WARP_MMA;
    const bool do_pv = !C::SPLIT_MMA || warp == WARP_PV;
    const uint32_t leader = elect_one();
    constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, false, false);
    constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, false, true);
    const uint64_t k_desc = sdesc_sw128(sbase + C::OFF_K, 16, 1024);
    const uint64_t v_desc = sdesc_sw128(sbase + C::OFF_V, CHUNK_BYTES, 1024);
    // Q reaches TMEM through the softmax threads.
    bool ok = warp_wait(bars.q_tmem(), 0, p.err, abort, W_QTMEM);
    if (ok) tc_fence_after();
    int jq = do_qk ? 0 : n_kv;
    for (int j = -2; j < n_kv && ok; ++j) {
      const int jq_end = C::SPLIT_MMA ? n_kv : min(n_kv, j + 3);
      for (; jq < jq_end; ++jq) {
        const int st = jq % C::STAGES;
        if (!warp_wait(bars.k_full(st), (jq / C::STAGES) & 1, p.err, abort, W_KFULL) ||
            (jq >= 2 &&
             !warp_wait(bars.s_free(jq & 1), ((jq - 2) >> 1) & 1, p.err, abort, W_SFREE))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_s = tmem + TM_S0 + (jq & 1) * BN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * CHUNK_BYTES + (kk & 3) * 32;
          mma_ts_if(leader, d_s, tmem + TM_Q + kk * 8, sdesc_add(k_desc, st * C::TILE + off),
                    IDESC_QK, kk > 0);
        }
        tc_commit_if(leader, bars.s_full(jq & 1));
        tc_commit_if(leader, bars.k_empty(st));
      }
      if (!ok || !do_pv) break;
      if (j < 0) continue;
      const int st = j % C::STAGES;
      if (!warp_wait(bars.v_full(st), (j / C::STAGES) & 1, p.err, abort, W_VFULL)) break;
      if (v_tail && j == n_kv - 1 && !warp_wait(bars.v_fix(), 0, p.err, abort, W_VFIX)) break;
      if (!warp_wait(bars.p_ready(), j & 1, p.err, abort, W_PREADY)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        mma_ts_if(leader, tmem + TM_O, tmem + TM_P + kk * 8,
                  sdesc_add(v_desc, st * C::TILE + kk * 2048), IDESC_PV,
                  (j > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit_if(leader, bars.v_empty(st));
      tc_commit_if(leader, bars.pv_done(j & 1));
    }
  } else {
    // ---------------------------------------------------------- softmax ---
    const int g = warp >> 2;            // softmax group: key tiles g, g+2, ...
    const int quarter = warp & 3;       // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    // Row r is query token r / g (position len - q_len + r / g of the
    // sequence) of query head hk * g + r % g. lim: last visible key of this
    // row (-1: none); out_row: row index of O / LSE in units of heads.
    const bool row_ok = row < dec.n_rows;
    const int pos = len - dec.q_len + row / dec.g;
    const int lim = !row_ok ? -1 : (p.causal ? min(pos, len - 1) : len - 1);
    const size_t out_row =
        static_cast<size_t>(b * dec.q_len + row / dec.g) * p.H + hk * dec.g + row % dec.g;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float c2 = p.scale_log2;   // log2 units per raw score
    float* mref_s = reinterpret_cast<float*>(smem + C::OFF_MREF);
    float* fin_s = reinterpret_cast<float*>(smem + C::OFF_FIN);
    float m_g = -INFINITY;  // reference of this group's last tile (log2 units)
    float l_g = 0.f;        // this group's row sum, in that reference
    bool ok = true;
    if (g == 0) {
      // Copy this row of Q from the swizzled shared tile into TMEM as packed
      // bf16 (even element in the low half): the A operand of S = Q K^T.
      ok = warp_wait(bars.q(), 0, p.err, abort, W_Q);
      if (ok) {
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c) {
          const uint8_t* rowp = smem + C::OFF_Q + c * CHUNK_BYTES + row * 128;
          uint32_t w[32];
#pragma unroll
          for (int k16 = 0; k16 < 8; ++k16) {
            // Rows past the q_len x g block were never loaded: zeros.
            const uint4 v = !row_ok
                                ? make_uint4(0, 0, 0, 0)
                                : *reinterpret_cast<const uint4*>(rowp + ((k16 ^ (row & 7)) << 4));
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
    } else {
      // The Q tile's shared memory is reused for the exchange words below:
      // group 1 writes none before group 0 has finished copying Q out of it.
      ok = warp_wait(bars.q_tmem(), 0, p.err, abort, W_QTMEM);
    }
    // Warps whose 32 rows are all padding (q_len x g < 128) keep the
    // barrier protocol - the same waits and arrivals, in the same order, so
    // no barrier phase ever mixes two tiles - but load, exponentiate and
    // store nothing: their rows are never written out.
    const bool idle = __all_sync(FULL, !row_ok);
    for (int j = g; j < n_kv && ok; j += 2) {
      const uint32_t s_col = TM_S0 + g * BN;
      if (!warp_wait(bars.s_full(g), (j >> 1) & 1, p.err, abort, W_SFULL)) {
        ok = false;
        break;
      }
      if (idle) {
        mbar_arrive(bars.s_free(g));
        if (j > 0 && !warp_wait(bars.mref(g ^ 1), ((j - 1) >> 1) & 1, p.err, abort, W_MREF)) {
          ok = false;
          break;
        }
        mbar_arrive(bars.mref(g));
        if (j > 0 &&
            !warp_wait(bars.pv_done(g ^ 1), ((j - 1) >> 1) & 1, p.err, abort, W_PVDONE)) {
          ok = false;
          break;
        }
        mbar_arrive(bars.p_ready());
        continue;
      }
      tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + s_col + 32 * c, r[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(r[c]);
      // The scores are in registers: the tensor core may overwrite this buffer.
      tc_fence_before();
      mbar_arrive(bars.s_free(g));

      const int nvalid = lim - (j0 + j) * BN + 1;  // visible keys in this tile
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
      // Reference of tile j-1, published by the other group.
      float m_prev = -INFINITY;
      if (j > 0) {
        if (!warp_wait(bars.mref(g ^ 1), ((j - 1) >> 1) & 1, p.err, abort, W_MREF)) {
          ok = false;
          break;
        }
        m_prev = mref_s[(g ^ 1) * BM + row];
      }
      // The reference only moves when the row max exceeds it by more than
      // RESCALE_LOG2 (log2 units): P = 2^(s c - m_ref) then stays below
      // 2^RESCALE_LOG2, and O / l is the same for any consistent reference.
      const float m_cand = mx * c2;
      const bool grow = m_cand > m_prev + RESCALE_LOG2;   // always true on tile 0
      const float m_new = grow ? m_cand : m_prev;
      mref_s[g * BM + row] = m_new;
      mbar_arrive(bars.mref(g));
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[2][32];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float p0 = ex2_approx(fmaf(__uint_as_float(r[c][i]), c2, -m_use));
          const float p1 = ex2_approx(fmaf(__uint_as_float(r[c][i + 1]), c2, -m_use));
          sum4[(i >> 1) & 3] += p0 + p1;
          pk[c >> 1][(c & 1) * 16 + i / 2] = pack_bf16x2(p0, p1);
        }
      const float sum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      // This group's partial sum moves to the new reference.
      l_g = (m_g == m_new) ? l_g + sum : l_g * ex2_approx(m_g - m_use) + sum;
      m_g = m_new;
      if (j > 0) {
        // PV_{j-1} (the other group's tile; the tensor core runs PVs in
        // order) has finished reading P and adding into O once its pv_done
        // phase completes: P_j may then be stored and O moved to the new
        // reference before PV_j.
        if (!warp_wait(bars.pv_done(g ^ 1), ((j - 1) >> 1) & 1, p.err, abort, W_PVDONE)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      tmem_st32(tmem + lane_off + TM_P, pk[0]);
      tmem_st32(tmem + lane_off + TM_P + 32, pk[1]);
      if (j > 0 && __any_sync(FULL, grow)) {
        const float alpha = grow ? ex2_approx(m_prev - m_use) : 1.f;
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
    }
    // ----------------------------------------------------------- epilogue ---
    // Merge the two partial sums in the final reference (the larger of the
    // two groups' last references: references never decrease), then each
    // group writes half of the columns of O / l.
    if (ok) {
      fin_s[(2 * g) * BM + row] = m_g;
      fin_s[(2 * g + 1) * BM + row] = l_g;
      mbar_arrive(bars.fin());
      ok = warp_wait(bars.fin(), 0, p.err, abort, W_FIN);
    }
    const int last = n_kv - 1;
    if (ok && !idle &&
        warp_wait(bars.pv_done(last & 1), (last >> 1) & 1, p.err, abort, W_PVDONE)) {
      tc_fence_after();
      const float m_o = fin_s[(2 * (g ^ 1)) * BM + row];
      const float l_o = fin_s[(2 * (g ^ 1) + 1) * BM + row];
      const float m_fin = fmaxf(m_g, m_o);
      float l = 0.f;
      if (m_g != -INFINITY) l += (m_g == m_fin) ? l_g : l_g * ex2_approx(m_g - m_fin);
      if (m_o != -INFINITY) l += (m_o == m_fin) ? l_o : l_o * ex2_approx(m_o - m_fin);
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      const float lse = (l > 0.f) ? (m_fin + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      // Split partials (several splits) stay fp32 for the merge.
      const bool part = dec.n_split > 1;
      const size_t prow = static_cast<size_t>(split) * p.total * p.H + out_row;
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        const int c = g * (D / 64) + cc;   // this group's 32-column chunks
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + TM_O + 32 * c, o);
        tmem_ld_wait();
        reg_fence(o);
        if (row_ok && part) {
          float4* dst = reinterpret_cast<float4*>(dec.o_part + prow * D + 32 * c);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            dst[v4] = make_float4(__uint_as_float(o[4 * v4 + 0]) * inv_l,
                                  __uint_as_float(o[4 * v4 + 1]) * inv_l,
                                  __uint_as_float(o[4 * v4 + 2]) * inv_l,
                                  __uint_as_float(o[4 * v4 + 3]) * inv_l);
        } else if (row_ok) {
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
      if (row_ok && g == 0) {
        if (part)
          dec.lse_part[prow] = lse;
        else
          p.lse[out_row] = lse;
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

// Merge of the split partials of one output row per warp: LSE = ln sum_s
// exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s (agentalpha.top "flash attention"
// answer, follow-up 2: the splits are merged with the online-softmax update).
template <int D>
__global__ void __launch_bounds__(256)
    decode_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                          __nv_bfloat16* __restrict__ o, float* __restrict__ lse, long long rows,
                          int n_split) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  float m = -INFINITY;
  for (int s = lane; s < n_split; s += 32) m = fmaxf(m, lse_part[s * rows + row]);
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, d));
  constexpr int PER = D / 32;   // columns per lane
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float tot = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < n_split; ++s) {
      const float ls = lse_part[s * rows + row];
      if (ls == -INFINITY) continue;
      const float w = expf(ls - m);
      tot += w;
      const float* src = o_part + (s * rows + row) * D + lane * PER;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] += w * src[i];
    }
  }
  const float inv = (tot > 0.f) ? 1.f / tot : 0.f;
  __nv_bfloat16* dst = o + row * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; i += 2)
    *reinterpret_cast<uint32_t*>(dst + i) = pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
  if (lane == 0) lse[row] = (tot > 0.f) ? m + logf(tot) : -INFINITY;
}

template <int D>
cudaError_t launch_decode_d(const AttnParams& p, const DecodeArgs& d, cudaStream_t stream) {
  using C = Cfg<D>;
  const long long ctas = static_cast<long long>(p.B) * p.H_kv * d.n_split;
  if (ctas == 0) return cudaSuccess;
  if (ctas > INT_MAX) return cudaErrorInvalidConfiguration;
  CUtensorMap tq, tk, tv;
  const unsigned box_rows = (d.block_table != nullptr) ? static_cast<unsigned>(min(d.page, BN)) : BN;
  if (!make_tmap_bf16_3d(&tq, p.q, p.total, p.H, D, static_cast<unsigned>(d.g),
                         static_cast<unsigned>(d.q_len)) ||
      !make_tmap_bf16_2d(&tk, p.k, d.cache_rows, static_cast<unsigned long long>(p.H_kv) * D, 64,
                         box_rows) ||
      !make_tmap_bf16_2d(&tv, p.v, d.cache_rows, static_cast<unsigned long long>(p.H_kv) * D, 64,
                         box_rows))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  decode_split_kernel<D><<<static_cast<unsigned>(ctas), C::THREADS, C::SMEM, stream>>>(
      tq, tk, tv, p, d);
  e = cudaGetLastError();
  if (e != cudaSuccess || d.n_split == 1) return e;
  const long long rows = p.total * p.H;
  decode_combine_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      d.o_part, d.lse_part, static_cast<__nv_bfloat16*>(p.o), p.lse, rows, d.n_split);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_bf16(const AttnParams& p, const DecodeArgs& d, cudaStream_t stream) {
  if (p.D == 64) return launch_decode_d<64>(p, d, stream);
  if (p.D == 128) return launch_decode_d<128>(p, d, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fa
