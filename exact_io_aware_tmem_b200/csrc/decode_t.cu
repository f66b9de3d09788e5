// Balanced split-KV decode at D = 128 for at most 64 query rows per kv head:
// one persistent CTA per SM, the keys on the TMEM lanes.
//
// What it computes is the decode of fa_decode (agentalpha.top "flash
// attention" answer, follow-up 2): the KV cache of each (sequence, kv head)
// is cut into pieces, each piece gives a partial O and LSE by the
// online-softmax recurrence of aiqz.cc "Flash Attention V2/V3 optimization",
// section "V2 algorithm optimisation", and the partials of a segment are
// merged with the same update. Two things differ from the one-CTA-per-split
// kernel in decode_split.cu.
//
// The cut. The units (sequence b, kv head, 128-key tile) are numbered in
// that order and cut into one contiguous range of equal size per SM, so
// every SM streams the same number of tiles whatever the mix of lengths. A
// CTA walks its range tile by tile; the pipeline does not drain at a piece
// boundary (the next piece's Q is loaded while the current one runs), so a
// CTA pays its start-up once. A segment that lies inside one range is
// written out directly; the others leave partials for the merge kernel.
//
// The transposed products. With R = q_len * g query rows (a few, for
// decode), a 128-row query tile would spend nearly all of its exponentials
// and TMEM reads on padding. Here
//     S^T  = K_j Q^T     (M = 128 keys, N = NQ >= R query columns, K = D)
//     O^T += V_j^T P^T   (M = D = 128, N = NQ, K = 128 keys)
// so thread t of the softmax warps owns key t of the tile (TMEM lane t) and
// takes R exponentials per tile. The reference max of a query row is shared
// by all 128 threads; it only moves (a reduction over the threads) on a
// piece's first tile and on tiles where some score exceeds it by more than
// 2^8, which keeps every P <= 2^8 before the bf16 cast. Row sums stay in
// each thread until the end of the piece.
//
// Roles (192 threads):
//   warps 0-3  softmax: thread t = key t of a tile; at the end of a piece,
//              row d = t of O^T (output column d of every query row).
//   warp 4     TMA producer: Q per piece (two buffers when they fit), K and
//              V through three-stage rings, paged or contiguous cache; it
//              zeroes the V rows past a sequence's end in its last tile.
//   warp 5     MMA warp: S^T_0, S^T_1, then per tile P_j V_j and S^T_{j+2},
//              across piece boundaries.
// TMEM: S^T buffers [0, NQ) and [NQ, 2 NQ), O^T [2 NQ, 3 NQ).
#include <limits.h>
#include <math.h>

#include "decode_t.h"

namespace fa {
namespace {
namespace dect {

constexpr int D = 128;
constexpr int BN = 128;                   // keys per tile
constexpr int CHUNKS = D / 64;            // 128-byte column blocks of a bf16 row
constexpr int STAGES = 3;
constexpr int SOFTMAX_THREADS = 256;
constexpr int THREADS = SOFTMAX_THREADS + 64;
constexpr int WARP_TMA = 8;
constexpr int WARP_MMA = 9;
constexpr uint32_t KV_SPAN = BN * 128;    // one column block of a K / V tile
constexpr uint32_t TILE = BN * D * 2;     // K / V tile
constexpr float RESCALE_LOG2 = 8.f;
constexpr unsigned FULL = 0xffffffffu;

// NQ: query columns of the products (R <= NQ).
template <int NQ>
struct Cfg {
  static_assert(NQ == 16 || NQ == 32 || NQ == 64, "query columns");
  static constexpr int QBUF = NQ <= 32 ? 2 : 1;     // Q buffers
  static constexpr int PBUF = NQ <= 32 ? 2 : 1;     // P buffers
  static constexpr uint32_t SPAN = NQ * 128;        // one column block of a Q or P tile
  static constexpr uint32_t QP_BYTES = CHUNKS * SPAN;
  static constexpr uint32_t OFF_K = 0;
  static constexpr uint32_t OFF_V = STAGES * TILE;
  static constexpr uint32_t OFF_Q = 2 * STAGES * TILE;
  static constexpr uint32_t OFF_P = OFF_Q + QBUF * QP_BYTES;  // P: NQ rows x 128 keys, K-major
  static constexpr uint32_t OFF_MREF = OFF_P + PBUF * QP_BYTES;  // float [NQ]: reference max
  static constexpr uint32_t OFF_ALPHA = OFF_MREF + NQ * 4;    // float [NQ]: its last move
  static constexpr uint32_t OFF_RED = OFF_ALPHA + NQ * 4;     // float [4][NQ]: per-warp max / sum
  static constexpr uint32_t OFF_ROWS = OFF_RED + 4 * NQ * 4;  // int [8][8]: paged rows per tile
  static constexpr uint32_t OFF_BAR = OFF_ROWS + 8 * 8 * 4;
  // k_full[S], k_empty[S], v_full[S], v_empty[S], q_full[QBUF], q_empty[QBUF],
  // s_full[2], s_free[2], p_ready[PBUF], pv_done[PBUF], v_land
  static constexpr int NBAR = 4 * STAGES + 2 * QBUF + 4 + 2 * PBUF + 1;
  // tmem slot, abort, first tile (b, hk, t), u0, u1
  static constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr uint32_t SMEM = OFF_MISC + 48 + 1024;   // + alignment slack
  static_assert(SMEM <= 232448, "shared memory budget");
  static constexpr uint32_t TMEM_COLS = NQ == 16 ? 64 : NQ == 32 ? 128 : 256;
  static constexpr uint32_t TM_S = 0;
  static constexpr uint32_t TM_O = 2 * NQ;
};

template <int NQ>
struct Bars {
  using C = Cfg<NQ>;
  uint32_t b;
  __device__ uint32_t k_full(int s) const { return b + 8u * s; }
  __device__ uint32_t k_empty(int s) const { return b + 8u * (STAGES + s); }
  __device__ uint32_t v_full(int s) const { return b + 8u * (2 * STAGES + s); }
  __device__ uint32_t v_empty(int s) const { return b + 8u * (3 * STAGES + s); }
  __device__ uint32_t q_full(int i) const { return b + 8u * (4 * STAGES + i); }
  __device__ uint32_t q_empty(int i) const { return b + 8u * (4 * STAGES + C::QBUF + i); }
  __device__ uint32_t s_full(int i) const { return b + 8u * (4 * STAGES + 2 * C::QBUF + i); }
  __device__ uint32_t s_free(int i) const { return b + 8u * (4 * STAGES + 2 * C::QBUF + 2 + i); }
  __device__ uint32_t p_ready(int i) const { return b + 8u * (4 * STAGES + 2 * C::QBUF + 4 + i); }
  __device__ uint32_t pv_done(int i) const {
    return b + 8u * (4 * STAGES + 2 * C::QBUF + 4 + C::PBUF + i);
  }
  __device__ uint32_t v_land() const {
    return b + 8u * (4 * STAGES + 2 * C::QBUF + 4 + 2 * C::PBUF);
  }
};

// Event kinds of the debug build's stamps (index: the CTA's tile counter),
// and of its per-CTA records (index: the CTA): the SM it ran on, and the
// global timer (ns) at its start and end.
enum : int {
  T_P_K = 0, T_P_V = 1, T_M_S = 2, T_M_PV = 3, T_W_SFULL = 4, T_W_ARR = 5, T_W_EPI = 6,
  T_CTA_SM = 29, T_CTA_START = 30, T_CTA_END = 31
};

// Debug builds only: every CTA (below 1024) records its SM and the global
// timer at its start and end into the trace buffer, whichever CTA is traced.
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
#endif
}

// Codes recorded in the device error word.
enum : unsigned {
  W_QFULL = 0x70100, W_QEMPTY = 0x70200, W_KEMPTY = 0x70300, W_VEMPTY = 0x70400,
  W_KFULL = 0x70500, W_VFULL = 0x70600, W_SFULL = 0x70700, W_SFREE = 0x70800,
  W_PREADY = 0x70900, W_PVDONE = 0x70A00, W_VLAND = 0x70B00, BAD_CACHE_LEN = 0x70F01,
  BAD_PAGE = 0x70F02, BAD_MERGE = 0x70F03
};

__device__ __forceinline__ void record(const DevErr& e, unsigned where) {
  atomicOr(e.word, ERR_BOUNDS);
  atomicExch(e.word + 1, where);
}

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

// The eight softmax warps (256 threads) meet at named barrier 1. The AND
// form also tells every thread whether all of them are still on track, so
// that a failed wait in one warp ends the loop of all eight at the same
// barrier; the OR form gathers a vote.
__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ bool softmax_sync_and(bool ok) {
  uint32_t all;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(all)
      : "r"(ok ? 1u : 0u)
      : "memory");
  return all != 0;
}

__device__ __forceinline__ bool softmax_sync_or(bool v) {
  uint32_t any;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(any)
      : "r"(v ? 1u : 0u)
      : "memory");
  return any != 0;
}

// 32 lanes x 16 consecutive 32-bit TMEM columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16p(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// N (8, 16, 32) consecutive columns of this thread's TMEM lane, valid on
// return.
template <int N>
__device__ __forceinline__ void tmem_row_ld(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 8) {
    tmem_ld8(taddr, r);
  } else {
#pragma unroll
    for (int c = 0; c < N / 16; ++c) tmem_ld16(taddr + 16 * c, r + 16 * c);
  }
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

template <int N>
__device__ __forceinline__ void tmem_row_st(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 8) {
    tmem_st8(taddr, r);
  } else {
#pragma unroll
    for (int c = 0; c < N / 16; ++c) tmem_st16p(taddr + 16 * c, r + 16 * c);
  }
  tmem_st_wait();
}

// Tiles of sequence b; a length outside [0, max_len] counts as no key (the
// start scan reports it). Host-callable, like Walk, so the walk can be
// checked on the CPU.
__host__ __device__ __forceinline__ int seq_tiles(const int* lens, int b, int max_len, int& len) {
#ifdef __CUDA_ARCH__
  const int l = __ldg(lens + b);
#else
  const int l = lens[b];
#endif
  len = (l >= 0 && l <= max_len) ? l : 0;
  return (len + BN - 1) / BN;
}

// Position of a role in the CTA's range of units: key tile t of kv head hk of
// sequence b, unit u. Every role walks the same sequence of tiles.
struct Walk {
  int b, t;
  int n, len;               // tiles and keys of sequence b
  long long u, u0, u1;      // current unit, the CTA's range [u0, u1)
  __host__ __device__ bool done() const { return u >= u1; }
  // First / last tile of its piece (the part of a segment inside the range).
  __host__ __device__ bool first() const { return t == 0 || u == u0; }
  __host__ __device__ bool last() const { return t + 1 == n || u + 1 == u1; }
  __host__ __device__ bool seg_end() const { return t + 1 == n; }
  __host__ __device__ void next(const int* lens, int B, int max_len) {
    ++u;
    ++t;
    if (u >= u1 || t < n) return;
    t = 0;
    do {
      if (++b >= B) {
        u = u1;
        return;
      }
      n = seq_tiles(lens, b, max_len, len);
    } while (n == 0);
  }
  // To the first tile of the next piece.
  __host__ __device__ void next_piece(const int* lens, int B, int max_len) {
    const long long step = (n - t < u1 - u) ? static_cast<long long>(n - t) : u1 - u;
    u += step - 1;
    t += static_cast<int>(step - 1);
    next(lens, B, max_len);
  }
};

template <int NQ>
__global__ void __launch_bounds__(THREADS, 1)
    decode_t_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p,
                    const DecodeArgs dec, const DecodeTArgs dt) {
  using C = Cfg<NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const Bars<NQ> bars{sbase + C::OFF_BAR};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* start = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
  long long* range = reinterpret_cast<long long*>(smem + C::OFF_MISC + 24);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int* lens = dec.cache_seqlens;
  const int R = dec.n_rows;

  if (threadIdx.x == 0) {
    cta_span(p, T_CTA_START);
    *abort = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bars.k_full(s), 1);
      mbar_init(bars.k_empty(s), 1);
      mbar_init(bars.v_full(s), 1);
      mbar_init(bars.v_empty(s), 1);
    }
    for (int i = 0; i < C::QBUF; ++i) {
      mbar_init(bars.q_full(i), 1);
      mbar_init(bars.q_empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars.s_full(i), 1);
      mbar_init(bars.s_free(i), SOFTMAX_THREADS);
    }
    for (int i = 0; i < C::PBUF; ++i) {
      mbar_init(bars.p_ready(i), SOFTMAX_THREADS);
      mbar_init(bars.pv_done(i), 1);
    }
    mbar_init(bars.v_land(), 1);
    fence_mbar_init();
  }
  // CTA c serves kv head c % H_kv over range c / H_kv of the groups.
  const int groups = dt.ctas / p.H_kv;
  const int grp = blockIdx.x / p.H_kv;
  const int hk = blockIdx.x % p.H_kv;
  if (warp == WARP_TMA) {
    // This CTA's range [u0, u1) of the U = sum_b n_b units, and the tile at
    // u0: a scan of the lengths, 32 sequences per step.
    long long tot = 0;
    for (int b0 = 0; b0 < p.B; b0 += 32) {
      const int b = b0 + lane;
      if (b < p.B) {
        int len;
        const int l = __ldg(lens + b);
        if (l < 0 || l > p.max_seqlen) record(p.err, BAD_CACHE_LEN);
        tot += seq_tiles(lens, b, p.max_seqlen, len);
      }
    }
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) tot += __shfl_xor_sync(FULL, tot, sh);
    const long long u0 = tot * grp / groups;
    const long long u1 = tot * (grp + 1) / groups;
    int sb = 0;
    long long base = 0;
    if (u0 < tot) {
      long long acc = 0;
      for (int b0 = 0; b0 < p.B; b0 += 32) {
        const int b = b0 + lane;
        int len = 0;
        const long long units = (b < p.B) ? seq_tiles(lens, b, p.max_seqlen, len) : 0;
        long long incl = units;
#pragma unroll
        for (int sh = 1; sh < 32; sh <<= 1) {
          const long long v = __shfl_up_sync(FULL, incl, sh);
          if (lane >= sh) incl += v;
        }
        incl += acc;
        const long long excl = incl - units;
        const unsigned hit = __ballot_sync(FULL, units > 0 && excl <= u0 && u0 < incl);
        if (hit != 0) {
          const int src = __ffs(hit) - 1;
          sb = b0 + src;
          base = __shfl_sync(FULL, excl, src);
          break;
        }
        acc = __shfl_sync(FULL, incl, 31);
      }
    }
    const long long off = u0 - base;   // < n_sb when u0 < tot
    if (lane == 0) {
      start[0] = sb;
      start[1] = static_cast<int>(u0 < tot ? off : 0);
      range[0] = u0;
      range[1] = u1;
    }
    if (u0 == u1 && u0 < tot && off != 0) {
      // An empty range strictly inside a segment (more groups than tiles):
      // the segment's pieces lie on both sides, so the merge reads this
      // CTA's slot too. It holds no key: LSE -inf.
      const size_t slot = static_cast<size_t>((sb + grp) * p.H_kv + hk) * R;
      for (int r = lane; r < R; r += 32) dt.lse_part[slot + r] = -INFINITY;
    }
  }
  if (warp == WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  // Q rows R .. NQ - 1 are never loaded: zero, so that the score columns of
  // the rows past R are exactly 0 and need no mask.
  for (int k = threadIdx.x; k < C::QBUF * CHUNKS * (NQ - R) * 8; k += THREADS) {
    const int unit = k % 8, row = R + (k / 8) % (NQ - R), blk = k / (8 * (NQ - R));
    *reinterpret_cast<uint4*>(smem + C::OFF_Q + blk * C::SPAN + row * 128 + unit * 16) =
        make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Walk w0;
  w0.b = start[0];
  w0.t = start[1];
  w0.u0 = range[0];
  w0.u1 = range[1];
  w0.u = w0.u0;
  w0.n = 0;
  w0.len = 0;
  if (w0.u0 < w0.u1) w0.n = seq_tiles(lens, w0.b, p.max_seqlen, w0.len);
  auto advance = [&](Walk& w) { w.next(lens, p.B, p.max_seqlen); };

  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ producer ---
    // The whole warp runs the loop; lane 0 issues Q and contiguous tiles,
    // lane u box u of a paged tile. Three independent streams: Q per piece
    // (once the buffer's last score MMA is done), K and V per tile; K leads.
    // Paged cache: the K stream reads the page ids of its sequence 32 at a
    // time (lane L holding page base + L, the next batch in flight), takes a
    // tile's ids by shuffle and leaves the tile's rows in a ring of 8 for the
    // V stream, which reads the same rows.
    const bool paged = dec.block_table != nullptr;
    const int box = paged ? min(dec.page, BN) : BN;   // rows per TMA box
    const int n_box = BN / box;                       // boxes (pages) per tile
    const int tpp = paged ? max(dec.page / BN, 1) : 1;   // tiles per page, pages >= 128 rows
    int* rows_s = reinterpret_cast<int*>(smem + C::OFF_ROWS);
    struct PageBatch {
      int base, cur, nxt;
    };
    auto page_id = [&](const Walk& w, int pg) -> int {
      const int n_pages = (w.len + dec.page - 1) / max(dec.page, 1);
      return (pg < n_pages && pg < dec.max_blocks)
                 ? __ldg(dec.block_table + static_cast<size_t>(w.b) * dec.max_blocks + pg)
                 : -1;
    };
    // Cache row of box `lane` (< n_box) of the K stream's tile: pages past the
    // sequence's end load from beyond the cache (zeros). A tile's n_box pages
    // start at a multiple of n_box, and n_box divides 32, so they lie in one
    // batch.
    PageBatch kpb{0, -1, -1};
    auto tile_row = [&](const Walk& w) -> int {
      const int pg0 = (box < BN) ? w.t * n_box : w.t / tpp;
      if (w.first()) {
        kpb.base = pg0;
        kpb.cur = page_id(w, pg0 + lane);
        kpb.nxt = page_id(w, pg0 + 32 + lane);
      }
      while (pg0 >= kpb.base + 32) {
        kpb.base += 32;
        kpb.cur = kpb.nxt;
        kpb.nxt = page_id(w, kpb.base + 32 + lane);
      }
      const int blk = __shfl_sync(FULL, kpb.cur, (pg0 + min(lane, n_box - 1) - kpb.base) & 31);
      int row = static_cast<int>(dec.cache_rows);
      if (lane < n_box && w.t * BN + lane * box < w.len) {
        if (blk >= 0 && static_cast<long long>(blk + 1) * dec.page <= dec.cache_rows)
          row = blk * dec.page + (box < BN ? 0 : (w.t - pg0 * tpp) * BN);
        else
          record(p.err, BAD_PAGE);
      }
      return row;
    };
    // Tile w of K (j: the K stream's tile count) or V (its rows from the ring).
    auto load_kv = [&](uint32_t dst, const CUtensorMap* map, uint32_t bar, const Walk& w, int j,
                       bool is_k) {
      if (!paged) {
        if (lane == 0) {
          const int row = w.b * dec.page + w.t * BN;
#pragma unroll
          for (int c = 0; c < CHUNKS; ++c)
            tma_load_2d(dst + c * KV_SPAN, map, bar, hk * D + c * 64, row);
        }
      } else {
        int row;
        if (is_k) {
          row = tile_row(w);
          if (lane < 8) rows_s[(j & 7) * 8 + lane] = row;
        } else {
          row = (lane < 8) ? rows_s[(j & 7) * 8 + lane] : 0;
        }
        if (lane < n_box) {
#pragma unroll
          for (int c = 0; c < CHUNKS; ++c)
            tma_load_2d(dst + c * KV_SPAN + lane * box * 128, map, bar, hk * D + c * 64, row);
        }
      }
    };
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    Walk kw = w0, vw = w0, qw = w0;
    int jk = 0, jv = 0, pq = 0, nland = 0;
    bool ok = true;
    long long t_last = clock64();
    while (!kw.done() || !vw.done() || !qw.done()) {
      bool progress = false;
      if (!qw.done()) {
        const int qb = pq % C::QBUF;
        if (pq < C::QBUF || warp_test(bars.q_empty(qb), ((pq / C::QBUF) - 1) & 1)) {
          // The q_len tokens x g heads of this piece's sequence and kv head:
          // one (64, g, q_len) box per column block, rows token * g + head.
          if (lane == 0) {
            mbar_arrive_expect_tx(bars.q_full(qb), R * 128 * CHUNKS);
#pragma unroll
            for (int c = 0; c < CHUNKS; ++c)
              tma_load_3d(sbase + C::OFF_Q + qb * C::QP_BYTES + c * C::SPAN, &tm_q,
                          bars.q_full(qb), c * 64, hk * dec.g, qw.b * dec.q_len);
          }
          ++pq;
          qw.next_piece(lens, p.B, p.max_seqlen);
          progress = true;
        }
      }
      // (K stays fewer than 8 tiles ahead of V: the rows ring.)
      if (!kw.done() && jk - jv < 8 &&
          warp_test(bars.k_empty(jk % STAGES), ((jk / STAGES) & 1) ^ 1)) {
        const int st = jk % STAGES;
        if (lane == 0) mbar_arrive_expect_tx(bars.k_full(st), TILE);
        __syncwarp();
        load_kv(sbase + C::OFF_K + st * TILE, &tm_k, bars.k_full(st), kw, jk, true);
        if (lane == 0) FA_STAMP(p, T_P_K, jk);
        ++jk;
        advance(kw);
        progress = true;
      }
      if (!vw.done() && jv < jk &&
          warp_test(bars.v_empty(jv % STAGES), ((jv / STAGES) & 1) ^ 1)) {
        const int st = jv % STAGES;
        const uint32_t dst = sbase + C::OFF_V + st * TILE;
        if (!(vw.seg_end() && (vw.len % BN) != 0)) {
          if (lane == 0) mbar_arrive_expect_tx(bars.v_full(st), TILE);
          __syncwarp();
          load_kv(dst, &tm_v, bars.v_full(st), vw, jv, false);
        } else {
          // A sequence's last, partly filled tile: its rows past the end may
          // hold anything (0 * NaN in P V would not be 0). It lands on
          // v_land; the rows are zeroed here and published on v_full.
          if (lane == 0) mbar_arrive_expect_tx(bars.v_land(), TILE);
          __syncwarp();
          load_kv(dst, &tm_v, bars.v_land(), vw, jv, false);
          if (!warp_wait(bars.v_land(), nland & 1, p.err, abort, W_VLAND)) {
            ok = false;
            break;
          }
          ++nland;
          const int first = vw.len - vw.t * BN;   // rows [first, 128) are past the end
          uint8_t* tile = smem + C::OFF_V + st * TILE;
          for (int i = lane; i < (BN - first) * 8 * CHUNKS; i += 32) {
            const int c = i / ((BN - first) * 8);
            const int rr = first + (i / 8) % (BN - first);
            *reinterpret_cast<uint4*>(tile + c * KV_SPAN + rr * 128 + (i % 8) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bars.v_full(st));
        }
        if (lane == 0) FA_STAMP(p, T_P_V, jv);
        ++jv;
        advance(vw);
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
          atomicExch(p.err.word + 1, !qw.done() ? W_QEMPTY : !kw.done() ? W_KEMPTY : W_VEMPTY);
        }
        ok = false;
        break;
      }
          }
    if (ok && lane == 0) {
      // Drain: the tensor core's last arrivals on the empty barriers must
      // land before the CTA's shared memory is released.
      for (int j = max(0, jk - STAGES); j < jk; ++j)
        if (!mbar_wait(bars.k_empty(j % STAGES), (j / STAGES) & 1, p.err, abort, W_KEMPTY)) break;
      for (int j = max(0, jv - STAGES); j < jv; ++j)
        if (!mbar_wait(bars.v_empty(j % STAGES), (j / STAGES) & 1, p.err, abort, W_VEMPTY)) break;
      for (int j = max(0, pq - C::QBUF); j < pq; ++j)
        if (!mbar_wait(bars.q_empty(j % C::QBUF), (j / C::QBUF) & 1, p.err, abort, W_QEMPTY))
          break;
    }
  } else if (warp == WARP_MMA) {
    // ---------------------------------------------------------- MMA issuer ---
    // The whole warp runs the loop; one elected lane issues and commits.
    const uint32_t leader = elect_one();
    constexpr uint32_t IDESC_S = idesc_bf16(BN, NQ, false, false);   // S^T = K Q^T
    constexpr uint32_t IDESC_O = idesc_bf16(D, NQ, true, false);     // O^T += V^T P^T
    const uint64_t k_desc = sdesc_sw128(sbase + C::OFF_K, 16, 1024);   // keys x D, K-major
    const uint64_t q_desc = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);   // queries x D, K-major
    // V^T as A: M = D runs along each V row (two 64-column blocks KV_SPAN
    // apart), K = keys down the rows: MN-major.
    const uint64_t v_desc = sdesc_sw128(sbase + C::OFF_V, KV_SPAN, 1024);
    const uint64_t p_desc = sdesc_sw128(sbase + C::OFF_P, 16, 1024);   // queries x keys, K-major
    // Polls its two streams and issues whichever is ready:
    //   S^T_is once K_is has landed, the softmax has loaded S^T_{is-2} from
    //   the buffer and (first tile of a piece) the piece's Q has landed;
    //   P_ip V_ip once V_ip has landed and P_ip is published.
    // Each barrier polled here completes its next phase only after this warp
    // has acted on the current one, so a parity test never sees two phases.
    Walk sw = w0, pw = w0;
    int is = 0, ip = 0, ps = 0;
    long long t_last = clock64();
    while (!pw.done()) {
      bool progress = false;
      if (!sw.done()) {
        const int st = is % STAGES;
        const bool first = sw.first();
        if ((!first || warp_test(bars.q_full(ps % C::QBUF), (ps / C::QBUF) & 1)) &&
            warp_test(bars.k_full(st), (is / STAGES) & 1) &&
            (is < 2 || warp_test(bars.s_free(is & 1), ((is - 2) >> 1) & 1))) {
          if (first) ++ps;
          const int qb = (ps - 1) % C::QBUF;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss_if(leader, tmem + C::TM_S + (is & 1) * NQ,
                      sdesc_add(k_desc, st * TILE + (kk >> 2) * KV_SPAN + (kk & 3) * 32),
                      sdesc_add(q_desc, qb * C::QP_BYTES + (kk >> 2) * C::SPAN + (kk & 3) * 32),
                      IDESC_S, kk > 0);
          tc_commit_if(leader, bars.s_full(is & 1));
          tc_commit_if(leader, bars.k_empty(st));
          if (sw.last()) tc_commit_if(leader, bars.q_empty(qb));
          if (lane == 0) FA_STAMP(p, T_M_S, is);
          ++is;
          advance(sw);
          progress = true;
        }
      }
      if (ip < is) {
        const int st = ip % STAGES;
        const int pb = ip % C::PBUF;
        if (warp_test(bars.v_full(st), (ip / STAGES) & 1) &&
            warp_test(bars.p_ready(pb), (ip / C::PBUF) & 1)) {
          tc_fence_after();
          const bool fresh = pw.first();   // a piece's first tile starts O^T afresh
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)   // K = 128 keys in steps of 16
            mma_ss_if(leader, tmem + C::TM_O, sdesc_add(v_desc, st * TILE + kk * 2048),
                      sdesc_add(p_desc, pb * C::QP_BYTES + (kk >> 2) * C::SPAN + (kk & 3) * 32),
                      IDESC_O, (fresh && kk == 0) ? 0u : 1u);
          tc_commit_if(leader, bars.v_empty(st));
          tc_commit_if(leader, bars.pv_done(pb));
          if (lane == 0) FA_STAMP(p, T_M_PV, ip);
          ++ip;
          advance(pw);
          progress = true;
        }
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
    // Warp w owns TMEM lanes 32 (w % 4) .. +31 (keys of a tile; rows of O^T
    // at the end of a piece) and query rows [NH (w / 4), NH (w / 4 + 1)).
    constexpr int NH = NQ / 2;
    const int sid = threadIdx.x;                 // 0 .. 255
    const int quarter = warp & 3;
    const int kt = quarter * 32 + lane;          // key of the tile / row d of O^T
    const int r0 = (warp >> 2) * NH;             // this thread's first query row
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    float* mref = reinterpret_cast<float*>(smem + C::OFF_MREF);
    float* alpha_s = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);   // [quarter][row]
    const float c2 = p.scale_log2;
    const int g = dec.g;
    // This thread's P word for a row pair holds keys (kt & ~1, kt | 1) of
    // row r (even thread) or r + 1 (odd thread): the pair's column block,
    // 16-byte unit (swizzled by the row below) and byte in the unit.
    const int kp = kt & ~1;
    const uint32_t p_chunk = C::OFF_P + (kp >> 6) * C::SPAN;
    const int p_unit = (kp & 63) >> 3;
    const int p_byte = (kp & 7) * 2;
    const bool odd = (lane & 1) != 0;
    // Rows past R: scores 0 (zero Q rows) or -inf (masked), reference +inf
    // and no move, so their P is 2^-inf = 0 and the per-row loops below run
    // over all of this thread's rows without a branch.
    if (sid < NQ) {
      mref[sid] = sid < R ? 0.f : INFINITY;
      alpha_s[sid] = 1.f;
    }
    softmax_sync();
    // This thread's rows' references: the move threshold m + 8 and the
    // exponent offset (0 while a row has seen no key, m = -inf), kept in
    // registers up to 16 rows a thread, read from shared memory beyond.
    constexpr bool REF_REGS = NH <= 16;
    float mt[REF_REGS ? NH : 1], mu[REF_REGS ? NH : 1];
    auto load_ref = [&]() {
      if constexpr (REF_REGS) {
#pragma unroll
        for (int r = 0; r < NH; ++r) {
          const float m = mref[r0 + r];
          mt[r] = m + RESCALE_LOG2;
          mu[r] = (m == -INFINITY) ? 0.f : m;
        }
      }
    };
    auto thr = [&](int r) -> float {
      if constexpr (REF_REGS) return mt[r];
      else return mref[r0 + r] + RESCALE_LOG2;
    };
    auto off = [&](int r) -> float {
      if constexpr (REF_REGS) {
        return mu[r];
      } else {
        const float m = mref[r0 + r];
        return (m == -INFINITY) ? 0.f : m;
      }
    };
    load_ref();
    Walk w = w0;
    float l[NH];   // this thread's part of its rows' sums, in the current reference
#pragma unroll
    for (int r = 0; r < NH; ++r) l[r] = 0.f;
    int i = 0;     // the CTA's tile counter
    int t0 = 0;    // first tile of the current piece
    bool ok = true;
    while (!w.done()) {
      const bool first = w.first();
      const bool last = w.last();
      if (first) {
        t0 = w.t;
#pragma unroll
        for (int r = 0; r < NH; ++r) l[r] = 0.f;
      }
      uint32_t s[NH];
      ok = ok && warp_wait(bars.s_full(i & 1), (i >> 1) & 1, p.err, abort, W_SFULL);
      if (ok) {
        if (warp == 0 && lane == 0) FA_STAMP(p, T_W_SFULL, i);
        tc_fence_after();
        tmem_row_ld<NH>(tmem + lane_off + C::TM_S + (i & 1) * NQ + r0, s);
        tc_fence_before();
        mbar_arrive(bars.s_free(i & 1));
      }
      // Query row r sees key `key` when key < len and, causally, key <=
      // len - q_len + r / g, i.e. r >= g * (key - len + q_len). Only a tile
      // that reaches past len - q_len (causal) or len - 1 needs the mask.
      float x[NH];
      if ((w.t + 1) * BN <= (p.causal ? w.len - dec.q_len + 1 : w.len)) {
#pragma unroll
        for (int r = 0; r < NH; ++r) x[r] = __uint_as_float(s[r]) * c2;
      } else {
        const int key = w.t * BN + kt;
        const int rmin = p.causal ? max(0, g * (key - (w.len - dec.q_len))) : 0;
        const int rlim = key < w.len ? R : 0;
#pragma unroll
        for (int r = 0; r < NH; ++r)
          x[r] = (r0 + r >= rmin && r0 + r < rlim) ? __uint_as_float(s[r]) * c2 : -INFINITY;
      }
      bool ex = false;
      if (!first) {
#pragma unroll
        for (int r = 0; r < NH; ++r) ex |= x[r] > thr(r);
      }
      // Does any score move its row's reference (or has a wait failed)? The
      // rare yes takes a second barrier that tells the two apart.
      const bool any = softmax_sync_or(ex || !ok);
      if (any && !softmax_sync_and(ok)) break;
      const bool move = first || any;
      bool rescale = false;
      if (move) {
        // Row maxima over the 128 keys: per warp by shuffles, then thread r
        // combines the four quarters and moves row r's reference.
#pragma unroll
        for (int r = 0; r < NH; ++r) {
          if (r0 + r < R) {
            float v = x[r];
#pragma unroll
            for (int sh = 16; sh > 0; sh >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, sh));
            if (lane == 0) red[quarter * NQ + r0 + r] = v;
          }
        }
        softmax_sync();
        if (sid < R) {
          const float tmax = fmaxf(fmaxf(red[sid], red[NQ + sid]),
                                   fmaxf(red[2 * NQ + sid], red[3 * NQ + sid]));
          const float mo = first ? -INFINITY : mref[sid];
          float mn = mo, a = 1.f;
          if (tmax > mo + RESCALE_LOG2) {
            mn = tmax;
            a = (mo == -INFINITY) ? 0.f : ex2_approx(mo - tmax);
          }
          mref[sid] = mn;
          alpha_s[sid] = a;
        }
        softmax_sync();
        load_ref();
        if (!first) {
#pragma unroll
          for (int r = 0; r < NH; ++r) {
            const float a = alpha_s[r0 + r];
            l[r] *= a;
            rescale |= a != 1.f;
          }
        }
      }
      // P = 2^(x - m) for this key and each of its rows; adjacent keys'
      // values are paired into one bf16x2 word per row by a shuffle.
      uint32_t pk[NH / 2];
#pragma unroll
      for (int r = 0; r < NH; r += 2) {
        const float p0 = ex2_approx(x[r] - off(r));
        const float p1 = ex2_approx(x[r + 1] - off(r + 1));
        l[r] += p0;
        l[r + 1] += p1;
        const float recv = __shfl_xor_sync(FULL, odd ? p0 : p1, 1);
        pk[r >> 1] = odd ? pack_bf16x2(recv, p1) : pack_bf16x2(p0, recv);
      }
      // P buffer i % PBUF is free once P_{i-PBUF} V_{i-PBUF} is done; O^T may
      // be rescaled once P_{i-1} V_{i-1} is (the same wait when PBUF = 1).
      const int pb = i % C::PBUF;
      if (i >= C::PBUF)
        ok = ok && warp_wait(bars.pv_done(pb), ((i - C::PBUF) / C::PBUF) & 1, p.err, abort,
                             W_PVDONE);
      if (rescale && C::PBUF > 1)
        ok = ok && warp_wait(bars.pv_done((i - 1) % C::PBUF), ((i - 1) / C::PBUF) & 1, p.err,
                             abort, W_PVDONE);
      if (ok) {
        tc_fence_after();
        uint8_t* pbase = smem + p_chunk + pb * C::QP_BYTES;
#pragma unroll
        for (int r = 0; r < NH; r += 2) {
          const int row = r0 + (odd ? r + 1 : r);
          *reinterpret_cast<uint32_t*>(pbase + row * 128 + ((p_unit ^ (row & 7)) << 4) + p_byte) =
              pk[r >> 1];
        }
        if (rescale) {
          // Row kt of O^T, this thread's columns: column r moves to row r's
          // new reference.
          uint32_t o[NH];
          tmem_row_ld<NH>(tmem + lane_off + C::TM_O + r0, o);
#pragma unroll
          for (int r = 0; r < NH; ++r)
            o[r] = __float_as_uint(__uint_as_float(o[r]) * alpha_s[r0 + r]);
          tmem_row_st<NH>(tmem + lane_off + C::TM_O + r0, o);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bars.p_ready(pb));
        if (warp == 0 && lane == 0) FA_STAMP(p, T_W_ARR, i);
      }
      if (last) {
        // ------------------------------------------------ end of a piece ---
        // Row sums over the 128 keys, then O = O^T / l and the LSE, as the
        // final output when the piece is the whole segment, else as a
        // partial for the merge.
#pragma unroll
        for (int r = 0; r < NH; ++r) {
          if (r0 + r < R) {
            float v = l[r];
#pragma unroll
            for (int sh = 16; sh > 0; sh >>= 1) v += __shfl_xor_sync(FULL, v, sh);
            if (lane == 0) red[quarter * NQ + r0 + r] = v;
          }
        }
        if (!softmax_sync_and(ok)) break;
        ok = warp_wait(bars.pv_done(i % C::PBUF), (i / C::PBUF) & 1, p.err, abort, W_PVDONE);
        if (ok) {
          tc_fence_after();
          uint32_t o[NH];
          tmem_row_ld<NH>(tmem + lane_off + C::TM_O + r0, o);
          tc_fence_before();
          const int seg = w.b * p.H_kv + hk;
          const bool whole = t0 == 0 && w.seg_end();
          const size_t slot = static_cast<size_t>((w.b + grp) * p.H_kv + hk) * R;
#pragma unroll
          for (int rr = 0; rr < NH; ++rr) {
            const int r = r0 + rr;
            if (r < R) {
              const float lt = (red[r] + red[NQ + r]) + (red[2 * NQ + r] + red[3 * NQ + r]);
              const float v = __uint_as_float(o[rr]) * (lt > 0.f ? 1.f / lt : 0.f);
              if (whole) {
                const size_t orow = static_cast<size_t>(w.b * dec.q_len + r / g) * p.H +
                                    hk * g + r % g;
                static_cast<__nv_bfloat16*>(p.o)[orow * D + kt] = __float2bfloat16_rn(v);
              } else {
                dt.o_part[(slot + r) * D + kt] = v;
              }
            }
          }
          if (sid < R) {
            const float lt =
                (red[sid] + red[NQ + sid]) + (red[2 * NQ + sid] + red[3 * NQ + sid]);
            const float lse =
                (lt > 0.f) ? (mref[sid] + __log2f(lt)) * 0.69314718055994531f : -INFINITY;
            if (whole) {
              const size_t orow = static_cast<size_t>(w.b * dec.q_len + sid / g) * p.H +
                                  hk * g + sid % g;
              p.lse[orow] = lse;
            } else {
              dt.lse_part[slot + sid] = lse;
            }
          }
          if (sid == 0) {
            if (t0 == 0) dt.seg_first[seg] = grp;
            if (w.seg_end()) dt.seg_last[seg] = grp;
          }
          if (warp == 0 && lane == 0) FA_STAMP(p, T_W_EPI, i);
        }
      }
      ++i;
      advance(w);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0) cta_span(p, T_CTA_END);
}

// Merge of the partials of one output row per warp: LSE = ln sum_c exp(LSE_c),
// O = sum_c exp(LSE_c - LSE) O_c over the pieces c of its segment
// (agentalpha.top "flash attention" answer, follow-up 2). Segments inside
// one CTA's range were written by that CTA; empty sequences get O = 0 and
// LSE = -inf here.
__global__ void __launch_bounds__(256)
    decode_t_merge_kernel(const AttnParams p, const DecodeArgs dec, const DecodeTArgs dt) {
  const long long rid = static_cast<long long>(blockIdx.x) * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int R = dec.n_rows;
  if (rid >= static_cast<long long>(p.B) * p.H_kv * R) return;
  const int seg = static_cast<int>(rid / R);
  const int r = static_cast<int>(rid % R);
  const int b = seg / p.H_kv;
  const int hk = seg % p.H_kv;
  const int len = __ldg(dec.cache_seqlens + b);
  if (len < 0 || len > p.max_seqlen) return;   // reported by the partials kernel
  const size_t orow = static_cast<size_t>(b * dec.q_len + r / dec.g) * p.H + hk * dec.g +
                      r % dec.g;
  constexpr int PER = D / 32;   // columns per lane
  static_assert(PER == 4, "one float4 per lane");
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.o) + orow * D + lane * PER;
  float acc[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) acc[k] = 0.f;
  float m = -INFINITY, tot = 0.f;
  if (len > 0) {
    const int c0 = dt.seg_first[seg];
    const int c1 = dt.seg_last[seg];
    if (c0 == c1) return;   // one piece: its CTA wrote the row
    if (c0 < 0 || c1 >= dt.ctas / p.H_kv || c0 > c1) {
      if (lane == 0) record(p.err, BAD_MERGE);
      return;
    }
    // Group c's piece of the segment sits in slot (b + c) H_kv + hk.
    for (int c = c0 + lane; c <= c1; c += 32)
      m = fmaxf(m, dt.lse_part[static_cast<size_t>((b + c) * p.H_kv + hk) * R + r]);
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, sh));
    if (m != -INFINITY) {
      for (int c = c0; c <= c1; ++c) {
        const size_t prow = static_cast<size_t>((b + c) * p.H_kv + hk) * R + r;
        const float ls = dt.lse_part[prow];
        if (ls == -INFINITY) continue;
        const float wgt = expf(ls - m);
        tot += wgt;
        const float4 v = *reinterpret_cast<const float4*>(dt.o_part + prow * D + lane * PER);
        acc[0] += wgt * v.x;
        acc[1] += wgt * v.y;
        acc[2] += wgt * v.z;
        acc[3] += wgt * v.w;
      }
    }
  }
  const float inv = (tot > 0.f) ? 1.f / tot : 0.f;
  uint2 wv;
  wv.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  wv.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  *reinterpret_cast<uint2*>(dst) = wv;
  if (lane == 0) p.lse[orow] = (tot > 0.f) ? m + logf(tot) : -INFINITY;
}

template <int NQ>
cudaError_t launch_nq(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                      const AttnParams& p, const DecodeArgs& d, const DecodeTArgs& t,
                      cudaStream_t stream) {
  using C = Cfg<NQ>;
  const cudaError_t e = cudaFuncSetAttribute(
      decode_t_kernel<NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  decode_t_kernel<NQ><<<static_cast<unsigned>(t.ctas), THREADS, C::SMEM, stream>>>(tq, tk, tv,
                                                                                   p, d, t);
  return cudaGetLastError();
}

}  // namespace dect
}  // namespace

int decode_t_ctas(int H_kv) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0) {
    cudaGetLastError();
    sms = 148;
  }
  const int groups = (H_kv > 0 && sms >= H_kv) ? sms / H_kv : 1;
  return groups * (H_kv > 0 ? H_kv : 1);
}

size_t decode_t_workspace(long long B, int H_kv, long long n_rows, int ctas) {
  auto r256 = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t segs = static_cast<size_t>(B) * H_kv;
  const size_t rows = (segs + static_cast<size_t>(ctas)) * static_cast<size_t>(n_rows);
  return r256(rows * dect::D * 4) + r256(rows * 4) + 2 * r256(segs * 4);
}

void decode_t_carve(DecodeTArgs& t, void* workspace, long long B, int H_kv, long long n_rows) {
  auto r256 = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t segs = static_cast<size_t>(B) * H_kv;
  const size_t rows = (segs + static_cast<size_t>(t.ctas)) * static_cast<size_t>(n_rows);
  char* w = static_cast<char*>(workspace);
  t.o_part = reinterpret_cast<float*>(w);
  w += r256(rows * dect::D * 4);
  t.lse_part = reinterpret_cast<float*>(w);
  w += r256(rows * 4);
  t.seg_first = reinterpret_cast<int*>(w);
  w += r256(segs * 4);
  t.seg_last = reinterpret_cast<int*>(w);
}

cudaError_t launch_decode_t(const AttnParams& p, const DecodeArgs& d, const DecodeTArgs& t,
                            cudaStream_t stream) {
  using namespace dect;
  if (p.D != D || d.n_rows < 1 || d.n_rows > 64 || p.H_kv <= 0 || t.ctas <= 0 ||
      t.ctas % p.H_kv != 0)
    return cudaErrorInvalidValue;
  const long long segs = static_cast<long long>(p.B) * p.H_kv;
  if (segs == 0) return cudaSuccess;
  CUtensorMap tq, tk, tv;
  const unsigned box_rows =
      (d.block_table != nullptr) ? static_cast<unsigned>(min(d.page, BN)) : BN;
  if (!make_tmap_bf16_3d(&tq, p.q, p.total, p.H, D, static_cast<unsigned>(d.g),
                         static_cast<unsigned>(d.q_len)) ||
      !make_tmap_bf16_2d(&tk, p.k, d.cache_rows, static_cast<unsigned long long>(p.H_kv) * D, 64,
                         box_rows) ||
      !make_tmap_bf16_2d(&tv, p.v, d.cache_rows, static_cast<unsigned long long>(p.H_kv) * D, 64,
                         box_rows))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if (d.n_rows <= 16)
    e = launch_nq<16>(tq, tk, tv, p, d, t, stream);
  else if (d.n_rows <= 32)
    e = launch_nq<32>(tq, tk, tv, p, d, t, stream);
  else
    e = launch_nq<64>(tq, tk, tv, p, d, t, stream);
  if (e != cudaSuccess) return e;
  const long long rows = segs * d.n_rows;
  if ((rows + 7) / 8 > INT_MAX) return cudaErrorInvalidConfiguration;
  decode_t_merge_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(p, d, t);
  return cudaGetLastError();
}

}  // namespace fa
