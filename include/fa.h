/*
 * fa.h - C ABI of the B200 (sm_100a) exact-attention library libfa_b200.so.
 *
 * The library computes exact scaled dot-product attention
 *     O = softmax(scale * Q K^T) V
 * tile by tile with the online-softmax recurrence (running row max m, running
 * exponential sum l, rescaling of the output accumulator, one division by l at
 * the end), and saves the row log-sum-exp for the backward pass. The backward
 * pass recomputes S and P from Q, K and the saved log-sum-exp and forms dV, dP,
 * dS, dQ and dK; no N x N matrix is ever written to global memory. Two more
 * paths reuse the forward: split-KV decode over a contiguous or paged KV cache
 * (fa_decode) and the two-pass FP8 (E4M3) forward (fa_fp8_quantize,
 * fa_fwd_fp8); their sections below state their sources and conventions.
 *
 * Sources for what is computed:
 *   - aiqz.cc "Flash Attention V2/V3 optimization", section "IO bottleneck
 *     analysis" (the attention definition) and section "V2 algorithm
 *     optimisation", update steps 1-5 (m, l and O recurrence, final O / l);
 *   - airsota.com interview card (p=1562), section 3 (safe, online softmax)
 *     and section 4 items 1-3 (deferred normalisation, recomputation from the
 *     saved statistics, grouped-query attention);
 *   - agentalpha.top "flash attention" answer, section 2 (recomputation in
 *     the backward pass);
 *   - "Flash Attention self-test" (book.bogosort.top), sections C and D, which
 *     ask for causal masks, variable-length batches, the 1/sqrt(d) scale and
 *     the dV/dP/dS/dQ/dK relations without answering them; the readings used
 *     are stated at each entry point below.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout (token-major, contiguous, row-major):
 *   q, o, dout, dq : [T, H, D]      k, v, dk, dv : [T, H_kv, D]
 *   where T = B * N for a dense batch, or T = total_tokens (= cu_seqlens[B])
 *   for a packed variable-length batch.
 *   lse : float32, [B, H, N] for a dense batch, [H, T] for a packed batch.
 * Element type (dtype): FA_BF16 (bf16 in and out, fp32 accumulation, tensor
 *   cores; D must be 64 or 128) or FA_F32 (fp32 everywhere, CUDA cores;
 *   1 <= D <= 128).
 * Grouped-query attention: H % H_kv == 0; query head h reads key/value head
 *   h / (H / H_kv). H_kv == 1 is multi-query attention.
 * Causal mask: key j is visible to query i iff j <= i, with i and j counted
 *   from the start of their own sequence. The diagonal is kept.
 * Variable length: cu_seqlens (device int32, B + 1 non-decreasing entries,
 *   cu_seqlens[0] == 0) gives sequence b the rows [cu[b], cu[b+1]) of every
 *   tensor; attention never crosses a sequence boundary; empty sequences are
 *   allowed. max_seqlen must be >= every length; total_tokens == cu[B].
 *   With cu_seqlens == NULL the batch is dense and N is the length.
 * scale: multiplies Q K^T before the row max. scale <= 0 (or NaN) selects
 *   1 / sqrt(D).
 * LSE: natural-log log-sum-exp of the scaled logits of each query row,
 *   LSE_i = m_i + ln(l_i).
 * Pointers: device pointers, 16-byte aligned (tensor-memory-accelerator
 *   copies need it). Buffers are owned by the caller; the library allocates
 *   no device memory and keeps no per-call state (fa_bwd_noalloc's built-in
 *   scratch array is part of the loaded library, see its section).
 * Device state: the library looks up, once per device and with that device
 *   current, the device addresses of its own module variables (the error word
 *   and fa_bwd_noalloc's scratch) and keeps them for the life of the process.
 *   Do not use the library across a cudaDeviceReset, or from a context other
 *   than the device's primary context: the kept addresses would be stale.
 * Streams: every entry point only enqueues work on ``stream`` (NULL = the
 *   legacy default stream) and returns without synchronising, except
 *   fa_check_device_error.
 * Errors: argument errors are detected on the host before anything is
 *   enqueued and return FA_ERR_INVALID_ARG or FA_ERR_UNSUPPORTED. Launch
 *   failures return FA_ERR_CUDA. Every wait inside a kernel is bounded; a wait
 *   that runs out sets a device error word, which fa_check_device_error
 *   reports as FA_ERR_DEVICE_TIMEOUT. Nothing traps.
 */
#ifndef EXACT_IO_AWARE_TMEM_FA_H
#define EXACT_IO_AWARE_TMEM_FA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,    /* bad pointer, size, alignment or layout       */
  FA_ERR_UNSUPPORTED = 2,    /* valid request this build has no kernel for  */
  FA_ERR_CUDA = 3,           /* a CUDA runtime call or kernel launch failed  */
  FA_ERR_DEVICE_TIMEOUT = 4  /* a bounded in-kernel wait ran out            */
} fa_status;

typedef enum { FA_BF16 = 0, FA_F32 = 1 } fa_dtype;

/* Same object as cudaStream_t; declared here so the header needs no CUDA
 * include. */
typedef struct CUstream_st* fa_stream_t;

/*
 * fa_fwd - attention forward pass.
 *
 * Inputs q, k, v; outputs o (same dtype as q) and lse (float32). Implements
 * the online-softmax forward of aiqz.cc "Flash Attention V2/V3 optimization",
 * section "V2 algorithm optimisation" (steps 1-5) with the log-sum-exp saved
 * as the airsota.com card, section 4 item 2, keeps "m, l" for the backward.
 *
 *   B            batch size (number of sequences when cu_seqlens != NULL)
 *   H, H_kv      query heads and key/value heads (H % H_kv == 0)
 *   N            sequence length of a dense batch (ignored when packed)
 *   D            head dimension
 *   causal       0 or 1
 *   cu_seqlens   NULL (dense) or device int32[B + 1] (packed)
 *   max_seqlen   packed only: upper bound on every sequence length
 *   total_tokens packed only: cu_seqlens[B], the row count of every tensor
 *
 * Returns FA_OK once the work is enqueued.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int H_kv, int N, int D, fa_dtype dtype, int causal, float scale,
                 const int* cu_seqlens, int max_seqlen, long long total_tokens,
                 fa_stream_t stream);

/*
 * Backward phases. fa_bwd enqueues FA_BWD_FUSED: the preprocess, the fused
 * kernel that forms every product of the method once per (query tile, key
 * tile) pair and adds the dQ partials into an fp32 accumulator, and the dQ
 * conversion. FA_BWD_SPLIT is the same backward as two kernels that share
 * no accumulator: one for dK / dV and one for dQ, which recomputes S and dP
 * (seven products per tile pair instead of five). It needs less workspace and
 * gives bitwise reproducible dQ; the fused path's dQ is reproducible only to
 * rounding, because the order of its fp32 additions over key tiles is not
 * fixed (dK and dV are reproducible on both paths).
 */
#define FA_BWD_PHASE_PREPROCESS 0x01u /* D_i = dO_i . O_i; zeroes the dQ accumulator */
#define FA_BWD_PHASE_DKDV 0x02u       /* split path: dK, dV                          */
#define FA_BWD_PHASE_DQ 0x04u         /* split path: dQ                              */
#define FA_BWD_PHASE_FUSED 0x08u      /* fused path: dK, dV, dQ accumulator          */
#define FA_BWD_PHASE_DQ_CONVERT 0x10u /* fused path: dQ = bf16(scale * accumulator)  */
#define FA_BWD_SPLIT 0x07u
#define FA_BWD_FUSED 0x19u
#define FA_BWD_ALL 0x1Fu

/*
 * fa_bwd_phases_workspace_size - bytes of device scratch fa_bwd_phases needs
 * for ``mask``, T tokens and H query heads: the float32 row terms
 * D_i = dO_i . O_i [H, T], rounded up to 256 bytes, plus, for bf16 when the
 * mask has FA_BWD_PHASE_FUSED or FA_BWD_PHASE_DQ_CONVERT, the float32 dQ
 * accumulator [T, H, D] rounded up to 256 bytes; plus 256. Returns 0 for
 * invalid sizes or masks.
 *
 * fa_bwd_workspace_size - the same for fa_bwd (mask FA_BWD_FUSED).
 */
size_t fa_bwd_phases_workspace_size(unsigned mask, long long total_tokens, int H, int D,
                                    fa_dtype dtype);
size_t fa_bwd_workspace_size(long long total_tokens, int H, int D, fa_dtype dtype);

/*
 * fa_bwd - attention backward pass for the loss sum(O * dO).
 *
 * Recomputes S = scale Q K^T and P = exp(S - LSE) tile by tile from q, k and
 * the lse that fa_fwd wrote (agentalpha.top "flash attention" answer, section
 * 2; airsota.com card, section 4 item 2), then forms
 *   dV = P^T dO, dP = dO V^T, D_i = dO_i . O_i, dS = P * (dP - D_i),
 *   dQ = scale dS K, dK = scale dS^T Q
 * (the relations the "Flash Attention self-test", section D, asks for). With
 * grouped-query attention dk and dv of a key/value head are summed over the
 * query heads that share it. Runs the FA_BWD_FUSED phases.
 *
 *   q, k, v, o, lse, dout   inputs, as written / read by fa_fwd
 *   dq, dk, dv              outputs, same dtype and layout as q, k, v
 *   workspace, ws_bytes     caller-owned device scratch of at least
 *                           fa_bwd_workspace_size(T, H, D, dtype) bytes,
 *                           256-byte aligned; its contents on entry do not
 *                           matter and are undefined on return
 * The remaining arguments mean what they mean for fa_fwd and must match the
 * forward call that produced o and lse.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N,
                 int D, fa_dtype dtype, int causal, float scale, const int* cu_seqlens,
                 int max_seqlen, long long total_tokens, void* workspace, size_t ws_bytes,
                 fa_stream_t stream);

/*
 * fa_bwd_phases - fa_bwd restricted to the phases in ``mask`` (the
 * FA_BWD_PHASE_* bits), enqueued in bit order; FA_BWD_SPLIT selects the
 * split backward, and single bits let each kernel be timed by itself. Every
 * phase after the preprocess reads D_i, so the preprocess must have run on
 * the same workspace first; it also zeroes the dQ accumulator whenever the
 * workspace is large enough to hold one (bf16), which the fused kernel
 * requires. ws_bytes must be at least
 * fa_bwd_phases_workspace_size(mask, T, H, D, dtype). For FA_F32 only the
 * masks FA_BWD_FUSED and FA_BWD_SPLIT are accepted (both run the one fp32
 * backward; FA_ERR_UNSUPPORTED otherwise). Other arguments as for fa_bwd.
 */
fa_status fa_bwd_phases(unsigned mask, const void* q, const void* k, const void* v,
                        const void* o, const float* lse, const void* dout, void* dq, void* dk,
                        void* dv, int B, int H, int H_kv, int N, int D, fa_dtype dtype, int causal,
                        float scale, const int* cu_seqlens, int max_seqlen, long long total_tokens,
                        void* workspace, size_t ws_bytes, fa_stream_t stream);

/*
 * fa_bwd_noalloc - fa_bwd for callers that cannot allocate device memory.
 *
 * The pages describe no such call; it exists for callers that are handed only
 * their input and output buffers and may not call cudaMalloc themselves (a
 * kernel plugin inside a framework that owns every device allocation, or a
 * latency-critical path where an allocation would synchronise the device or
 * break a fixed memory budget). Instead of a caller workspace it uses a
 * scratch array built into the library: FA_NOALLOC_SCRATCH_BYTES (32 MiB) of
 * device memory that every GPU loading the library holds until the process
 * exits. It calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments and layouts are those of fa_bwd without workspace and ws_bytes.
 * It runs the split backward (FA_BWD_SPLIT), whose only scratch is the D_i
 * rows, so its results are identical to fa_bwd_phases(FA_BWD_SPLIT, ...)
 * and agree with fa_bwd within rounding. The sizes are checked as fa_bwd
 * checks them first (same status for the same mistake). Limit:
 * fa_bwd_phases_workspace_size(FA_BWD_SPLIT, T, H, D, dtype) must not exceed
 * FA_NOALLOC_SCRATCH_BYTES (about T * H * 4 bytes, so T * H <= 8,388,000);
 * larger problems return FA_ERR_UNSUPPORTED before anything is enqueued. A
 * failed address lookup returns FA_ERR_CUDA and sets
 * fa_last_cuda_error_string.
 *
 * The scratch is shared by every call on a device and keeps the last call's
 * contents; each call re-initialises what it reads. Calls whose kernels can
 * overlap on the GPU (different streams without ordering between them, or
 * several host threads) race on the scratch and give wrong results: order
 * them on one stream. The first call on each device looks up the scratch's
 * device address (cudaGetSymbolAddress) once, with that device current; make
 * that first call before any stream capture begins.
 */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                         int H, int H_kv, int N, int D, fa_dtype dtype, int causal, float scale,
                         const int* cu_seqlens, int max_seqlen, long long total_tokens,
                         fa_stream_t stream);

/* fa_get_error_string - static, human-readable name of a status code. */
const char* fa_get_error_string(fa_status status);

/*
 * fa_last_cuda_error_string - the CUDA runtime's description of the most
 * recent CUDA error behind an FA_ERR_CUDA returned on the calling host
 * thread ("no error" if there was none). Static storage; do not free.
 */
const char* fa_last_cuda_error_string(void);

/*
 * fa_check_device_error - synchronises ``stream``, then reports and clears
 * the device error word of the current device: FA_ERR_DEVICE_TIMEOUT if a
 * kernel's bounded wait ran out since the last check, FA_ERR_CUDA if the
 * synchronisation failed, else FA_OK. ``where`` (nullable) receives the code
 * of the wait that gave up.
 */
fa_status fa_check_device_error(fa_stream_t stream, unsigned* where);

/*
 * fa_set_wait_budget - how many SM clock cycles one in-kernel wait may spin
 * before it gives up (default 4e9, about two seconds). Values <= 0 restore
 * the default. Applies to launches enqueued after the call.
 */
void fa_set_wait_budget(long long cycles);

/*
 * fa_selftest_wait_timeout - enqueues one small kernel that waits on an
 * mbarrier no thread ever arrives on, with a budget of ``cycles``, so that
 * the bounded-wait path can be exercised without faulting or hanging the
 * GPU. After it, fa_check_device_error must return FA_ERR_DEVICE_TIMEOUT.
 */
fa_status fa_selftest_wait_timeout(long long cycles, fa_stream_t stream);

/*
 * fa_selftest_exp2 - y[i] = 2^x[i] for n device floats, by the FMA-pipe
 * exponential that the D = 64 forward and the fused backward use for a
 * share of their softmax exponentials (range reduction x = n + f, |f| <= 1/2,
 * and a degree-3 minimax polynomial for 2^f: relative error at most 7.5e-5
 * for -125 <= x <= 127; x <= -126, -inf included, gives about 2^-126).
 * Enqueued on ``stream``. FA_ERR_INVALID_ARG for n < 0 or null pointers
 * with n > 0.
 */
fa_status fa_selftest_exp2(const float* x, float* y, long long n, fa_stream_t stream);

/*
 * Debug build. The library built with -DFA_DEBUG (libfa_b200_debug.so, same
 * entry points) checks indices in its kernels against the buffers they
 * address, recording a failed check in the device error word
 * (fa_check_device_error reports FA_ERR_INVALID_ARG, ``where`` names the
 * check) and skipping the access, and can record, for one CTA of each launch,
 * the SM clock at the events of its roles (waits passed, products issued,
 * signals sent): per kind of event, one 64-bit stamp per step.
 *
 * fa_debug_build - 1 in the debug build, 0 otherwise.
 *
 * fa_debug_set_trace - launches enqueued after the call stamp their events
 * into ``buffer`` (device memory of at least FA_DEBUG_TRACE_BYTES, 8-byte
 * aligned, owned by the caller: [32 kinds][1024 steps] unsigned 64-bit
 * clocks, entries of events that did not happen left as they were) for the
 * CTA with blockIdx.x == ``cta``. A null buffer stops stamping. The kinds of
 * each kernel are listed in exact_io_aware_tmem_b200/trace.py. Returns
 * FA_ERR_UNSUPPORTED in the ordinary build.
 */
#define FA_DEBUG_TRACE_BYTES (32u * 1024u * 8u)
int fa_debug_build(void);
fa_status fa_debug_set_trace(void* buffer, size_t bytes, int cta);

/*
 * ---------------------------------------------------------------- decode ---
 * Split-KV decode (FlashDecoding) over a contiguous or paged key/value cache.
 *
 * At inference the method keeps its tiling and drops recomputation
 * (agentalpha.top "flash attention" answer, section 2). The cache is split
 * into blocks whose attention is computed independently and merged with the
 * online-softmax update; a paged cache is read page by page (same answer,
 * follow-up 2). Result: attention of the q_len newest tokens of each of B
 * sequences against that sequence's cache prefix. The query token i of q_len
 * sits at position cache_seqlens[b] - q_len + i. With causal = 1 it sees keys
 * at positions <= its own; with causal = 0 it sees the whole prefix. A token
 * that sees no key (for instance when cache_seqlens[b] == 0) gets O = 0 and
 * LSE = -inf.
 *
 * fa_decode_num_splits - number of key splits fa_decode uses: ``requested``
 * when > 0, else a count aiming at about four CTAs per SM of a 148-SM B200.
 * In both cases it is clamped to the 128-key tiles of max_seqlen_k and then
 * to the fewest splits with the same tiles per split. Host only.
 */
int fa_decode_num_splits(int B, int H_kv, int max_seqlen_k, int requested);

/*
 * fa_decode_workspace_size - bytes of device workspace fa_decode needs for
 * these sizes and split request: 0 when it uses one split; otherwise fp32
 * split partials of O and LSE (n_split * B * q_len * H * (D + 1) * 4 bytes,
 * each array rounded up to 256 bytes). Host only. Returns 0 for invalid
 * sizes as well; fa_decode reports those.
 */
size_t fa_decode_workspace_size(int B, int q_len, int H, int H_kv, int D, int max_seqlen_k,
                                int n_split);

/*
 * fa_decode - bf16 split-KV decode attention.
 *   q             bf16 [B * q_len, H, D], token-major: the q_len newest tokens
 *                 of sequence b are rows b * q_len .. b * q_len + q_len - 1.
 *   k_cache,      bf16 [cache_rows, H_kv, D] each.
 *   v_cache       Contiguous cache (block_table NULL): position j of sequence
 *                 b is row b * page_size + j, so page_size is the rows per
 *                 sequence (>= max_seqlen_k). Paged cache: position j is row
 *                 block_table[b * max_blocks + j / page_size] * page_size +
 *                 j % page_size. Rows no position of a sequence maps to may
 *                 hold anything (NaN included); they never reach O.
 *   o             bf16 [B * q_len, H, D] out.
 *   lse           fp32 [B * q_len, H] out: natural-log LSE of the scaled
 *                 logits, -inf for a token that sees no key.
 *   cache_seqlens device int32 [B]: keys in each sequence's cache, each in
 *                 [0, max_seqlen_k] (a value outside is reported by
 *                 fa_check_device_error and that sequence is left unwritten).
 *   block_table   device int32 [B, max_blocks] page ids (entries past a
 *                 sequence's last page are never read), or NULL.
 *   page_size     paged: rows per page, a multiple of 16 that divides 128 or
 *                 is a multiple of 128; contiguous: rows per sequence.
 *   max_blocks    paged: row length of block_table (>= ceil(max_seqlen_k /
 *                 page_size)); ignored when block_table is NULL.
 *   cache_rows    rows of k_cache / v_cache (>= 1 and < 2^31; paged: a multiple of
 *                 page_size; contiguous: >= (B - 1) * page_size + max_seqlen_k).
 *   max_seqlen_k  host-side bound on cache_seqlens.
 *   H, H_kv       query / key-value heads, H % H_kv == 0. The q_len tokens x
 *                 H / H_kv query heads that share a key/value head form one
 *                 128-row tile: q_len * (H / H_kv) <= 128.
 *   D             64 or 128. scale <= 0 means 1 / sqrt(D).
 *   n_split       key splits (0: automatic, see fa_decode_num_splits).
 *   workspace     device, 16-byte aligned, ws_bytes >=
 *                 fa_decode_workspace_size(...) (may be NULL when that is 0).
 * Ownership, stream and errors as for fa_fwd: nothing is allocated; argument
 * errors return FA_ERR_INVALID_ARG / FA_ERR_UNSUPPORTED before any launch.
 */
fa_status fa_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                    const int* cache_seqlens, const int* block_table, int B, int q_len, int H,
                    int H_kv, int D, int page_size, int max_blocks, long long cache_rows,
                    int max_seqlen_k, int causal, float scale, int n_split, void* workspace,
                    size_t ws_bytes, fa_stream_t stream);

/*
 * ------------------------------------------------------------------ FP8 ---
 * FP8 (E4M3) forward (aiqz.cc "Flash Attention V2/V3 optimization" article,
 * section "FP8 low precision"): pass 1 (fa_fp8_quantize) takes each block's
 * largest |x|, its step Delta = max|x| / 448, and stores round(x / Delta) as
 * E4M3 codes; pass 2 (fa_fwd_fp8) multiplies the quantised Q and K on the
 * tensor cores with an fp32 accumulator and otherwise runs the forward above
 * (P V in bf16 with fp32 accumulation, bf16 O, fp32 LSE). A block is 128
 * consecutive tokens of one head of one sequence (the last block of a
 * sequence may be shorter); Delta and x / Delta are IEEE single-precision
 * divisions; rounding is to nearest even with saturation at +-448; a block of
 * zeros gets Delta = 1. Dense batches only (no cu_seqlens).
 *
 * fa_fp8_quantize - pass 1 for one tensor.
 *   x      bf16 [B * N, Hx, D] (token-major, as q or k of fa_fwd)
 *   x8     out: E4M3 codes, one byte per element, same layout as x
 *   scale  out: fp32 [B, Hx, ceil(N / 128)] steps Delta
 *   D      a multiple of 8, at most 256. Pointers 16-byte aligned.
 */
fa_status fa_fp8_quantize(const void* x, void* x8, float* scale, int B, int N, int Hx, int D,
                          fa_stream_t stream);

/*
 * fa_fwd_fp8 - pass 2: causal or full attention on the quantised Q and K.
 *   q8, k8     E4M3 codes [B * N, H, D] / [B * N, H_kv, D] from fa_fp8_quantize
 *   v          bf16 [B * N, H_kv, D]
 *   q_scale,   fp32 [B, H, ceil(N / 128)] / [B, H_kv, ceil(N / 128)] steps
 *   k_scale
 *   o, lse     as for fa_fwd with cu_seqlens NULL (o bf16 [B * N, H, D],
 *              lse fp32 [B, H, N])
 *   D          128 (one 128-byte E4M3 row per token). scale <= 0: 1 / sqrt(D).
 * Errors as for fa_fwd.
 */
fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v, const float* q_scale,
                     const float* k_scale, void* o, float* lse, int B, int H, int H_kv, int N,
                     int D, int causal, float scale, fa_stream_t stream);

/* fa_version - library version as major * 10000 + minor * 100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_IO_AWARE_TMEM_FA_H */
