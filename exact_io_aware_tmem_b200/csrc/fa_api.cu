// C ABI of libfa_b200.so (declared in include/fa.h): host-side argument
// checks, dispatch to the kernels, tensor-map encoding and the device error
// word that bounded in-kernel waits report through.
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "../../include/fa.h"
#include "decode_t.h"
#include "fwd_d64.h"
#include "ex2_fma.cuh"
#include "params.h"

namespace fa {

// Word 0: error bits (ERR_TIMEOUT, ERR_BOUNDS); word 1: code of the wait or
// check that failed. Every kernel receives its address in AttnParams::err.
__device__ unsigned g_err_word[2];

namespace {

constexpr long long kDefaultBudget = 4000000000LL;  // ~2 s at 1.9 GHz

// Last CUDA error behind an FA_ERR_CUDA on this host thread.
thread_local cudaError_t g_last_cuda = cudaSuccess;

fa_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return FA_OK;
  g_last_cuda = e;
  return FA_ERR_CUDA;
}
long long g_budget = kDefaultBudget;

// Debug builds: the stamp buffer and traced CTA of the next launches.
unsigned long long* g_trace = nullptr;
int g_trace_cta = 0;

constexpr int kMaxDevices = 64;
unsigned* g_err_ptr[kMaxDevices] = {};
std::mutex g_mu;

// Device address of g_err_word on the current device (looked up once).
unsigned* err_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_err_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_err_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<unsigned*>(ptr);
  }
  return g_err_ptr[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Shared checks of fa_fwd / fa_bwd; fills the size fields of ``p``.
fa_status check_common(AttnParams& p, int B, int H, int H_kv, int N, int D, fa_dtype dtype,
                       int causal, float scale, const int* cu_seqlens, int max_seqlen,
                       long long total_tokens) {
  if (B < 0 || H <= 0 || H_kv <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (H % H_kv != 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_F32) return FA_ERR_INVALID_ARG;
  if (dtype == FA_BF16 && D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (dtype == FA_F32 && D > 128) return FA_ERR_UNSUPPORTED;
  if (H > 65535 || B > 65535) return FA_ERR_UNSUPPORTED;  // grid y / z limits
  if (cu_seqlens != nullptr) {
    if (max_seqlen < 0 || total_tokens < 0 || total_tokens > INT32_MAX) return FA_ERR_INVALID_ARG;
    if (B == 0 && total_tokens != 0) return FA_ERR_INVALID_ARG;
    p.max_seqlen = max_seqlen;
    p.total = total_tokens;
    p.N = 0;
  } else {
    if (N < 0) return FA_ERR_INVALID_ARG;
    const long long total = static_cast<long long>(B) * N;
    if (total > INT32_MAX) return FA_ERR_UNSUPPORTED;
    p.max_seqlen = N;
    p.total = total;
    p.N = N;
  }
  p.cu_seqlens = cu_seqlens;
  p.B = B;
  p.H = H;
  p.H_kv = H_kv;
  p.D = D;
  p.causal = causal;
  if (!(scale > 0.f) || !isfinite(scale)) scale = 1.f / sqrtf(static_cast<float>(D));
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err.word = nullptr;
  p.err.budget = g_budget;
  p.trace = g_trace;
  p.trace_cta = g_trace_cta;
  return FA_OK;
}

}  // namespace

fa_status record_cuda(cudaError_t e) { return cuda_status(e); }

fa_status check_bwd_sizes(int B, int H, int H_kv, int N, int D, fa_dtype dtype, int causal,
                          const int* cu_seqlens, int max_seqlen, long long total_tokens,
                          long long* rows) {
  AttnParams p = {};
  const fa_status st = check_common(p, B, H, H_kv, N, D, dtype, causal, -1.f, cu_seqlens,
                                    max_seqlen, total_tokens);
  if (st == FA_OK && rows != nullptr) *rows = p.total;
  return st;
}

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, unsigned long long rows,
                       unsigned long long cols, unsigned box_cols, unsigned box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};  // bytes between rows
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_u8_2d(CUtensorMap* map, const void* base, unsigned long long rows,
                     unsigned long long cols, unsigned box_cols, unsigned box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};  // bytes between rows
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_f32_2d(CUtensorMap* map, const void* base, unsigned long long rows,
                      unsigned long long cols, unsigned box_cols, unsigned box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 4};  // bytes between rows
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, long long rows, int heads, int D,
                       unsigned box_heads, unsigned box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(heads) * D * 2};
  const cuuint32_t box[3] = {64, box_heads, box_rows};
  const cuuint32_t estride[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

__global__ void wait_selftest_kernel(DevErr e) {
  __shared__ alignas(8) unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on ``bar``: the wait must give up on its own.
  mbar_wait(smem_u32(&bar), 0, e, &abort_flag, 0x5e1f7e57u);
}

}  // namespace

cudaError_t launch_wait_selftest(DevErr err, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(err);
  return cudaGetLastError();
}

namespace {

__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y,
                                     long long n) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += stride)
    y[i] = ex2_fma(x[i]);
}

}  // namespace

cudaError_t launch_exp2_selftest(const float* x, float* y, long long n, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const long long blocks = std::min<long long>((n + 255) / 256, 148 * 8);
  exp2_selftest_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(x, y, n);
  return cudaGetLastError();
}

}  // namespace fa

using fa::AttnParams;

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int H_kv, int N, int D, fa_dtype dtype, int causal, float scale,
                 const int* cu_seqlens, int max_seqlen, long long total_tokens,
                 fa_stream_t stream) {
  AttnParams p = {};
  fa_status st = fa::check_common(p, B, H, H_kv, N, D, dtype, causal, scale, cu_seqlens,
                                  max_seqlen, total_tokens);
  if (st != FA_OK) return st;
  if (p.total == 0 || p.max_seqlen == 0 || B == 0) return FA_OK;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!fa::aligned16(q) || !fa::aligned16(k) || !fa::aligned16(v) || !fa::aligned16(o))
    return FA_ERR_INVALID_ARG;
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.lse = lse;
  p.err.word = fa::err_word();
  if (p.err.word == nullptr) return FA_ERR_CUDA;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e = (dtype == FA_F32) ? fa::launch_fwd_f32(p, s)
                        : (D == 64)       ? fa::launch_fwd_d64(p, s)
                                          : fa::launch_fwd_pair(p, s);
  return fa::cuda_status(e);
}

int fa_decode_num_splits(int B, int H_kv, int max_seqlen_k, int requested) {
  if (B <= 0 || H_kv <= 0 || max_seqlen_k <= 0) return 1;
  const long long tiles = (static_cast<long long>(max_seqlen_k) + 127) / 128;
  long long n = requested;
  if (n <= 0) {
    const long long units = static_cast<long long>(B) * H_kv;
    n = (4 * 148 + units - 1) / units;   // about four CTAs per SM of a 148-SM B200
  }
  n = std::max<long long>(1, std::min(n, tiles));
  const long long chunk = (tiles + n - 1) / n;
  return static_cast<int>((tiles + chunk - 1) / chunk);
}

size_t fa_decode_workspace_size(int B, int q_len, int H, int H_kv, int D, int max_seqlen_k,
                                int n_split) {
  if (B <= 0 || q_len <= 0 || H <= 0 || H_kv <= 0 || D <= 0 || max_seqlen_k < 0) return 0;
  if (n_split == 0 && H % H_kv == 0 &&
      fa::decode_t_eligible(D, static_cast<long long>(q_len) * (H / H_kv)))
    return fa::decode_t_workspace(B, H_kv, static_cast<long long>(q_len) * (H / H_kv),
                                  fa::decode_t_ctas(H_kv));
  const int ns = fa_decode_num_splits(B, H_kv, max_seqlen_k, n_split);
  if (ns <= 1) return 0;
  const size_t rows = static_cast<size_t>(ns) * B * q_len * H;
  return fa::round256(rows * D * 4) + fa::round256(rows * 4);
}

fa_status fa_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                    const int* cache_seqlens, const int* block_table, int B, int q_len, int H,
                    int H_kv, int D, int page_size, int max_blocks, long long cache_rows,
                    int max_seqlen_k, int causal, float scale, int n_split, void* workspace,
                    size_t ws_bytes, fa_stream_t stream) {
  if (B < 0 || q_len <= 0 || H <= 0 || H_kv <= 0 || D <= 0 || max_seqlen_k < 0 ||
      cache_rows < 0 || n_split < 0)
    return FA_ERR_INVALID_ARG;
  if (H % H_kv != 0 || (causal != 0 && causal != 1)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  const int g = H / H_kv;
  if (static_cast<long long>(q_len) * g > 128) return FA_ERR_UNSUPPORTED;
  if (cache_rows >= (1ll << 31) || static_cast<long long>(B) * q_len > INT32_MAX ||
      static_cast<long long>(B) * H_kv > (1ll << 24))
    return FA_ERR_UNSUPPORTED;
  if (B == 0) return FA_OK;
  if (page_size <= 0 || cache_rows < 1) return FA_ERR_INVALID_ARG;
  if (block_table == nullptr) {
    if (page_size < max_seqlen_k) return FA_ERR_INVALID_ARG;
    if (cache_rows < static_cast<long long>(B - 1) * page_size + max_seqlen_k)
      return FA_ERR_INVALID_ARG;
  } else {
    if (page_size % 16 != 0 || !(128 % page_size == 0 || page_size % 128 == 0))
      return FA_ERR_UNSUPPORTED;
    if (max_blocks < (max_seqlen_k + page_size - 1) / page_size || cache_rows % page_size != 0)
      return FA_ERR_INVALID_ARG;
  }
  if (!q || !k_cache || !v_cache || !o || !lse || !cache_seqlens) return FA_ERR_INVALID_ARG;
  if (!fa::aligned16(q) || !fa::aligned16(k_cache) || !fa::aligned16(v_cache) ||
      !fa::aligned16(o))
    return FA_ERR_INVALID_ARG;
  const int ns = fa_decode_num_splits(B, H_kv, max_seqlen_k, n_split);
  const size_t need = fa_decode_workspace_size(B, q_len, H, H_kv, D, max_seqlen_k, n_split);
  if (need > 0 && (workspace == nullptr || ws_bytes < need || !fa::aligned16(workspace)))
    return FA_ERR_INVALID_ARG;

  AttnParams p = {};
  p.q = q;
  p.k = k_cache;
  p.v = v_cache;
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.H_kv = H_kv;
  p.D = D;
  p.N = 0;
  p.causal = causal;
  p.max_seqlen = max_seqlen_k;
  p.total = static_cast<long long>(B) * q_len;
  if (!(scale > 0.f) || !isfinite(scale)) scale = 1.f / sqrtf(static_cast<float>(D));
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err.budget = fa::g_budget;
  p.err.word = fa::err_word();
  if (p.err.word == nullptr) return FA_ERR_CUDA;
  p.trace = fa::g_trace;
  p.trace_cta = fa::g_trace_cta;

  fa::DecodeArgs d = {};
  d.cache_seqlens = cache_seqlens;
  d.block_table = block_table;
  d.page = page_size;
  d.max_blocks = (block_table != nullptr) ? max_blocks : 0;
  d.cache_rows = cache_rows;
  d.q_len = q_len;
  d.g = g;
  d.n_rows = q_len * g;
  d.n_split = ns;
  const int tiles = std::max(1, (max_seqlen_k + 127) / 128);
  d.chunk = (tiles + ns - 1) / ns;
  if (ns > 1) {
    const size_t rows = static_cast<size_t>(ns) * B * q_len * H;
    d.o_part = static_cast<float*>(workspace);
    d.lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                          fa::round256(rows * D * 4));
  }
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (n_split == 0 && fa::decode_t_eligible(D, d.n_rows)) {
    // Balanced partition over one persistent CTA per SM (decode_t.cu); the
    // workspace size above was computed for the same device.
    fa::DecodeTArgs t = {};
    t.ctas = fa::decode_t_ctas(H_kv);
    fa::decode_t_carve(t, workspace, B, H_kv, d.n_rows);
    return fa::cuda_status(fa::launch_decode_t(p, d, t, s));
  }
  return fa::cuda_status(fa::launch_decode_bf16(p, d, s));
}

fa_status fa_fp8_quantize(const void* x, void* x8, float* scale, int B, int N, int Hx, int D,
                          fa_stream_t stream) {
  if (B < 0 || N < 0 || Hx <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (D % 8 != 0 || D > 256) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * N > INT32_MAX) return FA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0) return FA_OK;
  if (!x || !x8 || !scale) return FA_ERR_INVALID_ARG;
  if (!fa::aligned16(x) || !fa::aligned16(x8)) return FA_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return fa::cuda_status(fa::launch_fp8_quantize(x, x8, scale, B, N, Hx, D, s));
}

fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v, const float* q_scale,
                     const float* k_scale, void* o, float* lse, int B, int H, int H_kv, int N,
                     int D, int causal, float scale, fa_stream_t stream) {
  AttnParams p = {};
  fa_status st = fa::check_common(p, B, H, H_kv, N, D, FA_BF16, causal, scale, nullptr, N,
                                  static_cast<long long>(B) * N);
  if (st != FA_OK) return st;
  if (D != 128) return FA_ERR_UNSUPPORTED;
  if (p.total == 0 || B == 0) return FA_OK;
  if (!q8 || !k8 || !v || !q_scale || !k_scale || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!fa::aligned16(q8) || !fa::aligned16(k8) || !fa::aligned16(v) || !fa::aligned16(o))
    return FA_ERR_INVALID_ARG;
  p.q = q8;
  p.k = k8;
  p.v = v;
  p.o = o;
  p.lse = lse;
  p.err.word = fa::err_word();
  if (p.err.word == nullptr) return FA_ERR_CUDA;
  fa::Fp8Args f = {q_scale, k_scale, (N + 127) / 128};
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return fa::cuda_status(fa::launch_fwd_pair_fp8(p, f, s));
}

size_t fa_bwd_phases_workspace_size(unsigned mask, long long total_tokens, int H, int D,
                                    fa_dtype dtype) {
  if (total_tokens < 0 || H <= 0 || D <= 0) return 0;
  if (dtype != FA_BF16 && dtype != FA_F32) return 0;
  if (mask == 0 || (mask & ~FA_BWD_ALL) != 0) return 0;
  const size_t T = static_cast<size_t>(total_tokens);
  const size_t delta = fa::round256(T * H * sizeof(float));
  // The fused kernel and the dQ conversion also need the fp32 dQ accumulator.
  const bool acc = dtype == FA_BF16 && (mask & (FA_BWD_PHASE_FUSED | FA_BWD_PHASE_DQ_CONVERT));
  return delta + (acc ? fa::round256(T * H * D * sizeof(float)) : 0) + 256;
}

size_t fa_bwd_workspace_size(long long total_tokens, int H, int D, fa_dtype dtype) {
  return fa_bwd_phases_workspace_size(FA_BWD_FUSED, total_tokens, H, D, dtype);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N,
                 int D, fa_dtype dtype, int causal, float scale, const int* cu_seqlens,
                 int max_seqlen, long long total_tokens, void* workspace, size_t ws_bytes,
                 fa_stream_t stream) {
  return fa_bwd_phases(FA_BWD_FUSED, q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, D, dtype,
                       causal, scale, cu_seqlens, max_seqlen, total_tokens, workspace, ws_bytes,
                       stream);
}

fa_status fa_bwd_phases(unsigned mask, const void* q, const void* k, const void* v,
                        const void* o, const float* lse, const void* dout, void* dq, void* dk,
                        void* dv, int B, int H, int H_kv, int N, int D, fa_dtype dtype, int causal,
                        float scale, const int* cu_seqlens, int max_seqlen, long long total_tokens,
                        void* workspace, size_t ws_bytes, fa_stream_t stream) {
  if (mask == 0 || (mask & ~FA_BWD_ALL) != 0) return FA_ERR_INVALID_ARG;
  // The fp32 path is one backward of its own: only the two whole-pass masks.
  if (dtype == FA_F32 && mask != FA_BWD_FUSED && mask != FA_BWD_SPLIT) return FA_ERR_UNSUPPORTED;
  AttnParams p = {};
  fa_status st = fa::check_common(p, B, H, H_kv, N, D, dtype, causal, scale, cu_seqlens,
                                  max_seqlen, total_tokens);
  if (st != FA_OK) return st;
  if (p.total == 0 || p.max_seqlen == 0 || B == 0) return FA_OK;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return FA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, dout, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!fa::aligned16(ptr)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  if (ws_bytes < fa_bwd_phases_workspace_size(mask, p.total, H, D, dtype))
    return FA_ERR_INVALID_ARG;
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = const_cast<void*>(o);
  p.lse = const_cast<float*>(lse);
  p.dout = dout;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.delta = static_cast<float*>(workspace);
  // The accumulator follows the D_i rows whenever the workspace holds it, so
  // that a preprocess enqueued on its own (bit 0 alone) zeroes it for a fused
  // kernel enqueued by a later call on the same workspace.
  const size_t delta_bytes = fa::round256(static_cast<size_t>(p.total) * H * sizeof(float));
  const size_t acc_bytes = static_cast<size_t>(p.total) * H * D * sizeof(float);
  if (dtype == FA_BF16 && ws_bytes >= delta_bytes + acc_bytes)
    p.dq_accum = reinterpret_cast<float*>(static_cast<char*>(workspace) + delta_bytes);
  p.err.word = fa::err_word();
  if (p.err.word == nullptr) return FA_ERR_CUDA;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (dtype == FA_F32) {
    e = fa::launch_bwd_f32(p, s);
  } else {
    if (mask & (FA_BWD_PHASE_PREPROCESS | FA_BWD_PHASE_DKDV | FA_BWD_PHASE_DQ))
      e = fa::launch_bwd_bf16(p, s, mask & 7u);
    if (e == cudaSuccess && (mask & FA_BWD_PHASE_FUSED)) e = fa::launch_bwd_fused(p, s);
    if (e == cudaSuccess && (mask & FA_BWD_PHASE_DQ_CONVERT)) e = fa::launch_dq_convert(p, s);
  }
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return fa::cuda_status(e);
}

const char* fa_get_error_string(fa_status status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: bad pointer, size, alignment or layout";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: no kernel for this dtype / head dim / size";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA runtime call or kernel launch failed";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT: a bounded in-kernel wait ran out";
  }
  return "unknown fa_status";
}

fa_status fa_check_device_error(fa_stream_t stream, unsigned* where) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FA_ERR_CUDA;
  unsigned w[2] = {0, 0};
  if (cudaMemcpyFromSymbol(w, fa::g_err_word, sizeof(w)) != cudaSuccess) return FA_ERR_CUDA;
  if (where != nullptr) *where = w[1];
  if (w[0] == 0) return FA_OK;
  const unsigned zero[2] = {0, 0};
  if (cudaMemcpyToSymbol(fa::g_err_word, zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
  if (w[0] & fa::ERR_TIMEOUT) return FA_ERR_DEVICE_TIMEOUT;
  return FA_ERR_INVALID_ARG;  // ERR_BOUNDS: cu_seqlens inconsistent with the sizes
}

void fa_set_wait_budget(long long cycles) {
  fa::g_budget = cycles > 0 ? cycles : fa::kDefaultBudget;
}

fa_status fa_selftest_wait_timeout(long long cycles, fa_stream_t stream) {
  fa::DevErr e{fa::err_word(), cycles > 0 ? cycles : 1000000};
  if (e.word == nullptr) return FA_ERR_CUDA;
  return fa::launch_wait_selftest(e, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FA_OK
             : FA_ERR_CUDA;
}

fa_status fa_selftest_exp2(const float* x, float* y, long long n, fa_stream_t stream) {
  if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return FA_ERR_INVALID_ARG;
  return fa::cuda_status(fa::launch_exp2_selftest(x, y, n, reinterpret_cast<cudaStream_t>(stream)));
}

const char* fa_last_cuda_error_string(void) { return cudaGetErrorString(fa::g_last_cuda); }

fa_status fa_debug_set_trace(void* buffer, size_t bytes, int cta) {
#ifdef FA_DEBUG
  if (buffer == nullptr) {
    fa::g_trace = nullptr;
    return FA_OK;
  }
  if (bytes < static_cast<size_t>(FA_DEBUG_TRACE_BYTES) || cta < 0 ||
      (reinterpret_cast<uintptr_t>(buffer) & 7u) != 0)
    return FA_ERR_INVALID_ARG;
  fa::g_trace = static_cast<unsigned long long*>(buffer);
  fa::g_trace_cta = cta;
  return FA_OK;
#else
  (void)buffer;
  (void)bytes;
  (void)cta;
  return FA_ERR_UNSUPPORTED;
#endif
}

int fa_debug_build(void) {
#ifdef FA_DEBUG
  return 1;
#else
  return 0;
#endif
}

int fa_version(void) { return 100; }

}  // extern "C"
