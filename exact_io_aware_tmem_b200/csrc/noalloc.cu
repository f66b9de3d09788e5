// fa_bwd_noalloc: the backward pass with its scratch memory built into the
// library, for callers that cannot allocate device memory themselves.
//
// Who needs it: code that is handed only its input and output buffers and may
// not call cudaMalloc - for example a kernel plugin inside a host framework
// that owns every device allocation, or a latency-critical path where an
// allocation would synchronise the device or fail under a fixed memory
// budget. fa_bwd needs a caller-provided workspace (the D_i row terms); this
// entry point supplies it from a fixed, file-scope device array instead, and
// allocates nothing.
//
// The array is part of the loaded library: every GPU that loads the library
// holds FA_NOALLOC_SCRATCH_BYTES of device memory for it until the process
// exits. All calls on a device share it.
#include <mutex>

#include "../../include/fa.h"
#include "params.h"

namespace fa {
namespace {

// The shared scratch. Its contents persist from call to call; the backward
// pass re-initialises everything it reads (the preprocess kernel writes every
// D_i the later kernels use) before using it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device. In host code
// the name g_noalloc_scratch is only a host-side stand-in, so the address is
// looked up once per device with that device current.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace fa

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                    const float* lse, const void* dout, void* dq, void* dk,
                                    void* dv, int B, int H, int H_kv, int N, int D,
                                    fa_dtype dtype, int causal, float scale,
                                    const int* cu_seqlens, int max_seqlen,
                                    long long total_tokens, fa_stream_t stream) {
  // The sizes are checked exactly as fa_bwd checks them (same status for the
  // same mistake) before the scratch limit is applied.
  long long T = 0;
  const fa_status st = fa::check_bwd_sizes(B, H, H_kv, N, D, dtype, causal, cu_seqlens,
                                           max_seqlen, total_tokens, &T);
  if (st != FA_OK) return st;
  // The split backward needs only the D_i rows as scratch (the fused one
  // would also need a T x H x D fp32 dQ accumulator).
  const size_t need = fa_bwd_phases_workspace_size(FA_BWD_SPLIT, T, H, D, dtype);
  if (need == 0) return FA_ERR_INVALID_ARG;
  if (need > static_cast<size_t>(FA_NOALLOC_SCRATCH_BYTES)) return FA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const cudaError_t e = fa::scratch_address(&scratch);
  if (e != cudaSuccess) return fa::record_cuda(e);
  // ws_bytes = need (not the array's size), so the path never takes the
  // scratch for a dQ accumulator.
  return fa_bwd_phases(FA_BWD_SPLIT, q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, D, dtype,
                       causal, scale, cu_seqlens, max_seqlen, total_tokens, scratch, need, stream);
}
