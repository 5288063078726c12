// kvtc_decode_attention_noalloc: decode attention for callers that cannot allocate
// device memory themselves.
//
// Some hosts embed this library where no allocator is reachable: a caller inside an
// inference runtime that owns every device allocation through its own pool, a plugin
// that may only use buffers handed to it, or code that runs while the device heap is
// frozen for graph replay.  Such callers can pass the query, the cache and the output,
// but not the split-K scratch buffer that kvtc_decode_attention takes.  This entry point
// uses a scratch array that lives in the library itself instead: a file-scope
// __device__ array of fixed size, created once per device when the library's kernels
// are loaded and kept until the process exits.  Nothing is allocated per call.
#include <cuda_runtime.h>

#include <mutex>

#include "kvtc_internal.h"

namespace kvtc {
namespace {

// 16 MiB: the arrival tickets and split-K partials of seven 131072-token sequences of a
// 32-query-head model (kvtc_decode_workspace_bytes gives the exact need of a call).  The
// array is zero when the module loads and every call returns its tickets to zero.
constexpr size_t kScratchBytes = 16u << 20;
constexpr int kMaxDevices = 64;

// In host code this name is only a handle for cudaGetSymbolAddress; it is not a device
// address and must never be passed to a kernel directly.  The address found for a device
// is kept for the life of the process (it does not survive cudaDeviceReset).
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once per device).
kvtc_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(KVTC_EINVAL, "device index beyond the supported range");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress (decode scratch)");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KVTC_OK;
}

}  // namespace
}  // namespace kvtc

using namespace kvtc;

extern "C" kvtc_status kvtc_decode_attention_noalloc(const kvtc_plan* plan, const kvtc_cache* cache, int layer,
                                                     const void* q, kvtc_dtype q_dtype, const int32_t* seq_lens,
                                                     int max_seq_len, float softmax_scale, void* out,
                                                     kvtc_dtype out_dtype, void* stream) {
  if (!plan || !cache) return fail(KVTC_EINVAL, "null argument");
  const uint64_t need = kvtc_decode_workspace_bytes(plan, cache->n_seq, max_seq_len);
  if (need > kScratchBytes)
    return fail(KVTC_ECAPACITY,
                "decode needs more scratch than the library's fixed 16 MiB array holds; "
                "pass a workspace to kvtc_decode_attention instead");
  void* scratch = nullptr;
  kvtc_status st = scratch_address(&scratch);
  if (st != KVTC_OK) return st;
  return kvtc_decode_attention(plan, cache, layer, q, q_dtype, seq_lens, max_seq_len, softmax_scale, out,
                               out_dtype, scratch, kScratchBytes, stream);
}
