// Decode attention without a caller-provided workspace.
//
// Some callers cannot hand the library device memory for its scratch: a
// plain C host that links only libtq and has no device allocator of its own,
// a decode loop that must not call cudaMalloc (which can synchronise the
// whole device and stall every other stream), or an engine that reserved
// all free device memory for its own pool at start-up.  For them this file
// keeps the decode scratch (rotated queries and split-K partial states) in
// one fixed, file-scope device array.  The array lives in every GPU that
// loads the library until the process exits.
#include <atomic>
#include <mutex>

#include "tq_common.cuh"
#include "tq_kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = TQ_NOALLOC_SCRATCH_BYTES;

// The shared scratch.  In host code this symbol is only a host-side stand-in;
// its device address comes from cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of g_decode_scratch on the current device, looked up once
// per device (with that device current) and cached.
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
      e = cudaGetSymbolAddress(&p, g_decode_scratch);
      if (e != cudaSuccess) return e;
      g_scratch_addr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" tq_status tq_decode_attention_noalloc(const tq_params *p, const tq_cache *c,
                                                 const void *q, tq_dtype q_dtype, int h_q,
                                                 const int32_t *len_dev, int max_len,
                                                 float softmax_scale, float *out,
                                                 tq_stream_t stream) {
  // The same validation as tq_decode_attention (every argument is checked on
  // the host before the scratch address is looked up or anything launches);
  // a request whose scratch need exceeds the array returns TQ_ERR_WORKSPACE.
  // Every byte of the scratch that the kernels read is written earlier in the
  // same call, so nothing needs clearing between calls.
  const tq_status pre = tq::decode_common(p, c, q, q_dtype, h_q, len_dev, max_len, nullptr, nullptr,
                                          TQ_BF16, nullptr, 0, softmax_scale, out, nullptr, 0,
                                          nullptr, /*validate_only=*/true);
  if (pre != TQ_OK) return pre;
  void *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess || scratch == nullptr) return TQ_ERR_CUDA;
  return tq::decode_common(p, c, q, q_dtype, h_q, len_dev, max_len, nullptr, nullptr, TQ_BF16, nullptr,
                           0, softmax_scale, out, scratch, kNoAllocScratchBytes, (cudaStream_t)stream);
}
