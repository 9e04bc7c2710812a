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
#include <cmath>
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

bool aligned_to(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int sm_count_current() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

}  // namespace

extern "C" tq_status tq_decode_attention_noalloc(const tq_params *p, const tq_cache *c,
                                                 const void *q, tq_dtype q_dtype, int h_q,
                                                 const int32_t *len_dev, int max_len,
                                                 float softmax_scale, float *out,
                                                 tq_stream_t stream) {
  if (!p || !c) return TQ_ERR_INVALID_ARGUMENT;
  if (p->d != tq::kD || p->group != tq::kGroup) return TQ_ERR_UNSUPPORTED;
  if (p->key_bits < 2 || p->key_bits > 4 || p->value_bits < 2 || p->value_bits > 4)
    return TQ_ERR_UNSUPPORTED;
  if (!p->pi || !p->s || !p->centroids || !p->boundaries) return TQ_ERR_INVALID_ARGUMENT;
  if (!c->data || c->batch < 1 || c->h_kv < 1 || c->capacity < tq::kTile ||
      c->capacity % tq::kTile || !aligned_to(c->data, 256))
    return TQ_ERR_INVALID_ARGUMENT;
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_UNSUPPORTED;
  if (!q || !len_dev || !out) return TQ_ERR_INVALID_ARGUMENT;
  if (h_q < c->h_kv || h_q % c->h_kv) return TQ_ERR_INVALID_ARGUMENT;
  if (h_q / c->h_kv > 8) return TQ_ERR_UNSUPPORTED;
  if (max_len < 0 || max_len > c->capacity) return TQ_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(softmax_scale)) return TQ_ERR_INVALID_ARGUMENT;
  if (!aligned_to(q, 16) || !aligned_to(out, 16) || !aligned_to(len_dev, 4))
    return TQ_ERR_INVALID_ARGUMENT;
  const int sms = sm_count_current();
  if (sms <= 0) return TQ_ERR_CUDA;
  const tq::DecodePlan P = tq::make_decode_plan(c->batch, c->h_kv, h_q, max_len, sms, p->key_bits, p->value_bits);
  if (P.total_bytes > kNoAllocScratchBytes) return TQ_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess || scratch == nullptr) return TQ_ERR_CUDA;
  tq::DecodeArgs a;
  a.pi = p->pi; a.s = p->s; a.centroids = p->centroids;
  a.data = c->data; a.q = q; a.q_dtype = q_dtype; a.len = len_dev;
  a.batch = c->batch; a.h_kv = c->h_kv; a.h_q = h_q; a.ntiles = c->capacity / tq::kTile;
  a.max_len = max_len; a.key_bits = p->key_bits; a.value_bits = p->value_bits;
  a.softmax_scale = softmax_scale; a.nsplit = P.nsplit; a.tiles_per_split = P.tiles_per_split;
  a.part_stride = P.nsplit;
  a.win_k = nullptr; a.win_v = nullptr; a.win_dtype = TQ_BF16; a.win_len = nullptr; a.win_cap = 0;
  a.qt = 1; a.q_tstride = 1; a.q_t0 = 0; a.len_sub = 0;
  a.num_sms = sms;
  tq::bind_workspace(a, P, scratch);
  a.out = out;
  // Every byte of the scratch that the kernels read is written earlier in the
  // same call, so nothing needs clearing between calls.
  if (tq::launch_decode(a, (cudaStream_t)stream) != cudaSuccess) return TQ_ERR_CUDA;
  return TQ_OK;
}
