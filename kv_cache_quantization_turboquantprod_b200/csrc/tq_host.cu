// C-ABI entry points (include/tq.h): host-side validation, the Lloyd-Max
// codebook, workspace planning and kernel launches.  Nothing here allocates
// device memory or synchronises.
#include <math.h>
#include <string.h>

#include <atomic>
#include <cmath>
#include <mutex>
#include <vector>

#include "tq_common.cuh"
#include "tq_kernels.h"

namespace {

using tq::kD;
using tq::kGroup;
using tq::kTile;

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];  // 0 = not yet queried

// SM count of the current device (cached per device).
cudaError_t current_sm_count(int *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices) {
    int v = g_sm_count[dev].load(std::memory_order_relaxed);
    if (v > 0) { *out = v; return cudaSuccess; }
  }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices) g_sm_count[dev].store(sms, std::memory_order_relaxed);
  *out = sms;
  return cudaSuccess;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Bound of the kernels' pipeline waits (tq_set_wait_limit_ns).
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;
std::atomic<unsigned long long> g_wait_ns{kDefaultWaitNs};
// Tests of the timeout path (tq_test_withhold_handoffs).
std::atomic<int> g_withhold{0};
// Tests of the sign refinement (tq_test_sign_refine_threshold).
std::atomic<float> g_refine_z{tq::kSignRefineZ};

// Sticky per-device error word (TQ_ERRF_* bits) that kernels set when they
// give up on a bounded wait, and the per-device count of QJL sign bits the
// append kernels re-decided in float64 (tq_test_refine_count); their device
// addresses are looked up once per device.
__device__ unsigned int g_error_word;
__device__ unsigned long long g_refine_count;
std::atomic<unsigned int *> g_error_addr[kMaxDevices];
std::atomic<unsigned long long *> g_refine_addr[kMaxDevices];
std::mutex g_symbol_mutex;

template <class T>
cudaError_t cached_symbol_address(const T &symbol, std::atomic<T *> (&cache)[kMaxDevices], T **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  T *p = cache[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_symbol_mutex);
    p = cache[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
      void *v = nullptr;
      e = cudaGetSymbolAddress(&v, symbol);
      if (e != cudaSuccess) return e;
      p = static_cast<T *>(v);
      cache[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return cudaSuccess;
}

cudaError_t error_word_address(unsigned int **out) {
  return cached_symbol_address(g_error_word, g_error_addr, out);
}

cudaError_t refine_count_address(unsigned long long **out) {
  return cached_symbol_address(g_refine_count, g_refine_addr, out);
}

// Wait limits and error word of a launch on the current device.
template <class Args>
cudaError_t set_wait_fields(Args &a) {
  const unsigned long long ns = g_wait_ns.load(std::memory_order_relaxed);
  a.wait_ns = ns;
  a.wait_hint_ns = (unsigned int)(ns < 1000000ull ? ns : 1000000ull);
  a.test_withhold = g_withhold.load(std::memory_order_relaxed);
  return error_word_address(&a.errors);
}

tq_status check_params(const tq_params *p) {
  if (!p) return TQ_ERR_INVALID_ARGUMENT;
  if ((p->d != 64 && p->d != 128 && p->d != 256) || p->group != kGroup) return TQ_ERR_UNSUPPORTED;
  if (p->key_bits < 2 || p->key_bits > 4) return TQ_ERR_UNSUPPORTED;
  if (p->value_bits < 2 || p->value_bits > 4) return TQ_ERR_UNSUPPORTED;
  if (!p->pi || !p->s || !p->centroids || !p->boundaries) return TQ_ERR_INVALID_ARGUMENT;
  if (!aligned(p->pi, 16) || !aligned(p->s, 16)) return TQ_ERR_INVALID_ARGUMENT;
  if (p->value_mode != TQ_VALUES_GROUP && p->value_mode != TQ_VALUES_MSE) return TQ_ERR_UNSUPPORTED;
  if (p->value_mode == TQ_VALUES_MSE && (!p->v_centroids || !p->v_boundaries)) return TQ_ERR_INVALID_ARGUMENT;
  return TQ_OK;
}

tq_status check_cache(const tq_cache *c) {
  if (!c || !c->data) return TQ_ERR_INVALID_ARGUMENT;
  if (c->batch < 1 || c->h_kv < 1 || c->capacity < kTile || c->capacity % kTile)
    return TQ_ERR_INVALID_ARGUMENT;
  if (!aligned(c->data, 256)) return TQ_ERR_INVALID_ARGUMENT;
  return TQ_OK;
}

bool dtype_ok(tq_dtype d) { return d == TQ_F32 || d == TQ_BF16; }

double phi(double x) { return std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI); }

// P(a < Z <= b), Z standard normal; infinite ends allowed.
double normal_mass(double a, double b) {
  const double fa = std::isinf(a) ? (a < 0 ? 0.0 : 1.0) : 0.5 * std::erfc(-a / std::sqrt(2.0));
  const double fb = std::isinf(b) ? (b < 0 ? 0.0 : 1.0) : 0.5 * std::erfc(-b / std::sqrt(2.0));
  return fb - fa;
}

}  // namespace

extern "C" {

const char *tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_INVALID_ARGUMENT: return "TQ_ERR_INVALID_ARGUMENT";
    case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
    case TQ_ERR_CAPACITY: return "TQ_ERR_CAPACITY";
    case TQ_ERR_WORKSPACE: return "TQ_ERR_WORKSPACE";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
    case TQ_ERR_INTERNAL: return "TQ_ERR_INTERNAL";
  }
  return "TQ_UNKNOWN_STATUS";
}

tq_status tq_make_codebook(int mse_bits, int d, double *centroids, double *boundaries) {
  if (!centroids || (!boundaries && mse_bits > 0)) return TQ_ERR_INVALID_ARGUMENT;
  if (mse_bits < 1 || mse_bits > 4 || d < 1) return TQ_ERR_UNSUPPORTED;
  const int levels = 1 << mse_bits;
  const double sigma = 1.0 / std::sqrt((double)d);
  // Lloyd's iteration: cell boundaries at midpoints, centroids at the
  // conditional means of N(0, sigma^2) over the cells.
  std::vector<double> c(levels), t(levels - 1), cn(levels);
  for (int i = 0; i < levels; ++i) c[i] = sigma * (-2.0 + 4.0 * i / (levels - 1));
  for (int it = 0; it < 100000; ++it) {
    for (int i = 0; i + 1 < levels; ++i) t[i] = 0.5 * (c[i] + c[i + 1]);
    double delta = 0.0;
    for (int i = 0; i < levels; ++i) {
      const double a = (i == 0) ? -INFINITY : t[i - 1] / sigma;
      const double b = (i == levels - 1) ? INFINITY : t[i] / sigma;
      const double pa = std::isinf(a) ? 0.0 : phi(a);
      const double pb = std::isinf(b) ? 0.0 : phi(b);
      cn[i] = sigma * (pa - pb) / normal_mass(a, b);
      delta = std::fmax(delta, std::fabs(cn[i] - c[i]));
    }
    c.swap(cn);
    if (delta < 1e-14 * sigma) break;
  }
  // the law is symmetric: make the fixed point exactly antisymmetric (the
  // iteration leaves last-bit differences), c_i = -c_{n-1-i}
  for (int i = 0; i < levels / 2; ++i) {
    const double m = 0.5 * (c[levels - 1 - i] - c[i]);
    c[i] = -m;
    c[levels - 1 - i] = m;
  }
  for (int i = 0; i + 1 < levels; ++i) t[i] = 0.5 * (c[i] + c[i + 1]);
  for (int i = 0; i < levels; ++i) centroids[i] = c[i];
  for (int i = 0; i + 1 < levels; ++i) boundaries[i] = t[i];
  return TQ_OK;
}

tq_status tq_sketch_product(const tq_params *p, double *s_pit, tq_stream_t stream) {
  if (!p || !s_pit || !aligned(s_pit, 16)) return TQ_ERR_INVALID_ARGUMENT;
  if (p->d != 64 && p->d != 128 && p->d != 256) return TQ_ERR_UNSUPPORTED;
  if (!p->pi || !p->s || !aligned(p->pi, 16) || !aligned(p->s, 16)) return TQ_ERR_INVALID_ARGUMENT;
  return tq::launch_sketch_product(p->pi, p->s, p->d, s_pit, (cudaStream_t)stream) == cudaSuccess ? TQ_OK
                                                                                               : TQ_ERR_CUDA;
}

tq_status tq_prepare_operands(const tq_params *p, void *dst, tq_stream_t stream) {
  if (!p || !dst || !aligned(dst, 128)) return TQ_ERR_INVALID_ARGUMENT;
  if (p->d != 128) return TQ_ERR_UNSUPPORTED;
  if (!p->pi || !p->s_pit || !aligned(p->pi, 16) || !aligned(p->s_pit, 16)) return TQ_ERR_INVALID_ARGUMENT;
  return tq::launch_prepare_operands(p->pi, p->s_pit, dst, (cudaStream_t)stream) == cudaSuccess ? TQ_OK
                                                                                                : TQ_ERR_CUDA;
}

size_t tq_record_bytes(const tq_params *p) {
  if (check_params(p) != TQ_OK) return 0;
  return (size_t)tq::TileLayout::make(p->key_bits, p->value_bits, p->value_mode, p->d).record_bytes();
}

size_t tq_cache_bytes(const tq_params *p, int batch, int h_kv, int capacity) {
  if (check_params(p) != TQ_OK) return 0;
  if (batch < 1 || h_kv < 1 || capacity < kTile || capacity % kTile) return 0;
  const tq::TileLayout L = tq::TileLayout::make(p->key_bits, p->value_bits, p->value_mode, p->d);
  return (size_t)batch * h_kv * (size_t)(capacity / kTile) * (size_t)L.tile_bytes;
}

tq_status tq_quantize_append(const tq_params *p, const tq_cache *c, const void *k,
                             const void *v, tq_dtype dtype, int T, const int32_t *len_host,
                             const int32_t *n_new_host, tq_stream_t stream) {
  tq_status st = check_params(p);
  if (st != TQ_OK) return st;
  if ((st = check_cache(c)) != TQ_OK) return st;
  if (!dtype_ok(dtype)) return TQ_ERR_UNSUPPORTED;
  if (T < 0 || !len_host) return TQ_ERR_INVALID_ARGUMENT;
  if (c->batch > TQ_MAX_BATCH) return TQ_ERR_CAPACITY;
  if (T == 0) return TQ_OK;
  if (!k || !v || !aligned(k, 16) || !aligned(v, 16)) return TQ_ERR_INVALID_ARGUMENT;
  if (!p->s_pit || !aligned(p->s_pit, 16)) return TQ_ERR_INVALID_ARGUMENT;
  tq::AppendArgs a;
  memset(&a, 0, sizeof(a));
  for (int b = 0; b < c->batch; ++b) {
    const int len = len_host[b];
    const int nn = n_new_host ? n_new_host[b] : T;
    if (len < 0 || nn < 0 || nn > T) return TQ_ERR_INVALID_ARGUMENT;
    if ((long long)len + nn > c->capacity) return TQ_ERR_CAPACITY;
    a.lens[b] = len;
    a.nnew[b] = nn;
  }
  a.d = p->d;
  a.pi = p->pi; a.s = p->s; a.centroids = p->centroids; a.boundaries = p->boundaries;
  a.value_mode = p->value_mode; a.v_centroids = p->v_centroids; a.v_boundaries = p->v_boundaries;
  a.data = c->data; a.k = k; a.v = v;
  a.batch = c->batch; a.h_kv = c->h_kv; a.ntiles = c->capacity / kTile; a.T = T;
  a.key_bits = p->key_bits; a.value_bits = p->value_bits; a.dtype = dtype;
  int sms = 0;
  if (current_sm_count(&sms) != cudaSuccess) return TQ_ERR_CUDA;
  if (set_wait_fields(a) != cudaSuccess) return TQ_ERR_CUDA;
  a.refine_z = g_refine_z.load(std::memory_order_relaxed);
  a.s_pit = p->s_pit;
  a.tc_ops = p->d == 128 ? p->tc_operands : nullptr;
  if (refine_count_address(&a.refine_count) != cudaSuccess) return TQ_ERR_CUDA;
  const cudaError_t e = tq::quantize_tc_supported(a) ? tq::launch_quantize_tc(a, sms, (cudaStream_t)stream)
                                                    : tq::launch_quantize_simt(a, sms, (cudaStream_t)stream);
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  return TQ_OK;
}

size_t tq_decode_workspace_size(const tq_params *p, const tq_cache *c, int h_q, int max_len) {
  if (check_params(p) != TQ_OK || check_cache(c) != TQ_OK) return 0;
  if (h_q < c->h_kv || h_q % c->h_kv || max_len < 0 || max_len > c->capacity) return 0;
  int sms = 0;
  if (current_sm_count(&sms) != cudaSuccess) return 0;
  return tq::make_decode_plan(c->batch, c->h_kv, h_q, max_len, sms, p->key_bits, p->value_bits,
                              p->value_mode, p->d).total_bytes;
}

namespace {

// Query tokens of a prefill chunk that one decode pass takes together: the
// largest power of two ts <= t_chunk with G * ts <= 4 that the tensor-core
// kernel builds (so the pass reads every KV tile once for ts tokens), else 1.
// Wider passes (8 heads per worker thread) measured slower per token than
// single-token passes at GQA 4.
int prefill_tokens_per_pass(const tq_params *p, int gqa, int t_chunk) {
  int ts = 1;
  while (2 * ts <= t_chunk && gqa * 2 * ts <= 4 &&
         tq::decode_tc_supported(p->key_bits, p->value_bits, gqa * 2 * ts, p->value_mode, p->d))
    ts *= 2;
  return ts;
}

}  // namespace

int tq_prefill_tokens_per_pass(const tq_params *p, int h_q, int h_kv, int t_chunk) {
  if (check_params(p) != TQ_OK || h_kv < 1 || h_q < h_kv || h_q % h_kv || t_chunk < 1) return 0;
  return prefill_tokens_per_pass(p, h_q / h_kv, t_chunk);
}

size_t tq_prefill_workspace_size(const tq_params *p, const tq_cache *c, int h_q, int t_chunk,
                                 int max_len) {
  if (check_params(p) != TQ_OK || check_cache(c) != TQ_OK) return 0;
  if (h_q < c->h_kv || h_q % c->h_kv || t_chunk < 1 || max_len < t_chunk || max_len > c->capacity)
    return 0;
  int sms = 0;
  if (current_sm_count(&sms) != cudaSuccess) return 0;
  const int ts = prefill_tokens_per_pass(p, h_q / c->h_kv, t_chunk);
  return tq::make_decode_plan(c->batch, c->h_kv, h_q * ts, max_len, sms, p->key_bits, p->value_bits,
                              p->value_mode, p->d)
      .total_bytes;
}

tq_status tq_prefill_attention(const tq_params *p, const tq_cache *c, const void *q, tq_dtype q_dtype,
                               int h_q, int t_chunk, const int32_t *len_dev, int max_len,
                               float softmax_scale, float *out, void *workspace, size_t workspace_bytes,
                               tq_stream_t stream) {
  tq_status st = check_params(p);
  if (st != TQ_OK) return st;
  if ((st = check_cache(c)) != TQ_OK) return st;
  if (!dtype_ok(q_dtype)) return TQ_ERR_UNSUPPORTED;
  if (!q || !len_dev || !out) return TQ_ERR_INVALID_ARGUMENT;
  if (h_q < c->h_kv || h_q % c->h_kv) return TQ_ERR_INVALID_ARGUMENT;
  if (h_q / c->h_kv > 8) return TQ_ERR_UNSUPPORTED;
  if (t_chunk < 1 || max_len < t_chunk || max_len > c->capacity) return TQ_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(softmax_scale)) return TQ_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(len_dev, 4)) return TQ_ERR_INVALID_ARGUMENT;
  if (!workspace || !aligned(workspace, 256)) return TQ_ERR_WORKSPACE;
  int sms = 0;
  if (current_sm_count(&sms) != cudaSuccess) return TQ_ERR_CUDA;
  const int G = h_q / c->h_kv;
  const int ts = prefill_tokens_per_pass(p, G, t_chunk);
  if (workspace_bytes < tq::make_decode_plan(c->batch, c->h_kv, h_q * ts, max_len, sms, p->key_bits,
                                             p->value_bits, p->value_mode, p->d).total_bytes)
    return TQ_ERR_WORKSPACE;
  // passes of ts tokens (the last one of the largest power of two that is
  // left); pass tokens t0 .. t0 + n - 1 see len - (t_chunk - 1 - t) tokens
  for (int t0 = 0; t0 < t_chunk;) {
    int n = ts;
    while (n > t_chunk - t0) n >>= 1;
    const int len_sub = t_chunk - t0 - n;
    const int ml = max_len - len_sub;
    const tq::DecodePlan P = tq::make_decode_plan(c->batch, c->h_kv, h_q * n, ml, sms, p->key_bits, p->value_bits,
                                                  p->value_mode, p->d);
    tq::DecodeArgs a;
    a.d = p->d;
    a.pi = p->pi; a.s = p->s; a.centroids = p->centroids;
    a.value_mode = p->value_mode; a.v_centroids = p->v_centroids;
    a.data = c->data; a.q = q; a.q_dtype = q_dtype; a.len = len_dev;
    a.batch = c->batch; a.h_kv = c->h_kv; a.h_q = h_q * n; a.ntiles = c->capacity / kTile;
    a.max_len = ml; a.key_bits = p->key_bits; a.value_bits = p->value_bits;
    a.softmax_scale = softmax_scale; a.nsplit = P.nsplit; a.tiles_per_split = P.tiles_per_split;
    a.part_stride = P.nsplit;
    a.win_k = nullptr; a.win_v = nullptr; a.win_dtype = TQ_BF16; a.win_len = nullptr; a.win_cap = 0;
    a.qt = n; a.q_tstride = t_chunk; a.q_t0 = t0; a.len_sub = len_sub;
    a.num_sms = sms;
    if (set_wait_fields(a) != cudaSuccess) return TQ_ERR_CUDA;
    tq::bind_workspace(a, P, workspace);
    a.out = out;
    if (tq::launch_decode(a, (cudaStream_t)stream) != cudaSuccess) return TQ_ERR_CUDA;
    t0 += n;
  }
  return TQ_OK;
}

}  // extern "C"

namespace tq {

// Shared by tq_decode_attention, tq_decode_attention_window (win_k null: no
// window) and tq_decode_attention_noalloc (the library's scratch as workspace).
tq_status decode_common(const tq_params *p, const tq_cache *c, const void *q, tq_dtype q_dtype,
                        int h_q, const int32_t *len_dev, int max_len, const void *win_k,
                        const void *win_v, tq_dtype win_dtype, const int32_t *win_len_dev,
                        int win_cap, float softmax_scale, float *out, void *workspace,
                        size_t workspace_bytes, cudaStream_t stream, bool validate_only) {
  tq_status st = check_params(p);
  if (st != TQ_OK) return st;
  if ((st = check_cache(c)) != TQ_OK) return st;
  if (!dtype_ok(q_dtype)) return TQ_ERR_UNSUPPORTED;
  if (!q || !len_dev || !out) return TQ_ERR_INVALID_ARGUMENT;
  if (h_q < c->h_kv || h_q % c->h_kv) return TQ_ERR_INVALID_ARGUMENT;
  if (h_q / c->h_kv > 8) return TQ_ERR_UNSUPPORTED;
  if (max_len < 0 || max_len > c->capacity) return TQ_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(softmax_scale)) return TQ_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(len_dev, 4)) return TQ_ERR_INVALID_ARGUMENT;
  if (win_k) {
    if (!dtype_ok(win_dtype)) return TQ_ERR_UNSUPPORTED;
    if (!win_v || !win_len_dev || win_cap < 1 || win_cap > kTile) return TQ_ERR_INVALID_ARGUMENT;
    if (!aligned(win_k, 16) || !aligned(win_v, 16) || !aligned(win_len_dev, 4))
      return TQ_ERR_INVALID_ARGUMENT;
  }
  if (validate_only) return TQ_OK;
  if (!workspace || !aligned(workspace, 256)) return TQ_ERR_WORKSPACE;
  int sms = 0;
  if (current_sm_count(&sms) != cudaSuccess) return TQ_ERR_CUDA;
  const tq::DecodePlan P = tq::make_decode_plan(c->batch, c->h_kv, h_q, max_len, sms, p->key_bits, p->value_bits,
                                                p->value_mode, p->d);
  if (workspace_bytes < P.total_bytes) return TQ_ERR_WORKSPACE;
  tq::DecodeArgs a;
  a.d = p->d;
  a.pi = p->pi; a.s = p->s; a.centroids = p->centroids;
  a.value_mode = p->value_mode; a.v_centroids = p->v_centroids;
  a.data = c->data; a.q = q; a.q_dtype = q_dtype; a.len = len_dev;
  a.batch = c->batch; a.h_kv = c->h_kv; a.h_q = h_q; a.ntiles = c->capacity / kTile;
  a.max_len = max_len; a.key_bits = p->key_bits; a.value_bits = p->value_bits;
  a.softmax_scale = softmax_scale; a.nsplit = P.nsplit; a.tiles_per_split = P.tiles_per_split;
  a.part_stride = win_k ? P.nsplit + 1 : P.nsplit;
  a.win_k = win_k; a.win_v = win_v; a.win_dtype = win_dtype; a.win_len = win_len_dev;
  a.win_cap = win_cap;
  a.qt = 1; a.q_tstride = 1; a.q_t0 = 0; a.len_sub = 0;
  a.num_sms = sms;
  if (set_wait_fields(a) != cudaSuccess) return TQ_ERR_CUDA;
  tq::bind_workspace(a, P, workspace);
  a.out = out;
  if (tq::launch_decode(a, stream) != cudaSuccess) return TQ_ERR_CUDA;
  return TQ_OK;
}

}  // namespace tq

extern "C" {

tq_status tq_decode_attention(const tq_params *p, const tq_cache *c, const void *q,
                              tq_dtype q_dtype, int h_q, const int32_t *len_dev, int max_len,
                              float softmax_scale, float *out, void *workspace,
                              size_t workspace_bytes, tq_stream_t stream) {
  return tq::decode_common(p, c, q, q_dtype, h_q, len_dev, max_len, nullptr, nullptr, TQ_BF16, nullptr,
                           0, softmax_scale, out, workspace, workspace_bytes, (cudaStream_t)stream);
}

tq_status tq_decode_attention_window(const tq_params *p, const tq_cache *c, const void *q,
                                     tq_dtype q_dtype, int h_q, const int32_t *len_dev,
                                     int max_len, const void *win_k, const void *win_v,
                                     tq_dtype win_dtype, const int32_t *win_len_dev, int win_cap,
                                     float softmax_scale, float *out, void *workspace,
                                     size_t workspace_bytes, tq_stream_t stream) {
  if (!win_k) return TQ_ERR_INVALID_ARGUMENT;
  return tq::decode_common(p, c, q, q_dtype, h_q, len_dev, max_len, win_k, win_v, win_dtype,
                           win_len_dev, win_cap, softmax_scale, out, workspace, workspace_bytes,
                           (cudaStream_t)stream);
}

tq_status tq_set_wait_limit_ns(unsigned long long ns) {
  g_wait_ns.store(ns == 0 ? kDefaultWaitNs : ns, std::memory_order_relaxed);
  return TQ_OK;
}

tq_status tq_test_withhold_handoffs(int on) {
  g_withhold.store(on ? 1 : 0, std::memory_order_relaxed);
  return TQ_OK;
}

tq_status tq_test_sign_refine_threshold(double z) {
  if (!(z >= 0.0)) return TQ_ERR_INVALID_ARGUMENT;
  g_refine_z.store(z == 0.0 ? tq::kSignRefineZ : (float)z, std::memory_order_relaxed);
  return TQ_OK;
}

tq_status tq_test_refine_count(unsigned long long *count, int clear) {
  if (!count) return TQ_ERR_INVALID_ARGUMENT;
  unsigned long long *p = nullptr;
  if (refine_count_address(&p) != cudaSuccess) return TQ_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return TQ_ERR_CUDA;
  unsigned long long v = 0;
  if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return TQ_ERR_CUDA;
  *count = v;
  if (clear && cudaMemset(p, 0, sizeof(v)) != cudaSuccess) return TQ_ERR_CUDA;
  if (clear && cudaDeviceSynchronize() != cudaSuccess) return TQ_ERR_CUDA;
  return TQ_OK;
}

tq_status tq_device_errors(uint32_t *flags, int clear) {
  if (!flags) return TQ_ERR_INVALID_ARGUMENT;
  unsigned int *p = nullptr;
  if (error_word_address(&p) != cudaSuccess) return TQ_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return TQ_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return TQ_ERR_CUDA;
  *flags = v;
  if (clear && cudaMemset(p, 0, sizeof(v)) != cudaSuccess) return TQ_ERR_CUDA;
  if (clear && cudaDeviceSynchronize() != cudaSuccess) return TQ_ERR_CUDA;
  return TQ_OK;
}

tq_status tq_dequantize(const tq_params *p, const tq_cache *c, int b, int start, int count,
                        float *k_out, float *v_out, tq_stream_t stream) {
  tq_status st = check_params(p);
  if (st != TQ_OK) return st;
  if ((st = check_cache(c)) != TQ_OK) return st;
  if (b < 0 || b >= c->batch || start < 0 || count < 0) return TQ_ERR_INVALID_ARGUMENT;
  if ((long long)start + count > c->capacity) return TQ_ERR_INVALID_ARGUMENT;
  if (count == 0) return TQ_OK;
  if (!k_out || !v_out || !aligned(k_out, 4) || !aligned(v_out, 4)) return TQ_ERR_INVALID_ARGUMENT;
  tq::DequantArgs a;
  a.d = p->d;
  a.pi = p->pi; a.s = p->s; a.centroids = p->centroids; a.data = c->data;
  a.value_mode = p->value_mode; a.v_centroids = p->v_centroids;
  a.h_kv = c->h_kv; a.ntiles = c->capacity / kTile; a.b = b; a.start = start; a.count = count;
  a.key_bits = p->key_bits; a.value_bits = p->value_bits; a.k_out = k_out; a.v_out = v_out;
  if (tq::launch_dequantize(a, (cudaStream_t)stream) != cudaSuccess) return TQ_ERR_CUDA;
  return TQ_OK;
}

}  // extern "C"
