// Internal launch interface between the C-ABI host layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>
#include <utility>

#include "tq.h"

namespace tq {

// Launch `kernel` on `stream` with programmatic stream serialization: it may
// start while its predecessor in the stream is still running and must call
// pdl_wait() (sm100.cuh) before it reads that predecessor's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Arguments of one quantize_append launch.  Passed by value as a
// __grid_constant__ kernel parameter (12 KB of per-sequence lengths and tile
// offsets; CUDA 12.1+ allows kernel parameters up to 32764 bytes).
struct AppendArgs {
  int d;                                 // head dim (64, 128 or 256)
  const float *pi, *s, *centroids, *boundaries;
  int value_mode;                        // tq_value_mode
  const float *v_centroids, *v_boundaries;  // MSE values' codebook
  void *data;
  const void *k, *v;
  int batch, h_kv, ntiles, T;
  int key_bits, value_bits;
  tq_dtype dtype;
  int lens[TQ_MAX_BATCH];
  int nnew[TQ_MAX_BATCH];
  // tensor-core path: 128-token tiles per (sequence, head); sequence b owns
  // tiles [tstart[b], tstart[b + 1])
  int tstart[TQ_MAX_BATCH + 1];
  int total_tiles;
  // bounded pipeline waits (tensor-core path): limit, suspend hint, and the
  // sticky per-device error word a timeout sets (TQ_ERRF_QUANTIZE_WAIT)
  unsigned long long wait_ns;
  unsigned int wait_hint_ns;
  unsigned int *errors;
  // tests of the timeout path: the loader withholds its operand hand-offs
  int test_withhold;
  // QJL signs with |(S r)_j| below this are re-decided in float64 (with
  // s_pit = S Pi^T in float64); the number re-decided is added to
  // *refine_count
  float refine_z;
  const double *s_pit;
  unsigned long long *refine_count;
  // the tensor-core append's prepared operand images (tq_prepare_operands),
  // or nullptr: then every CTA builds them from pi and s_pit
  const void *tc_ops;
};

// Split-K plan of one decode call (host-computed, identical in the
// workspace-size query and the launch).
struct DecodePlan {
  int nsplit;          // splits per (b, h_kv)
  int tiles_per_split; // 128-token tiles per split
  size_t status_bytes; // status word (nonzero: a kernel gave up on a bounded wait)
  size_t qrot_bytes;   // [B][H_q][2][d] fp32
  size_t part_bytes;   // [B][H_q][nsplit + 1][d + 2] fp32 (acc, m, l); the extra slot
                       // holds the recent-token window's partial state
  size_t qblock_bytes; // per (b, h_kv) query block of the tensor-core kernel (0: SIMT path)
  size_t order_bytes;  // the tensor-core kernel's work items, largest first (0: SIMT path)
  size_t total_bytes;
};

struct DecodeArgs {
  int d;                       // head dim (64, 128 or 256)
  const float *pi, *s, *centroids;
  int value_mode;              // tq_value_mode (MSE: partials in the rotated space)
  const float *v_centroids;    // MSE values' codebook
  const void *data;
  const void *q;
  tq_dtype q_dtype;
  const int32_t *len;
  int batch, h_kv, h_q, ntiles, max_len;
  int key_bits, value_bits;
  float softmax_scale;
  int nsplit, tiles_per_split;
  int part_stride;  // partial slots per (b, hq): nsplit, or nsplit + 1 with a window
  // recent-token window kept exactly (win_k == nullptr: none)
  const void *win_k, *win_v;
  tq_dtype win_dtype;
  const int32_t *win_len;
  int win_cap;
  // workspace words: status[0] nonzero once a kernel of this call gave up on a
  // bounded wait (combine then writes NaN rows); status[1] nonzero when the
  // codebook needs the SIMT split-K kernel (set by the query-block kernel)
  int *status;
  float *qrot;   // workspace: [B][H_q][2][d]
  float *part;   // workspace: [B][H_q][part_stride][d+2]
  uint8_t *qblocks;  // workspace: [B][H_kv] query blocks (tensor-core path)
  // workspace: the tensor-core kernel's work items {split * B * H_kv + b *
  // H_kv + h, the sequence's length clamped to [0, max_len]}, ordered by tile
  // count, largest first (written by the query-block kernel; CTA i takes
  // item order[i])
  int2 *order;
  int num_sms;
  float *out;    // [B][H_q][d]
  // Chunked prefill (qt > 1 or q_tstride > 1): the h_q heads of a sequence
  // are qt query tokens x (h_q / qt) heads; q and out are [B][q_tstride][H][d]
  // blocks (H = h_q / qt) of which this call covers tokens q_t0 .. q_t0 + qt
  // - 1.  The call attends over len[b] - len_sub cache tokens; query token t
  // of it sees the first len[b] - len_sub - (qt - 1 - t).  Decode: qt = 1,
  // q_tstride = 1, q_t0 = 0, len_sub = 0.
  int qt, q_tstride, q_t0, len_sub;
  // bounded pipeline waits: limit, suspend hint, sticky per-device error word
  // a timeout sets (TQ_ERRF_DECODE_WAIT)
  unsigned long long wait_ns;
  unsigned int wait_hint_ns;
  unsigned int *errors;
  // tests of the timeout path: the producer withholds the tile copies
  int test_withhold;
};

// Element offset of virtual head hv's row of sequence b in q / out (rows of
// a.d elements).  Virtual heads of KV head h are h * G' + t * (G' / qt) + g
// (G' = h_q / h_kv).
__host__ __device__ inline size_t qrow_offset(const DecodeArgs &a, int b, int hv) {
  if (a.qt == 1 && a.q_tstride == 1) return ((size_t)b * a.h_q + hv) * a.d;
  const int gv = a.h_q / a.h_kv, greal = gv / a.qt, hreal = a.h_q / a.qt;
  const int h = hv / gv, r = hv % gv, t = r / greal, g = r % greal;
  return (((size_t)b * a.q_tstride + a.q_t0 + t) * hreal + (size_t)h * greal + g) * a.d;
}

struct DequantArgs {
  int d;
  const float *pi, *s, *centroids;
  int value_mode;
  const float *v_centroids;
  const void *data;
  int h_kv, ntiles, b, start, count;
  int key_bits, value_bits;
  float *k_out, *v_out;
};

DecodePlan make_decode_plan(int batch, int h_kv, int h_q, int max_len, int num_sms,
                            int key_bits, int value_bits, int value_mode = 0, int d = 128);

cudaError_t launch_quantize_simt(const AppendArgs &a, int num_sms, cudaStream_t stream);
// Tensor-core quantize-append (bf16 K/V, appends of 64+ tokens).
bool quantize_tc_supported(const AppendArgs &a);
cudaError_t launch_quantize_tc(AppendArgs &a, int num_sms, cudaStream_t stream);
// Group quantization of values alone (bandwidth-bound), run by the
// tensor-core append path before its key kernel.
cudaError_t launch_value_quant(const AppendArgs &a, int num_sms, cudaStream_t stream);
// Warp-per-vector append for small appends (decode steps).
cudaError_t launch_quantize_warp(const AppendArgs &a, int num_sms, cudaStream_t stream);
// W = S Pi^T in float64 (d x d, row-major by sketch row j).
cudaError_t launch_sketch_product(const float *pi, const float *s, int d, double *out, cudaStream_t stream);
cudaError_t launch_prepare_operands(const float *pi, const double *s_pit, void *dst, cudaStream_t stream);
cudaError_t launch_decode_simt(const DecodeArgs &a, cudaStream_t stream);
// Tensor-core split-K kernel (qprep and combine are shared with the SIMT path).
bool decode_tc_supported(int key_bits, int value_bits, int gqa, int value_mode = 0, int d = 128);

size_t decode_tc_qblock_bytes(int key_bits, int gqa);
cudaError_t launch_decode_tc(const DecodeArgs &a, cudaStream_t stream);
// qprep -> split-K (tensor-core kernel where built, SIMT otherwise) -> combine
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);
// Fill DecodeArgs' workspace pointers from a plan.
void bind_workspace(DecodeArgs &a, const DecodePlan &P, void *workspace);
// Validate one decode call (tq_decode_attention's contract) and launch it
// with the given scratch; shared by the workspace and no-allocation entry
// points.  win_k == nullptr: no recent window.  validate_only: return after
// the argument checks that need no device (before the workspace checks).
tq_status decode_common(const tq_params *p, const tq_cache *c, const void *q, tq_dtype q_dtype,
                        int h_q, const int32_t *len_dev, int max_len, const void *win_k,
                        const void *win_v, tq_dtype win_dtype, const int32_t *win_len_dev,
                        int win_cap, float softmax_scale, float *out, void *workspace,
                        size_t workspace_bytes, cudaStream_t stream, bool validate_only = false);
cudaError_t launch_dequantize(const DequantArgs &a, cudaStream_t stream);

}  // namespace tq
