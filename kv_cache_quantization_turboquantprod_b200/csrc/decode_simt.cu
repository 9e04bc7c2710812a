// Decode attention over the compressed cache, SIMT form (head dims 64, 128
// and 256): qprep (rotate the query once), split-K one-pass attention,
// log-sum-exp combine; the combine and the recent-token window are shared
// with the tensor-core path.
//
// Score of a cached key ("turboquant/audit_claims.py" attention_score,
// AUDIT 3/5/6; "TurboQuant" explainer, troisinh.com, "Ý tưởng cốt lõi"):
//   score = ||k|| * ( <Pi q, c[idx]> + sqrt(pi/2)/d * ||r|| * <S q, 2 sign - 1> )
// One pass per split ("03. Results & Benchmarks", turboquant_cutile,
// "Latency Benchmarks": score, QJL correction, online softmax and V
// accumulation in one pass): logits = score * softmax_scale, online softmax
// (base 2), acc += p * (code * scale + zero).
#include <math.h>

#include "decode_splitk.cuh"
#include "sm100.cuh"
#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

namespace {

using sm100::pdl_trigger;
using sm100::pdl_wait;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxG = 8;

// ---------------------------------------------------------------------------
// qprep: qrot[b][hq][0][:] = Pi q, qrot[b][hq][1][:] = S q   (fp32), head dim D
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) qprep_kernel(DecodeArgs a) {
  constexpr int C = D / 32;
  pdl_trigger();
  const int bh = blockIdx.x;  // b * h_q + hq
  if (bh == 0 && threadIdx.x == 0 && a.status) *a.status = 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float qv[C];
#pragma unroll
  for (int m = 0; m < C; ++m) qv[m] = load_elem(a.q, a.q_dtype, qrow_offset(a, bh / a.h_q, bh % a.h_q) + lane + 32 * m);
  float *dst = a.qrot + (size_t)bh * 2 * D;
  for (int o = warp; o < 2 * D; o += 8) {
    const float *row = (o < D) ? (a.pi + (size_t)o * D) : (a.s + (size_t)(o - D) * D);
    float acc = 0.f;
#pragma unroll
    for (int m = 0; m < C; ++m) acc = fmaf(row[lane + 32 * m], qv[m], acc);
    acc = warp_sum(acc);
    if (lane == 0) dst[o] = acc;
  }
  // launched as a dependent of the call's predecessor (reads only the
  // queries and Pi, S; writes only the workspace): wait for it before
  // finishing, so the split-K kernel's wait covers both
  pdl_wait();
}

// ---------------------------------------------------------------------------
// split-K, SIMT form (every bit width and GQA <= 8; see decode_splitk.cuh)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) decode_splitk_simt_kernel(DecodeArgs a) {
  pdl_wait();
  __shared__ __align__(16) uint8_t smem[SplitkSmem<kMaxG, D>::kBytes];
  splitk_simt_body<kMaxG, D>(a, blockIdx.x, blockIdx.y, blockIdx.z, threadIdx.x, smem, 0);
}

// ---------------------------------------------------------------------------
// combine: out[b][hq][:] = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s
// (TurboQuant-MSE values: the partials are in the rotated space and the
// merged accumulator is rotated back once, Pi^T acc).  A call whose kernels
// gave up on a bounded wait (status word nonzero) gets NaN rows, so a
// timeout never comes back as a plausible result.
// 256 threads: M from one split per thread, then warp w sums splits w,
// w + 8, ... (lane l holding dims 64u + 2l, 64u + 2l + 1), so the loads of
// every split are in flight at once; the eight warp sums meet in shared
// memory and thread j finishes dim j.
// ---------------------------------------------------------------------------
constexpr int kCombThreads = 256;
constexpr int kCombWarps = kCombThreads / 32;

template <int D>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(DecodeArgs a) {
  static_assert(D % 64 == 0 && D <= kCombThreads, "combine layout");
  constexpr int U = D / 64;  // float2 loads per lane and split
  __shared__ float smax[kCombWarps], sden[kCombWarps];
  __shared__ __align__(8) float snum[kCombWarps][D];
  __shared__ float acc[D];
  pdl_wait();
  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t orow = qrow_offset(a, bh / a.h_q, bh % a.h_q);
  if (a.status[0] != 0) {
    if (tid < D) a.out[orow + tid] = __int_as_float(0x7fc00000);
    return;
  }
  const int ns = a.part_stride;
  const float *src = a.part + (size_t)bh * ns * (D + 2);
  float m = -INFINITY;
  for (int s = tid; s < ns; s += kCombThreads) m = fmaxf(m, src[(size_t)s * (D + 2) + D]);
  m = warp_max(m);
  if (lane == 0) smax[warp] = m;
  __syncthreads();
  float M = smax[0];
#pragma unroll
  for (int w = 1; w < kCombWarps; ++w) M = fmaxf(M, smax[w]);
  float2 num[U];
#pragma unroll
  for (int u = 0; u < U; ++u) num[u] = make_float2(0.f, 0.f);
  float den = 0.f;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int s = warp; s < ns; s += kCombWarps) {
      const float *row = src + (size_t)s * (D + 2);
      const float2 ml = *reinterpret_cast<const float2 *>(row + D);  // (m_s, l_s)
      if (ml.x == -INFINITY) continue;  // empty split
      const float f = exp2f(ml.x - M);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float2 v = *reinterpret_cast<const float2 *>(row + 64 * u + 2 * lane);
        num[u].x = fmaf(v.x, f, num[u].x);
        num[u].y = fmaf(v.y, f, num[u].y);
      }
      den = fmaf(ml.y, f, den);
    }
  }
#pragma unroll
  for (int u = 0; u < U; ++u) *reinterpret_cast<float2 *>(&snum[warp][64 * u + 2 * lane]) = num[u];
  if (lane == 0) sden[warp] = den;
  __syncthreads();
  float o = 0.f, dsum = 0.f;
#pragma unroll
  for (int w = 0; w < kCombWarps; ++w) dsum += sden[w];
  if (tid < D) {
#pragma unroll
    for (int w = 0; w < kCombWarps; ++w) o += snum[w][tid];
  }
  if (a.value_mode == TQ_VALUES_MSE) {
    // the merged accumulator is in the rotated space: out_j = (Pi^T acc)_j
    if (tid < D) acc[tid] = o;
    __syncthreads();
    if (tid < D) {
      o = 0.f;
      for (int i = 0; i < D; ++i) o = fmaf(a.pi[(size_t)i * D + tid], acc[i], o);
    }
  }
  if (tid < D) a.out[orow + tid] = dsum > 0.f ? o / dsum : 0.f;
}

// ---------------------------------------------------------------------------
// Recent-token window: exact attention of the G query heads of (b, h_kv)
// over win_len[b] window tokens, written as partial slot nsplit (acc, m in
// log2 units, l), so the combine merges it with the compressed splits.
// One CTA per (h_kv, b); thread t scores window slot t, then sums dims
// t, t + 128, ... over the slots.  (TurboQuant-MSE values: the partial is
// rotated like the compressed splits, Pi acc.)
// Launched as a programmatic dependent of the split-K kernel, whose CTAs
// signal only after their own wait on the call's predecessors (or which
// signals by finishing), so the queries and the window rows are complete
// when this grid starts; it reads nothing the split-K kernel writes, so it
// runs beside that kernel's last CTAs and waits for it only before it
// finishes (the combine's wait then covers both).
// ---------------------------------------------------------------------------
template <int G, int D>
__global__ void __launch_bounds__(128) window_kernel(DecodeArgs a) {
  constexpr int J = (D + 127) / 128;
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  __shared__ float qs[G][D];
  __shared__ float ps[G][kTile];
  __shared__ float red[G][4];
  int wl = a.win_len[b];
  wl = wl < 0 ? 0 : (wl > a.win_cap ? a.win_cap : wl);
  for (int i = t; i < G * D; i += 128)
    qs[i / D][i % D] = load_elem(a.q, a.q_dtype, ((size_t)b * a.h_q + (size_t)h * G) * D + i);
  __syncthreads();
  const size_t row0 = ((size_t)b * a.h_kv + h) * (size_t)a.win_cap;
  const float scale2 = a.softmax_scale * 1.4426950408889634f;
  float lg[G];
#pragma unroll
  for (int g = 0; g < G; ++g) lg[g] = -INFINITY;
  if (t < wl) {
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = 0.f;
    // the slot's key row with 16-byte loads (8 bf16 or 4 fp32 at a time)
    if (a.win_dtype == TQ_BF16) {
      const uint4 *kr = reinterpret_cast<const uint4 *>(
          reinterpret_cast<const __nv_bfloat16 *>(a.win_k) + (row0 + t) * D);
#pragma unroll 4
      for (int c = 0; c < D / 8; ++c) {
        const uint4 w = kr[c];
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
#pragma unroll
          for (int g = 0; g < G; ++g)
            acc[g] = fmaf(qs[g][8 * c + 2 * e + 1], f.y, fmaf(qs[g][8 * c + 2 * e], f.x, acc[g]));
        }
      }
    } else {
      const float4 *kr = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.win_k) +
                                                          (row0 + t) * D);
#pragma unroll 4
      for (int c = 0; c < D / 4; ++c) {
        const float4 f = kr[c];
#pragma unroll
        for (int g = 0; g < G; ++g)
          acc[g] = fmaf(qs[g][4 * c + 3], f.w, fmaf(qs[g][4 * c + 2], f.z,
                   fmaf(qs[g][4 * c + 1], f.y, fmaf(qs[g][4 * c], f.x, acc[g]))));
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) lg[g] = acc[g] * scale2;
  }
  const int warp = t >> 5, lane = t & 31;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float m = warp_max(lg[g]);
    if (lane == 0) red[g][warp] = m;
  }
  __syncthreads();
  float mx[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    mx[g] = fmaxf(fmaxf(red[g][0], red[g][1]), fmaxf(red[g][2], red[g][3]));
    ps[g][t] = (t < wl) ? exp2f(lg[g] - mx[g]) : 0.f;
  }
  __syncthreads();
  // thread t now sums dims t, t + 128, ... over the window slots
  float num[G][J], den[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    den[g] = 0.f;
#pragma unroll
    for (int u = 0; u < J; ++u) num[g][u] = 0.f;
  }
  // kWinBatch slots at a time, every load of the batch issued before any
  // is used (the slots' rows are independent), then the tail one by one
  constexpr int kWinBatch = 16;
  int i = 0;
  for (; i + kWinBatch <= wl; i += kWinBatch) {
    float v[kWinBatch][J];
#pragma unroll
    for (int k = 0; k < kWinBatch; ++k)
#pragma unroll
      for (int u = 0; u < J; ++u)
        v[k][u] = (t + 128 * u < D) ? load_elem(a.win_v, a.win_dtype, (row0 + i + k) * D + t + 128 * u) : 0.f;
#pragma unroll
    for (int k = 0; k < kWinBatch; ++k) {
#pragma unroll
      for (int u = 0; u < J; ++u)
#pragma unroll
        for (int g = 0; g < G; ++g) num[g][u] = fmaf(ps[g][i + k], v[k][u], num[g][u]);
#pragma unroll
      for (int g = 0; g < G; ++g) den[g] += ps[g][i + k];
    }
  }
  for (; i < wl; ++i) {
#pragma unroll
    for (int u = 0; u < J; ++u) {
      if (t + 128 * u >= D) continue;
      const float v = load_elem(a.win_v, a.win_dtype, (row0 + i) * D + t + 128 * u);
#pragma unroll
      for (int g = 0; g < G; ++g) num[g][u] = fmaf(ps[g][i], v, num[g][u]);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) den[g] += ps[g][i];
  }
  if (a.value_mode == TQ_VALUES_MSE) {
    // the compressed splits accumulate in the rotated space: rotate this
    // partial too, (Pi num)_j  (qs is free again: the scores are done)
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int u = 0; u < J; ++u)
        if (t + 128 * u < D) qs[g][t + 128 * u] = num[g][u];
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int u = 0; u < J; ++u) {
        const int j = t + 128 * u;
        if (j >= D) continue;
        float o = 0.f;
        for (int k = 0; k < D; ++k) o = fmaf(a.pi[(size_t)j * D + k], qs[g][k], o);
        num[g][u] = o;
      }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float *dst = a.part + (((size_t)b * a.h_q + (size_t)h * G + g) * a.part_stride + a.nsplit) * (D + 2);
#pragma unroll
    for (int u = 0; u < J; ++u)
      if (t + 128 * u < D) dst[t + 128 * u] = num[g][u];
    if (t == 0) {
      dst[D] = wl > 0 ? mx[g] : -INFINITY;
      dst[D + 1] = den[g];
    }
  }
  pdl_wait();
}

template <int D>
cudaError_t launch_window_d(const DecodeArgs &a, cudaStream_t stream) {
  const dim3 grid(a.h_kv, a.batch);
  switch (a.h_q / a.h_kv) {
    case 1: return launch_pdl(window_kernel<1, D>, grid, dim3(128), 0, stream, a);
    case 2: return launch_pdl(window_kernel<2, D>, grid, dim3(128), 0, stream, a);
    case 3: return launch_pdl(window_kernel<3, D>, grid, dim3(128), 0, stream, a);
    case 4: return launch_pdl(window_kernel<4, D>, grid, dim3(128), 0, stream, a);
    case 5: return launch_pdl(window_kernel<5, D>, grid, dim3(128), 0, stream, a);
    case 6: return launch_pdl(window_kernel<6, D>, grid, dim3(128), 0, stream, a);
    case 7: return launch_pdl(window_kernel<7, D>, grid, dim3(128), 0, stream, a);
    case 8: return launch_pdl(window_kernel<8, D>, grid, dim3(128), 0, stream, a);
    default: return cudaErrorNotSupported;
  }
}

cudaError_t launch_window(const DecodeArgs &a, cudaStream_t stream) {
  switch (a.d) {
    case 64: return launch_window_d<64>(a, stream);
    case 128: return launch_window_d<128>(a, stream);
    case 256: return launch_window_d<256>(a, stream);
    default: return cudaErrorNotSupported;
  }
}

template <int D>
cudaError_t launch_decode_simt_d(const DecodeArgs &a, cudaStream_t stream) {
  const int bhq = a.batch * a.h_q;
  cudaError_t e = launch_pdl(qprep_kernel<D>, dim3(bhq), dim3(256), 0, stream, a);
  if (e != cudaSuccess) return e;
  e = launch_pdl(decode_splitk_simt_kernel<D>, dim3(a.nsplit, a.h_kv, a.batch), dim3(128), 0, stream, a);
  if (e != cudaSuccess) return e;
  if (a.win_k) {
    e = launch_window(a, stream);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(combine_kernel<D>, dim3(bhq), dim3(kCombThreads), 0, stream, a);
}

}  // namespace

DecodePlan make_decode_plan(int batch, int h_kv, int h_q, int max_len, int num_sms,
                            int key_bits, int value_bits, int value_mode, int d) {
  DecodePlan P;
  const int ntile = (max_len + kTile - 1) / kTile;
  const long long units = (long long)batch * h_kv;
  // CTAs per SM the split plan aims at: with at least one (sequence, head)
  // unit per SM, about two (fewer, longer CTAs amortise each CTA's pipeline
  // fill, and the split-major grid runs every unit's first split before any
  // ragged last one); with fewer, longer units, about eight, so the last wave
  // of CTAs is a small part of the call (measured on 4 x 131,072-token
  // sequences: 0.299 ms at two, 0.270 ms at eight) -- but no split shorter
  // than 32 tiles, whose pipeline fill and merge would dominate (measured on
  // 8 sequences of 16K-32K tokens, 64 units: 123 us with 19 splits of ~10
  // tiles, 110 us with 6), unless that leaves SMs without a CTA (a few short
  // sequences: there more, shorter splits are what keeps the call short)
#ifndef TQ_DECODE_CTAS_PER_SM
#define TQ_DECODE_CTAS_PER_SM 2
#endif
#ifndef TQ_DECODE_CTAS_PER_SM_FEW_UNITS
#define TQ_DECODE_CTAS_PER_SM_FEW_UNITS 8
#endif
#ifndef TQ_DECODE_MIN_TILES_PER_SPLIT
#define TQ_DECODE_MIN_TILES_PER_SPLIT 32
#endif
  const long long cps = units >= num_sms ? TQ_DECODE_CTAS_PER_SM : TQ_DECODE_CTAS_PER_SM_FEW_UNITS;
  const long long target = cps * num_sms;
  long long ns = (target + units - 1) / units;
  ns = std::min(ns, std::max((long long)std::max(ntile / TQ_DECODE_MIN_TILES_PER_SPLIT, 1),
                              ((long long)num_sms + units - 1) / units));
  ns = std::max(1LL, std::min(ns, (long long)std::max(ntile, 1)));
  int tps = ntile > 0 ? (int)((ntile + ns - 1) / ns) : 0;
  int nsplit = tps > 0 ? (ntile + tps - 1) / tps : 1;
  P.nsplit = nsplit;
  P.tiles_per_split = tps;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  P.status_bytes = 256;
  P.qrot_bytes = al((size_t)batch * h_q * 2 * d * sizeof(float));
  P.part_bytes = al((size_t)batch * h_q * (nsplit + 1) * (d + 2) * sizeof(float));
  const int G = h_q / h_kv;
  P.qblock_bytes =
      decode_tc_supported(key_bits, value_bits, G, value_mode, d) ? decode_tc_qblock_bytes(key_bits, G) : 0;
  P.order_bytes = P.qblock_bytes ? al((size_t)batch * h_kv * nsplit * sizeof(int2)) : 0;
  P.total_bytes =
      P.status_bytes + P.qrot_bytes + P.part_bytes + al((size_t)batch * h_kv * P.qblock_bytes) + P.order_bytes;
  return P;
}

void bind_workspace(DecodeArgs &a, const DecodePlan &P, void *workspace) {
  uint8_t *w = reinterpret_cast<uint8_t *>(workspace);
  a.status = reinterpret_cast<int *>(w);
  a.qrot = reinterpret_cast<float *>(w + P.status_bytes);
  a.part = reinterpret_cast<float *>(w + P.status_bytes + P.qrot_bytes);
  a.qblocks = w + P.status_bytes + P.qrot_bytes + P.part_bytes;
  // the work list is the last region
  a.order = P.order_bytes ? reinterpret_cast<int2 *>(w + P.total_bytes - P.order_bytes) : nullptr;
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
  if (!decode_tc_supported(a.key_bits, a.value_bits, a.h_q / a.h_kv, a.value_mode, a.d))
    return launch_decode_simt(a, stream);
  const int bhq = a.batch * a.h_q;
  // query blocks (which clear the status word) + the tensor-core kernel
  cudaError_t e = launch_decode_tc(a, stream);
  if (e != cudaSuccess) return e;
  if (a.win_k) {
    e = launch_window(a, stream);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(combine_kernel<kD>, dim3(bhq), dim3(kCombThreads), 0, stream, a);
}

cudaError_t launch_decode_simt(const DecodeArgs &a, cudaStream_t stream) {
  switch (a.d) {
    case 64: return launch_decode_simt_d<64>(a, stream);
    case 128: return launch_decode_simt_d<128>(a, stream);
    case 256: return launch_decode_simt_d<256>(a, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace tq
