// Decode attention over the compressed cache, SIMT form: qprep (rotate the
// query once), split-K one-pass attention, log-sum-exp combine.
//
// Score of a cached key ("turboquant/audit_claims.py" attention_score,
// AUDIT 3/5/6; "TurboQuant" explainer, troisinh.com, "Ý tưởng cốt lõi"):
//   score = ||k|| * ( <Pi q, c[idx]> + sqrt(pi/2)/d * ||r|| * <S q, 2 sign - 1> )
// One pass per split ("03. Results & Benchmarks", turboquant_cutile,
// "Latency Benchmarks": score, QJL correction, online softmax and V
// accumulation in one pass): logits = score * softmax_scale, online softmax
// (base 2), acc += p * (code * scale + zero).
#include <math.h>

#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxG = 8;

// ---------------------------------------------------------------------------
// qprep: qrot[b][hq][0][:] = Pi q, qrot[b][hq][1][:] = S q   (fp32)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) qprep_kernel(DecodeArgs a) {
  const int bh = blockIdx.x;  // b * h_q + hq
  if (bh == 0 && threadIdx.x == 0 && a.status) *a.status = 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float qv[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) qv[m] = load_elem(a.q, a.q_dtype, qrow_offset(a, bh / a.h_q, bh % a.h_q) + lane + 32 * m);
  float *dst = a.qrot + (size_t)bh * 2 * kD;
  for (int o = warp; o < 2 * kD; o += 8) {
    const float *row = (o < kD) ? (a.pi + (size_t)o * kD) : (a.s + (size_t)(o - kD) * kD);
    float acc = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) acc = fmaf(row[lane + 32 * m], qv[m], acc);
    acc = warp_sum(acc);
    if (lane == 0) dst[o] = acc;
  }
}

// ---------------------------------------------------------------------------
// split-K: one CTA per (split, h_kv, b); 4 warps stride over the split's
// tokens; a lane owns 4 consecutive dims (one nibble of every plane row).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) decode_splitk_simt_kernel(DecodeArgs a) {
  // behind the tensor-core kernel: only for a codebook that kernel left to us
  if (a.fallback_gate && a.status[1] == 0) return;
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = a.h_q / a.h_kv;
  const TileLayout L = TileLayout::make(a.key_bits, a.value_bits, a.value_mode);
  const float kappa = qjl_kappa();
  const float scale2 = a.softmax_scale * kLog2e;

  __shared__ float cent[16], vcent[16];
  __shared__ float sm_m[4][kMaxG], sm_l[4][kMaxG];
  __shared__ float sm_acc[4][kMaxG][kD];
  if (threadIdx.x < (1 << L.mb)) cent[threadIdx.x] = a.centroids[threadIdx.x];
  if (L.mse && threadIdx.x < (1 << L.vb)) vcent[threadIdx.x] = a.v_centroids[threadIdx.x];

  float qt[kMaxG][4], sh[kMaxG][4], acc[kMaxG][4], mrun[kMaxG], lrun[kMaxG];
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) {
    mrun[g] = -INFINITY;
    lrun[g] = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[g][k] = 0.f;
      if (g < G) {
        const float *src = a.qrot + ((size_t)b * a.h_q + h * G + g) * 2 * kD;
        qt[g][k] = src[4 * lane + k];
        sh[g][k] = src[kD + 4 * lane + k];
      } else {
        qt[g][k] = sh[g][k] = 0.f;
      }
    }
  }
  __syncthreads();

  int len = a.len[b] - a.len_sub;
  len = len < 0 ? 0 : (len > a.max_len ? a.max_len : len);
  const int t0 = s * a.tiles_per_split * kTile;
  const int t1 = min(len, (s + 1) * a.tiles_per_split * kTile);
  const int byte = lane >> 1, shift = (lane & 1) * 4;
  const int grp = lane >> 3;

  for (int n = t0 + warp; n < t1; n += 4) {
    const uint8_t *tp = tile_ptr(const_cast<void *>(a.data), L, a.h_kv, a.ntiles, b, h, n / kTile);
    const int slot = n % kTile;
    int idx[4] = {0, 0, 0, 0};
    for (int p = 0; p < L.mb; ++p) {
      const int nib = (tp[L.kplanes + p * kPlaneBytes + slot * kRowBytes + byte] >> shift) & 0xF;
#pragma unroll
      for (int k = 0; k < 4; ++k) idx[k] |= ((nib >> k) & 1) << p;
    }
    const int snib = (tp[L.signs + slot * kRowBytes + byte] >> shift) & 0xF;
    int code[4] = {0, 0, 0, 0};
    if (L.vb == 2 && !L.mse) {
      const int pk = tp[L.vplanes + slot * kPackedRowBytes + lane];  // channels 4 lane .. 4 lane + 3
#pragma unroll
      for (int k = 0; k < 4; ++k) code[k] = (pk >> (2 * k)) & 3;
    } else {
      for (int p = 0; p < L.vb; ++p) {
        const int nib = (tp[L.vplanes + p * kPlaneBytes + slot * kRowBytes + byte] >> shift) & 0xF;
#pragma unroll
        for (int k = 0; k < 4; ++k) code[k] |= ((nib >> k) & 1) << p;
      }
    }
    const __half2 nr = *reinterpret_cast<const __half2 *>(tp + L.norms + slot * 4);
    const float nk = __low2float(nr), rn = __high2float(nr);
    float c[4], sg[4], vh[4];
    if (L.mse) {
      // TurboQuant-MSE values, kept in the rotated space: ||v|| c[cell]
      const float nv = __half2float(*reinterpret_cast<const __half *>(tp + L.vsz + slot * 2));
#pragma unroll
      for (int k = 0; k < 4; ++k) vh[k] = nv * vcent[code[k]];
    } else {
      const __half2 sz = *reinterpret_cast<const __half2 *>(tp + L.vsz + (slot * kGroups + grp) * 4);
      const float vs = __low2float(sz), vz = __high2float(sz);
#pragma unroll
      for (int k = 0; k < 4; ++k) vh[k] = fmaf((float)code[k], vs, vz);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      c[k] = cent[idx[k]];
      sg[k] = ((snib >> k) & 1) ? 1.f : -1.f;
    }
    const float krn = kappa * rn;
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) {
      if (g >= G) break;
      float mse = 0.f, qjl = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        mse = fmaf(qt[g][k], c[k], mse);
        qjl = fmaf(sh[g][k], sg[k], qjl);
      }
      const float part = warp_sum(fmaf(krn, qjl, mse));
      const float l2 = nk * part * scale2;
      const float mnew = fmaxf(mrun[g], l2);
      const float corr = exp2f(mrun[g] - mnew);
      const float p = exp2f(l2 - mnew);
      lrun[g] = fmaf(lrun[g], corr, p);
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[g][k] = fmaf(acc[g][k], corr, p * vh[k]);
      mrun[g] = mnew;
    }
  }

  // merge the 4 warps' states
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) {
    if (g >= G) break;
    if (lane == 0) { sm_m[warp][g] = mrun[g]; sm_l[warp][g] = lrun[g]; }
#pragma unroll
    for (int k = 0; k < 4; ++k) sm_acc[warp][g][4 * lane + k] = acc[g][k];
  }
  __syncthreads();
  const int j = threadIdx.x;  // one dim per thread
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w][g]);
    float Lsum = 0.f, A = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float f = exp2f(sm_m[w][g] - M);
        Lsum = fmaf(sm_l[w][g], f, Lsum);
        A = fmaf(sm_acc[w][g][j], f, A);
      }
    }
    float *dst = a.part + (((size_t)b * a.h_q + h * G + g) * a.part_stride + s) * (kD + 2);
    dst[j] = A;
    if (j == 0) { dst[kD] = M; dst[kD + 1] = Lsum; }
  }
}

// ---------------------------------------------------------------------------
// combine: out[b][hq][:] = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s
// (TurboQuant-MSE values: the partials are in the rotated space and the
// merged accumulator is rotated back once, Pi^T acc).  A call whose kernels gave up on a bounded wait (status word nonzero) gets
// NaN rows, so a timeout never comes back as a plausible result.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) combine_kernel(DecodeArgs a) {
  const int bh = blockIdx.x;
  const int j = threadIdx.x;
  if (a.status[0] != 0) {
    a.out[qrow_offset(a, bh / a.h_q, bh % a.h_q) + j] = __int_as_float(0x7fc00000);
    return;
  }
  const float *src = a.part + (size_t)bh * a.part_stride * (kD + 2);
  float M = -INFINITY;
  for (int s = 0; s < a.part_stride; ++s) M = fmaxf(M, src[s * (kD + 2) + kD]);
  float num = 0.f, den = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < a.part_stride; ++s) {
      const float ms = src[s * (kD + 2) + kD];
      if (ms == -INFINITY) continue;  // empty split
      const float f = exp2f(ms - M);
      num = fmaf(src[s * (kD + 2) + j], f, num);
      den = fmaf(src[s * (kD + 2) + kD + 1], f, den);
    }
  }
  if (a.value_mode == TQ_VALUES_MSE) {
    // the merged accumulator is in the rotated space: out_j = (Pi^T acc)_j
    __shared__ float acc[kD];
    acc[j] = num;
    __syncthreads();
    float o = 0.f;
    for (int i = 0; i < kD; ++i) o = fmaf(a.pi[(size_t)i * kD + j], acc[i], o);
    num = o;
  }
  a.out[qrow_offset(a, bh / a.h_q, bh % a.h_q) + j] = den > 0.f ? num / den : 0.f;
}

// ---------------------------------------------------------------------------
// Recent-token window: exact attention of the G query heads of (b, h_kv)
// over win_len[b] window tokens, written as partial slot nsplit (acc, m in
// log2 units, l), so the combine merges it with the compressed splits.
// One CTA per (h_kv, b); thread t scores window slot t, thread j then sums
// dimension j over the slots.
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(128) window_kernel(DecodeArgs a) {
  const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
  __shared__ float qs[G][kD];
  __shared__ float ps[G][kTile];
  __shared__ float red[G][4];
  int wl = a.win_len[b];
  wl = wl < 0 ? 0 : (wl > a.win_cap ? a.win_cap : wl);
  for (int i = t; i < G * kD; i += 128)
    qs[i / kD][i % kD] = load_elem(a.q, a.q_dtype, ((size_t)b * a.h_q + (size_t)h * G) * kD + i);
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
          reinterpret_cast<const __nv_bfloat16 *>(a.win_k) + (row0 + t) * kD);
#pragma unroll 4
      for (int c = 0; c < kD / 8; ++c) {
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
                                                          (row0 + t) * kD);
#pragma unroll 4
      for (int c = 0; c < kD / 4; ++c) {
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
  // thread t now sums dimension t over the window slots
  float num[G], den[G];
#pragma unroll
  for (int g = 0; g < G; ++g) num[g] = den[g] = 0.f;
  for (int i = 0; i < wl; ++i) {
    const float v = load_elem(a.win_v, a.win_dtype, (row0 + i) * kD + t);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      num[g] = fmaf(ps[g][i], v, num[g]);
      den[g] += ps[g][i];
    }
  }
  if (a.value_mode == TQ_VALUES_MSE) {
    // the compressed splits accumulate in the rotated space: rotate this
    // partial too, (Pi num)_t
#pragma unroll
    for (int g = 0; g < G; ++g) qs[g][t] = num[g];
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float o = 0.f;
      for (int j = 0; j < kD; ++j) o = fmaf(a.pi[(size_t)t * kD + j], qs[g][j], o);
      num[g] = o;
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float *dst = a.part + (((size_t)b * a.h_q + (size_t)h * G + g) * a.part_stride + a.nsplit) * (kD + 2);
    dst[t] = num[g];
    if (t == 0) {
      dst[kD] = wl > 0 ? mx[g] : -INFINITY;
      dst[kD + 1] = den[g];
    }
  }
}

cudaError_t launch_window(const DecodeArgs &a, cudaStream_t stream) {
  const dim3 grid(a.h_kv, a.batch);
  switch (a.h_q / a.h_kv) {
    case 1: window_kernel<1><<<grid, 128, 0, stream>>>(a); break;
    case 2: window_kernel<2><<<grid, 128, 0, stream>>>(a); break;
    case 3: window_kernel<3><<<grid, 128, 0, stream>>>(a); break;
    case 4: window_kernel<4><<<grid, 128, 0, stream>>>(a); break;
    case 5: window_kernel<5><<<grid, 128, 0, stream>>>(a); break;
    case 6: window_kernel<6><<<grid, 128, 0, stream>>>(a); break;
    case 7: window_kernel<7><<<grid, 128, 0, stream>>>(a); break;
    case 8: window_kernel<8><<<grid, 128, 0, stream>>>(a); break;
    default: return cudaErrorNotSupported;
  }
  return cudaGetLastError();
}

}  // namespace

DecodePlan make_decode_plan(int batch, int h_kv, int h_q, int max_len, int num_sms,
                            int key_bits, int value_bits, int value_mode) {
  DecodePlan P;
  const int ntile = (max_len + kTile - 1) / kTile;
  const long long units = (long long)batch * h_kv;
  // about two CTAs per SM: fewer, longer CTAs amortise each CTA's pipeline fill
#ifndef TQ_DECODE_CTAS_PER_SM
#define TQ_DECODE_CTAS_PER_SM 2
#endif
  const long long target = (long long)TQ_DECODE_CTAS_PER_SM * num_sms;
  long long ns = (target + units - 1) / units;
  ns = std::max(1LL, std::min(ns, (long long)std::max(ntile, 1)));
  int tps = ntile > 0 ? (int)((ntile + ns - 1) / ns) : 0;
  int nsplit = tps > 0 ? (ntile + tps - 1) / tps : 1;
  P.nsplit = nsplit;
  P.tiles_per_split = tps;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  P.status_bytes = 256;
  P.qrot_bytes = al((size_t)batch * h_q * 2 * kD * sizeof(float));
  P.part_bytes = al((size_t)batch * h_q * (nsplit + 1) * (kD + 2) * sizeof(float));
  const int G = h_q / h_kv;
  P.qblock_bytes =
      decode_tc_supported(key_bits, value_bits, G, value_mode) ? decode_tc_qblock_bytes(key_bits, G) : 0;
  P.total_bytes = P.status_bytes + P.qrot_bytes + P.part_bytes + al((size_t)batch * h_kv * P.qblock_bytes);
  return P;
}

void bind_workspace(DecodeArgs &a, const DecodePlan &P, void *workspace) {
  uint8_t *w = reinterpret_cast<uint8_t *>(workspace);
  a.status = reinterpret_cast<int *>(w);
  a.qrot = reinterpret_cast<float *>(w + P.status_bytes);
  a.part = reinterpret_cast<float *>(w + P.status_bytes + P.qrot_bytes);
  a.qblocks = w + P.status_bytes + P.qrot_bytes + P.part_bytes;
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream) {
  if (!decode_tc_supported(a.key_bits, a.value_bits, a.h_q / a.h_kv, a.value_mode))
    return launch_decode_simt(a, stream);
  const int bhq = a.batch * a.h_q;
  // the query-block kernel (first in launch_decode_tc) clears the status word
  cudaError_t e = launch_decode_tc(a, stream);
  if (e != cudaSuccess) return e;
  if (decode_tc_needs_fallback(a.key_bits, a.value_bits, a.h_q / a.h_kv)) {
    // returns at once unless the codebook needs it (status[1], set on the device)
    DecodeArgs f = a;
    f.fallback_gate = 1;
    dim3 grid(a.nsplit, a.h_kv, a.batch);
    decode_splitk_simt_kernel<<<grid, 128, 0, stream>>>(f);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.win_k) {
    e = launch_window(a, stream);
    if (e != cudaSuccess) return e;
  }
  combine_kernel<<<bhq, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode_simt(const DecodeArgs &a, cudaStream_t stream) {
  const int bhq = a.batch * a.h_q;
  qprep_kernel<<<bhq, 256, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid(a.nsplit, a.h_kv, a.batch);
  decode_splitk_simt_kernel<<<grid, 128, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.win_k) {
    e = launch_window(a, stream);
    if (e != cudaSuccess) return e;
  }
  combine_kernel<<<bhq, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace tq
