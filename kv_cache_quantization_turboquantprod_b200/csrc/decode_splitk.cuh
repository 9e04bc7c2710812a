// Split-K decode attention over the compressed cache, SIMT form, as a block
// body that both the standalone SIMT kernel and the tensor-core kernel (for
// codebooks it leaves to this path) run with 128 threads.
//
// Score of a cached key ("turboquant/audit_claims.py" attention_score,
// AUDIT 3/5/6; "TurboQuant" explainer, troisinh.com, "Ý tưởng cốt lõi"):
//   score = ||k|| * ( <Pi q, c[idx]> + sqrt(pi/2)/d * ||r|| * <S q, 2 sign - 1> )
// One pass per split ("03. Results & Benchmarks", turboquant_cutile,
// "Latency Benchmarks": score, QJL correction, online softmax and V
// accumulation in one pass): logits = score * softmax_scale, online softmax
// (base 2), acc += p * v_hat, with v_hat = code * scale + zero for
// group-quantized values and ||v|| c_v[cell] (rotated space) for
// TurboQuant-MSE values.  4 warps stride over the split's tokens; a lane owns
// 4 consecutive dims (one nibble of every plane row).  The rotated queries
// (Pi q, S q) are read from the workspace.
#pragma once

#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

// Shared-memory scratch of one split-K block for up to MAXG query heads of
// head dim D.
template <int MAXG, int D = kD>
struct SplitkSmem {
  float cent[16], vcent[16];
  float m[4][MAXG], l[4][MAXG];
  float acc[4][MAXG][D];
  static constexpr int kBytes = (32 + 8 * MAXG + 4 * MAXG * D) * 4;
};

// `width` (<= 16) consecutive bits starting at bit `bit` of a row of bytes.
__device__ __forceinline__ uint32_t row_bits(const uint8_t *row, int bit, int width) {
  const uint8_t *p = row + (bit >> 3);
  const uint32_t w = width <= 8 - (bit & 7) ? (uint32_t)p[0] : (uint32_t)p[0] | ((uint32_t)p[1] << 8);
  return (w >> (bit & 7)) & ((1u << width) - 1u);
}

// Named-barrier sync of the 128 threads running the body (id 0 is the block
// barrier of a 128-thread block).
__device__ __forceinline__ void splitk_bar(int id) {
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}

// Partial state (acc[D], m in log2 units, l) of split s of (b, h) for the G
// query heads of KV head h.  Threads tid 0..127 call it together; smem holds
// SplitkSmem<MAXG, D>::kBytes bytes.  A lane owns C = D / 32 consecutive dims.
template <int MAXG, int D = kD>
__device__ __forceinline__ void splitk_simt_body(const DecodeArgs &a, int s, int h, int b, int tid,
                                              uint8_t *smem, int bar_id) {
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr int C = D / 32;
  SplitkSmem<MAXG, D> &S = *reinterpret_cast<SplitkSmem<MAXG, D> *>(smem);
  const int lane = tid & 31, warp = tid >> 5;
  const int G = a.h_q / a.h_kv;
  const TileLayout L = TileLayout::make(a.key_bits, a.value_bits, a.value_mode, D);
  const float kappa = qjl_kappa(D);
  const float scale2 = a.softmax_scale * kLog2e;

  if (tid < (1 << L.mb)) S.cent[tid] = a.centroids[tid];
  if (L.mse && tid < (1 << L.vb)) S.vcent[tid] = a.v_centroids[tid];

  float qt[MAXG][C], sh[MAXG][C], acc[MAXG][C], mrun[MAXG], lrun[MAXG];
#pragma unroll
  for (int g = 0; g < MAXG; ++g) {
    mrun[g] = -INFINITY;
    lrun[g] = 0.f;
#pragma unroll
    for (int k = 0; k < C; ++k) {
      acc[g][k] = 0.f;
      if (g < G) {
        const float *src = a.qrot + ((size_t)b * a.h_q + h * G + g) * 2 * D;
        qt[g][k] = src[C * lane + k];
        sh[g][k] = src[D + C * lane + k];
      } else {
        qt[g][k] = sh[g][k] = 0.f;
      }
    }
  }
  splitk_bar(bar_id);

  int len = a.len[b] - a.len_sub;
  len = len < 0 ? 0 : (len > a.max_len ? a.max_len : len);
  const int t0 = s * a.tiles_per_split * kTile;
  const int t1 = min(len, (s + 1) * a.tiles_per_split * kTile);
  const int grp = (C * lane) / kGroup;  // value group of this lane's dims

  for (int n = t0 + warp; n < t1; n += 4) {
    const uint8_t *tp = tile_ptr(const_cast<void *>(a.data), L, a.h_kv, a.ntiles, b, h, n / kTile);
    const int slot = n % kTile;
    int idx[C], code[C];
#pragma unroll
    for (int k = 0; k < C; ++k) idx[k] = code[k] = 0;
    for (int p = 0; p < L.mb; ++p) {
      const uint32_t bits = row_bits(tp + L.kplanes + p * L.plane_bytes + slot * L.row_bytes, C * lane, C);
#pragma unroll
      for (int k = 0; k < C; ++k) idx[k] |= (int)((bits >> k) & 1u) << p;
    }
    const uint32_t sbits = row_bits(tp + L.signs + slot * L.row_bytes, C * lane, C);
    if (L.vb == 2 && !L.mse) {
      // packed: channel 4i + m in bits 2m, 2m+1 of byte i
      const uint32_t pk = row_bits(tp + L.vplanes + slot * L.packed_row_bytes, 2 * C * lane, 2 * C);
#pragma unroll
      for (int k = 0; k < C; ++k) code[k] = (int)((pk >> (2 * k)) & 3u);
    } else {
      for (int p = 0; p < L.vb; ++p) {
        const uint32_t bits = row_bits(tp + L.vplanes + p * L.plane_bytes + slot * L.row_bytes, C * lane, C);
#pragma unroll
        for (int k = 0; k < C; ++k) code[k] |= (int)((bits >> k) & 1u) << p;
      }
    }
    const __half2 nr = *reinterpret_cast<const __half2 *>(tp + L.norms + slot * 4);
    const float nk = __low2float(nr), rn = __high2float(nr);
    float c[C], sg[C], vh[C];
    if (L.mse) {
      // TurboQuant-MSE values, kept in the rotated space: ||v|| c[cell]
      const float nv = __half2float(*reinterpret_cast<const __half *>(tp + L.vsz + slot * 2));
#pragma unroll
      for (int k = 0; k < C; ++k) vh[k] = nv * S.vcent[code[k]];
    } else {
      const __half2 sz = *reinterpret_cast<const __half2 *>(tp + L.vsz + (slot * L.groups + grp) * 4);
      const float vs = __low2float(sz), vz = __high2float(sz);
#pragma unroll
      for (int k = 0; k < C; ++k) vh[k] = fmaf((float)code[k], vs, vz);
    }
#pragma unroll
    for (int k = 0; k < C; ++k) {
      c[k] = S.cent[idx[k]];
      sg[k] = ((sbits >> k) & 1u) ? 1.f : -1.f;
    }
    const float krn = kappa * rn;
#pragma unroll
    for (int g = 0; g < MAXG; ++g) {
      if (g >= G) break;
      float mse = 0.f, qjl = 0.f;
#pragma unroll
      for (int k = 0; k < C; ++k) {
        mse = fmaf(qt[g][k], c[k], mse);
        qjl = fmaf(sh[g][k], sg[k], qjl);
      }
      const float part = warp_sum(fmaf(krn, qjl, mse));
      // prefill: query token g / (G / qt) of the pass sees len - (qt - 1 - that) tokens
      const int gq = g / (G / a.qt);
      const float l2 = (n + a.qt - 1 - gq < len) ? nk * part * scale2 : -INFINITY;
      const float mnew = fmaxf(mrun[g], l2);
      const float corr = mnew == -INFINITY ? 1.f : exp2f(mrun[g] - mnew);
      const float p = mnew == -INFINITY ? 0.f : exp2f(l2 - mnew);
      lrun[g] = fmaf(lrun[g], corr, p);
#pragma unroll
      for (int k = 0; k < C; ++k) acc[g][k] = fmaf(acc[g][k], corr, p * vh[k]);
      mrun[g] = mnew;
    }
  }

  // merge the 4 warps' states
#pragma unroll
  for (int g = 0; g < MAXG; ++g) {
    if (g >= G) break;
    if (lane == 0) {
      S.m[warp][g] = mrun[g];
      S.l[warp][g] = lrun[g];
    }
#pragma unroll
    for (int k = 0; k < C; ++k) S.acc[warp][g][C * lane + k] = acc[g][k];
  }
  splitk_bar(bar_id);
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, S.m[w][g]);
    float *dst = a.part + (((size_t)b * a.h_q + h * G + g) * a.part_stride + s) * (D + 2);
    for (int j = tid; j < D; j += 128) {  // dims
      float Lsum = 0.f, A = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float f = exp2f(S.m[w][g] - M);
          Lsum = fmaf(S.l[w][g], f, Lsum);
          A = fmaf(S.acc[w][g][j], f, A);
        }
      }
      dst[j] = A;
      if (j == 0) {
        dst[D] = M;
        dst[D + 1] = Lsum;
      }
    }
  }
}

}  // namespace tq
