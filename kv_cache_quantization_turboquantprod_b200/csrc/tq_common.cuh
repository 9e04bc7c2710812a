// Shared device-side definitions for the TurboQuant-prod kernels: the cache
// tile layout (documented in include/tq.h) and small helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq.h"

namespace tq {

constexpr int kD = 128;            // head dimension built
constexpr int kGroup = 32;         // value group
constexpr int kGroups = kD / kGroup;
constexpr int kTile = TQ_TILE_TOKENS;
constexpr int kRowBytes = kD / 8;  // one bit-plane row of a token
constexpr int kPlaneBytes = kTile * kRowBytes;  // 2048
constexpr int kPackedRowBytes = kD / 4;         // packed 2-bit value codes of a token

// Byte offsets of the sections inside one tile (head dim d: 64, 128 or 256;
// the tensor-core kernels are built for d = kD = 128 and use the constants
// above).
struct TileLayout {
  int mb;          // Lloyd-Max bits (key_bits - 1)
  int vb;          // value bits
  int d;           // head dim
  int row_bytes;   // one bit-plane row of a token (d / 8)
  int plane_bytes; // one bit-plane of a tile (128 rows)
  int packed_row_bytes;  // packed 2-bit value codes of a token (d / 4)
  int groups;      // value groups of a token (d / 32)
  int kplanes;     // offset of key planes
  int signs;       // offset of the sign plane
  int vplanes;     // offset of value planes
  int norms;       // offset of {||k||, ||r||} fp16 pairs
  int vsz;         // offset of {scale, zero} fp16 pairs (MSE values: fp16 norms)
  int tile_bytes;  // bytes of one tile
  bool mse;        // TurboQuant-MSE values: value cells as bit-planes + one fp16 norm

  __host__ __device__ static TileLayout make(int key_bits, int value_bits, int value_mode = 0,
                                             int d = kD) {
    TileLayout L;
    L.mb = key_bits - 1;
    L.vb = value_bits;
    L.d = d;
    L.row_bytes = d / 8;
    L.plane_bytes = kTile * L.row_bytes;
    L.packed_row_bytes = d / 4;
    L.groups = d / kGroup;
    L.mse = value_mode == TQ_VALUES_MSE;
    L.kplanes = 0;
    L.signs = L.mb * L.plane_bytes;
    L.vplanes = L.signs + L.plane_bytes;
    L.norms = L.vplanes + L.vb * L.plane_bytes;
    L.vsz = L.norms + kTile * 4;
    L.tile_bytes = L.vsz + (L.mse ? kTile * 2 : kTile * 4 * L.groups);
    return L;
  }
  __host__ __device__ int record_bytes() const { return tile_bytes / kTile; }
};

// Base pointer of tile t of (b, h).
__device__ __forceinline__ uint8_t *tile_ptr(void *data, const TileLayout &L,
                                             int h_kv, int ntiles, int b, int h,
                                             int t) {
  size_t idx = ((size_t)b * h_kv + h) * (size_t)ntiles + (size_t)t;
  return reinterpret_cast<uint8_t *>(data) + idx * (size_t)L.tile_bytes;
}

// Value code of channel j of token slot `slot`: packed 2-bit codes (channel
// 4i + m in bits 2m, 2m+1 of byte i) for 2-bit group-quantized values,
// bit-planes otherwise (MSE values: the cell of rotated coordinate j).
__device__ __forceinline__ int value_code(const uint8_t *tile, const TileLayout &L, int slot, int j) {
  if (L.vb == 2 && !L.mse) return (tile[L.vplanes + slot * L.packed_row_bytes + (j >> 2)] >> (2 * (j & 3))) & 3;
  int code = 0;
  for (int p = 0; p < L.vb; ++p)
    code |= ((tile[L.vplanes + p * L.plane_bytes + slot * L.row_bytes + (j >> 3)] >> (j & 7)) & 1) << p;
  return code;
}

__device__ __forceinline__ float load_elem(const void *p, tq_dtype dt, size_t i) {
  if (dt == TQ_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
  return reinterpret_cast<const float *>(p)[i];
}

// Bits 0..15 of x moved to the even positions 0, 2, .., 30.
__device__ __forceinline__ uint32_t spread_bits16(uint32_t x) {
  x &= 0xFFFFu;
  x = (x | (x << 8)) & 0x00FF00FFu;
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  x = (x | (x << 2)) & 0x33333333u;
  x = (x | (x << 1)) & 0x55555555u;
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_min(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Copy a row-major D x D fp32 matrix (16-byte aligned) into shared memory
// with a row stride of `pad` floats.  Eight 16-byte loads per thread are in
// flight at a time, so staging is bandwidth- rather than latency-bound.
template <int D = kD>
__device__ __forceinline__ void stage_matrix(float *dst, int pad, const float *src, int tid, int nthr) {
  const float4 *s4 = reinterpret_cast<const float4 *>(src);
  constexpr int kN4 = D * D / 4;
  for (int base = tid; base < kN4; base += 8 * nthr) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * nthr;
      v[u] = i < kN4 ? s4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * nthr;
      if (i < kN4) {
        float *d = dst + ((4 * i) / D) * pad + (4 * i) % D;
        d[0] = v[u].x;
        d[1] = v[u].y;
        d[2] = v[u].z;
        d[3] = v[u].w;
      }
    }
  }
}

// QJL constant sqrt(pi/2) / d.
__host__ __device__ constexpr float qjl_kappa(int d = kD) { return 1.2533141373155003f / d; }

// Sketch components |(S r)_j| below this are re-decided in float64: the
// single-precision paths (tensor-core hi/lo products, fp32 norms) can be off
// by up to ~1e-6 there, and the sign of such a component is the key's stored
// QJL bit.
constexpr float kSignRefineZ = 1e-5f;

__device__ __forceinline__ double warp_sum_f64(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Warp-cooperative float64 re-decision of QJL sign bits of one key row, head
// dim D (all 32 lanes call it together with the same arguments).  The row's
// key starts at element kbase of k; pl holds its Lloyd-Max code bit-planes
// (three planes of D/32 32-coordinate words, planes beyond the code width
// zero) and nw the mask of coordinates to re-decide.  In float64: ||k||,
// u = k / ||k|| and, for every masked j,
//   z_j = S_j . u - sum_m c_m W[j][m]     (W = S Pi^T, c = centroids of the codes)
// which is (S (u - Pi^T c))_j; bit j of the returned words is [z_j >= 0]
// (zero outside the mask).  A lane holds D/32 consecutive coordinates; S and
// W rows are read from global memory.
template <int D = kD>
__device__ __forceinline__ void refine_row_f64(const float *s, const double *s_pit, const float *cent,
                                               const void *k, tq_dtype dt, size_t kbase,
                                               const uint32_t (&pl)[3][D / 32], const uint32_t (&nw)[D / 32],
                                               uint32_t (&res)[D / 32]) {
  constexpr int W = D / 32;   // 32-coordinate words of a row
  constexpr int C = D / 32;   // coordinates per lane
  const int lane = threadIdx.x & 31;
  double x[C], ss = 0.0;
#pragma unroll
  for (int m = 0; m < C; ++m) {
    x[m] = (double)load_elem(k, dt, kbase + C * lane + m);
    ss = fma(x[m], x[m], ss);
  }
  const double nk = sqrt(warp_sum_f64(ss));
  // centroids of this lane's coordinates C lane .. C lane + C - 1
  const int wi = (C * lane) >> 5, sh = (C * lane) & 31;
  uint32_t b0 = 0u, b1 = 0u, b2 = 0u;
#pragma unroll
  for (int w = 0; w < W; ++w)
    if (w == wi) {
      b0 = pl[0][w] >> sh;
      b1 = pl[1][w] >> sh;
      b2 = pl[2][w] >> sh;
    }
  double u[C], c[C];
#pragma unroll
  for (int m = 0; m < C; ++m) {
    u[m] = x[m] / nk;
    c[m] = (double)cent[((b0 >> m) & 1u) | (((b1 >> m) & 1u) << 1) | (((b2 >> m) & 1u) << 2)];
  }
#pragma unroll
  for (int w = 0; w < W; ++w) {
    res[w] = 0u;
    uint32_t bits = nw[w];
    while (bits) {
      const int j = 32 * w + __ffs(bits) - 1;
      bits &= bits - 1;
      const float *srow = s + (size_t)j * D + C * lane;
      const double *wrow = s_pit + (size_t)j * D + C * lane;
      double part = 0.0;
#pragma unroll
      for (int m = 0; m < C; ++m) part = fma((double)srow[m], u[m], part);
#pragma unroll
      for (int m = 0; m < C; ++m) part = fma(-wrow[m], c[m], part);
      if (warp_sum_f64(part) >= 0.0) res[w] |= 1u << (j & 31);
    }
  }
}

// The same for the key row of lane `src`: lane src passes its planes, mask,
// key offset and sign words (sw), and gets the sign words back corrected.
template <int D = kD>
__device__ __forceinline__ void refine_signs_f64(const float *s, const double *s_pit, const float *cent,
                                                 const void *k, tq_dtype dt, size_t kbase,
                                                 const uint32_t (&planes)[3][D / 32],
                                                 const uint32_t (&near)[D / 32], uint32_t (&sw)[D / 32],
                                                 int src) {
  constexpr int W = D / 32;
  const int lane = threadIdx.x & 31;
  uint32_t pl[3][W], nw[W], res[W];
#pragma unroll
  for (int w = 0; w < W; ++w) {
#pragma unroll
    for (int p = 0; p < 3; ++p) pl[p][w] = __shfl_sync(0xffffffffu, planes[p][w], src);
    nw[w] = __shfl_sync(0xffffffffu, near[w], src);
  }
  const unsigned long long kb = __shfl_sync(0xffffffffu, (unsigned long long)kbase, src);
  refine_row_f64<D>(s, s_pit, cent, k, dt, kb, pl, nw, res);
  if (lane == src)
#pragma unroll
    for (int w = 0; w < W; ++w) sw[w] = (sw[w] & ~nw[w]) | res[w];
}

}  // namespace tq
