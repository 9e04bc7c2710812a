// Pieces shared by the SIMT quantize-append kernels (quantize_simt.cu, the
// CTA-per-pass form for large appends, and quantize_warp.cu, the
// warp-per-vector form for small ones).
#pragma once

#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

// (sequence, token, head) of vector slot id = (b T + t) H_kv + h of an append;
// valid when the slot exists and t < n_new[b].
__device__ __forceinline__ void vec_coords(const AppendArgs &a, long long id, int &b,
                                           int &t, int &h, bool &valid) {
  const long long per_b = (long long)a.T * a.h_kv;
  const long long total = (long long)a.batch * per_b;
  valid = id < total;
  if (!valid) { b = t = h = 0; return; }
  b = (int)(id / per_b);
  long long rem = id - (long long)b * per_b;
  t = (int)(rem / a.h_kv);
  h = (int)(rem - (long long)t * a.h_kv);
  valid = t < a.nnew[b];
}

// Group quantization of one value vector by a converged warp
// ("turboquant/audit_claims.py", AUDIT 1: value_bits, value_group_size):
// group m = channels 32m .. 32m + 31, one channel per lane; zero = fp16(min),
// scale = fp16((max - min) / (2^vb - 1)) rounded once from the float64
// quotient, code = clamp(rint((v - zero) / scale)) of the exact quotient
// (single precision decides unless the quotient is next to a half-integer,
// then float64 does).  Writes the record's value codes and (scale, zero) at
// token slot `slot` of `tile`; the value starts at element `base` of a.v.
// Groups m0, m0 + mstep, ... (all of them by default).
template <int D>
__device__ __forceinline__ void quantize_value_groups(const AppendArgs &a, const TileLayout &L, uint8_t *tile,
                                                      int slot, size_t base, float vlevels, int m0 = 0,
                                                      int mstep = 1) {
  constexpr int C = D / 32;
  const int lane = threadIdx.x & 31;
  for (int m = m0; m < C; m += mstep) {
    const float vv = load_elem(a.v, a.dtype, base + lane + 32 * m);
    const float mn = warp_min(vv);
    const float mx = warp_max(vv);
    const __half zero16 = __float2half_rn(mn);
    const __half scale16 = __double2half(((double)mx - (double)mn) / (double)vlevels);
    const float z32 = __half2float(zero16);
    const float sc32 = __half2float(scale16);
    int code = 0;
    if (sc32 != 0.f) {
      const float t32 = __fdiv_rn(__fsub_rn(vv, z32), sc32);
      float tq = rintf(t32);
      if (fabsf(t32 - tq) > 0.5f - 1e-5f) tq = (float)rint(((double)vv - (double)z32) / (double)sc32);
      tq = fminf(fmaxf(tq, 0.f), vlevels);
      code = (int)tq;
    }
    if (L.vb == 2) {
      // packed codes: channel 4i + m' of a row in bits 2m', 2m'+1 of byte i
      const unsigned lo = __ballot_sync(0xffffffffu, code & 1);
      const unsigned hi = __ballot_sync(0xffffffffu, (code >> 1) & 1);
      if (lane == 0) {
        uint32_t *dst = reinterpret_cast<uint32_t *>(tile + L.vplanes + slot * L.packed_row_bytes + 8 * m);
        dst[0] = spread_bits16(lo & 0xFFFFu) | (spread_bits16(hi & 0xFFFFu) << 1);
        dst[1] = spread_bits16(lo >> 16) | (spread_bits16(hi >> 16) << 1);
      }
    } else {
      for (int p = 0; p < L.vb; ++p) {
        const unsigned word = __ballot_sync(0xffffffffu, (code >> p) & 1);
        if (lane == 0)
          *reinterpret_cast<uint32_t *>(tile + L.vplanes + p * L.plane_bytes + slot * L.row_bytes + 4 * m) = word;
      }
    }
    if (lane == 0)
      *reinterpret_cast<__half2 *>(tile + L.vsz + (slot * L.groups + m) * 4) = __halves2half2(scale16, zero16);
  }
}

}  // namespace tq
