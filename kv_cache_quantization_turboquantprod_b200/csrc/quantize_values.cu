// Group quantization of values for the tensor-core append path, as its own
// bandwidth-bound kernel ("turboquant/audit_claims.py", AUDIT 1:
// value_bits, value_group_size): per group of 32 channels of one token's
// head vector, zero = fp16(min), scale = fp16((max - min) / (2^vb - 1))
// rounded once from the exact quotient, code = clamp(rint((v - zero) /
// scale)) of the exact quotient.
//
// Memory-level parallelism decides the speed of this streaming kernel: a
// half-warp takes one vector (16 lanes x 8 channels, one 16-byte load of
// bf16 per lane), a warp two, and every iteration issues the loads of four
// such pairs (eight vectors) before it quantizes any.  A group of 32
// channels is 4 lanes (min and max by two shuffles).  Codes use the
// reciprocal of the fp16 scale and are redone in float64 where the product
// sits next to a half-integer, so every code is the rounded exact quotient.
// The records' value sections (codes, scale, zero) are written in place;
// the key sections are the tensor-core kernel's.  Grid-stride over all
// B x T x H_kv vector slots; head dim 128, bf16 input (the tensor-core append
// path).
#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

namespace {

constexpr int kVqThreads = 256;
constexpr int kVqUnroll = 4;  // vector pairs in flight per warp

__global__ void __launch_bounds__(kVqThreads) value_quant_kernel(const __grid_constant__ AppendArgs a) {
  const TileLayout L = TileLayout::make(a.key_bits, a.value_bits, a.value_mode, kD);
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4, hl = lane & 15;  // vector of the pair, lane within it
  const long long per_b = (long long)a.T * a.h_kv;
  const long long total = (long long)a.batch * per_b;
  const long long npairs = (total + 1) / 2;
  const long long nwarps = (long long)gridDim.x * (kVqThreads / 32);
  const float vlevels = (float)((1 << a.value_bits) - 1);
  const int ilev = (1 << a.value_bits) - 1;
  for (long long p0 = ((long long)blockIdx.x * (kVqThreads / 32) + (threadIdx.x >> 5)) * kVqUnroll;
       p0 < npairs; p0 += nwarps * kVqUnroll) {
    // issue every load of the iteration first
    uint4 raw[kVqUnroll];
    int vb_[kVqUnroll], vt_[kVqUnroll], vh_[kVqUnroll];
    bool ok[kVqUnroll];
#pragma unroll
    for (int u = 0; u < kVqUnroll; ++u) {
      const long long id = 2 * (p0 + u) + half;
      ok[u] = id < total;
      int b = 0, t = 0, h = 0;
      if (ok[u]) {
        b = (int)(id / per_b);
        const long long rem = id - (long long)b * per_b;
        t = (int)(rem / a.h_kv);
        h = (int)(rem - (long long)t * a.h_kv);
        ok[u] = t < a.nnew[b];
      }
      vb_[u] = b; vt_[u] = t; vh_[u] = h;
      const size_t base = (((size_t)b * a.T + t) * a.h_kv + h) * kD + 8 * hl;
      raw[u] = ok[u] ? *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(a.v) + base)
                     : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kVqUnroll; ++u) {
      float x[8];
      const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&raw[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p2[e]);
        x[2 * e] = f.x;
        x[2 * e + 1] = f.y;
      }
      float mn = x[0], mx = x[0];
#pragma unroll
      for (int e = 1; e < 8; ++e) {
        mn = fminf(mn, x[e]);
        mx = fmaxf(mx, x[e]);
      }
      // a group of 32 channels = 4 consecutive lanes
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const __half zero16 = __float2half_rn(mn);
      const __half scale16 = __double2half(((double)mx - (double)mn) / (double)vlevels);
      const float z32 = __half2float(zero16), sc32 = __half2float(scale16);
      int code[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) code[e] = 0;
      if (sc32 != 0.f) {
        const float rsc = 1.f / sc32;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float tq = (x[e] - z32) * rsc;
          float r = rintf(tq);
          if (fabsf(tq - r) > 0.5f - 1e-5f) r = (float)rint(((double)x[e] - (double)z32) / (double)sc32);
          code[e] = min(max((int)r, 0), ilev);
        }
      }
      if (!ok[u]) continue;  // uniform within each half-warp; no collectives follow
      const int pos = a.lens[vb_[u]] + vt_[u];
      uint8_t *tile = tile_ptr(a.data, L, a.h_kv, a.ntiles, vb_[u], vh_[u], pos / kTile);
      const int slot = pos % kTile;
      if (L.vb == 2) {
        // packed: channel 4i + m in bits 2m, 2m+1 of byte i; this lane's 8
        // channels are bytes 2 hl and 2 hl + 1
        uint32_t w = 0u;
#pragma unroll
        for (int e = 0; e < 8; ++e) w |= (uint32_t)code[e] << (2 * e);
        *reinterpret_cast<uint16_t *>(tile + L.vplanes + slot * L.packed_row_bytes + 2 * hl) = (uint16_t)w;
      } else {
        // plane p: byte hl of the row holds bit p of this lane's 8 channels
        for (int p = 0; p < L.vb; ++p) {
          uint32_t byte = 0u;
#pragma unroll
          for (int e = 0; e < 8; ++e) byte |= (uint32_t)((code[e] >> p) & 1) << e;
          tile[L.vplanes + p * L.plane_bytes + slot * L.row_bytes + hl] = (uint8_t)byte;
        }
      }
      if ((hl & 3) == 0)
        *reinterpret_cast<__half2 *>(tile + L.vsz + (slot * L.groups + (hl >> 2)) * 4) =
            __halves2half2(scale16, zero16);
    }
  }
}

}  // namespace

cudaError_t launch_value_quant(const AppendArgs &a, int num_sms, cudaStream_t stream) {
  const long long total = (long long)a.batch * a.T * a.h_kv;
  if (total == 0) return cudaSuccess;
  const long long per_block = 2LL * kVqUnroll * (kVqThreads / 32);  // vectors per block iteration
  const long long blocks = (total + per_block - 1) / per_block;
  const int grid = (int)std::min<long long>(blocks, 8LL * num_sms);
  value_quant_kernel<<<grid, kVqThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace tq
