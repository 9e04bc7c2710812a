// Group quantization of values for the tensor-core append path, as its own
// bandwidth-bound kernel ("turboquant/audit_claims.py", AUDIT 1:
// value_bits, value_group_size): per group of 32 channels of one token's
// head vector, zero = fp16(min), scale = fp16((max - min) / (2^vb - 1))
// rounded once from the exact quotient, code = clamp(rint((v - zero) /
// scale)) of the exact quotient.
//
// One warp per (token, KV head) vector: lane i holds channels 4i .. 4i+3
// (one 8-byte load of bf16 or 16 bytes of fp32), a group is 8 lanes, min and
// max by three shuffles.  Codes use the reciprocal of the fp16 scale and are
// redone in float64 where the product sits next to a half-integer, so every
// code is the rounded exact quotient.  The records' value sections (codes,
// scale, zero) are written in place; the key sections are the tensor-core
// kernel's.  Grid-stride over all B x T x H_kv vector slots.
#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

namespace {

constexpr int kVqThreads = 256;

__global__ void __launch_bounds__(kVqThreads) value_quant_kernel(const __grid_constant__ AppendArgs a) {
  const TileLayout L = TileLayout::make(a.key_bits, a.value_bits, a.value_mode);
  const int lane = threadIdx.x & 31;
  const long long per_b = (long long)a.T * a.h_kv;
  const long long total = (long long)a.batch * per_b;
  const long long nwarps = (long long)gridDim.x * (kVqThreads / 32);
  const float vlevels = (float)((1 << a.value_bits) - 1);
  const int ilev = (1 << a.value_bits) - 1;
  const unsigned gmask = 0xFFu << (lane & 24);  // the 8 lanes of this lane's group
  for (long long id = (long long)blockIdx.x * (kVqThreads / 32) + (threadIdx.x >> 5); id < total;
       id += nwarps) {
    const int b = (int)(id / per_b);
    const long long rem = id - (long long)b * per_b;
    const int t = (int)(rem / a.h_kv), h = (int)(rem - (long long)t * a.h_kv);
    if (t >= a.nnew[b]) continue;  // warp-uniform
    const size_t base = (((size_t)b * a.T + t) * a.h_kv + h) * kD + 4 * lane;
    float x[4];
    if (a.dtype == TQ_BF16) {
      const uint2 raw = *reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(a.v) + base);
      const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
      const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
      x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y;
    } else {
      const float4 f = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.v) + base);
      x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
    }
    float mn = fminf(fminf(x[0], x[1]), fminf(x[2], x[3]));
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const __half zero16 = __float2half_rn(mn);
    const __half scale16 = __double2half(((double)mx - (double)mn) / (double)vlevels);
    const float z32 = __half2float(zero16), sc32 = __half2float(scale16);
    int code[4] = {0, 0, 0, 0};
    if (sc32 != 0.f) {
      const float rsc = 1.f / sc32;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float tq = (x[k] - z32) * rsc;
        float r = rintf(tq);
        if (fabsf(tq - r) > 0.5f - 1e-5f) r = (float)rint(((double)x[k] - (double)z32) / (double)sc32);
        code[k] = min(max((int)r, 0), ilev);
      }
    }
    const int pos = a.lens[b] + t;
    uint8_t *tile = tile_ptr(a.data, L, a.h_kv, a.ntiles, b, h, pos / kTile);
    const int slot = pos % kTile;
    if (L.vb == 2) {
      // packed: channel 4i + m of the row in bits 2m, 2m+1 of byte i
      tile[L.vplanes + slot * kPackedRowBytes + lane] =
          (uint8_t)(code[0] | (code[1] << 2) | (code[2] << 4) | (code[3] << 6));
    } else {
      // plane p, word w holds bit p of channels 32w .. 32w+31
      for (int p = 0; p < L.vb; ++p) {
        uint32_t nib = 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k) nib |= (uint32_t)((code[k] >> p) & 1) << k;
        const uint32_t word = __reduce_or_sync(gmask, nib << (4 * (lane & 7)));
        if ((lane & 7) == 0)
          *reinterpret_cast<uint32_t *>(tile + L.vplanes + p * kPlaneBytes + slot * kRowBytes + 4 * (lane >> 3)) =
              word;
      }
    }
    if ((lane & 7) == 0)
      *reinterpret_cast<__half2 *>(tile + L.vsz + (slot * kGroups + (lane >> 3)) * 4) =
          __halves2half2(scale16, zero16);
  }
}

}  // namespace

cudaError_t launch_value_quant(const AppendArgs &a, int num_sms, cudaStream_t stream) {
  const long long total = (long long)a.batch * a.T * a.h_kv;
  if (total == 0) return cudaSuccess;
  const long long blocks = (total + kVqThreads / 32 - 1) / (kVqThreads / 32);
  const int grid = (int)std::min<long long>(blocks, 8LL * num_sms);
  value_quant_kernel<<<grid, kVqThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace tq
