// Group quantization of values for the tensor-core append path, as its own
// bandwidth-bound kernel ("turboquant/audit_claims.py", AUDIT 1:
// value_bits, value_group_size): per group of 32 channels of one token's
// head vector, zero = fp16(min), scale = fp16((max - min) / (2^vb - 1))
// rounded once from the exact quotient, code = clamp(rint((v - zero) /
// scale)) of the exact quotient (half to even).
//
// A lane takes one group (four 16-byte loads of bf16), so four lanes take a
// vector and a warp streams eight consecutive vectors (2 KB) per round; two
// rounds' loads are issued before either is quantized.  The vector slot
// id = (b T + t) H_kv + h gives the input offset directly; the division into
// (b, t, h) and the record address are computed by one lane per vector and
// handed to its group lanes by shuffles.
//
// Codes.  For 2-bit values the code is the number of the group's three
// rounding thresholds z + (k + 1/2) s below v, compared on bf16 pairs: each
// threshold rounded down to bf16, or for an odd k (a tie rounds up to the
// even code) whose threshold is a bf16, the bf16 just below it.  That is the
// rounded exact quotient by comparisons alone.  For 3 and 4 bits the code is
// rint of the float32 quotient, redone in float64 where it sits within 1e-5
// of a half-integer.  The records' value sections (codes, scale, zero) are
// written in place; the key sections are the tensor-core kernel's.  Head dim
// 128, bf16 input.
#include "sm100.cuh"
#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

namespace {

constexpr int kVqThreads = 256;
constexpr int kVqRounds = 2;  // rounds of 8 vectors per warp iteration

// fp16 scale of a group: the float64 difference and quotient, rounded once
// to fp16 (the same operations as the float64 definition).
__device__ __forceinline__ __half group_scale(float mn, float mx, int levels) {
  return __double2half(((double)mx - (double)mn) / (double)levels);
}

// The largest bf16 below a finite bf16 b (as raw bits).
__device__ __forceinline__ unsigned short bf16_below(unsigned short b) {
  if ((b & 0x7fffu) == 0u) return 0x8001u;  // below +-0: the negative of the least subnormal
  return (b & 0x8000u) ? (unsigned short)(b + 1u) : (unsigned short)(b - 1u);
}

// The three rounding thresholds of 2-bit codes as bf16 pairs.  Threshold k
// is t = z + (k + 1/2) s; one FMA rounded down and one rounded up bracket it
// and agree exactly when t is a float.  A bf16 value v is above t iff it is
// above t rounded down to bf16; for odd k, where a tie rounds up to the even
// code, v counts when it equals t, i.e. when it is above the bf16 below t.
__device__ __forceinline__ void thresholds2(__half zero16, __half scale16, __nv_bfloat162 (&thr)[3]) {
  const float z = __half2float(zero16), s = __half2float(scale16);
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    unsigned short tb;
    if (s == 0.f) {
      tb = 0x7f80u;  // +inf: zero scale, every code 0
    } else {
      const float tlo = __fmaf_rd((float)k + 0.5f, s, z), thi = __fmaf_ru((float)k + 0.5f, s, z);
      const __nv_bfloat16 b = __float2bfloat16_rd(tlo);
      tb = __bfloat16_as_ushort(b);
      // odd k: a value equal to the threshold rounds up (to the even code)
      if ((k & 1) && tlo == thi && __bfloat162float(b) == tlo) tb = bf16_below(tb);
    }
    const __nv_bfloat16 bt = __ushort_as_bfloat16(tb);
    thr[k] = __halves2bfloat162(bt, bt);
  }
}

// Packed 2-bit codes of 16 bf16 channels (8 words of channel pairs; channel
// 4i + m in bits 2m, 2m+1 of byte i): the number of thresholds below each
// value, two channels per comparison.  With the masks m_k (0xffff where a
// channel is above threshold k), bit 1 of the code is m_1 and bit 0 is
// m_0 ^ m_1 ^ m_2 (the thresholds ascend).
__device__ __forceinline__ uint32_t codes2_word(const uint32_t *xw, const __nv_bfloat162 (&thr)[3]) {
  uint32_t w = 0u;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const __nv_bfloat162 x2 = *reinterpret_cast<const __nv_bfloat162 *>(&xw[j]);
    const uint32_t m0 = __hgt2_mask(x2, thr[0]), m1 = __hgt2_mask(x2, thr[1]), m2 = __hgt2_mask(x2, thr[2]);
    // channel 2j in bits 0-1, channel 2j + 1 in bits 16-17
    const uint32_t c = ((m0 ^ m1 ^ m2) & 0x00010001u) | (m1 & 0x00020002u);
    w |= ((c | (c >> 14)) & 0xfu) << (4 * j);
  }
  return w;
}

template <int VB>
__global__ void __launch_bounds__(kVqThreads) value_quant_kernel(const __grid_constant__ AppendArgs a) {
  const TileLayout L = TileLayout::make(a.key_bits, VB, a.value_mode, kD);
  sm100::pdl_trigger();  // see the tensor-core append kernel
  const int lane = threadIdx.x & 31;
  const int vl = lane >> 2, g = lane & 3;  // vector of the round, its value group
  const long long total = (long long)a.batch * a.T * a.h_kv;
  const unsigned per_b = (unsigned)a.T * (unsigned)a.h_kv;  // < 2^31 (the host checks)
  const long long nwarps = (long long)gridDim.x * (kVqThreads / 32);
  constexpr int kLevels = (1 << VB) - 1;
  constexpr int kVecs = 8 * kVqRounds;  // vectors per warp iteration
  for (long long id0 = ((long long)blockIdx.x * (kVqThreads / 32) + (threadIdx.x >> 5)) * kVecs; id0 < total;
       id0 += nwarps * kVecs) {
    // lane j < kVecs: where vector id0 + j goes (record offset, slot; -1: none)
    long long roff = -1;
    int rslot = 0;
    if (lane < kVecs && id0 + lane < total) {
      const long long id = id0 + lane;
      const int b = (int)(id / per_b);
      const unsigned rem = (unsigned)(id - (long long)b * per_b);
      const unsigned t = rem / (unsigned)a.h_kv;
      const unsigned h = rem - t * (unsigned)a.h_kv;
      if ((int)t < a.nnew[b]) {
        const int pos = a.lens[b] + (int)t;
        roff = (long long)((((size_t)b * a.h_kv + h) * (size_t)a.ntiles + (size_t)(pos / kTile)) *
                           (size_t)L.tile_bytes);
        rslot = pos % kTile;
      }
    }
    // issue every load of the iteration first: this lane's group of 32
    // channels (64 bytes) of each round's vector
    uint4 raw[kVqRounds][4];
#pragma unroll
    for (int u = 0; u < kVqRounds; ++u) {
      const long long id = id0 + 8 * u + vl;
      const bool in = id < total;
      const uint4 *src = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(a.v) +
                                                         (size_t)(in ? id : 0) * kD + 32 * g);
#pragma unroll
      for (int c = 0; c < 4; ++c) raw[u][c] = in ? src[c] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kVqRounds; ++u) {
      const long long off = __shfl_sync(0xffffffffu, roff, 8 * u + vl);
      const int slot = __shfl_sync(0xffffffffu, rslot, 8 * u + vl);
      const uint32_t *xw = reinterpret_cast<const uint32_t *>(&raw[u][0]);  // 16 bf16 pairs
      float mn, mx;
      {
        __nv_bfloat162 lo2 = *reinterpret_cast<const __nv_bfloat162 *>(&xw[0]), hi2 = lo2;
#pragma unroll
        for (int k = 1; k < 16; ++k) {
          const __nv_bfloat162 x2 = *reinterpret_cast<const __nv_bfloat162 *>(&xw[k]);
          lo2 = __hmin2(lo2, x2);
          hi2 = __hmax2(hi2, x2);
        }
        mn = fminf(__low2float(lo2), __high2float(lo2));
        mx = fmaxf(__low2float(hi2), __high2float(hi2));
      }
      const __half zero16 = __float2half_rn(mn);
      const __half scale16 = group_scale(mn, mx, kLevels);
      if (off < 0) continue;  // no collectives follow
      uint8_t *tile = reinterpret_cast<uint8_t *>(a.data) + off;
      if constexpr (VB == 2) {
        // packed: the group's 32 channels are bytes 8 g .. 8 g + 7 of the row
        __nv_bfloat162 thr[3];
        thresholds2(zero16, scale16, thr);
        *reinterpret_cast<uint2 *>(tile + L.vplanes + slot * L.packed_row_bytes + 8 * g) =
            make_uint2(codes2_word(xw, thr), codes2_word(xw + 8, thr));
      } else {
        const float z32 = __half2float(zero16), sc32 = __half2float(scale16);
        const float rsc = sc32 != 0.f ? 1.f / sc32 : 0.f;
        uint32_t pw[VB];
#pragma unroll
        for (int p = 0; p < VB; ++p) pw[p] = 0u;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float x = __uint_as_float(e & 1 ? (xw[e >> 1] & 0xffff0000u) : (xw[e >> 1] << 16));
          const float tq = (x - z32) * rsc;
          float r = rintf(tq);
          if (fabsf(tq - r) > 0.5f - 1e-5f) r = (float)rint(((double)x - (double)z32) / (double)sc32);
          const uint32_t code = sc32 != 0.f ? (uint32_t)min(max((int)r, 0), kLevels) : 0u;
#pragma unroll
          for (int p = 0; p < VB; ++p) pw[p] |= ((code >> p) & 1u) << e;
        }
        // plane p: bytes 4 g .. 4 g + 3 of the row hold bit p of the group's channels
#pragma unroll
        for (int p = 0; p < VB; ++p)
          *reinterpret_cast<uint32_t *>(tile + L.vplanes + p * L.plane_bytes + slot * L.row_bytes + 4 * g) = pw[p];
      }
      *reinterpret_cast<__half2 *>(tile + L.vsz + (slot * L.groups + g) * 4) = __halves2half2(scale16, zero16);
    }
  }
}

}  // namespace

cudaError_t launch_value_quant(const AppendArgs &a, int num_sms, cudaStream_t stream) {
  const long long total = (long long)a.batch * a.T * a.h_kv;
  if (total == 0) return cudaSuccess;
  const long long per_block = 8LL * kVqRounds * (kVqThreads / 32);  // vectors per block iteration
  const long long blocks = (total + per_block - 1) / per_block;
  const int grid = (int)std::min<long long>(blocks, 8LL * num_sms);
  switch (a.value_bits) {
    case 2: value_quant_kernel<2><<<grid, kVqThreads, 0, stream>>>(a); break;
    case 3: value_quant_kernel<3><<<grid, kVqThreads, 0, stream>>>(a); break;
    case 4: value_quant_kernel<4><<<grid, kVqThreads, 0, stream>>>(a); break;
    default: return cudaErrorNotSupported;
  }
  return cudaGetLastError();
}

}  // namespace tq
