// Explicit reconstruction of cached tokens (the audit's
// quantizer.dequantize(prod_q), "turboquant/audit_claims.py", AUDIT 2):
//   k_hat = ||k|| * (Pi^T c + sqrt(pi/2)/d * ||r|| * S^T (2 sign - 1))
//   v_hat = code * scale + zero     (TurboQuant-MSE values: ||v|| Pi^T c[cell])
// One CTA per (token, KV head); thread j produces output coordinate j by
// walking column j of Pi and S (coalesced across threads).
#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

namespace {

// head dim D: one thread per output coordinate
template <int D>
__global__ void __launch_bounds__(D) dequantize_kernel(DequantArgs a) {
  const int i = blockIdx.x;   // token offset in [0, count)
  const int h = blockIdx.y;
  const int j = threadIdx.x;
  const TileLayout L = TileLayout::make(a.key_bits, a.value_bits, a.value_mode, D);
  const int n = a.start + i;
  const uint8_t *tp = tile_ptr(const_cast<void *>(a.data), L, a.h_kv, a.ntiles, a.b, h, n / kTile);
  const int slot = n % kTile;
  __shared__ float c[D], sg[D], cv[D];
  const int byte = j >> 3, bit = j & 7;
  int idx = 0;
  for (int p = 0; p < L.mb; ++p)
    idx |= ((tp[L.kplanes + p * L.plane_bytes + slot * L.row_bytes + byte] >> bit) & 1) << p;
  const int sbit = (tp[L.signs + slot * L.row_bytes + byte] >> bit) & 1;
  const int code = value_code(tp, L, slot, j);
  c[j] = a.centroids[idx];
  sg[j] = sbit ? 1.f : -1.f;
  if (L.mse) cv[j] = a.v_centroids[code];
  __syncthreads();
  const __half2 nr = *reinterpret_cast<const __half2 *>(tp + L.norms + slot * 4);
  const float nk = __low2float(nr), rn = __high2float(nr);
  float mse = 0.f, qjl = 0.f;
  for (int r = 0; r < D; ++r) {
    mse = fmaf(a.pi[(size_t)r * D + j], c[r], mse);
    qjl = fmaf(a.s[(size_t)r * D + j], sg[r], qjl);
  }
  const size_t o = ((size_t)i * a.h_kv + h) * D + j;
  a.k_out[o] = nk * fmaf(qjl_kappa(D) * rn, qjl, mse);
  if (L.mse) {
    float v = 0.f;
    for (int r = 0; r < D; ++r) v = fmaf(a.pi[(size_t)r * D + j], cv[r], v);
    a.v_out[o] = __half2float(*reinterpret_cast<const __half *>(tp + L.vsz + slot * 2)) * v;
    return;
  }
  const __half2 sz = *reinterpret_cast<const __half2 *>(tp + L.vsz + (slot * L.groups + j / kGroup) * 4);
  a.v_out[o] = fmaf((float)code, __low2float(sz), __high2float(sz));
}

}  // namespace

cudaError_t launch_dequantize(const DequantArgs &a, cudaStream_t stream) {
  if (a.count <= 0) return cudaSuccess;
  dim3 grid(a.count, a.h_kv);
  switch (a.d) {
    case 64: dequantize_kernel<64><<<grid, 64, 0, stream>>>(a); break;
    case 128: dequantize_kernel<128><<<grid, 128, 0, stream>>>(a); break;
    case 256: dequantize_kernel<256><<<grid, 256, 0, stream>>>(a); break;
    default: return cudaErrorNotSupported;
  }
  return cudaGetLastError();
}

}  // namespace tq
