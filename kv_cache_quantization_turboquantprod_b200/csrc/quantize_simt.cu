// quantize_append, SIMT form: TurboQuant-prod key encoding and value
// quantization of new tokens, written straight into the tiled cache, for
// head dims 64, 128 and 256.
//
// Keys ("TurboQuant" explainer, troisinh.com, "Ý tưởng cốt lõi";
// "turboquant/audit_claims.py", AUDIT 1 / AUDIT 5): u = k/||k||, y = Pi u,
// idx = #{boundaries < y}, r = u - Pi^T c, signs = [S r >= 0], ||r||.
// Values (AUDIT 1, value_bits / value_group_size): per 32-channel group
// min/max, fp16 zero = min, fp16 scale = (max-min)/(2^vb - 1) rounded once
// from the exact quotient, code = clamp(rint((v - zero)/scale)) of the exact
// quotient (float64 where single precision could round it the other way).
// TurboQuant-MSE values ("03. Results & Benchmarks", "At a Glance ->
// Compression"): the value's norm and the Lloyd-Max cells of Pi v / ||v||.
//
// This form serves large appends (small ones take quantize_warp.cu).
// A persistent CTA encodes kNV vectors per pass: three D x D mat-vecs per
// vector (Pi u, Pi^T c, S r; and Pi w for MSE values) in fp32 with a fixed
// accumulation order per output.  Up to D = 128, Pi and S sit in shared
// memory (rows padded to D + 1 floats so row and column walks are
// bank-conflict free); at D = 256 they are read from global memory (L2).  A
// sketch component within 1e-5 of zero has its sign decided again in float64.
#include <stddef.h>

#include "quantize_common.cuh"
#include "sm100.cuh"
#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

namespace {

constexpr int kThreads = 256;

template <int kNV, int D>
struct QuantSmem {
  static constexpr bool kMatsInSmem = D <= 128;
  static constexpr int kPad = D + 1;
  static constexpr int kMatFloats = kMatsInSmem ? D * kPad : 1;
  // arrays read with 16-byte vector loads start on 16-byte boundaries
  alignas(16) float pi[kMatFloats];
  alignas(16) float s[kMatFloats];
  alignas(16) float u[kNV][D];
  alignas(16) float c[kNV][D];
  alignas(16) float r[kNV][D];
  float rn2[kNV][D / 32];
  float nk[kNV];
  float cent[16];
  float bnd[16];
  uint32_t nearw[kNV][D / 32];  // sketch components to re-decide in float64
  // TurboQuant-MSE values: unit value vectors, norms, the values' codebook
  alignas(16) float w[kNV][D];
  float nv[kNV];
  float vcent[16];
  float vbnd[16];
};

// Element (i, j) of a row-major D x D matrix: shared memory (padded rows) up
// to D = 128, global memory above.
template <int kNV, int D>
__device__ __forceinline__ float mat_at(const float *sm, const float *gm, int i, int j) {
  if constexpr (QuantSmem<kNV, D>::kMatsInSmem) return sm[i * QuantSmem<kNV, D>::kPad + j];
  else return __ldg(gm + (size_t)i * D + j);
}

template <int kNV, int D>
__global__ void __launch_bounds__(kThreads, 1)
quantize_append_simt_kernel(const __grid_constant__ AppendArgs a) {
  using SM = QuantSmem<kNV, D>;
  constexpr int C = D / 32;                // elements per lane of one vector
  constexpr int NG = kThreads / D;         // thread groups (one coordinate each)
  constexpr int VPT = kNV / NG;            // vectors per thread in the mat-vec phases
  static_assert(VPT >= 1 && kNV % NG == 0, "vectors per pass");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SM &S = *reinterpret_cast<SM *>(smem_raw);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const TileLayout L = TileLayout::make(a.key_bits, a.value_bits, a.value_mode, D);
  const int ncent = 1 << L.mb;
  const int nvcent = 1 << L.vb;
  // a decode call's query kernel may start now: it reads none of this
  // kernel's output and waits for this grid before it finishes
  sm100::pdl_trigger();

  if constexpr (SM::kMatsInSmem) {
    stage_matrix<D>(S.pi, SM::kPad, a.pi, tid, kThreads);
    stage_matrix<D>(S.s, SM::kPad, a.s, tid, kThreads);
  }
  if (tid < ncent) S.cent[tid] = a.centroids[tid];
  if (tid < ncent - 1) S.bnd[tid] = a.boundaries[tid];
  if (L.mse && tid < nvcent) S.vcent[tid] = a.v_centroids[tid];
  if (L.mse && tid < nvcent - 1) S.vbnd[tid] = a.v_boundaries[tid];
  __syncthreads();

  const long long total = (long long)a.batch * a.T * a.h_kv;
  const long long nchunks = (total + kNV - 1) / kNV;
  const float vlevels = (float)((1 << a.value_bits) - 1);
  // the mat-vec phases: thread -> coordinate i, vectors v0 .. v0 + VPT - 1
  const int i = tid % D;
  const int v0 = (tid / D) * VPT;

  for (long long chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x) {
    const long long id0 = chunk * kNV;

    if (tid < kNV * C) S.nearw[tid / C][tid % C] = 0u;
    // ---- phase 0: load, normalise keys; quantize values ----------------
    for (int vi = warp; vi < kNV; vi += kThreads / 32) {
      int b, t, h;
      bool valid;
      vec_coords(a, id0 + vi, b, t, h, valid);
      float x[C];
      float ss = 0.f;
      const size_t base = valid ? ((((size_t)b * a.T + t) * a.h_kv + h) * D) : 0;
#pragma unroll
      for (int m = 0; m < C; ++m) {
        x[m] = valid ? load_elem(a.k, a.dtype, base + lane + 32 * m) : 0.f;
        ss = fmaf(x[m], x[m], ss);
      }
      ss = warp_sum(ss);
      const float nk = sqrtf(ss);
#pragma unroll
      for (int m = 0; m < C; ++m) S.u[vi][lane + 32 * m] = nk > 0.f ? __fdiv_rn(x[m], nk) : 0.f;
      if (lane == 0) S.nk[vi] = nk;

      if (L.mse) {
        // TurboQuant-MSE values: the unit vector (rotated and bucketized in
        // phase 1b) and its norm
        float y[C], sv = 0.f;
#pragma unroll
        for (int m = 0; m < C; ++m) {
          y[m] = valid ? load_elem(a.v, a.dtype, base + lane + 32 * m) : 0.f;
          sv = fmaf(y[m], y[m], sv);
        }
        const float nv = sqrtf(warp_sum(sv));
#pragma unroll
        for (int m = 0; m < C; ++m) S.w[vi][lane + 32 * m] = nv > 0.f ? __fdiv_rn(y[m], nv) : 0.f;
        if (lane == 0) S.nv[vi] = nv;
      } else if (valid) {
        const int pos = a.lens[b] + t;
        quantize_value_groups<D>(a, L, tile_ptr(a.data, L, a.h_kv, a.ntiles, b, h, pos / kTile), pos % kTile,
                                 base, vlevels);
      }
    }
    __syncthreads();

    // ---- phase 1: y = Pi u, bucketize, pack code planes ------------------
    {
      float acc[VPT];
#pragma unroll
      for (int v = 0; v < VPT; ++v) acc[v] = 0.f;
      for (int j = 0; j < D; j += 4) {
        const float w0 = mat_at<kNV, D>(S.pi, a.pi, i, j), w1 = mat_at<kNV, D>(S.pi, a.pi, i, j + 1);
        const float w2 = mat_at<kNV, D>(S.pi, a.pi, i, j + 2), w3 = mat_at<kNV, D>(S.pi, a.pi, i, j + 3);
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
          const float4 uu = *reinterpret_cast<const float4 *>(&S.u[v0 + v][j]);
          acc[v] = fmaf(w0, uu.x, acc[v]);
          acc[v] = fmaf(w1, uu.y, acc[v]);
          acc[v] = fmaf(w2, uu.z, acc[v]);
          acc[v] = fmaf(w3, uu.w, acc[v]);
        }
      }
#pragma unroll
      for (int v = 0; v < VPT; ++v) {
        const int vi = v0 + v;
        int b, t, h;
        bool valid;
        vec_coords(a, id0 + vi, b, t, h, valid);
        int idx = 0;
        for (int q = 0; q < ncent - 1; ++q) idx += (S.bnd[q] < acc[v]) ? 1 : 0;
        const bool zero = !(S.nk[vi] > 0.f);
        if (zero) idx = 0;
        S.c[vi][i] = zero ? 0.f : S.cent[idx];
        if (valid) {
          const int pos = a.lens[b] + t;
          uint8_t *tile = tile_ptr(a.data, L, a.h_kv, a.ntiles, b, h, pos / kTile);
          const int slot = pos % kTile;
          for (int p = 0; p < L.mb; ++p) {
            const unsigned word = __ballot_sync(0xffffffffu, (idx >> p) & 1);
            if (lane == 0)
              *reinterpret_cast<uint32_t *>(tile + L.kplanes + p * L.plane_bytes + slot * L.row_bytes +
                                            4 * (i >> 5)) = word;
          }
        }
      }
    }
    // ---- phase 1b (MSE values): y = Pi w, value cells, value norm ---------
    if (L.mse) {
      float acc[VPT];
#pragma unroll
      for (int v = 0; v < VPT; ++v) acc[v] = 0.f;
      for (int j = 0; j < D; j += 4) {
        const float w0 = mat_at<kNV, D>(S.pi, a.pi, i, j), w1 = mat_at<kNV, D>(S.pi, a.pi, i, j + 1);
        const float w2 = mat_at<kNV, D>(S.pi, a.pi, i, j + 2), w3 = mat_at<kNV, D>(S.pi, a.pi, i, j + 3);
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
          const float4 ww = *reinterpret_cast<const float4 *>(&S.w[v0 + v][j]);
          acc[v] = fmaf(w0, ww.x, acc[v]);
          acc[v] = fmaf(w1, ww.y, acc[v]);
          acc[v] = fmaf(w2, ww.z, acc[v]);
          acc[v] = fmaf(w3, ww.w, acc[v]);
        }
      }
#pragma unroll
      for (int v = 0; v < VPT; ++v) {
        const int vi = v0 + v;
        int b, t, h;
        bool valid;
        vec_coords(a, id0 + vi, b, t, h, valid);
        int idx = 0;
        for (int q = 0; q < nvcent - 1; ++q) idx += (S.vbnd[q] < acc[v]) ? 1 : 0;
        if (!(S.nv[vi] > 0.f)) idx = 0;
        if (valid) {
          const int pos = a.lens[b] + t;
          uint8_t *tile = tile_ptr(a.data, L, a.h_kv, a.ntiles, b, h, pos / kTile);
          const int slot = pos % kTile;
          for (int p = 0; p < L.vb; ++p) {
            const unsigned word = __ballot_sync(0xffffffffu, (idx >> p) & 1);
            if (lane == 0)
              *reinterpret_cast<uint32_t *>(tile + L.vplanes + p * L.plane_bytes + slot * L.row_bytes +
                                            4 * (i >> 5)) = word;
          }
          if (i == 0) *reinterpret_cast<__half *>(tile + L.vsz + slot * 2) = __float2half_rn(S.nv[vi]);
        }
      }
    }
    __syncthreads();

    // ---- phase 2: r = u - Pi^T c, partial ||r||^2 -------------------------
    {
      const int j = i;
      float acc[VPT];
#pragma unroll
      for (int v = 0; v < VPT; ++v) acc[v] = 0.f;
      for (int k = 0; k < D; k += 4) {
        const float w0 = mat_at<kNV, D>(S.pi, a.pi, k, j), w1 = mat_at<kNV, D>(S.pi, a.pi, k + 1, j);
        const float w2 = mat_at<kNV, D>(S.pi, a.pi, k + 2, j), w3 = mat_at<kNV, D>(S.pi, a.pi, k + 3, j);
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
          const float4 cc = *reinterpret_cast<const float4 *>(&S.c[v0 + v][k]);
          acc[v] = fmaf(w0, cc.x, acc[v]);
          acc[v] = fmaf(w1, cc.y, acc[v]);
          acc[v] = fmaf(w2, cc.z, acc[v]);
          acc[v] = fmaf(w3, cc.w, acc[v]);
        }
      }
#pragma unroll
      for (int v = 0; v < VPT; ++v) {
        const int vi = v0 + v;
        const float rr = S.u[vi][j] - acc[v];
        S.r[vi][j] = rr;
        const float part = warp_sum(rr * rr);
        if (lane == 0) S.rn2[vi][j >> 5] = part;
      }
    }
    __syncthreads();

    // ---- phase 3: z = S r, sign plane, norms ------------------------------
    {
      float acc[VPT];
#pragma unroll
      for (int v = 0; v < VPT; ++v) acc[v] = 0.f;
      for (int j = 0; j < D; j += 4) {
        const float w0 = mat_at<kNV, D>(S.s, a.s, i, j), w1 = mat_at<kNV, D>(S.s, a.s, i, j + 1);
        const float w2 = mat_at<kNV, D>(S.s, a.s, i, j + 2), w3 = mat_at<kNV, D>(S.s, a.s, i, j + 3);
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
          const float4 rr = *reinterpret_cast<const float4 *>(&S.r[v0 + v][j]);
          acc[v] = fmaf(w0, rr.x, acc[v]);
          acc[v] = fmaf(w1, rr.y, acc[v]);
          acc[v] = fmaf(w2, rr.z, acc[v]);
          acc[v] = fmaf(w3, rr.w, acc[v]);
        }
      }
#pragma unroll
      for (int v = 0; v < VPT; ++v) {
        const int vi = v0 + v;
        int b, t, h;
        bool valid;
        vec_coords(a, id0 + vi, b, t, h, valid);
        const bool zero = !(S.nk[vi] > 0.f);
        const int bit = (!zero && acc[v] >= 0.f) ? 1 : 0;
        const unsigned word = __ballot_sync(0xffffffffu, bit);
        const unsigned nearb = __ballot_sync(0xffffffffu, valid && !zero && fabsf(acc[v]) < a.refine_z);
        if (lane == 0 && nearb) S.nearw[vi][i >> 5] = nearb;
        if (valid) {
          const int pos = a.lens[b] + t;
          uint8_t *tile = tile_ptr(a.data, L, a.h_kv, a.ntiles, b, h, pos / kTile);
          const int slot = pos % kTile;
          if (lane == 0) *reinterpret_cast<uint32_t *>(tile + L.signs + slot * L.row_bytes + 4 * (i >> 5)) = word;
          if (i == 0) {
            float rs = 0.f;
#pragma unroll
            for (int w = 0; w < C; ++w) rs += S.rn2[vi][w];
            const float rn = zero ? 0.f : sqrtf(rs);
            __half2 nr = __halves2half2(__float2half_rn(S.nk[vi]), __float2half_rn(rn));
            *reinterpret_cast<__half2 *>(tile + L.norms + slot * 4) = nr;
          }
        }
      }
    }
    __syncthreads();

    // ---- phase 4: sketch components next to zero, signs again in float64 --
    for (int vi = warp; vi < kNV; vi += kThreads / 32) {
      uint32_t nw[C];
      uint32_t any = 0u;
#pragma unroll
      for (int w = 0; w < C; ++w) {
        nw[w] = S.nearw[vi][w];
        any |= nw[w];
      }
      if (!any) continue;
      int b, t, h;
      bool valid;
      vec_coords(a, id0 + vi, b, t, h, valid);  // flagged vectors are valid
      const int pos = a.lens[b] + t;
      uint8_t *tile = tile_ptr(a.data, L, a.h_kv, a.ntiles, b, h, pos / kTile);
      const int slot = pos % kTile;
      uint32_t planes[3][C], sw[C];
#pragma unroll
      for (int w = 0; w < C; ++w) {
#pragma unroll
        for (int p = 0; p < 3; ++p)
          planes[p][w] = p < L.mb ? *reinterpret_cast<const uint32_t *>(tile + L.kplanes + p * L.plane_bytes +
                                                                        slot * L.row_bytes + 4 * w)
                                  : 0u;
        sw[w] = *reinterpret_cast<const uint32_t *>(tile + L.signs + slot * L.row_bytes + 4 * w);
      }
      const size_t kbase = (((size_t)b * a.T + t) * a.h_kv + h) * D;
      refine_signs_f64<D>(a.s, a.s_pit, S.cent, a.k, a.dtype, kbase, planes, nw, sw, 0);
      if (lane == 0) {
        int nbits = 0;
#pragma unroll
        for (int w = 0; w < C; ++w) {
          *reinterpret_cast<uint32_t *>(tile + L.signs + slot * L.row_bytes + 4 * w) = sw[w];
          nbits += __popc(nw[w]);
        }
        if (a.refine_count) atomicAdd(a.refine_count, (unsigned long long)nbits);
      }
    }
    __syncthreads();
  }
}

template <int kNV, int D>
cudaError_t launch_simt_nv(const AppendArgs &a, int num_sms, cudaStream_t stream) {
  const size_t smem = sizeof(QuantSmem<kNV, D>);
  static_assert(sizeof(QuantSmem<kNV, D>) <= 227 * 1024, "shared memory per CTA");
  using SMT = QuantSmem<kNV, D>;
  static_assert(offsetof(SMT, w) % 16 == 0 && offsetof(SMT, r) % 16 == 0, "16-byte loads of the vector arrays");
  cudaError_t e = cudaFuncSetAttribute(quantize_append_simt_kernel<kNV, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long total = (long long)a.batch * a.T * a.h_kv;
  const long long nchunks = (total + kNV - 1) / kNV;
  const int grid = (int)std::min<long long>(nchunks, (long long)num_sms);
  if (grid <= 0) return cudaSuccess;
  quantize_append_simt_kernel<kNV, D><<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

// 16 vectors per pass (small appends take the warp-per-vector kernel)
template <int D>
cudaError_t launch_simt_d(const AppendArgs &a, int num_sms, cudaStream_t stream) {
  return launch_simt_nv<16, D>(a, num_sms, stream);
}

}  // namespace

// W = S Pi^T in float64: one thread per entry (j, m), the d products of the
// float32 entries summed in float64 in index order.  A one-off per layer.
__global__ void sketch_product_kernel(const float *__restrict__ pi, const float *__restrict__ s, int d,
                                      double *__restrict__ out) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= d * d) return;
  const int j = e / d, m = e - j * d;
  const float *srow = s + (size_t)j * d, *prow = pi + (size_t)m * d;
  double acc = 0.0;
  for (int i = 0; i < d; ++i) acc = fma((double)srow[i], (double)prow[i], acc);
  out[e] = acc;
}

cudaError_t launch_sketch_product(const float *pi, const float *s, int d, double *out, cudaStream_t stream) {
  const int n = d * d;
  sketch_product_kernel<<<(n + 255) / 256, 256, 0, stream>>>(pi, s, d, out);
  return cudaGetLastError();
}

cudaError_t launch_quantize_simt(const AppendArgs &a, int num_sms, cudaStream_t stream) {
  // Up to eight vector slots per SM (a decode step appends one token per
  // sequence and head) the warp-per-vector kernel, which stages nothing, is
  // faster than staging Pi and S in every CTA.
  const long long total = (long long)a.batch * a.T * a.h_kv;
  if (total <= 8LL * num_sms) return launch_quantize_warp(a, num_sms, stream);
  switch (a.d) {
    case 64: return launch_simt_d<64>(a, num_sms, stream);
    case 128: return launch_simt_d<128>(a, num_sms, stream);
    case 256: return launch_simt_d<256>(a, num_sms, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace tq
