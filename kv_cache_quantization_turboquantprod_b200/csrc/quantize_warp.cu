// quantize_append for small appends (a decode step's one token per sequence
// and head): four warps per vector, each taking a quarter of every mat-vec.  Up to d = 128 the CTA first copies Pi and
// S into shared memory as they are (row-major, 16-byte asynchronous copies,
// all in flight at once); at d = 256 they are read from global memory
// (L1/L2).  Same encoding as the other append kernels ("TurboQuant"
// explainer, troisinh.com, "Ý tưởng cốt lõi"; "turboquant/audit_claims.py",
// AUDIT 1 / AUDIT 5): u = k/||k||, y = Pi u, idx = #{boundaries < y},
// r = u - Pi^T c, signs = [S r >= 0], ||r||; group-quantized values, or
// TurboQuant-MSE values ("03. Results & Benchmarks", "At a Glance ->
// Compression": the Lloyd-Max cells of Pi v/||v|| and ||v||).
//
// Layout in a warp.  A vector (u, r, the unit value) is held as lane l ->
// coordinates C l .. C l + C - 1 (C = D/32), so every row of Pi or S is one
// coalesced read.  M x for a block of 32 rows is the lanes' partial dot
// products reduced by recursive halving (31 shuffles for 32 rows), which
// leaves row r0 + l in lane l: exactly the order of a code-plane word, so
// one ballot per plane packs it.  The four warps of a quad take the 32-row
// blocks of Pi u and S r in turn, a quarter of the rows of Pi^T c each (the
// c_i and the partial sums meet in shared memory), and the value groups in
// turn.  Sketch components within 1e-5 of zero have their sign decided
// again in float64 (with W = S Pi^T).
#include "quantize_common.cuh"
#include "sm100.cuh"
#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

namespace {

constexpr int kWarpsPerCta = 8;

using sm100::cp_async16;
using sm100::cp_async_wait_all;

// C consecutive floats of row `row` of a row-major D x D matrix, this lane's
// coordinates C lane .. C lane + C - 1.
template <int D>
__device__ __forceinline__ void load_row_chunk(const float *__restrict__ M, int row, float (&w)[D / 32]) {
  constexpr int C = D / 32;
  const float *p = M + (size_t)row * D + C * (threadIdx.x & 31);
  if constexpr (C == 2) {
    const float2 t = *reinterpret_cast<const float2 *>(p);
    w[0] = t.x;
    w[1] = t.y;
  } else {
#pragma unroll
    for (int q = 0; q < C / 4; ++q) {
      const float4 t = *reinterpret_cast<const float4 *>(p + 4 * q);
      w[4 * q] = t.x;
      w[4 * q + 1] = t.y;
      w[4 * q + 2] = t.z;
      w[4 * q + 3] = t.w;
    }
  }
}

// (M x)[r0 + lane] for rows r0 .. r0 + 31 of M, x held as lane l -> x[C l ..].
template <int D>
__device__ __forceinline__ float rows32_dot(const float *__restrict__ M, int r0, const float (&x)[D / 32]) {
  constexpr int C = D / 32;
  constexpr int kBatch = 32 / C;  // rows whose loads are in flight together (32 floats a lane)
  const int lane = threadIdx.x & 31;
  float p[32];
#pragma unroll
  for (int r = 0; r < 32; r += kBatch) {
    float w[kBatch][C];
#pragma unroll
    for (int e = 0; e < kBatch; ++e) load_row_chunk<D>(M, r0 + r + e, w[e]);
#pragma unroll
    for (int e = 0; e < kBatch; ++e) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < C; ++m) acc = fmaf(w[e][m], x[m], acc);
      p[r + e] = acc;
    }
  }
  // recursive halving: after the step of width s, lane l keeps the sums of
  // the rows whose index agrees with l in the bits above and at s
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int q = 0; q < s; ++q) {
      const float send = upper ? p[q] : p[q + s];
      const float keep = upper ? p[q + s] : p[q];
      p[q] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return p[0];
}

// #{boundaries < y} over NB ascending boundaries (unused ones +inf).
template <int NB>
__device__ __forceinline__ int bucketize(const float (&bnd)[NB], float y) {
  int idx = 0;
#pragma unroll
  for (int q = 0; q < NB; ++q) idx += (bnd[q] < y) ? 1 : 0;
  return idx;
}

// Pi and S in shared memory up to d = 128 (2 d^2 floats), else in global memory.
template <int D>
__host__ __device__ constexpr bool stage_mats() { return D <= 128; }

// Scratch of a group of four warps that encodes one vector together: the
// centroids c_i of the key's codes, the four warps' partial sums of Pi^T c,
// and the 32-bit words of the code planes, signs and refinement mask.
template <int D>
struct QuadScratch {
  float c[D];
  float part[4][D];
  uint32_t planes[3][D / 32];
  uint32_t sw[D / 32], nw[D / 32];
};

constexpr int kQuads = kWarpsPerCta / 4;  // vectors in flight per CTA

template <int D>
__host__ __device__ constexpr size_t warp_kernel_smem() {
  return (stage_mats<D>() ? 2 * D * D * sizeof(float) : 0) + kQuads * sizeof(QuadScratch<D>);
}

// Named barrier of the 128 threads of quad q (id 1 + q; id 0 is the CTA's).
__device__ __forceinline__ void quad_sync(int q) {
  asm volatile("bar.sync %0, 128;" ::"r"(1 + q) : "memory");
}

// One vector, by the four converged warps of quad `quad` (qw = 0..3 within
// it); Pi and S at pim and sm (shared or global memory), Q its scratch.
// The 32-row blocks of every mat-vec are spread over the four warps.
template <int D>
__device__ __forceinline__ void encode_vector(const AppendArgs &a, long long id, const float *__restrict__ pim,
                                              const float *__restrict__ sm, QuadScratch<D> &Q, int quad, int qw) {
  constexpr int C = D / 32;  // coordinates per lane; also 32-coordinate words per row
  const int lane = threadIdx.x & 31;
  int b, t, h;
  bool valid;
  vec_coords(a, id, b, t, h, valid);
  if (!valid) return;  // uniform over the quad
  const TileLayout L = TileLayout::make(a.key_bits, a.value_bits, a.value_mode, D);
  const size_t base = (((size_t)b * a.T + t) * a.h_kv + h) * D;
  const int pos = a.lens[b] + t;
  uint8_t *tile = tile_ptr(a.data, L, a.h_kv, a.ntiles, b, h, pos / kTile);
  const int slot = pos % kTile;
  const int ncent = 1 << L.mb;
  float bnd[7], cent[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    cent[q] = q < ncent ? a.centroids[q] : 0.f;
    if (q < 7) bnd[q] = q < ncent - 1 ? a.boundaries[q] : INFINITY;
  }

  // ---- key: u = k / ||k|| (every warp of the quad) ---------------------------
  float u[C], ss = 0.f;
#pragma unroll
  for (int m = 0; m < C; ++m) {
    u[m] = load_elem(a.k, a.dtype, base + C * lane + m);
    ss = fmaf(u[m], u[m], ss);
  }
  const float nk = sqrtf(warp_sum(ss));
  const bool zero = !(nk > 0.f);
#pragma unroll
  for (int m = 0; m < C; ++m) u[m] = zero ? 0.f : __fdiv_rn(u[m], nk);

  // ---- y = Pi u, codes: block k leaves coordinate 32 k + l in lane l -------
  for (int k = qw; k < C; k += 4) {
    const float y = rows32_dot<D>(pim, 32 * k, u);
    const int idx = zero ? 0 : bucketize(bnd, y);
    float c = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) c = (q == idx) ? cent[q] : c;
    Q.c[32 * k + lane] = zero ? 0.f : c;
#pragma unroll
    for (int p = 0; p < 3; ++p) {
      const uint32_t word = p < L.mb ? __ballot_sync(0xffffffffu, (idx >> p) & 1) : 0u;
      if (lane == 0) Q.planes[p][k] = word;
    }
  }
  quad_sync(quad);

  // ---- r = u - Pi^T c (rows split over the warps), ||r|| ----------------------
  float r[C];
  {
    float acc[C];
#pragma unroll
    for (int m = 0; m < C; ++m) acc[m] = 0.f;
#pragma unroll 8
    for (int i = qw * (D / 4); i < (qw + 1) * (D / 4); ++i) {
      const float ci = Q.c[i];
      float w[C];
      load_row_chunk<D>(pim, i, w);
#pragma unroll
      for (int m = 0; m < C; ++m) acc[m] = fmaf(w[m], ci, acc[m]);
    }
#pragma unroll
    for (int m = 0; m < C; ++m) Q.part[qw][C * lane + m] = acc[m];
    quad_sync(quad);
    float rr = 0.f;
#pragma unroll
    for (int m = 0; m < C; ++m) {
      const int j = C * lane + m;
      r[m] = u[m] - (((Q.part[0][j] + Q.part[1][j]) + Q.part[2][j]) + Q.part[3][j]);
      rr = fmaf(r[m], r[m], rr);
    }
    rr = warp_sum(rr);
    if (qw == 0 && lane == 0)
      *reinterpret_cast<__half2 *>(tile + L.norms + slot * 4) =
          __halves2half2(__float2half_rn(nk), __float2half_rn(zero ? 0.f : sqrtf(rr)));
  }

  // ---- z = S r: signs, and the components to re-decide in float64 ----------
  for (int k = qw; k < C; k += 4) {
    const float z = rows32_dot<D>(sm, 32 * k, r);
    const uint32_t sw = __ballot_sync(0xffffffffu, !zero && z >= 0.f);
    const uint32_t nw = __ballot_sync(0xffffffffu, !zero && fabsf(z) < a.refine_z);
    if (lane == 0) {
      Q.sw[k] = sw;
      Q.nw[k] = nw;
    }
  }
  quad_sync(quad);
  if (qw == 0) {
    uint32_t planes[3][C], sw[C], nw[C];
    uint32_t anynear = 0u;
#pragma unroll
    for (int k = 0; k < C; ++k) {
#pragma unroll
      for (int p = 0; p < 3; ++p) planes[p][k] = Q.planes[p][k];
      sw[k] = Q.sw[k];
      nw[k] = Q.nw[k];
      anynear |= nw[k];
    }
    if (anynear) {
      uint32_t res[C];
      refine_row_f64<D>(a.s, a.s_pit, a.centroids, a.k, a.dtype, base, planes, nw, res);
      int nbits = 0;
#pragma unroll
      for (int k = 0; k < C; ++k) {
        sw[k] = (sw[k] & ~nw[k]) | res[k];
        nbits += __popc(nw[k]);
      }
      if (lane == 0 && a.refine_count) atomicAdd(a.refine_count, (unsigned long long)nbits);
    }
    if (lane < C) {  // lane k writes word k of every plane and of the signs
      uint32_t pw[3] = {0u, 0u, 0u}, sk = 0u;
#pragma unroll
      for (int k = 0; k < C; ++k)
        if (lane == k) {
          pw[0] = planes[0][k];
          pw[1] = planes[1][k];
          pw[2] = planes[2][k];
          sk = sw[k];
        }
#pragma unroll
      for (int p = 0; p < 3; ++p)
        if (p < L.mb)
          *reinterpret_cast<uint32_t *>(tile + L.kplanes + p * L.plane_bytes + slot * L.row_bytes + 4 * lane) =
              pw[p];
      *reinterpret_cast<uint32_t *>(tile + L.signs + slot * L.row_bytes + 4 * lane) = sk;
    }
  }

  // ---- values (the groups / 32-row blocks spread over the warps) -------------
  if (!L.mse) {
    quantize_value_groups<D>(a, L, tile, slot, base, (float)((1 << a.value_bits) - 1), qw, 4);
  } else {
    // TurboQuant-MSE: the cells of Pi w, w = v / ||v||, and ||v||
    const int nvc = 1 << L.vb;
    float vbnd[15];
#pragma unroll
    for (int q = 0; q < 15; ++q) vbnd[q] = q < nvc - 1 ? a.v_boundaries[q] : INFINITY;
    float w[C], sv = 0.f;
#pragma unroll
    for (int m = 0; m < C; ++m) {
      w[m] = load_elem(a.v, a.dtype, base + C * lane + m);
      sv = fmaf(w[m], w[m], sv);
    }
    const float nv = sqrtf(warp_sum(sv));
    const bool vzero = !(nv > 0.f);
#pragma unroll
    for (int m = 0; m < C; ++m) w[m] = vzero ? 0.f : __fdiv_rn(w[m], nv);
    for (int k = qw; k < C; k += 4) {
      const float y = rows32_dot<D>(pim, 32 * k, w);
      const int idx = vzero ? 0 : bucketize(vbnd, y);
      for (int p = 0; p < L.vb; ++p) {
        const uint32_t word = __ballot_sync(0xffffffffu, (idx >> p) & 1);
        if (lane == 0)
          *reinterpret_cast<uint32_t *>(tile + L.vplanes + p * L.plane_bytes + slot * L.row_bytes + 4 * k) = word;
      }
    }
    if (qw == 0 && lane == 0) *reinterpret_cast<__half *>(tile + L.vsz + slot * 2) = __float2half_rn(nv);
  }
  quad_sync(quad);  // the scratch is reused by the quad's next vector
}

template <int D>
__global__ void __launch_bounds__(32 * kWarpsPerCta, 1) quantize_append_warp_kernel(const __grid_constant__ AppendArgs a) {
  extern __shared__ __align__(16) float mats[];
  // a decode call's query kernel may start now: it reads none of this
  // kernel's output and waits for this grid before it finishes
  sm100::pdl_trigger();
  const float *pim = a.pi, *sm = a.s;
  constexpr int kMatFloats = stage_mats<D>() ? 2 * D * D : 0;
  if constexpr (stage_mats<D>()) {
    constexpr int kChunks = D * D / 4;  // 16-byte chunks per matrix
    for (int i = threadIdx.x; i < kChunks; i += 32 * kWarpsPerCta) {
      cp_async16(mats + 4 * i, a.pi + 4 * i);
      cp_async16(mats + D * D + 4 * i, a.s + 4 * i);
    }
    cp_async_wait_all();
    __syncthreads();
    pim = mats;
    sm = mats + D * D;
  }
  const int warp = threadIdx.x >> 5, quad = warp >> 2, qw = warp & 3;
  QuadScratch<D> &Q = reinterpret_cast<QuadScratch<D> *>(mats + kMatFloats)[quad];
  const long long total = (long long)a.batch * a.T * a.h_kv;
  for (long long id = (long long)blockIdx.x * kQuads + quad; id < total; id += (long long)gridDim.x * kQuads)
    encode_vector<D>(a, id, pim, sm, Q, quad, qw);
}

template <int D>
cudaError_t launch_warp_d(const AppendArgs &a, int num_sms, cudaStream_t stream) {
  const long long total = (long long)a.batch * a.T * a.h_kv;
  const long long blocks = std::min<long long>((total + kQuads - 1) / kQuads, num_sms);
  if (blocks == 0) return cudaSuccess;
  const int smem = (int)warp_kernel_smem<D>();
  cudaError_t e = cudaFuncSetAttribute(quantize_append_warp_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  quantize_append_warp_kernel<D><<<(unsigned)blocks, 32 * kWarpsPerCta, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_warp(const AppendArgs &a, int num_sms, cudaStream_t stream) {
  switch (a.d) {
    case 64: return launch_warp_d<64>(a, num_sms, stream);
    case 128: return launch_warp_d<128>(a, num_sms, stream);
    case 256: return launch_warp_d<256>(a, num_sms, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace tq
