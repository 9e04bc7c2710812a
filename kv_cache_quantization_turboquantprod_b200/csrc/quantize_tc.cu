// quantize_append on the 5th-generation tensor cores (tcgen05 kind::f16):
// the TurboQuant-prod key encoding of "TurboQuant" explainer (troisinh.com,
// "Ý tưởng cốt lõi") and "turboquant/audit_claims.py" (AUDIT 1 / AUDIT 5),
// with the d x d products of every key vector as tensor-core GEMMs over
// 128-vector tiles and everything else fused in their epilogues:
//   GEMM1  Y = K Pi^T            y = Y / ||k||, bucketize -> codes, c = c[idx],
//                                E = y - c, ||r|| = ||E||
//   GEMM2  Z = E W^T             signs = [z >= 0]
// with W = S Pi^T (float64, formed once per layer).  Pi is orthogonal, so
// the residual r = u - Pi^T c equals Pi^T (y - c): its norm is that of
// E = y - c and its sketch is S r = S Pi^T E = W E.  No r is formed and no
// key row is read twice.
// Values are group-quantized (per 32 channels, fp16 scale/zero) by a
// separate bandwidth-bound kernel launched just before this one
// (quantize_values.cu).
//
// Precision.  A bf16 key is exact in fp16 once scaled per vector by 2^s
// (largest |k| 2^s in [2^14, 2^15)); Pi, W and E are split into fp16 hi +
// lo parts (scaled so no part is subnormal where it matters), and each
// product takes the significant hi/lo terms with f32 accumulation: about 22
// bits per operand, the error of an fp32 mat-vec.  E is formed from the
// accumulator in one rounding (fma(Y, 2^13 / (2^(s+10) ||k||), -c 2^13)).
//
// Tiles are 128 consecutive new tokens of one (sequence, KV head), so every
// record section a tile writes is one contiguous run of the cache.
//
// Pipeline.  Tensor memory holds the accumulators D1 (columns 0-127) and D2
// (128-255) and GEMM2's A operand E (256-383: fp16 hi and lo parts, 16
// columns a K-step).  The epilogue hands E to the issuer a K-step at a time
// (one barrier per K-step), so GEMM2 runs under E1, and the next tile's
// GEMM1 runs while this tile's signs are read.
//
// Warp roles (768 threads, by warpgroup):
//   WG0  warp 0       MMA issuer (one elected lane), sleeping in blocking
//                     waits on the operand barriers; warp 1 idles
//        warps 2, 3   sign refiners: sketch components the epilogue found next
//                     to zero (|S r| < 1e-5, about one key in 300) get their
//                     sign again in float64, off the pipeline's critical path;
//                     each epilogue warp hands such rows over through its own
//                     ring in shared memory and a refiner patches the stored
//                     sign words
//   WG1  warps 4-7    loader: K rows -> scaled fp16 A operand + norms in
//                     shared memory (two buffers); the epilogue releases a
//                     buffer as soon as GEMM1 has read it
//   WG2-WG5           epilogue: thread = tile row = TMEM lane; warp w takes
//                     lane quarter w % 4 and one quarter of the columns
// setmaxnreg moves registers from WG0 and WG1 to the epilogue warpgroups.
// Every mbarrier wait between roles is bounded (2 s unless the host set another
// limit) and answers warp-uniformly; on timeout the CTA raises its abort flag
// and the device's sticky error word, stops, lets its own MMAs finish, frees
// TMEM and marks the records it owns with NaN norms.
#include <math.h>

#include <type_traits>

#include "sm100.cuh"
#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

namespace {

using namespace sm100;

constexpr int kQtThreads = 768;  // 6 warpgroups
constexpr int kQtRegs = 80;      // registers a thread at launch (65536 / 768, rounded down to 8)
// setmaxnreg shares: WG0 (issuers, refiners), WG1 (loader), WG2-5 (epilogue)
constexpr int kIssRegs = 56, kLoadRegs = 72, kEpiRegs = 88;
constexpr int kRingCap = 8;      // refinement requests per epilogue warp in flight
constexpr int kMat16 = 128 * 128 * 2;  // one fp16 128 x 128 operand (32 KB)
constexpr float kPiScale = 1024.f;     // Pi parts are stored x 2^10
constexpr double kWScale = 256.0;     // W = S Pi^T parts x 2^8
constexpr float kEScale = 8192.f;      // E = y - c parts x 2^13

// byte offset of element (row, col) of a 128 x 128 fp16 matrix in the
// canonical no-swizzle layout: 8 x 8 blocks, block (row / 8, col / 8) at
// (col / 8) * 2048 + (row / 8) * 128.  Read K-major (K = col) with
// LBO 2048 / SBO 128, or MN-major (K = row, N = col) with LBO 128 / SBO 2048.
__host__ __device__ constexpr int blk_off(int row, int col) {
  return (col >> 3) * 2048 + (row >> 3) * 128 + (row & 7) * 16 + (col & 7) * 2;
}

// A key row whose sketch has components next to zero: the mask of
// components to re-decide, its key's element offset, and the addresses of
// its stored code-plane rows (plane p at planes + p * plane bytes) and sign
// row.  The requesting thread stored those rows itself before the hand-off.
struct RefineReq {
  uint32_t near[4];
  unsigned long long kbase;
  unsigned long long planes;
  unsigned long long signs;
};

struct QtSmem {
  alignas(1024) uint8_t pi[2][kMat16];  // Pi x 2^10: hi, lo
  alignas(1024) uint8_t w[2][kMat16];   // W = S Pi^T x 2^8: hi, lo
  alignas(1024) uint8_t a1[2][kMat16];  // K rows x 2^s (fp16), double-buffered by tile
  float nk[2][128];
  int sh[2][128];
  float cent[8];
  float cent13[8];               // centroids x 2^13
  float bnd[8];                  // ascending, padded with +inf
  int sym;                       // boundaries exactly antisymmetric (b[i] == -b[nb - 1 - i])
  // a1_full / a1_free: a K operand buffer is loaded / read by GEMM1 and its
  // norms taken; d1_full / d2_full: a tile's GEMM1 / GEMM2 is complete;
  // d_free: the epilogue has read D2; kc[c]: K-step c of the tile's E
  // operand is in tensor memory; fin: the issuer's last commit (every MMA
  // it issued is done)
  uint64_t a1_full[2], a1_free[2], d1_full, d2_full, d_free, kc[8], fin;
  uint32_t tmem_base;
  volatile int abort_flag;
  // refinement rings, one per epilogue warp (single producer, the refiner
  // the single consumer): requests [head, tail) are pending
  RefineReq ring[16][kRingCap];
  volatile int ring_head[16], ring_tail[16];
  volatile int epi_done;  // epilogue warps past their last tile
  // [tile parity][column quarter][row]: ||r||^2 x 2^26 over a quarter of a
  // row (by parity, so a warp that runs a tile ahead cannot overwrite a value
  // that is yet to be read: that would take the reader's next hand-over)
  float rrq[2][4][128];
  uint64_t pair[4];         // [lane quarter]: the four column quarters of a row block meet
  volatile int progress;  // changes whenever an epilogue warp finishes a tile
};

struct TileInfo {
  int b, h, t0, nrow;
};

__device__ __forceinline__ TileInfo tile_info(const AppendArgs &a, int gt) {
  // batch b owns tiles [tstart[b], tstart[b + 1])
  int lo = 0, hi = a.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.tstart[mid] <= gt) lo = mid; else hi = mid - 1;
  }
  TileInfo ti;
  ti.b = lo;
  const int rem = gt - a.tstart[lo];
  const int ntb = (a.nnew[lo] + 127) >> 7;
  ti.h = rem / ntb;
  const int tb = rem - ti.h * ntb;
  ti.t0 = tb * 128;
  ti.nrow = min(128, a.nnew[lo] - ti.t0);
  return ti;
}

// Bounded pipeline wait (limit a.wait_ns, 2 s by default) with one answer for
// the whole converged warp; a timeout raises the CTA's abort flag and the
// device's sticky error word.
__device__ __forceinline__ bool qwait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                      const AppendArgs &a) {
  bool timed_out = false;
  const bool ok = pipe_wait(bar, parity, abort_flag, a.wait_ns, a.wait_hint_ns, &timed_out);
  if (timed_out && a.errors) atomicOr(a.errors, (unsigned int)TQ_ERRF_QUANTIZE_WAIT);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait until epilogue warp ew's refinement ring has room for the
// requests before index `upto` (upto - head <= kRingCap); one answer for the
// whole warp.
__device__ __forceinline__ bool ring_room(QtSmem &S, int ew, int upto, const AppendArgs &a) {
  bool ok = true;
  if (upto - S.ring_head[ew] > kRingCap) {
    const uint64_t t0 = globaltimer_ns();
    while (upto - S.ring_head[ew] > kRingCap) {
      if (S.abort_flag) {
        ok = false;
        break;
      }
      if (globaltimer_ns() - t0 > a.wait_ns) {
        S.abort_flag = 1;
        if (a.errors) atomicOr(a.errors, (unsigned int)TQ_ERRF_QUANTIZE_WAIT);
        ok = false;
        break;
      }
      __nanosleep(128);
    }
  }
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ uint32_t pack_h2(float lo_elem, float hi_elem) {
  const __half2 h = __floats2half2_rn(lo_elem, hi_elem);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// hi + lo fp16 parts of x (already scaled)
__device__ __forceinline__ void split16(float x, float &hi, float &lo) {
  hi = __half2float(__float2half_rn(x));
  lo = x - hi;
}

template <int MB>
__global__ void __launch_bounds__(kQtThreads, 1) quantize_tc_kernel(const __grid_constant__ AppendArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  QtSmem &S = *reinterpret_cast<QtSmem *>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const TileLayout L = TileLayout::make(a.key_bits, a.value_bits, a.value_mode);
  // a decode call's query kernel may start now: it reads none of this
  // kernel's output and waits for this grid before it finishes
  pdl_trigger();
  constexpr int ncent = 1 << MB;
  const int nlocal = a.total_tiles > (int)blockIdx.x
                         ? (a.total_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                         : 0;

  // ---- setup: split Pi and W = S Pi^T into fp16 parts, barriers, TMEM ---
  // eight elements (one 16-byte block row) per item, both matrices' loads
  // issued before any is used; W is split from its float64 values
  for (int it = tid; it < 128 * 16; it += kQtThreads) {
    const int i = it >> 4, j0 = (it & 15) * 8;
    const float4 *pp = reinterpret_cast<const float4 *>(a.pi + i * 128 + j0);
    const double2 *wp = reinterpret_cast<const double2 *>(a.s_pit + i * 128 + j0);
    const float4 p0 = pp[0], p1 = pp[1];
    const double2 w0 = wp[0], w1 = wp[1], w2 = wp[2], w3 = wp[3];
    const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    const double wv[8] = {w0.x, w0.y, w1.x, w1.y, w2.x, w2.y, w3.x, w3.y};
    uint32_t ph[4], pl[4], wh[4], wl[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float h0, l0, h1, l1;
      split16(pv[2 * e] * kPiScale, h0, l0);
      split16(pv[2 * e + 1] * kPiScale, h1, l1);
      ph[e] = pack_h2(h0, h1);
      pl[e] = pack_h2(l0, l1);
      const double x0 = wv[2 * e] * kWScale, x1 = wv[2 * e + 1] * kWScale;
      const __half hh0 = __double2half(x0), hh1 = __double2half(x1);
      const __half ll0 = __double2half(x0 - (double)__half2float(hh0));
      const __half ll1 = __double2half(x1 - (double)__half2float(hh1));
      const __half2 hw2 = __halves2half2(hh0, hh1), lw2 = __halves2half2(ll0, ll1);
      wh[e] = *reinterpret_cast<const uint32_t *>(&hw2);
      wl[e] = *reinterpret_cast<const uint32_t *>(&lw2);
    }
    *reinterpret_cast<uint4 *>(S.pi[0] + blk_off(i, j0)) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
    *reinterpret_cast<uint4 *>(S.pi[1] + blk_off(i, j0)) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
    *reinterpret_cast<uint4 *>(S.w[0] + blk_off(i, j0)) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    *reinterpret_cast<uint4 *>(S.w[1] + blk_off(i, j0)) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
  }
  if (tid < ncent) {
    S.cent[tid] = a.centroids[tid];
    S.cent13[tid] = a.centroids[tid] * kEScale;
  }
  if (tid < 8) S.bnd[tid] = tid < ncent - 1 ? a.boundaries[tid] : INFINITY;
  if (tid == 0) {
    int sym = 1;
    for (int i = 0; i < ncent - 1; ++i) sym &= (a.boundaries[i] == -a.boundaries[ncent - 2 - i]) ? 1 : 0;
    S.sym = sym;
  }
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.a1_full[b], 4);
      mbar_init(&S.a1_free[b], 16);
    }
    mbar_init(&S.d1_full, 1);
    mbar_init(&S.d2_full, 1);
    mbar_init(&S.d_free, 16);
    for (int c = 0; c < 8; ++c) mbar_init(&S.kc[c], 4);
    mbar_init(&S.fin, 1);
    S.abort_flag = 0;
    for (int w = 0; w < 16; ++w) S.ring_head[w] = S.ring_tail[w] = 0;
    for (int q = 0; q < 4; ++q) mbar_init(&S.pair[q], 4);
    S.epi_done = 0;
    S.progress = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&S.tmem_base, 512);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;

  // Registers move from the warpgroups that need few (issuers and refiners,
  // loader) to the four epilogue warpgroups: (56 + 72) x 128 + 88 x 512 =
  // 61440, exactly the 80 x 768 the CTA is launched with (the kernel's
  // register count is checked on the host before launch).
  const int wg = warp >> 2;
  if (wg == 0) {
    reg_dealloc<kIssRegs>();
    if (warp == 0) {
    // ---------------- MMA issuer -------------------------------------------
    // One warp issues every product, in order, sleeping in blocking waits on
    // the operand barriers (a polling issuer shares its sub-partition's
    // issue slots with the loader and epilogue warps).  GEMM2 goes out
    // K-step by K-step as the epilogue hands over the chunks of its A
    // operand, so it runs under the epilogue step that produces it.
    const bool leader = elect_one();
    const uint32_t id1 = idesc_f16(128, 128, false, false);
    const uint64_t dpk[2] = {smem_desc(S.pi[0], 2048, 128), smem_desc(S.pi[1], 2048, 128)};
    const uint64_t dwk[2] = {smem_desc(S.w[0], 2048, 128), smem_desc(S.w[1], 2048, 128)};
    const uint64_t da1[2] = {smem_desc(S.a1[0], 2048, 128), smem_desc(S.a1[1], 2048, 128)};
    const uint32_t d1col = tbase, d2col = tbase + 128;
    const uint32_t eop = tbase + 256;  // E operand: K-step c hi at 16 c, lo at 16 c + 8
    auto wait_all = [&](uint64_t *bar, uint32_t parity) { return qwait(bar, parity, &S.abort_flag, a); };
    for (int j = 0; j < nlocal; ++j) {
      const int buf = j & 1;
      const uint32_t ph = j & 1;
      // Y = K Pi^T: (K)(Pi_hi + Pi_lo), once K is in.  D1 of the previous
      // tile has been read: every warp loads its D1 columns before handing
      // over its first E chunk, and all were handed over.
      if (!wait_all(&S.a1_full[buf], (j >> 1) & 1)) break;
      tc_fence_after();
#pragma unroll
      for (int pr = 0; pr < 2; ++pr)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          if (leader)
            mma_f16_ss(d1col, da1[buf] + (uint64_t)((ks * 4096) >> 4), dpk[pr] + (uint64_t)((ks * 4096) >> 4), id1,
                       (pr | ks) ? 1u : 0u);
      if (leader) mma_commit(&S.d1_full);
      __syncwarp();
      // Z = E W^T: E_hi W_hi + E_hi W_lo + E_lo W_hi, once the previous
      // tile's D2 has been read; K-steps in the order the chunks are done
      // (every column quarter's first chunk, then every second one)
      if (j > 0 && !wait_all(&S.d_free, ph ^ 1u)) break;
      bool ok = true;
#pragma unroll 1
      for (int o = 0; o < 8; ++o) {
        const int ks = 2 * (o & 3) + (o >> 2);
        if (!wait_all(&S.kc[ks], ph)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int pr = 0; pr < 3; ++pr)
          if (leader)
            mma_f16_ts(d2col, eop + 16 * ks + (pr == 2 ? 8 : 0), dwk[pr == 1 ? 1 : 0] + (uint64_t)((ks * 4096) >> 4),
                       id1, (o | pr) ? 1u : 0u);
        __syncwarp();
      }
      if (!ok) break;
      if (leader) mma_commit(&S.d2_full);
      __syncwarp();
    }
    // never leave with an MMA in flight (also after a wait that gave up
    // between two K-steps): one more commit covers all of them
    if (leader) mma_commit(&S.fin);
    __syncwarp();
    mbar_wait(&S.fin, 0u);
    } else if (warp >= 2) {
    // ---------------- sign refiners ----------------------------------------
    // Warp 2 serves the rings of epilogue warps 0-7, warp 3 those of 8-15, in
    // turn, until every epilogue warp is done and its rings are empty.  Its
    // waits are on the epilogue warps, whose own waits are bounded; it is
    // bounded too (same limit, measured from the
    // last request or finished tile it saw) and gives up by raising the
    // abort flag.
    unsigned long long t_last = globaltimer_ns();
    int seen = S.progress;
    // idle polls back off from 256 ns to 2 us (a poll costs its
    // sub-partition ~40 issue slots; requests are rare)
    unsigned int nap = 256;
    while (true) {
      // shared words are read by lane 0 and broadcast, so the warp stays converged
      const int done = __shfl_sync(0xffffffffu, S.epi_done, 0);  // before the rings: no request after it is missed
      bool any = false;
#pragma unroll 1
      for (int ew = 8 * (warp - 2); ew < 8 * (warp - 2) + 8; ++ew) {
        int h = __shfl_sync(0xffffffffu, S.ring_head[ew], 0);
        const int t = __shfl_sync(0xffffffffu, S.ring_tail[ew], 0);
        if (h == t) continue;
        __threadfence_block();
        for (; h != t; ++h) {
          const RefineReq &q = S.ring[ew][h % kRingCap];
          uint32_t pl[3][4], nw[4], res[4];
          const uint8_t *prow = reinterpret_cast<const uint8_t *>(q.planes);
#pragma unroll
          for (int p = 0; p < 3; ++p) {
            const uint4 v = p < MB ? *reinterpret_cast<const uint4 *>(prow + p * kPlaneBytes) : make_uint4(0u, 0u, 0u, 0u);
            pl[p][0] = v.x;
            pl[p][1] = v.y;
            pl[p][2] = v.z;
            pl[p][3] = v.w;
          }
#pragma unroll
          for (int w = 0; w < 4; ++w) nw[w] = q.near[w];
          const unsigned long long kb = q.kbase;
          uint32_t *words = reinterpret_cast<uint32_t *>(q.signs);
          refine_row_f64<kD>(a.s, a.s_pit, S.cent, a.k, a.dtype, kb, pl, nw, res);
          uint32_t mn = 0u, mr = 0u;  // lane w < 4 patches word w
#pragma unroll
          for (int w = 0; w < 4; ++w)
            if (lane == w) {
              mn = nw[w];
              mr = res[w];
            }
          if (mn != 0u) {
            atomicAnd(words + lane, ~mn);
            atomicOr(words + lane, mr);
          }
          if (lane == 0 && a.refine_count)
            atomicAdd(a.refine_count,
                      (unsigned long long)(__popc(nw[0]) + __popc(nw[1]) + __popc(nw[2]) + __popc(nw[3])));
          __syncwarp();
          if (lane == 0) {
            __threadfence_block();
            S.ring_head[ew] = h + 1;  // the slot may be reused
          }
          __syncwarp();
        }
        any = true;
      }
      if (any) {
        t_last = globaltimer_ns();
        nap = 256;
        continue;
      }
      if (done == 16) break;
      if (__shfl_sync(0xffffffffu, S.abort_flag, 0)) break;
      const int prog = __shfl_sync(0xffffffffu, S.progress, 0);
      if (prog != seen) {
        seen = prog;
        t_last = globaltimer_ns();
      } else if (globaltimer_ns() - t_last > a.wait_ns) {
        if (lane == 0) {
          S.abort_flag = 1;
          if (a.errors) atomicOr(a.errors, (unsigned int)TQ_ERRF_QUANTIZE_WAIT);
        }
        __syncwarp();
        break;
      }
      __nanosleep(nap);
      nap = nap < 2048 ? 2 * nap : 2048;
    }
    }
  } else if (wg == 1) {
    reg_dealloc<kLoadRegs>();
    // ---------------- loader -----------------------------------------------
    // A warp takes 8 rows at a time (one 8-row group of the operand): lane
    // (row rr = lane / 4, channel quarter q = lane % 4) holds channels
    // 32q .. 32q + 31.  Values are quantized by their own kernel, so the
    // loader reads keys only; the rows of the next two steps are in flight
    // while this step's are converted.
    const int w = warp - 4, rr = lane >> 2, q = lane & 3;
    // rows of step u = 4 i + pass
    auto fetch = [&](int u, uint4 (&kr)[4]) {
      const int i = u >> 2, pass = u & 3;
      bool valid = i < nlocal;
      size_t base = 0;
      if (valid) {
        const TileInfo ti = tile_info(a, blockIdx.x + i * gridDim.x);
        const int r = 32 * pass + 8 * w + rr;
        valid = r < ti.nrow;
        base = ((((size_t)ti.b * a.T + ti.t0 + r) * a.h_kv + ti.h) * kD + 32 * q);
      }
      const uint4 *ks = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(a.k) + base);
#pragma unroll
      for (int c = 0; c < 4; ++c) kr[c] = valid ? ks[c] : make_uint4(0u, 0u, 0u, 0u);
    };
    uint4 kr[4], k1[4];
    fetch(0, kr);
    fetch(1, k1);
    for (int i = 0; i < nlocal; ++i) {
      const int g = i & 1;
      const TileInfo ti = tile_info(a, blockIdx.x + i * gridDim.x);
      uint8_t *a1 = S.a1[g];
      bool stop = false;
#pragma unroll 1
      for (int pass = 0; pass < 4; ++pass) {
        uint4 k2[4];
        fetch(4 * i + pass + 2, k2);
        if (pass == 0 && i >= 2 && !qwait(&S.a1_free[g], ((i - 2) >> 1) & 1, &S.abort_flag, a)) {
          stop = true;
          break;
        }
        const int r = 32 * pass + 8 * w + rr;
        // ---- key: norm, per-vector scale, fp16 operand ----
        float ss = 0.f, mx = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&kr[c]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(p2[e]);
            ss = fmaf(f.x, f.x, ss);
            ss = fmaf(f.y, f.y, ss);
            mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
          }
        }
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float nk = sqrtf(ss);
        const int sh = mx > 0.f ? min(14 - ilogbf(mx), 127) : 0;
        const float f2 = __uint_as_float((uint32_t)(sh + 127) << 23);  // 2^sh
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&kr[c]);
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(p2[e]);
            o[e] = pack_h2(f.x * f2, f.y * f2);
          }
          *reinterpret_cast<uint4 *>(a1 + blk_off(r, 32 * q + 8 * c)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        if (q == 0) {
          S.nk[g][r] = nk;
          S.sh[g][r] = sh;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          kr[c] = k1[c];
          k1[c] = k2[c];
        }
      }
      if (stop) break;
      fence_proxy_async_smem();
      __syncwarp();
      // (a test of the timeout path withholds the hand-off: the MMA issuer's
      // bounded wait on it then runs out)
      if (lane == 0 && !a.test_withhold) mbar_arrive(&S.a1_full[g]);
    }
  } else {
    reg_alloc<kEpiRegs>();
    // ---------------- epilogue ---------------------------------------------
    // Warp w of WG2-WG5 takes TMEM lane quarter w % 4 (tile rows 32 (w % 4)
    // .. + 31, a row per thread) and column quarter cq (coordinates 32 cq ..
    // 32 cq + 31, the K-steps 2 cq and 2 cq + 1 of GEMM2).  The four warps
    // of a lane quarter meet once per tile for ||r||^2.
    const int ew = warp - 8;  // epilogue warp 0 .. 15 (its refinement ring)
    const int cq = ew >> 2;
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;  // tile row == TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const uint32_t d1col = tbase + lane_off + 32 * cq, d2col = d1col + 128;
    const uint32_t ecol = tbase + lane_off + 256;  // E operand
    constexpr int NC = 1 << MB;
    // upper half of a symmetric codebook's boundaries, for the compare-count
    // bucketize: idx = NC/2 + #{ub < |y|} (y > 0) or NC/2 - 1 - #{ub < |y|}
    // (y <= 0), equal to #{b < y} except at exact ties (inside the band)
    constexpr int NU = NC / 2 - 1 > 0 ? NC / 2 - 1 : 1;
    float ub[NU];
#pragma unroll
    for (int k = 0; k < NU; ++k) ub[k] = (k < NC / 2 - 1) ? S.bnd[NC / 2 + k] : INFINITY;
    const bool sym = S.sym != 0;
    const float kNearZ = a.refine_z * 2097152.f;  // D2 = (S r) x 2^21 (E x 2^13 times W x 2^8)
    for (int j = 0; j < nlocal; ++j) {
      const int buf = j & 1;
      const uint32_t ph = j & 1;
      const TileInfo ti = tile_info(a, blockIdx.x + j * gridDim.x);
      const bool valid = r < ti.nrow;
      const int pos = a.lens[ti.b] + ti.t0 + r;
      uint8_t *tp = valid ? tile_ptr(a.data, L, a.h_kv, a.ntiles, ti.b, ti.h, pos / kTile) : nullptr;
      const int slot = pos % kTile;
      const size_t kbase = (((size_t)ti.b * a.T + ti.t0 + r) * a.h_kv + ti.h) * kD;  // this row's key
      if (!qwait(&S.d1_full, ph, &S.abort_flag, a)) break;
      tc_fence_after();
      const float nk = S.nk[buf][r];
      const int sh = S.sh[buf][r];
      // GEMM1 has read the K operand and the norms are in registers: the
      // loader may refill the buffer now
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.a1_free[buf]);
      const bool zero = !(nk > 0.f);
      const float rnk = zero ? 0.f : 1.f / nk;
      const float inv1 = ldexpf(rnk, -(sh + 10));  // y = Y 2^-(s+10) / ||k||
      const float inv13 = inv1 * kEScale;
      // a zero key gets y = -inf everywhere, which every bucketize below
      // maps to code 0; its E row is finite garbage (D1 = 0, scale 0) whose
      // products stay in its own row, and its signs and ||r|| are zeroed
      const float ybias = zero ? -INFINITY : 0.f;
      // ---- E1: y = Pi u, codes, E = (y - c) x 2^13 handed to GEMM2 a K-step
      // (16 coordinates) at a time, ||r||^2 = ||E||^2 ----
      uint32_t pw[3] = {0u, 0u, 0u};
      float rr = 0.f;  // ||r||^2 x 2^26 over this quarter
      uint32_t dA[16], dB[16];
      // The codebook's shape is decided once per tile, outside the element
      // loop: a branch per element would keep the compiler from interleaving
      // the elements' dependent chains.
      auto e1 = [&](auto sym_c) {
        constexpr bool SYM = decltype(sym_c)::value;
        tmem_ld16(d1col, dA);
        tmem_ld16(d1col + 16, dB);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const uint32_t(&d)[16] = cc ? dB : dA;
          uint32_t hl[16];  // hi parts (columns 0-7), lo parts (8-15)
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float ev[2];
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              const float dv = __uint_as_float(d[e + x]);
              const float y = fmaf(dv, inv1, ybias);
              int idx;  // #{boundaries < y}
              if constexpr (SYM) {
                const float ay = fabsf(y);
                int cnt = 0;
#pragma unroll
                for (int k = 0; k < NU; ++k) cnt += (ub[k] < ay) ? 1 : 0;
                idx = y > 0.f ? NC / 2 + cnt : NC / 2 - 1 - cnt;
              } else {  // any codebook: count the boundaries below y
                idx = 0;
#pragma unroll
                for (int k = 0; k < NC - 1; ++k) idx += (S.bnd[k] < y) ? 1 : 0;  // independent broadcast reads
              }
#pragma unroll
              for (int p = 0; p < MB; ++p) pw[p] |= (uint32_t)((idx >> p) & 1) << (16 * cc + e + x);
              // E = (y - c) 2^13 from D1 in one rounding
              ev[x] = fmaf(dv, inv13, -S.cent13[idx]);
              rr = fmaf(ev[x], ev[x], rr);
            }
            const __half2 hh = __floats2half2_rn(ev[0], ev[1]);
            const float2 hf = __half22float2(hh);
            const __half2 ll = __floats2half2_rn(ev[0] - hf.x, ev[1] - hf.y);
            hl[e >> 1] = *reinterpret_cast<const uint32_t *>(&hh);
            hl[8 + (e >> 1)] = *reinterpret_cast<const uint32_t *>(&ll);
          }
          tmem_st16(ecol + 16 * (2 * cq + cc), hl);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.kc[2 * cq + cc]);
        }
      };
      if (sym) e1(std::true_type{});
      else e1(std::false_type{});
      if (valid)  // this warp's word of every code plane row
#pragma unroll
        for (int p = 0; p < MB; ++p)
          *reinterpret_cast<uint32_t *>(tp + L.kplanes + p * kPlaneBytes + slot * kRowBytes + 4 * cq) = pw[p];
      S.rrq[ph][cq][r] = rr;
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.pair[q4]);  // this quarter's ||r||^2 is written
      // ---- E2: signs of z = S r = W (y - c), norms ----
      if (!qwait(&S.d2_full, ph, &S.abort_flag, a)) break;
      tc_fence_after();
      tmem_ld16(d2col, dA);
      tmem_ld16(d2col + 16, dB);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.d_free);  // D2 is in registers
      uint32_t sw = 0u;
      uint32_t nearw = 0u;  // |S r| below the refinement threshold
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const uint32_t(&d)[16] = cc ? dB : dA;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float z = __uint_as_float(d[e]);
          sw |= (z >= 0.f ? 1u : 0u) << (16 * cc + e);
          nearw |= (fabsf(z) < kNearZ ? 1u : 0u) << (16 * cc + e);
        }
      }
      if (zero) sw = 0u;
      if (zero || !valid) nearw = 0u;
      if (valid) *reinterpret_cast<uint32_t *>(tp + L.signs + slot * kRowBytes + 4 * cq) = sw;
      if (cq == 0) {
        // the other quarters' ||r||^2
        if (!qwait(&S.pair[q4], ph, &S.abort_flag, a)) break;
        if (valid) {
          const float rr2 = (rr + S.rrq[ph][1][r]) + (S.rrq[ph][2][r] + S.rrq[ph][3][r]);
          const float rn = zero ? 0.f : sqrtf(rr2) * (1.f / kEScale);
          *reinterpret_cast<__half2 *>(tp + L.norms + slot * 4) = __halves2half2(__float2half_rn(nk), __float2half_rn(rn));
        }
      }
      // sketch components next to zero: handed to the float64 refiner, which
      // patches the sign words stored above (at most kRingCap rows at a time)
      unsigned rest = __ballot_sync(0xffffffffu, nearw != 0u);
      bool stop = false;
      while (rest) {
        const int tail = S.ring_tail[ew];
        const int rank = __popc(rest & ((1u << lane) - 1u));
        const unsigned chunk = __ballot_sync(0xffffffffu, ((rest >> lane) & 1u) && rank < kRingCap);
        const int n = __popc(chunk);
        if (!ring_room(S, ew, tail + n, a)) {
          stop = true;
          break;
        }
        if ((chunk >> lane) & 1u) {
          RefineReq &q = S.ring[ew][(tail + rank) % kRingCap];
#pragma unroll
          for (int w = 0; w < 4; ++w) q.near[w] = w == cq ? nearw : 0u;
          q.kbase = kbase;
          q.planes = (unsigned long long)(tp + L.kplanes + slot * kRowBytes);
          q.signs = (unsigned long long)(tp + L.signs + slot * kRowBytes);
        }
        // the sign rows and the requests, then the new tail
        __threadfence_block();
        __syncwarp();
        if (lane == 0) S.ring_tail[ew] = tail + n;
        __syncwarp();
        rest &= ~chunk;
      }
      if (stop) break;
      if (lane == 0) S.progress = S.progress + 1;
    }
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      atomicAdd(const_cast<int *>(&S.epi_done), 1);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
    tmem_relinquish();
  }
  // A CTA that gave up on a wait leaves its tiles' records incomplete: mark
  // every record it owns with NaN norms, so that decode over them returns
  // NaN instead of a plausible result.
  if (S.abort_flag) {
    const uint32_t nan2 = 0x7E007E00u;  // two fp16 quiet NaNs (||k||, ||r||)
    for (int i = 0; i < nlocal; ++i) {
      const TileInfo ti = tile_info(a, blockIdx.x + i * gridDim.x);
      for (int r = tid; r < ti.nrow; r += kQtThreads) {
        const int pos = a.lens[ti.b] + ti.t0 + r;
        uint8_t *tp = tile_ptr(a.data, L, a.h_kv, a.ntiles, ti.b, ti.h, pos / kTile);
        *reinterpret_cast<uint32_t *>(tp + L.norms + (pos % kTile) * 4) = nan2;
      }
    }
  }
}

template <int MB>
cudaError_t launch_qt(const AppendArgs &a, int grid, cudaStream_t stream) {
  const size_t smem = sizeof(QtSmem);
  static_assert(sizeof(QtSmem) <= 227 * 1024, "shared memory per CTA");
  static_assert((kIssRegs + kLoadRegs) * 128 + kEpiRegs * 512 <= kQtRegs * kQtThreads &&
                    kQtRegs * kQtThreads <= 65536 && kIssRegs % 8 == 0 && kLoadRegs % 8 == 0 && kEpiRegs % 8 == 0,
                "warpgroup register targets must add up to at most the launch pool");
  cudaError_t e = cudaFuncSetAttribute(quantize_tc_kernel<MB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // The register targets assume the build gave the kernel exactly kQtRegs
  // registers a thread; refuse to launch otherwise (an increase beyond the
  // pool would wait forever).
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, quantize_tc_kernel<MB>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kQtRegs) return cudaErrorInvalidConfiguration;
  quantize_tc_kernel<MB><<<grid, kQtThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

bool quantize_tc_supported(const AppendArgs &a) {
  return a.d == kD && a.value_mode == TQ_VALUES_GROUP && a.dtype == TQ_BF16 && a.key_bits >= 2 && a.key_bits <= 4 && a.value_bits >= 2 &&
         a.value_bits <= 4 && a.T >= 64;
}

cudaError_t launch_quantize_tc(AppendArgs &a, int num_sms, cudaStream_t stream) {
  int total = 0;
  for (int b = 0; b < a.batch; ++b) {
    a.tstart[b] = total;
    total += a.h_kv * ((a.nnew[b] + 127) / 128);
  }
  a.tstart[a.batch] = total;
  a.total_tiles = total;
  if (total == 0) return cudaSuccess;
  const int grid = total < num_sms ? total : num_sms;
  const cudaError_t ev = launch_value_quant(a, num_sms, stream);
  if (ev != cudaSuccess) return ev;
  switch (a.key_bits - 1) {
    case 1: return launch_qt<1>(a, grid, stream);
    case 2: return launch_qt<2>(a, grid, stream);
    case 3: return launch_qt<3>(a, grid, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace tq
