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
// Precision.  GEMM1 multiplies the bf16 key rows by Pi split into three bf16
// parts whose sum is Pi exactly, so every product is exact and only the f32
// accumulation rounds.  W and E are split into fp16 hi + lo parts (scaled
// so no part is subnormal where it matters) and GEMM2 takes the three
// significant hi/lo terms with f32 accumulation: about 22 bits per operand,
// the error of an fp32 mat-vec.  E is formed from the accumulator in one
// rounding (fma(Y, 2^13 / ||k||, -c 2^13)).
//
// Tiles are 128 consecutive new tokens of one (sequence, KV head), so every
// record section a tile writes is one contiguous run of the cache.
//
// Pipeline.  Tensor memory holds the accumulator D1 (columns 0-127), two D2
// buffers (128-255, 256-383) and GEMM2's A operand E (384-511: fp16 hi and
// lo parts, 16 columns a K-step).  The epilogue hands E to the issuer a
// K-step at a time (one barrier per K-step), so GEMM2 runs under E1; the
// next tile's GEMM1 goes out as soon as every warp holds its D1 columns;
// and tile j's signs are read after E1 of tile j + 1, so the end of GEMM2
// runs while the epilogue works on the next tile.
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
//   WG1  warps 4-7    loader: the next tile's bf16 K rows -> the A operand
//                     buffer (TMA tensor copies) as soon as GEMM1 has read
//                     it, their norms and inverse norms, and where the
//                     tile's records go
//   WG2-WG5           epilogue: thread = tile row = TMEM lane; warp w takes
//                     lane quarter w % 4 and one quarter of the columns
// setmaxnreg moves registers from WG0 and WG1 to the epilogue warpgroups.
// Every mbarrier wait between roles is bounded (2 s unless the host set another
// limit) and answers warp-uniformly; on timeout the CTA raises its abort flag
// and the device's sticky error word, stops, lets its own MMAs finish, frees
// TMEM and marks the records it owns with NaN norms.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>
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
constexpr int kIssRegs = 72, kLoadRegs = 56, kEpiRegs = 88;
constexpr int kRingCap = 8;      // refinement requests per epilogue warp in flight
constexpr int kMat16 = 128 * 128 * 2;  // one 16-bit 128 x 128 operand (32 KB)
constexpr int kOperandBytes = 5 * kMat16;  // Pi's three bf16 parts, W's fp16 hi and lo
static_assert(kOperandBytes == TQ_TC_OPERAND_BYTES, "operand image size");
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

// Where a tile's rows go: rows below nrow are new tokens; row r is cache
// slot pos0 + r of the (sequence, head) whose records start at byte offset
// rec of the cache, its key at element kbase0 + r H_kv d of K.
struct TileRec {
  int nrow, pos0;
  long long rec, kbase0;
};

struct QtSmem {
  alignas(1024) uint8_t pi[3][kMat16];  // Pi as three bf16 parts (their sum is Pi exactly)
  alignas(1024) uint8_t w[2][kMat16];   // W = S Pi^T x 2^8: fp16 hi, lo
  alignas(1024) uint8_t a1[kMat16];     // the tile's bf16 K rows
  float nk[2][128];                     // ||k|| by tile parity
  float ninv[2][128];                   // 1 / ||k|| (0 for a zero key)
  TileRec trec[2];                      // by tile parity, written with the norms
  float cent[8];
  float ncent13[8];              // -(centroids x 2^13)
  float bnd[8];                  // ascending, padded with +inf
  int sym;                       // boundaries exactly antisymmetric (b[i] == -b[nb - 1 - i])
  // k_full: the tile's K rows have landed (TMA); a1_full / a1_free: the K
  // operand and its norms are in / it has been read by GEMM1; d1_full / d2_full[b]: a tile's GEMM1 / GEMM2 (into D2
  // buffer b) is complete; d1_read: every epilogue warp holds its D1
  // columns; d_free[b]: the epilogue has read D2 buffer b; kc[c]: K-step c
  // of the tile's E operand is in tensor memory; fin: the issuer's last
  // commit (every MMA it issued is done)
  uint64_t k_full, a1_full, a1_free, d1_full, d2_full[2], d1_read, d_free[2], kc[8], fin;
  uint64_t ops_full;  // the prepared operand images have landed
  uint32_t tmem_base;
  volatile int abort_flag;
  // refinement rings, one per epilogue warp (single producer, the refiner
  // the single consumer): requests [head, tail) are pending
  RefineReq ring[16][kRingCap];
  volatile int ring_head[16], ring_tail[16];
  volatile int epi_done;  // epilogue warps past their last tile
  // [tile mod 4][column quarter][row]: ||r||^2 x 2^26 over a quarter of a
  // row (the reader takes tile t's values while the others write t + 1's)
  float rrq[4][4][128];
  uint64_t pair[2][4];      // [tile parity][lane quarter]: the four column quarters of a row block meet
  volatile int progress;  // changes whenever an epilogue warp finishes a tile
};

static_assert(offsetof(QtSmem, w) == offsetof(QtSmem, pi) + 3 * kMat16, "operand images back to back");

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


// The shared-memory operand images of Pi (three bf16 parts, their sum Pi
// exactly) and W = S Pi^T (fp16 hi + lo of W x 2^8, split from its float64
// values), 32 KB each, back to back at dst in the canonical no-swizzle
// layout.  Item it (0 .. 2047) writes eight elements (one 16-byte block row)
// of each, both matrices' loads issued before any is used.
__device__ __forceinline__ void operand_item(const float *pi, const double *s_pit, int it, uint8_t *dst) {
  const int i = it >> 4, j0 = (it & 15) * 8;
  const float4 *pp = reinterpret_cast<const float4 *>(pi + i * 128 + j0);
  const double2 *wp = reinterpret_cast<const double2 *>(s_pit + i * 128 + j0);
  const float4 p0 = pp[0], p1 = pp[1];
  const double2 w0 = wp[0], w1 = wp[1], w2 = wp[2], w3 = wp[3];
  const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
  const double wv[8] = {w0.x, w0.y, w1.x, w1.y, w2.x, w2.y, w3.x, w3.y};
  uint32_t pp3[3][4], wh[4], wl[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    // x = p1 + p2 + p3 exactly: each remainder is exact in fp32 and the
    // last has at most 8 significant bits
    float r0 = pv[2 * e], r1 = pv[2 * e + 1];
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(r0, r1);
      pp3[q][e] = *reinterpret_cast<const uint32_t *>(&b2);
      r0 -= __low2float(b2);
      r1 -= __high2float(b2);
    }
    const double x0 = wv[2 * e] * kWScale, x1 = wv[2 * e + 1] * kWScale;
    const __half hh0 = __double2half(x0), hh1 = __double2half(x1);
    const __half ll0 = __double2half(x0 - (double)__half2float(hh0));
    const __half ll1 = __double2half(x1 - (double)__half2float(hh1));
    const __half2 hw2 = __halves2half2(hh0, hh1), lw2 = __halves2half2(ll0, ll1);
    wh[e] = *reinterpret_cast<const uint32_t *>(&hw2);
    wl[e] = *reinterpret_cast<const uint32_t *>(&lw2);
  }
#pragma unroll
  for (int q = 0; q < 3; ++q)
    *reinterpret_cast<uint4 *>(dst + q * kMat16 + blk_off(i, j0)) = make_uint4(pp3[q][0], pp3[q][1], pp3[q][2], pp3[q][3]);
  *reinterpret_cast<uint4 *>(dst + 3 * kMat16 + blk_off(i, j0)) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
  *reinterpret_cast<uint4 *>(dst + 4 * kMat16 + blk_off(i, j0)) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
}

// The operand images written once per layer into global memory.
__global__ void __launch_bounds__(256) prepare_operands_kernel(const float *pi, const double *s_pit, uint8_t *dst) {
  const int it = blockIdx.x * 256 + threadIdx.x;
  if (it < 128 * 16) operand_item(pi, s_pit, it, dst);
}

template <int MB>
__global__ void __launch_bounds__(kQtThreads, 1) quantize_tc_kernel(const __grid_constant__ AppendArgs a,
                                                                   const __grid_constant__ CUtensorMap kmap) {
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

  // ---- setup: the operand images of Pi and W, barriers, TMEM ------------
  if (a.tc_ops) {
    // prepared once per layer (tq_prepare_operands): one bulk copy
    if (tid == 0) {
      mbar_init(&S.ops_full, 1);
      fence_mbar_init();
      mbar_arrive_expect_tx(&S.ops_full, kOperandBytes);
#pragma unroll 1
      for (int c = 0; c < kOperandBytes / kMat16; ++c)
        bulk_g2s(S.pi[0] + c * kMat16, reinterpret_cast<const uint8_t *>(a.tc_ops) + c * kMat16, kMat16,
                 &S.ops_full);
    }
  } else {
    for (int it = tid; it < 128 * 16; it += kQtThreads) operand_item(a.pi, a.s_pit, it, S.pi[0]);
  }
  if (tid < ncent) {
    S.cent[tid] = a.centroids[tid];
    S.ncent13[tid] = -(a.centroids[tid] * kEScale);
  }
  if (tid < 8) S.bnd[tid] = tid < ncent - 1 ? a.boundaries[tid] : INFINITY;
  if (tid == 0) {
    int sym = 1;
    for (int i = 0; i < ncent - 1; ++i) sym &= (a.boundaries[i] == -a.boundaries[ncent - 2 - i]) ? 1 : 0;
    S.sym = sym;
  }
  if (tid == 0) {
    mbar_init(&S.k_full, 1);
    mbar_init(&S.a1_full, 4);
    mbar_init(&S.a1_free, 1);
    mbar_init(&S.d1_full, 1);
    mbar_init(&S.d1_read, 16);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.d2_full[b], 1);
      mbar_init(&S.d_free[b], 16);
    }
    for (int c = 0; c < 8; ++c) mbar_init(&S.kc[c], 4);
    mbar_init(&S.fin, 1);
    S.abort_flag = 0;
    for (int w = 0; w < 16; ++w) S.ring_head[w] = S.ring_tail[w] = 0;
    for (int q = 0; q < 4; ++q) {
      mbar_init(&S.pair[0][q], 4);
      mbar_init(&S.pair[1][q], 4);
    }
    S.epi_done = 0;
    S.progress = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&S.tmem_base, 512);
  // the MMA issuer (warp 0) sees the prepared images land itself; the copy
  // engine completes them, so the wait ends
  if (a.tc_ops && warp == 0) mbar_wait(&S.ops_full, 0);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;

  // Registers move from the warpgroups that need few (issuers and refiners,
  // loader) to the four epilogue warpgroups: (72 + 56) x 128 + 88 x 512 =
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
    const uint32_t idb = idesc_f16(128, 128, false, false) | (1u << 7) | (1u << 10);  // bf16 A and B
    const uint64_t dpk[3] = {smem_desc(S.pi[0], 2048, 128), smem_desc(S.pi[1], 2048, 128),
                             smem_desc(S.pi[2], 2048, 128)};
    const uint64_t dwk[2] = {smem_desc(S.w[0], 2048, 128), smem_desc(S.w[1], 2048, 128)};
    const uint64_t da1 = smem_desc(S.a1, 2048, 128);
    const uint32_t d1col = tbase;      // D1; D2 buffers at 128, 256
    const uint32_t eop = tbase + 384;  // E operand: K-step c hi at 16 c, lo at 16 c + 8
    auto wait_all = [&](uint64_t *bar, uint32_t parity) { return qwait(bar, parity, &S.abort_flag, a); };
    // non-blocking: has every lane seen the phase complete?
    auto ready = [&](uint64_t *bar, uint32_t parity) { return __all_sync(0xffffffffu, mbar_test(bar, parity)); };
    // Y = K Pi^T of tile t into D1: K (Pi_1 + Pi_2 + Pi_3), bf16 products
    // exact in the f32 accumulator; its commit also frees the K buffer
    auto gemm1 = [&](int t) {
      tc_fence_after();
#pragma unroll
      for (int pr = 0; pr < 3; ++pr)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          if (leader)
            mma_f16_ss(d1col, da1 + (uint64_t)((ks * 4096) >> 4), dpk[pr] + (uint64_t)((ks * 4096) >> 4), idb,
                       (pr | ks) ? 1u : 0u);
      if (leader) {
        mma_commit(&S.d1_full);
        mma_commit(&S.a1_free);
      }
      __syncwarp();
    };
    if (nlocal > 0 && wait_all(&S.a1_full, 0u)) gemm1(0);
    for (int j = 0; j < nlocal; ++j) {
      const int buf = j & 1;
      const uint32_t ph = j & 1;
      // GEMM1 of tile j + 1 goes out as soon as every warp holds its D1
      // columns of tile j and that tile's K is in: before GEMM2 of tile j
      // where it can, between its K-steps or after it otherwise
      if (!wait_all(&S.d1_read, ph)) break;
      bool g1 = j + 1 < nlocal;
      const uint32_t nph = (j + 1) & 1;
      if (g1 && ready(&S.a1_full, nph)) {
        gemm1(j + 1);
        g1 = false;
      }
      // Z = E W^T: E_hi W_hi + E_hi W_lo + E_lo W_hi into D2 buffer j % 2,
      // once tile j - 2's D2 has been read; K-steps in the order the chunks
      // are done (every column quarter's first chunk, then every second one)
      const uint32_t d2col = tbase + 128 + 128 * buf;
      if (j >= 2 && !wait_all(&S.d_free[buf], ((j - 2) >> 1) & 1)) break;
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
        if (g1 && ready(&S.a1_full, nph)) {
          gemm1(j + 1);
          g1 = false;
        }
      }
      if (!ok) break;
      if (leader) mma_commit(&S.d2_full[buf]);
      __syncwarp();
      if (g1) {
        if (!wait_all(&S.a1_full, nph)) break;
        gemm1(j + 1);
      }
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
    // Once GEMM1 has read the K buffer, one lane has the TMA engine copy the
    // next tile's bf16 rows into it: 16 boxes of 8 channels x 128 tokens of
    // the (channel, head, token, sequence) tensor map, each landing as one
    // 16-byte column of the canonical operand layout; tokens past the
    // sequence's end read as zeros.  Then warp w takes the norms of tile
    // rows 32 w .. 32 w + 31 (a row per lane).
    const int w = warp - 4;
    int in_flight = -1;  // a tile whose copies were issued and not yet seen landing
    for (int i = 0; i < nlocal; ++i) {
      const TileInfo ti = tile_info(a, blockIdx.x + i * gridDim.x);
      if (i >= 1 && !qwait(&S.a1_free, (i - 1) & 1, &S.abort_flag, a)) break;
      // (GEMM1 of tile i - 1 is done, so every epilogue warp has read the
      // record of tile i - 2 that this one replaces)
      if (w == 1 && lane == 0) {
        TileRec &tr = S.trec[i & 1];
        tr.nrow = ti.nrow;
        tr.pos0 = a.lens[ti.b] + ti.t0;
        tr.rec = ((long long)ti.b * a.h_kv + ti.h) * a.ntiles * (long long)L.tile_bytes;
        tr.kbase0 = (((long long)ti.b * a.T + ti.t0) * a.h_kv + ti.h) * kD;
      }
      if (w == 0 && lane == 0) {
        mbar_arrive_expect_tx(&S.k_full, 16 * 2048);
#pragma unroll 1
        for (int ch = 0; ch < 16; ++ch) tma_load_4d(S.a1 + ch * 2048, &kmap, 8 * ch, ti.h, ti.t0, ti.b, &S.k_full);
      }
      __syncwarp();
      in_flight = i;
      if (!qwait(&S.k_full, i & 1, &S.abort_flag, a)) break;
      in_flight = -1;
      const int row = 32 * w + lane;
      float ss = 0.f;
#pragma unroll 4
      for (int c = 0; c < 16; ++c) {
        const uint4 v = *reinterpret_cast<const uint4 *>(S.a1 + blk_off(row, 8 * c));
        const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(p2[e]);
          ss = fmaf(f.x, f.x, ss);
          ss = fmaf(f.y, f.y, ss);
        }
      }
      const float nrm = sqrtf(ss);
      S.nk[i & 1][row] = nrm;
      S.ninv[i & 1][row] = nrm > 0.f ? 1.f / nrm : 0.f;
      __syncwarp();
      // (a test of the timeout path withholds the hand-off: the MMA issuer's
      // bounded wait on it then runs out)
      if (lane == 0 && !a.test_withhold) mbar_arrive(&S.a1_full);
    }
    // never leave with a copy in flight (a role gave up while it ran): the
    // copy engine completes it, so this wait ends
    if (in_flight >= 0) mbar_wait(&S.k_full, in_flight & 1);
  } else {
    reg_alloc<kEpiRegs>();
    // ---------------- epilogue ---------------------------------------------
    // Warp w of WG2-WG5 takes TMEM lane quarter w % 4 (tile rows 32 (w % 4)
    // .. + 31, a row per thread) and column quarter cq (coordinates 32 cq ..
    // 32 cq + 31, the K-steps 2 cq and 2 cq + 1 of GEMM2).  Step j runs E1
    // of tile j and then E2 of tile j - 1, whose GEMM2 ran under E1 and has
    // finished by then.  The four warps of a lane quarter meet once per tile
    // for ||r||^2.
    const int ew = warp - 8;  // epilogue warp 0 .. 15 (its refinement ring)
    const int cq = ew >> 2;
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;  // tile row == TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const uint32_t d1col = tbase + lane_off + 32 * cq;
    const uint32_t ecol = tbase + lane_off + 384;  // E operand
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
    // the previous tile's row, for its E2
    bool pv_valid = false, pv_zero = true;
    uint8_t *pv_tp = nullptr;
    int pv_slot = 0;
    size_t pv_kbase = 0;
    float pv_nk = 0.f;
    for (int j = 0; j <= nlocal; ++j) {
      bool valid = false, zero = true;
      uint8_t *tp = nullptr;
      int slot = 0;
      size_t kbase = 0;
      float nk = 0.f;
      if (j < nlocal) {
        const int buf = j & 1;
        if (!qwait(&S.d1_full, j & 1, &S.abort_flag, a)) break;
        tc_fence_after();
        // the tile's record and norms, written by the loader before GEMM1
        {
          const TileRec &tr = S.trec[buf];
          valid = r < tr.nrow;
          const int pos = tr.pos0 + r;
          tp = valid ? reinterpret_cast<uint8_t *>(a.data) + tr.rec + (long long)((unsigned)pos / kTile) * L.tile_bytes
                     : nullptr;
          slot = (int)((unsigned)pos % kTile);
          kbase = (size_t)(tr.kbase0 + (long long)r * a.h_kv * kD);  // this row's key
        }
        nk = S.nk[buf][r];
        zero = !(nk > 0.f);
        const float inv1 = S.ninv[buf][r];  // y = Y / ||k||
        const float inv13 = inv1 * kEScale;
        // a zero key gets y = -inf everywhere, which every bucketize below
        // maps to code 0; its E row is finite garbage (D1 = 0, scale 0) whose
        // products stay in its own row, and its signs and ||r|| are zeroed
        const float ybias = zero ? -INFINITY : 0.f;
        // ---- E1: y = Pi u, codes, E = (y - c) x 2^13 handed to GEMM2 a
        // K-step (16 coordinates) at a time, ||r||^2 = ||E||^2 ----
        // code indices as nibbles, split into bit-planes once the quarter is
        // done: element e goes to word e / 8, nibble 2 b (b = e % 8 < 4) or
        // 2 (b - 4) + 1 (b >= 4), the order one multiply gathers bit p of
        // the eight nibbles in
        uint32_t nib[4] = {0u, 0u, 0u, 0u};
        float2 rr2 = make_float2(0.f, 0.f);  // ||r||^2 x 2^26 over this quarter, in two halves
        // The codebook's shape is decided once per tile, outside the element
        // loop: a branch per element would keep the compiler from
        // interleaving the elements' dependent chains.
        // GEMM1 of the next tile may overwrite D1 once every warp holds its
        // columns; E may be overwritten once the previous tile's GEMM2 is done
        auto e1 = [&](auto sym_c) -> bool {
          constexpr bool SYM = decltype(sym_c)::value;
          uint32_t d1[32];
          tmem_ld32(d1col, d1);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.d1_read);
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const uint32_t *d = d1 + 16 * cc;
            uint32_t hl[16];  // hi parts (columns 0-7), lo parts (8-15)
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              // two coordinates at a time, in paired f32 arithmetic
              const float2 dv2 = make_float2(__uint_as_float(d[e]), __uint_as_float(d[e + 1]));
              const float2 y2 = __ffma2_rn(dv2, make_float2(inv1, inv1), make_float2(ybias, ybias));
              float nc[2];  // -c x 2^13
#pragma unroll
              for (int x = 0; x < 2; ++x) {
                const float y = x ? y2.y : y2.x;
                // the code is #{boundaries < y} = NC/2 + xi
                int xi;
                if constexpr (SYM) {
                  // NC/2 + cnt above zero, NC/2 - 1 - cnt = NC/2 + ~cnt at or
                  // below it: one xor with the all-ones mask of y <= 0
                  const float ay = fabsf(y);
                  int cnt = 0;
#pragma unroll
                  for (int k = 0; k < NU; ++k) cnt += (ub[k] < ay) ? 1 : 0;
                  xi = cnt ^ -(int)!(y > 0.f);
                } else {  // any codebook: count the boundaries below y
                  xi = -NC / 2;
#pragma unroll
                  for (int k = 0; k < NC - 1; ++k) xi += (S.bnd[k] < y) ? 1 : 0;  // independent broadcast reads
                }
                // xi in [-NC/2, NC/2): the words hold sum xi 16^slot, and
                // NC/2 in every nibble is added at the end (the sums are exact
                // modulo 2^32, so the borrows cancel)
                const int el = 16 * cc + e + x, b = el & 7;
                nib[el >> 3] += (uint32_t)xi << (4 * (b < 4 ? 2 * b : 2 * b - 7));
                nc[x] = S.ncent13[NC / 2 + xi];
              }
              // E = (y - c) 2^13 from D1 in one rounding
              const float2 ev = __ffma2_rn(dv2, make_float2(inv13, inv13), make_float2(nc[0], nc[1]));
              rr2 = __ffma2_rn(ev, ev, rr2);
              const __half2 hh = __floats2half2_rn(ev.x, ev.y);
              // lo = E - hi, exact
              const float2 lo = __ffma2_rn(__half22float2(hh), make_float2(-1.f, -1.f), ev);
              const __half2 ll = __floats2half2_rn(lo.x, lo.y);
              hl[e >> 1] = *reinterpret_cast<const uint32_t *>(&hh);
              hl[8 + (e >> 1)] = *reinterpret_cast<const uint32_t *>(&ll);
            }
            if (cc == 0 && j >= 1) {
              if (!qwait(&S.d2_full[(j - 1) & 1], ((j - 1) >> 1) & 1, &S.abort_flag, a)) return false;
              tc_fence_after();
            }
            tmem_st16(ecol + 16 * (2 * cq + cc), hl);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.kc[2 * cq + cc]);
          }
          return true;
        };
        if (!(sym ? e1(std::true_type{}) : e1(std::false_type{}))) break;
#pragma unroll
        for (int q = 0; q < 4; ++q) nib[q] += (uint32_t)(NC / 2) * 0x11111111u;
        if (valid)  // this warp's word of every code plane row
#pragma unroll
          for (int p = 0; p < MB; ++p) {
            // bit p of nibble i sits at 4 i + p; times sum_k 2^(7 k + 3 - p)
            // it lands at 4 i + 7 k + 3, sixteen distinct positions for
            // k < 4 (no carries), with nibbles 0, 2, 4, 6 at bits 24-27
            // (k = 3 - i / 2) and 1, 3, 5, 7 at 28-31: byte 3 is elements
            // 8q .. 8q + 7 of the quarter in order
            uint32_t g[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) g[q] = (nib[q] & (0x11111111u << p)) * (0x00204081u << (3 - p));
            const uint32_t w = __byte_perm(__byte_perm(g[0], g[1], 0x0073u), __byte_perm(g[2], g[3], 0x0073u), 0x5410u);
            *reinterpret_cast<uint32_t *>(tp + L.kplanes + p * kPlaneBytes + slot * kRowBytes + 4 * cq) = w;
          }
        S.rrq[j & 3][cq][r] = rr2.x + rr2.y;
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.pair[j & 1][q4]);  // this quarter's ||r||^2 is written
      }
      if (j >= 1) {
        // ---- E2 of tile t = j - 1: signs of z = S r = W (y - c), norms ----
        const int t = j - 1, tb = t & 1;
        const uint32_t tph = (t >> 1) & 1;
        if (!qwait(&S.d2_full[tb], tph, &S.abort_flag, a)) break;
        tc_fence_after();
        uint32_t d2[32];
        tmem_ld32(d1col + 128 + 128 * tb, d2);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.d_free[tb]);  // D2 is in registers
        // sign bits: element e's sign bit shifted in last-first, so it ends
        // in bit e (one funnel shift an element); a set sign bit is z < 0
        // except at z = -0, which like every |z| < the refinement threshold
        // is re-decided by the refiner
        uint32_t neg = 0u;
#pragma unroll
        for (int e = 31; e >= 0; --e) neg = __funnelshift_l(d2[e], neg, 1);
        uint32_t sw = ~neg;
        // the smallest |z| of the row (three-input minima); the mask of the
        // components next to zero only where it is below the threshold
        float zmin = fabsf(__uint_as_float(d2[0]));
#pragma unroll
        for (int e = 1; e < 31; e += 2)
          zmin = min3f(zmin, fabsf(__uint_as_float(d2[e])),
                       fabsf(__uint_as_float(d2[e + 1])));
        zmin = fminf(zmin, fabsf(__uint_as_float(d2[31])));
        uint32_t nearw = 0u;  // |S r| below the refinement threshold
        if (zmin < kNearZ) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            nearw |= (fabsf(__uint_as_float(d2[e])) < kNearZ ? 1u : 0u) << e;
        }
        if (pv_zero) sw = 0u;
        if (pv_zero || !pv_valid) nearw = 0u;
        if (pv_valid) *reinterpret_cast<uint32_t *>(pv_tp + L.signs + pv_slot * kRowBytes + 4 * cq) = sw;
        if (cq == 0) {
          // the four quarters' ||r||^2
          if (!qwait(&S.pair[tb][q4], tph, &S.abort_flag, a)) break;
          if (pv_valid) {
            const float rr2 = (S.rrq[t & 3][0][r] + S.rrq[t & 3][1][r]) + (S.rrq[t & 3][2][r] + S.rrq[t & 3][3][r]);
            const float rn = pv_zero ? 0.f : sqrtf(rr2) * (1.f / kEScale);
            *reinterpret_cast<__half2 *>(pv_tp + L.norms + pv_slot * 4) =
                __halves2half2(__float2half_rn(pv_nk), __float2half_rn(rn));
          }
        }
        // sketch components next to zero: handed to the float64 refiner,
        // which patches the sign words stored above (at most kRingCap rows
        // at a time)
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
            q.kbase = pv_kbase;
            q.planes = (unsigned long long)(pv_tp + L.kplanes + pv_slot * kRowBytes);
            q.signs = (unsigned long long)(pv_tp + L.signs + pv_slot * kRowBytes);
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
      pv_valid = valid;
      pv_zero = zero;
      pv_tp = tp;
      pv_slot = slot;
      pv_kbase = kbase;
      pv_nk = nk;
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
  // launched as a dependent of the value kernel: this grid is not complete
  // before that one is
  pdl_wait();
}

template <int MB>
cudaError_t launch_qt(const AppendArgs &a, const CUtensorMap &kmap, int grid, cudaStream_t stream) {
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
  // a programmatic dependent of the value kernel, whose record bytes it
  // does not touch: it starts as that kernel's blocks drain and waits for
  // it only before it finishes
  return launch_pdl(quantize_tc_kernel<MB>, dim3(grid), dim3(kQtThreads), smem, stream, a, kmap);
}

// The driver's tensor-map encoder, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// K as a (channel, head, token, sequence) bf16 tensor, boxes of 8 channels
// x 1 head x 128 tokens x 1 sequence, no swizzle, zero fill out of range.
cudaError_t encode_k_map(const AppendArgs &a, CUtensorMap *map) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)a.h_kv, (cuuint64_t)a.T, (cuuint64_t)a.batch};
  const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)a.h_kv * kD * 2, (cuuint64_t)a.T * a.h_kv * kD * 2};
  const cuuint32_t box[4] = {8, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(a.k), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_prepare_operands(const float *pi, const double *s_pit, void *dst, cudaStream_t stream) {
  prepare_operands_kernel<<<128 * 16 / 256, 256, 0, stream>>>(pi, s_pit, reinterpret_cast<uint8_t *>(dst));
  return cudaGetLastError();
}

bool quantize_tc_supported(const AppendArgs &a) {
  // (the K tensor map wants a 16-byte aligned base; the value kernel splits
  // vector slots with 32-bit arithmetic below a sequence)
  return a.d == kD && a.value_mode == TQ_VALUES_GROUP && a.dtype == TQ_BF16 && a.key_bits >= 2 && a.key_bits <= 4 &&
         a.value_bits >= 2 && a.value_bits <= 4 && a.T >= 64 && (reinterpret_cast<uintptr_t>(a.k) & 15) == 0 &&
         (long long)a.T * a.h_kv < (1LL << 31);
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
  CUtensorMap kmap;
  const cudaError_t em = encode_k_map(a, &kmap);
  if (em != cudaSuccess) return em;
  const cudaError_t ev = launch_value_quant(a, num_sms, stream);
  if (ev != cudaSuccess) return ev;
  switch (a.key_bits - 1) {
    case 1: return launch_qt<1>(a, kmap, grid, stream);
    case 2: return launch_qt<2>(a, kmap, grid, stream);
    case 3: return launch_qt<3>(a, kmap, grid, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace tq
