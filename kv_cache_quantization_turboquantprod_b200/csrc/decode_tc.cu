// Decode attention over the compressed cache on the 5th-generation tensor
// cores (tcgen05, kind::i8), one CTA per (split, KV head, sequence).
//
// What it computes is the one-pass decode of "03. Results & Benchmarks"
// (turboquant_cutile, "Latency Benchmarks": score, QJL correction, online
// softmax and V accumulation in one pass) with the estimator of
// "turboquant/audit_claims.py" (attention_score):
//   score = ||k|| * ( <Pi q, c[idx]> + sqrt(pi/2)/d * ||r|| * <S q, 2 sign - 1> ).
//
// How.  Decode is HBM-bound on the packed records, but a SIMT
// implementation cannot retire a 128-coordinate dot product per (token,
// query head) inside the ~20 issue slots per record that full bandwidth
// allows.  The bit-planes are therefore fed to the tensor cores as exact
// 0/2^k integer operands: one LOP3 (w & (0x01010101 << k)) turns a 32-bit
// plane word into four u8 operands, and
//   * scores: D[token, (head, limb)] = A_k[token, plane bits] x B_q, where
//     B_q holds the rotated query (times the plane weight, divided by 2^k)
//     as four signed base-128 fixed-point limbs; s32 accumulation is exact;
//     the centroid lookup is exact because c(idx) is multilinear in the code
//     bits (2-bit codes) or a sum of threshold planes (3-bit codes);
//   * values: D[channel, (group, head, byte)] = A_v[channel, codes x tokens]
//     x B_p[tokens, p * scale_g as 22-bit fixed point]; 2-bit codes are
//     stored packed, so one mask (w & (0x03030303 << 2m)) yields code * 4^m
//     operands; wider codes are bit-planes whose B_p copies carry 2^plane.
//     The 4^m (or 2^k) weight of each operand row is undone per channel.
// Per 128-token tile the record bytes arrive by one 1-D bulk copy (TMA
// engine) into a ring of shared-memory stages.
//
// Warp roles (448 threads; each SM sub-partition gets one warp of each
// worker group, so the three per-token instruction streams overlap):
//   warp 0       bulk-copy producer; allocates / frees tensor memory
//   warp 1       single-thread MMA issuer (tcgen05.mma + commit)
//   warps 2-5    key group: key bit-planes -> A_k operand in tensor memory
//   warps 6-9    value group: V bit-planes -> A_v (MN-major, shared memory);
//                PV epilogue and the per-channel accumulators
//   warps 10-13  softmax group: score epilogue, online softmax (tile max by
//                warp redux + an mbarrier exchange), the P' operand, running
//                l and zero-point sums
// Every mbarrier wait is bounded (2 s); on timeout the CTA sets the status word in
// the workspace, stops, waits for its own copies and MMAs and frees TMEM.
#include <math.h>

#include "sm100.cuh"
#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

namespace {

using namespace sm100;

constexpr int kTcThreads = 448;
constexpr float kLog2e = 1.4426950408889634f;

// 2^n for n in [-126, 127]
__device__ __forceinline__ float exp2i(int n) { return __uint_as_float((uint32_t)(n + 127) << 23); }
// floor(log2(x)) for a positive normal float
__device__ __forceinline__ int ilog2f(float x) { return (int)((__float_as_uint(x) >> 23) & 0xFF) - 127; }

// Score constants that follow B_q in a query block (floats): cm[8] (c_0 sum
// q~), csum[8] (sum s^), coef_m[8][2], coef_s[8][2] (limb weights), then the
// skip flag of the product plane (int).
constexpr int kQConstBytes = 256;
struct QConst {
  float cm[8];
  float csum[8];
  float coef_m[8][2];
  float coef_s[8][2];
  int skip_product_plane;
};
static_assert(sizeof(QConst) <= kQConstBytes, "query constants");

template <int MB_, int VB_, int G_>
struct Cfg {
  static constexpr int MB = MB_, VB = VB_, G = G_;
  // operand planes of the MSE term: b0 (1 bit); b0, b1, b0&b1 (2 bits,
  // multilinear, exact for any 4-level codebook); [idx >= l], l = 1..7
  // (3 bits, threshold planes)
  static constexpr int NP = MB == 1 ? 1 : (MB == 2 ? 3 : 7);
  static constexpr int AK_COLS = (NP + 1) * 32;          // one A_k buffer
  static constexpr int NS = ((4 * G + 15) / 16) * 16;   // score N per accumulator
  static constexpr int NPV = 16 * G;                    // PV N: 4 groups x G heads x 4 bytes
  static constexpr int DS_COLS = 4 * NS;                // 2 buffers x (mse, qjl)
  static constexpr int DPV_COLS = 2 * NPV;              // 2 buffers
  static constexpr int AKB = (2 * AK_COLS + DS_COLS + DPV_COLS <= 512) ? 2 : 1;
  static constexpr int COL_AK = 0;
  static constexpr int COL_DS = AKB * AK_COLS;
  static constexpr int COL_DPV = COL_DS + DS_COLS;
  static constexpr int COLS_USED = COL_DPV + DPV_COLS;
  static constexpr int TMEM_COLS =
      COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64 : COLS_USED <= 128 ? 128
                                                    : COLS_USED <= 256 ? 256 : 512;
  static constexpr int REC = (MB + 1 + VB) * 16 + 20;
  static constexpr int TILE_BYTES = 128 * REC;
  static constexpr int OFF_SIGNS = MB * 2048;
  static constexpr int OFF_V = (MB + 1) * 2048;
  static constexpr int OFF_NORMS = (MB + 1 + VB) * 2048;
  static constexpr int OFF_VSZ = OFF_NORMS + 512;
  // value operands: 2-bit values are stored packed (one operand byte per
  // channel holds code * 4^m); wider values are bit-planes (one operand each)
  static constexpr bool PACKED_V = (VB == 2);
  static constexpr int VOPS = PACKED_V ? 1 : VB;
  static constexpr int AV_BYTES = VOPS * 128 * 128;     // [128 channels] x [VOPS*128 K]
  static constexpr int BP_BYTES = VOPS * 128 * NPV;     // [VOPS*128 K] x [NPV]
  static constexpr int BQ_BYTES = (NP + 1) * 128 * NS;  // [(NP+1)*128 K] x [NS]
  static constexpr int SBO_V = VOPS * 2048;             // MN-major stride of 16-byte chunks
  static constexpr int LBO_Q = (NS / 8) * 128;          // K-major stride of 16-byte K chunks
  static constexpr int QBLOCK = BQ_BYTES + kQConstBytes;  // per (sequence, KV head)
  static constexpr int FIXED = 2 * AV_BYTES + 2 * BP_BYTES + QBLOCK + 4096;
  static constexpr int STAGES_FIT = (220 * 1024 - FIXED) / TILE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  static_assert(COLS_USED <= 512, "tensor memory budget");
  static_assert(STAGES >= 2, "shared memory budget");
  static_assert(TILE_BYTES % 16 == 0, "bulk copy size");
};

template <class C>
struct TcSmem {
  alignas(128) uint8_t stage[C::STAGES][C::TILE_BYTES];
  alignas(128) uint8_t av[2][C::AV_BYTES];
  alignas(128) uint8_t bp[2][C::BP_BYTES];
  alignas(128) uint8_t bq[C::BQ_BYTES + kQConstBytes];  // B_q operand + score constants
  uint64_t full[C::STAGES];
  uint64_t empty[C::STAGES];
  uint64_t ak_ready[2], s_ready[2], s_free[2], av_ready[2], p_ready[2], pv_done[2], pv_free[2];
  uint64_t red_bar[2];
  uint64_t q_full;
  uint32_t tmem_base;
  volatile int abort_flag;
  uint32_t red[2][4][C::G + 1];
  float alpha[2][C::G];
  float pscale[2];
  float zsum[4][C::G][4];
  float lsum[4][C::G];
};

// Bounded wait (2 s of wall time) that also gives up when another role has
// aborted; a timeout raises the CTA's abort flag and the status word.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         int *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > 2000000000ull) break;
  }
  *abort_flag = 1;
  if (status) atomicOr(status, 1);
  return false;
}

// Operand plane `op` of the MSE term for one 32-bit word of each bit-plane.
template <int MB>
__device__ __forceinline__ uint32_t mse_plane_word(int op, const uint32_t (&bw)[3]) {
  if (MB == 1) return bw[0];
  if (MB == 2) return op == 0 ? bw[0] : (op == 1 ? bw[1] : (bw[0] & bw[1]));
  // MB == 3: threshold planes [idx >= op + 1]
  const uint32_t b0 = bw[0], b1 = bw[1], b2 = bw[2];
  switch (op) {
    case 0: return b0 | b1 | b2;
    case 1: return b1 | b2;
    case 2: return b2 | (b1 & b0);
    case 3: return b2;
    case 4: return b2 & (b1 | b0);
    case 5: return b2 & b1;
    default: return b2 & b1 & b0;
  }
}

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
  static_assert(N % 4 == 0, "multiple of 4 columns");
  int c = 0;
#pragma unroll
  for (; c + 32 <= N; c += 32) {
    uint32_t t[32];
    tmem_ld32(taddr + c, t);
#pragma unroll
    for (int x = 0; x < 32; ++x) r[c + x] = t[x];
  }
#pragma unroll
  for (; c + 16 <= N; c += 16) {
    uint32_t t[16];
    tmem_ld16(taddr + c, t);
#pragma unroll
    for (int x = 0; x < 16; ++x) r[c + x] = t[x];
  }
#pragma unroll
  for (; c + 8 <= N; c += 8) {
    uint32_t t[8];
    tmem_ld8(taddr + c, t);
#pragma unroll
    for (int x = 0; x < 8; ++x) r[c + x] = t[x];
  }
#pragma unroll
  for (; c + 4 <= N; c += 4) {
    uint32_t t[4];
    tmem_ld4(taddr + c, t);
#pragma unroll
    for (int x = 0; x < 4; ++x) r[c + x] = t[x];
  }
}

template <int MB, int VB, int G>
__global__ void __launch_bounds__(kTcThreads, 1) decode_tc_kernel(const __grid_constant__ DecodeArgs a) {
  using C = Cfg<MB, VB, G>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  TcSmem<C> &S = *reinterpret_cast<TcSmem<C> *>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;

  int len = a.len[b];
  len = len < 0 ? 0 : (len > a.max_len ? a.max_len : len);
  const int tile0 = split * a.tiles_per_split;
  const int t_begin = tile0 * kTile;
  const int t_end = min(len, (split + 1) * a.tiles_per_split * kTile);
  const int ntile = t_end > t_begin ? (t_end - t_begin + kTile - 1) / kTile : 0;
  auto part_row = [&](int g) {
    return a.part + (((size_t)b * a.h_q + (size_t)h * G + g) * a.nsplit + split) * (kD + 2);
  };
  if (ntile == 0) {  // empty split: neutral partial state
    for (int i = tid; i < G * (kD + 2); i += kTcThreads) {
      const int g = i / (kD + 2), j = i % (kD + 2);
      part_row(g)[j] = (j == kD) ? -INFINITY : 0.f;
    }
    return;
  }

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 12);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.ak_ready[i], 4);
      mbar_init(&S.s_ready[i], 1);
      mbar_init(&S.s_free[i], 4);
      mbar_init(&S.av_ready[i], 4);
      mbar_init(&S.p_ready[i], 4);
      mbar_init(&S.pv_done[i], 1);
      mbar_init(&S.pv_free[i], 4);
      mbar_init(&S.red_bar[i], 4);
    }
    mbar_init(&S.q_full, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&S.tmem_base, C::TMEM_COLS);

  const uint8_t *tiles = reinterpret_cast<const uint8_t *>(a.data) +
                         (((size_t)b * a.h_kv + h) * a.ntiles + tile0) * (size_t)C::TILE_BYTES;
  const QConst &Q = *reinterpret_cast<const QConst *>(S.bq + C::BQ_BYTES);

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;
  int *status = a.status;

  if (warp == 0) {
    // ---------------- producer --------------------------------------------
    if (lane == 0) {
      mbar_arrive_expect_tx(&S.q_full, C::QBLOCK);
      bulk_g2s(S.bq, a.qblocks + ((size_t)b * a.h_kv + h) * C::QBLOCK, C::QBLOCK, &S.q_full);
      int issued = 0;
      for (int i = 0; i < ntile; ++i) {
        const int s = i % C::STAGES;
        if (i >= C::STAGES &&
            !wait_bar(&S.empty[s], ((i / C::STAGES) - 1) & 1, &S.abort_flag, status))
          break;
        mbar_arrive_expect_tx(&S.full[s], C::TILE_BYTES);
        bulk_g2s(S.stage[s], tiles + (size_t)i * C::TILE_BYTES, C::TILE_BYTES, &S.full[s]);
        ++issued;
      }
      // never leave with a copy in flight
      mbar_wait(&S.q_full, 0);
      for (int i = max(0, issued - C::STAGES); i < issued; ++i)
        mbar_wait(&S.full[i % C::STAGES], (i / C::STAGES) & 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ------------------------------------------
    // Descriptors are built once; an instruction's operand offsets are
    // compile-time constants added to the 16-byte-unit address field.
    if (lane == 0) {
      const uint32_t id_s = idesc_i8(128, C::NS, false, true, false, false);
      const uint32_t id_p = idesc_i8(128, C::NPV, false, false, true, true);
      const bool qok = wait_bar(&S.q_full, 0, &S.abort_flag, status);
      const bool skip3 = Q.skip_product_plane != 0;
      const uint64_t dq0 = smem_desc(S.bq, C::LBO_Q, 128);
      const uint64_t dav[2] = {smem_desc(S.av[0], 128, C::SBO_V), smem_desc(S.av[1], 128, C::SBO_V)};
      const uint64_t dbp[2] = {smem_desc(S.bp[0], 128, C::SBO_V), smem_desc(S.bp[1], 128, C::SBO_V)};
      int last_s = -1, last_p = -1;
      for (int i = 0; qok && i <= ntile; ++i) {
        if (i < ntile) {
          const int kb = i & 1;
          if (!wait_bar(&S.ak_ready[kb], (i >> 1) & 1, &S.abort_flag, status)) break;
          if (i >= 2 && !wait_bar(&S.s_free[kb], ((i - 2) >> 1) & 1, &S.abort_flag, status)) break;
          tc_fence_after();
          const uint32_t a_base = tbase + C::COL_AK + (i % C::AKB) * C::AK_COLS;
          const uint32_t d_mse = tbase + C::COL_DS + kb * 2 * C::NS;
          const uint32_t d_qjl = d_mse + C::NS;
#pragma unroll
          for (int p = 0; p < C::NP; ++p) {
            if (MB == 2 && p == 2 && skip3) continue;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const int ins = p * 4 + kk;
              mma_i8_ts(d_mse, a_base + ins * 8, dq0 + (uint64_t)((2 * ins * C::LBO_Q) >> 4), id_s,
                        ins ? 1u : 0u);
            }
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int ins = C::NP * 4 + kk;
            mma_i8_ts(d_qjl, a_base + ins * 8, dq0 + (uint64_t)((2 * ins * C::LBO_Q) >> 4), id_s,
                      kk ? 1u : 0u);
          }
          mma_commit(&S.s_ready[kb]);
          last_s = i;
        }
        if (i >= 1) {
          const int jt = i - 1, pb = jt & 1;
          if (!wait_bar(&S.p_ready[pb], (jt >> 1) & 1, &S.abort_flag, status)) break;
          if (!wait_bar(&S.av_ready[pb], (jt >> 1) & 1, &S.abort_flag, status)) break;
          if (jt >= 2 && !wait_bar(&S.pv_free[pb], ((jt - 2) >> 1) & 1, &S.abort_flag, status)) break;
          tc_fence_after();
          const uint32_t d_pv = tbase + C::COL_DPV + pb * C::NPV;
          const uint64_t da = dav[pb], db = dbp[pb];
#pragma unroll
          for (int ins = 0; ins < C::VOPS * 4; ++ins)
            mma_i8_ss(d_pv, da + (uint64_t)(32 * ins), db + (uint64_t)(32 * ins), id_p, ins ? 1u : 0u);
          mma_commit(&S.pv_done[pb]);
          last_p = jt;
        }
      }
      // never leave with an MMA in flight
      if (last_s >= 0) mbar_wait(&S.s_ready[last_s & 1], (last_s >> 1) & 1);
      if (last_p >= 0) mbar_wait(&S.pv_done[last_p & 1], (last_p >> 1) & 1);
    }
  } else if (warp < 6) {
    // ---------------- key group: A_k expansion ----------------------------
    const int q4 = warp & 3;
    const int t = 32 * q4 + lane;  // token slot == TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const bool qok = wait_bar(&S.q_full, 0, &S.abort_flag, status);
    const bool skip3 = Q.skip_product_plane != 0;
    for (int i = 0; qok && i < ntile; ++i) {
      const int s = i % C::STAGES;
      if (!wait_bar(&S.full[s], (i / C::STAGES) & 1, &S.abort_flag, status)) break;
      // the A_k buffer of tile i was last read by the score MMA of tile i - AKB
      if (i >= C::AKB) {
        const int prev = i - C::AKB;
        if (!wait_bar(&S.s_ready[prev & 1], (prev >> 1) & 1, &S.abort_flag, status)) break;
      }
      const uint8_t *st = S.stage[s];
      uint32_t bw[4][3];
#pragma unroll
      for (int p = 0; p < MB; ++p) {
        const uint4 v = *reinterpret_cast<const uint4 *>(st + p * kPlaneBytes + t * kRowBytes);
        bw[0][p] = v.x; bw[1][p] = v.y; bw[2][p] = v.z; bw[3][p] = v.w;
      }
#pragma unroll
      for (int p = MB; p < 3; ++p) bw[0][p] = bw[1][p] = bw[2][p] = bw[3][p] = 0u;
      const uint4 sv = *reinterpret_cast<const uint4 *>(st + C::OFF_SIGNS + t * kRowBytes);
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[s]);
      const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
      const uint32_t a_base = tbase + lane_off + C::COL_AK + (i % C::AKB) * C::AK_COLS;
#pragma unroll
      for (int op = 0; op <= C::NP; ++op) {
        if (MB == 2 && op == 2 && skip3) continue;
        uint32_t r[32];
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          const uint32_t word = (op < C::NP) ? mse_plane_word<MB>(op, bw[wd]) : sw[wd];
#pragma unroll
          for (int k = 0; k < 8; ++k) r[wd * 8 + k] = word & (0x01010101u << k);
        }
        tmem_st32(a_base + op * 32, r);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.ak_ready[i & 1]);
    }
  } else if (warp < 10) {
    // ---------------- value group ------------------------------------------
    const int q4 = warp & 3;
    const int t = 32 * q4 + lane;  // token slot for expansion; M slot for PV
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    // channel of this M slot and the 2^kk weight its operand bytes carry
    const int kk = C::PACKED_V ? 2 * ((t >> 2) & 3) : (t & 31) >> 2;
    const int chan = C::PACKED_V ? 16 * (t >> 4) + 4 * (t & 3) + ((t >> 2) & 3)
                                 : 32 * q4 + 8 * (t & 3) + kk;
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = 0.f;
    for (int i = 0; i <= ntile; ++i) {
      if (i < ntile) {
        const int s = i % C::STAGES, vb = i & 1;
        if (!wait_bar(&S.full[s], (i / C::STAGES) & 1, &S.abort_flag, status)) break;
        const uint8_t *st = S.stage[s];
        uint8_t *av = S.av[vb];
        if constexpr (C::PACKED_V) {
          // packed row: word w holds channels 16w .. 16w+15; mask m keeps
          // channel 16w + 4i + m in byte i as code * 4^m (M slot 16w + 4m + i)
          const uint4 v0 = *reinterpret_cast<const uint4 *>(st + C::OFF_V + t * kPackedRowBytes);
          const uint4 v1 = *reinterpret_cast<const uint4 *>(st + C::OFF_V + t * kPackedRowBytes + 16);
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.empty[s]);
          const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
          uint8_t *row = av + (t >> 3) * 128 + (t & 7) * 16;
#pragma unroll
          for (int w = 0; w < 8; ++w)
            *reinterpret_cast<uint4 *>(row + w * C::SBO_V) =
                make_uint4(vw[w] & 0x03030303u, vw[w] & 0x0C0C0C0Cu, vw[w] & 0x30303030u,
                           vw[w] & 0xC0C0C0C0u);
        } else {
          uint4 vp[VB];
#pragma unroll
          for (int p = 0; p < VB; ++p)
            vp[p] = *reinterpret_cast<const uint4 *>(st + C::OFF_V + p * kPlaneBytes + t * kRowBytes);
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.empty[s]);
#pragma unroll
          for (int p = 0; p < VB; ++p) {
            const uint32_t vw[4] = {vp[p].x, vp[p].y, vp[p].z, vp[p].w};
            uint8_t *row = av + p * 2048 + (t >> 3) * 128 + (t & 7) * 16;
#pragma unroll
            for (int m16 = 0; m16 < 8; ++m16) {
              const uint32_t word = vw[m16 >> 1];
              const int k0 = (m16 & 1) * 4;
              *reinterpret_cast<uint4 *>(row + m16 * C::SBO_V) =
                  make_uint4(word & (0x01010101u << k0), word & (0x01010101u << (k0 + 1)),
                             word & (0x01010101u << (k0 + 2)), word & (0x01010101u << (k0 + 3)));
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.av_ready[vb]);
      }
      if (i >= 1) {
        const int jt = i - 1, pb = jt & 1;
        if (!wait_bar(&S.pv_done[pb], (jt >> 1) & 1, &S.abort_flag, status)) break;
        if (!wait_bar(&S.p_ready[pb], (jt >> 1) & 1, &S.abort_flag, status)) break;
        tc_fence_after();
        uint32_t d[4 * G];
        tmem_ld_cols<4 * G>(tbase + lane_off + C::COL_DPV + pb * C::NPV + q4 * 4 * G, d);
        tmem_wait_ld();
        tc_fence_before();
        float alpha[G];
#pragma unroll
        for (int g = 0; g < G; ++g) alpha[g] = S.alpha[pb][g];
        const float sc = S.pscale[pb] * exp2i(-kk);
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.pv_free[pb]);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float v = fmaf(16777216.f, (float)d[4 * g + 3],
                               fmaf(65536.f, (float)d[4 * g + 2],
                                    fmaf(256.f, (float)d[4 * g + 1], (float)d[4 * g])));
          acc[g] = fmaf(acc[g], alpha[g], v * sc);
        }
      }
    }
    named_bar_sync(3, 256);  // the softmax group's zero-point sums are in smem
    // unnormalised partial output: sum_t p_t (code * scale + zero)
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float z = 0.f;
#pragma unroll
      for (int wq = 0; wq < 4; ++wq) z += S.zsum[wq][g][q4];
      part_row(g)[chan] = acc[g] + z;
    }
  } else {
    // ---------------- softmax group ----------------------------------------
    const int q4 = warp & 3;
    const int t = 32 * q4 + lane;  // token slot == TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const float kappa = qjl_kappa();
    const float scale2 = a.softmax_scale * kLog2e;
    float mrun[G], lsum[G], zs[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mrun[g] = -INFINITY;
      lsum[g] = 0.f;
#pragma unroll
      for (int gg = 0; gg < 4; ++gg) zs[g][gg] = 0.f;
    }
    const bool qok = wait_bar(&S.q_full, 0, &S.abort_flag, status);
    for (int jt = 0; qok && jt < ntile; ++jt) {
      const int kb = jt & 1, pb = jt & 1, s = jt % C::STAGES;
      if (!wait_bar(&S.full[s], (jt / C::STAGES) & 1, &S.abort_flag, status)) break;
      if (!wait_bar(&S.s_ready[kb], (jt >> 1) & 1, &S.abort_flag, status)) break;
      tc_fence_after();
      uint32_t dm[4 * G], dq[4 * G];
      {
        const uint32_t base = tbase + lane_off + C::COL_DS + kb * 2 * C::NS;
        tmem_ld_cols<4 * G>(base, dm);
        tmem_ld_cols<4 * G>(base + C::NS, dq);
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.s_free[kb]);

      const uint8_t *st = S.stage[s];
      const bool valid = t_begin + jt * kTile + t < t_end;
      const __half2 nr = *reinterpret_cast<const __half2 *>(st + C::OFF_NORMS + t * 4);
      const float nk = __low2float(nr), rn = __high2float(nr);
      const uint4 szr = *reinterpret_cast<const uint4 *>(st + C::OFF_VSZ + t * 16);
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[s]);
      const __half2 *szh = reinterpret_cast<const __half2 *>(&szr);
      float vsc[4], vze[4];
      float msc = 0.f;
#pragma unroll
      for (int gg = 0; gg < 4; ++gg) {
        vsc[gg] = valid ? __low2float(szh[gg]) : 0.f;
        vze[gg] = valid ? __high2float(szh[gg]) : 0.f;
        msc = fmaxf(msc, vsc[gg]);
      }
      const float krn = kappa * rn;
      float lg[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int am = (int)dm[4 * g] + 128 * (int)dm[4 * g + 1];
        const int bm = (int)dm[4 * g + 2] + 128 * (int)dm[4 * g + 3];
        const int as = (int)dq[4 * g] + 128 * (int)dq[4 * g + 1];
        const int bs = (int)dq[4 * g + 2] + 128 * (int)dq[4 * g + 3];
        const float mse = fmaf(Q.coef_m[g][1], (float)bm, fmaf(Q.coef_m[g][0], (float)am, Q.cm[g]));
        const float qjl =
            fmaf(Q.coef_s[g][1], (float)bs, fmaf(Q.coef_s[g][0], (float)as, -Q.csum[g]));
        const float score = nk * fmaf(krn, qjl, mse);
        lg[g] = valid ? score * scale2 : -INFINITY;
      }
      // tile maxima (logits per head, value scale) over the 128 tokens
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const uint32_t u = __reduce_max_sync(0xffffffffu, float_to_ordered(lg[g]));
        if (lane == 0) S.red[pb][q4][g] = u;
      }
      {
        const uint32_t u = __reduce_max_sync(0xffffffffu, __float_as_uint(msc));
        if (lane == 0) S.red[pb][q4][G] = u;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.red_bar[pb]);
      if (!wait_bar(&S.red_bar[pb], (jt >> 1) & 1, &S.abort_flag, status)) break;
      float alpha[G];
      bool changed = false;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        uint32_t u = S.red[pb][0][g];
#pragma unroll
        for (int wq = 1; wq < 4; ++wq) u = max(u, S.red[pb][wq][g]);
        const float mnew = fmaxf(mrun[g], ordered_to_float(u));
        alpha[g] = exp2f(mrun[g] - mnew);
        changed |= (mnew != mrun[g]);
        mrun[g] = mnew;
      }
      uint32_t us = S.red[pb][0][G];
#pragma unroll
      for (int wq = 1; wq < 4; ++wq) us = max(us, S.red[pb][wq][G]);
      const float mscale = __uint_as_float(us);
      if (changed) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          lsum[g] *= alpha[g];
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) zs[g][gg] *= alpha[g];
        }
      }
      // p * scale <= mscale < 2^(e+1); fixed point with values < 2^21
      const int F = mscale > 0.f ? 20 - ilog2f(mscale) : 0;
      const float fscale = mscale > 0.f ? exp2i(F) : 0.f;
      uint32_t X[G][4];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float p = valid ? exp2f(lg[g] - mrun[g]) : 0.f;
        lsum[g] += p;
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
          zs[g][gg] = fmaf(p, vze[gg], zs[g][gg]);
          X[g][gg] = __float_as_uint(fmaf(p * vsc[gg], fscale, 12582912.f)) & 0x3FFFFFu;
        }
      }
      // P' operand of tile j: wait until the PV of tile j-2 has been read
      if (jt >= 2 && !wait_bar(&S.pv_free[pb], ((jt - 2) >> 1) & 1, &S.abort_flag, status)) break;
      uint8_t *bp = S.bp[pb];
#pragma unroll
      for (int p = 0; p < C::VOPS; ++p) {
        // n = group * 4G + head * 4 + byte: one u32 per (group, head); the
        // operand of bit-plane p carries the plane weight 2^p
        uint32_t wv[4 * G];
#pragma unroll
        for (int gg = 0; gg < 4; ++gg)
#pragma unroll
          for (int g = 0; g < G; ++g) wv[gg * G + g] = C::PACKED_V ? X[g][gg] : (X[g][gg] << p);
        uint8_t *row = bp + p * 2048 + (t >> 3) * 128 + (t & 7) * 16;
#pragma unroll
        for (int c = 0; c < G; ++c)
          *reinterpret_cast<uint4 *>(row + c * C::SBO_V) =
              make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
      }
      if (t == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) S.alpha[pb][g] = alpha[g];
        S.pscale[pb] = mscale > 0.f ? exp2i(-F) : 0.f;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.p_ready[pb]);
    }
    // reduce l and the zero-point sums over the 128 tokens
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float l = warp_sum(lsum[g]);
      if (lane == 0) S.lsum[q4][g] = l;
#pragma unroll
      for (int gg = 0; gg < 4; ++gg) {
        const float z = warp_sum(zs[g][gg]);
        if (lane == 0) S.zsum[q4][g][gg] = z;
      }
    }
    named_bar_sync(3, 256);  // publish to the value group
    if (t == 0) {
      // m (log2 units, as the SIMT path) and l of the split
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float l = 0.f;
#pragma unroll
        for (int wq = 0; wq < 4; ++wq) l += S.lsum[wq][g];
        part_row(g)[kD] = mrun[g];
        part_row(g)[kD + 1] = l;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
    tmem_relinquish();
  }
}


// ---------------------------------------------------------------------------
// Query blocks: for every (sequence, KV head) the score MMA's B operand
// (B_q in its shared-memory byte layout) and the score constants, built once
// per decode call.  A persistent CTA keeps Pi and S in shared memory (rows
// padded to 129 floats) and rotates the G query heads of each unit:
// q~ = Pi q, s^ = S q (fp32), then writes
//   B_q[kappa][head * 4 + limb] = limb of round(w_p q~_j 2^(F - k)) or of
//   round(2 s^_j 2^(F - k)), kappa <-> (plane p, word wd, mask k, byte i),
//   j = 32 wd + 8 i + k, four signed base-128 limbs,
// with F per head chosen so every operand stays below 2^26.
// ---------------------------------------------------------------------------
template <int MB, int VB, int G>
__global__ void __launch_bounds__(256, 1) qblock_kernel(const __grid_constant__ DecodeArgs a) {
  using C = Cfg<MB, VB, G>;
  constexpr int kPadQ = kD + 1;
  extern __shared__ __align__(16) float qsm[];
  float *mat = qsm;                         // [256][129]: rows of Pi then S
  float *qv = mat + 2 * kD * kPadQ;         // [G][128]
  float *rot = qv + G * kD;                 // [G][2][128]
  float *red = rot + G * 2 * kD;            // [8 warps][G][4]
  uint8_t *blk = reinterpret_cast<uint8_t *>(red + 8 * G * 4);  // QBLOCK staging
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int i = tid; i < 2 * kD * kD; i += 256) {
    const int r = i / kD, c = i % kD;
    mat[r * kPadQ + c] = (r < kD) ? a.pi[i] : a.s[i - kD * kD];
  }
  float cent[8];
#pragma unroll
  for (int i = 0; i < (1 << MB); ++i) cent[i] = a.centroids[i];
  float w[C::NP];
  if (MB == 1) {
    w[0] = cent[1] - cent[0];
  } else if (MB == 2) {
    w[0] = cent[1] - cent[0];
    w[1] = cent[2] - cent[0];
    w[2] = cent[3] - cent[2] - cent[1] + cent[0];
  } else {
#pragma unroll
    for (int l = 0; l < C::NP; ++l) w[l] = cent[l + 1] - cent[l];
  }
  float wmax = 0.f;
#pragma unroll
  for (int p = 0; p < C::NP; ++p) wmax = fmaxf(wmax, fabsf(w[p]));
  QConst *qc = reinterpret_cast<QConst *>(blk + C::BQ_BYTES);
  __syncthreads();

  const int units = a.batch * a.h_kv;
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int b = u / a.h_kv, h = u % a.h_kv;
    for (int i = tid; i < G * kD; i += 256)
      qv[i] = load_elem(a.q, a.q_dtype, ((size_t)b * a.h_q + (size_t)h * G) * kD + i);
    __syncthreads();
    {  // thread o rotates row o of [Pi; S] against the G queries
      const int o = tid;
      float acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = 0.f;
      for (int i = 0; i < kD; ++i) {
        const float m = mat[o * kPadQ + i];
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = fmaf(m, qv[g * kD + i], acc[g]);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) rot[g * 2 * kD + o] = acc[g];
    }
    __syncthreads();
    // per head: sum q~, max |q~|, sum s^, max |s^|
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int j = tid & (kD - 1);
      const float x = rot[g * 2 * kD + (tid < kD ? 0 : kD) + j];
      const float sm = warp_sum(x), mx = warp_max(fabsf(x));
      if (lane == 0) {
        red[(warp * G + g) * 4 + (tid < kD ? 0 : 2)] = sm;
        red[(warp * G + g) * 4 + (tid < kD ? 1 : 3)] = mx;
      }
    }
    __syncthreads();
    int fm[G], fs[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float sq = 0.f, mq = 0.f, ss = 0.f, ms = 0.f;
      for (int wq = 0; wq < 4; ++wq) {        // warps 0-3 hold q~, 4-7 hold s^
        sq += red[(wq * G + g) * 4 + 0];
        mq = fmaxf(mq, red[(wq * G + g) * 4 + 1]);
        ss += red[((wq + 4) * G + g) * 4 + 2];
        ms = fmaxf(ms, red[((wq + 4) * G + g) * 4 + 3]);
      }
      const float bm = wmax * mq, bs = 2.f * ms;
      fm[g] = bm > 0.f ? 25 - ilogbf(bm) : 0;
      fs[g] = bs > 0.f ? 25 - ilogbf(bs) : 0;
      if (tid == 0) {
        qc->cm[g] = cent[0] * sq;
        qc->csum[g] = ss;
        // limbs combine as (D0 + 128 D1) 2^-F + (D2 + 128 D3) 2^(14-F)
        qc->coef_m[g][0] = ldexpf(1.f, -fm[g]);
        qc->coef_m[g][1] = ldexpf(1.f, 14 - fm[g]);
        qc->coef_s[g][0] = ldexpf(1.f, -fs[g]);
        qc->coef_s[g][1] = ldexpf(1.f, 14 - fs[g]);
      }
    }
    if (tid == 0) qc->skip_product_plane = (MB == 2 && w[2] == 0.f) ? 1 : 0;
    for (int kappa = tid; kappa < (C::NP + 1) * 128; kappa += 256) {
      const int p = kappa >> 7, rem = kappa & 127;
      const int col = rem >> 2, bi = rem & 3;
      const int wd = col >> 3, k = col & 7;
      const int coord = 32 * wd + 8 * bi + k;
      uint8_t *dst0 = blk + (kappa >> 4) * C::LBO_Q + (kappa & 15);
      for (int n = 4 * G; n < C::NS; ++n) dst0[(n >> 3) * 128 + (n & 7) * 16] = 0;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float x;
        int F;
        if (p < C::NP) {
          x = w[p] * rot[g * 2 * kD + coord];
          F = fm[g];
        } else {
          x = 2.f * rot[g * 2 * kD + kD + coord];
          F = fs[g];
        }
        int X = __float2int_rn(ldexpf(x, F - k));
#pragma unroll
        for (int l = 0; l < 4; ++l) {
          const int dgt = (l < 3) ? (((X + 64) & 127) - 64) : X;
          X = (X - dgt) >> 7;
          const int n = g * 4 + l;
          dst0[(n >> 3) * 128 + (n & 7) * 16] = (uint8_t)(int8_t)dgt;
        }
      }
    }
    __syncthreads();
    uint4 *dst = reinterpret_cast<uint4 *>(a.qblocks + (size_t)u * C::QBLOCK);
    const uint4 *src = reinterpret_cast<const uint4 *>(blk);
    for (int i = tid; i < C::QBLOCK / 16; i += 256) dst[i] = src[i];
    __syncthreads();
  }
}

template <int MB, int VB, int G>
size_t qblock_smem_bytes() {
  using C = Cfg<MB, VB, G>;
  return sizeof(float) * (2 * kD * (kD + 1) + G * kD + G * 2 * kD + 8 * G * 4) + C::QBLOCK;
}

template <int MB, int VB, int G>
cudaError_t launch_tc(const DecodeArgs &a, cudaStream_t stream) {
  using C = Cfg<MB, VB, G>;
  const size_t smem = sizeof(TcSmem<C>);
  static_assert(sizeof(TcSmem<C>) <= 227 * 1024, "shared memory per CTA");
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<MB, VB, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const size_t qsmem = qblock_smem_bytes<MB, VB, G>();
  e = cudaFuncSetAttribute(qblock_kernel<MB, VB, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)qsmem);
  if (e != cudaSuccess) return e;
  const int units = a.batch * a.h_kv;
  const int qgrid = units < a.num_sms ? units : a.num_sms;
  qblock_kernel<MB, VB, G><<<qgrid, 256, qsmem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 grid(a.nsplit, a.h_kv, a.batch);
  decode_tc_kernel<MB, VB, G><<<grid, kTcThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t decode_tc_qblock_bytes(int key_bits, int G) {
  const int mb = key_bits - 1;
  const int np = mb == 1 ? 1 : (mb == 2 ? 3 : 7);
  const int ns = ((4 * G + 15) / 16) * 16;
  return (size_t)(np + 1) * 128 * ns + kQConstBytes;
}

bool decode_tc_supported(int key_bits, int value_bits, int G) {
  const int mb = key_bits - 1;
  if (value_bits == 2 && (G == 1 || G == 2 || G == 4 || G == 8) && (mb == 1 || mb == 2)) return true;
  if (value_bits == 2 && mb == 3 && G == 4) return true;
  if (value_bits == 3 && mb == 2 && G == 6) return true;
  return false;
}

cudaError_t launch_decode_tc(const DecodeArgs &a, cudaStream_t stream) {
  const int mb = a.key_bits - 1, vb = a.value_bits, G = a.h_q / a.h_kv;
#define TQ_TC(MB_, VB_, G_) \
  if (mb == MB_ && vb == VB_ && G == G_) return launch_tc<MB_, VB_, G_>(a, stream);
  TQ_TC(1, 2, 1) TQ_TC(1, 2, 2) TQ_TC(1, 2, 4) TQ_TC(1, 2, 8)
  TQ_TC(2, 2, 1) TQ_TC(2, 2, 2) TQ_TC(2, 2, 4) TQ_TC(2, 2, 8)
  TQ_TC(3, 2, 4) TQ_TC(2, 3, 6)
#undef TQ_TC
  return cudaErrorNotSupported;
}

}  // namespace tq
