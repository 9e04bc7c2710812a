// Decode attention over the compressed cache on the 5th-generation tensor
// cores (tcgen05), one CTA per (split, KV head, sequence).
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
// allows, so both contractions run on the tensor cores with exact operands.
//
//   Scores (kind::i8, A from tensor memory).  Write the code bits of
//   coordinate j as spins s_k = 2 b_k - 1.  Any codebook of 2^m levels is a
//   multilinear polynomial in the spins (its Walsh expansion),
//   c(idx) = a_0 + sum_S a_S prod_{k in S} s_k, and for the symmetric
//   Lloyd-Max codebooks only the odd subsets S survive (1, 2 and 4 planes at
//   m = 1, 2, 3).  A spin is 2 bit - 1, so each subset plane and the QJL sign
//   plane enter as 0/1 bits (the -1 halves are per-head constants).  One LOP3
//   (w & (0x01010101 << k)) turns a 32-bit plane word into four u8 operands
//   of weight 2^k; the worker groups store them straight into tensor memory, so
//   the score operands never touch shared memory.  The query side B holds
//   2 a_S Pi q / 2^k (and 2 S q / 2^k) in four signed base-128 limbs; the s32
//   accumulation is exact and the limbs are combined per (token, head).
//   Values (kind::i8): D[channel, (group, head, byte)] = A_v[channel, code
//   bytes x tokens] x B_p[tokens, p * scale_g as 22-bit fixed point].  Two-
//   bit codes are stored packed, so one mask (w & (0x03030303 << 2m))
//   yields code * 4^m operands; wider codes are assembled from their bit-
//   planes into one code byte.  The 4^m weight of each row is undone per
//   channel.
// Per 128-token tile the record bytes arrive by one 1-D bulk copy (TMA
// engine) into a ring of shared-memory stages.
// Chunked prefill runs through the same kernel: the query heads of a unit
// are then several query tokens of a chunk, each with its causal limit on
// the tokens it sees (applied per head in the softmax).
//
// Warp roles (608 threads):
//   warp 0        bulk-copy producer; allocates / frees tensor memory
//   warp 1        score MMA issuer, warp 18 P.V MMA issuer (one elected lane
//                 issues); each sleeps in blocking waits on its own queue
//   warps 2-17    four worker groups of four warps (one per TMEM lane
//                 quarter); group g takes tiles g, g + 4, ... through every
//                 SIMT step: plane operands -> tensor memory, value codes ->
//                 A_v (MN-major, shared memory), score epilogue, tile max by
//                 warp redux + an mbarrier exchange inside the group, online
//                 softmax with the group's own running max / sum, the P'
//                 operand, and the P.V read-back into per-channel
//                 accumulators.  The four states are merged at the end like
//                 four splits.  Every SM sub-partition runs one warp of each
//                 group, so the per-tile work is spread evenly.
// Every mbarrier wait between roles is bounded (2 s unless the host set another
// limit) and answers warp-uniformly; on timeout the CTA sets the call's status
// word in the workspace (the combine then writes NaN rows) and the device's
// sticky error word, stops, waits for its own copies and MMAs and frees TMEM.
#include <math.h>

#include "decode_splitk.cuh"
#include "sm100.cuh"
#include "tq_common.cuh"
#include "tq_kernels.h"

namespace tq {

namespace {

using namespace sm100;

// Worker groups of 4 warps; group g takes tiles g, g + kWorkGroups, ...
#ifndef TQ_DECODE_WORKER_GROUPS
#define TQ_DECODE_WORKER_GROUPS 4
#endif
constexpr int kWorkGroups = TQ_DECODE_WORKER_GROUPS;
constexpr int kPvWarp = 2 + 4 * kWorkGroups;      // the P.V MMA issuer, after the worker warps
constexpr int kTcThreads = 32 * (3 + 4 * kWorkGroups);
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTmemCols = 512;
constexpr int kPlaneCols = 32;  // one u8 operand plane: 128 coordinates per row = 32 TMEM columns

// 2^n for n in [-126, 127]
__device__ __forceinline__ float exp2i(int n) { return __uint_as_float((uint32_t)(n + 127) << 23); }
// floor(log2(x)) for a positive normal float
__device__ __forceinline__ int ilog2f(float x) { return (int)((__float_as_uint(x) >> 23) & 0xFF) - 127; }

// score N per accumulator: 4 limbs per query head
__host__ __device__ constexpr int score_n(int G) { return ((4 * G + 15) / 16) * 16; }
// all non-empty code-bit subsets + the sign plane
__host__ __device__ constexpr int max_planes(int MB) { return (1 << MB); }

// Score constants that follow B_q in a query block.
constexpr int kQConstBytes = 256;
struct QConst {
  float cm[8];     // (a_0 - sum of the active a_S) * sum_j q~_j
  float ncsum[8];  // -sum_j s^_j
  float fm[8];     // limb weight 2^-F of the MSE term (the upper limb pair carries 2^14 more)
  float fs[8];     // limb weight of the QJL term
  int n_mse;       // active subset planes (1 .. 2^m - 1)
  int subset[7];   // their code-bit masks
};
static_assert(sizeof(QConst) <= kQConstBytes, "query constants");

__host__ __device__ constexpr size_t qblock_bytes_for(int MB, int G) {
  return (size_t)max_planes(MB) * 128 * score_n(G) + kQConstBytes;
}

template <int MB_, int VB_, int G_>
struct Cfg {
  static constexpr int MB = MB_, VB = VB_, G = G_;
  // MSE planes of a symmetric codebook (the odd code-bit subsets)
  static constexpr int NSYM = MB == 1 ? 1 : (MB == 2 ? 2 : 4);
  static constexpr int NS = score_n(G);                 // score N per accumulator
  // P' bytes per (value group, head): the 22-bit fixed point needs 3; at
  // GQA 8 only 3 are stored, so two A_k buffers still fit in tensor memory
  static constexpr int PB = (G == 8) ? 3 : 4;
  static constexpr int NPV = 4 * G * PB;                // PV N: 4 groups x G heads x PB bytes
  static constexpr int NPL = max_planes(MB);            // operand planes, upper bound
  static constexpr int SYM_COLS = (NSYM + 1) * kPlaneCols;  // A_k of one tile, symmetric codebook
  // tensor memory: A_k planes | D_s (2 buffers x (mse, qjl)) | D_pv (NR buffers).
  // The P.V ring (A_v, B_p, D_pv) gets one slot per worker group when two
  // symmetric A_k buffers still fit (each group then owns its slot), else
  // as many as fit, at least 2.
  static constexpr int NR_FIT = (kTmemCols - 4 * NS - 2 * SYM_COLS) / NPV;
  static constexpr int NR = NR_FIT >= kWorkGroups ? kWorkGroups : (NR_FIT >= 2 ? NR_FIT : 2);
  static constexpr bool OWN_SLOT = NR == kWorkGroups;
  static constexpr int AK_COLS = kTmemCols - 4 * NS - NR * NPV;
  // A_k ring depth for a codebook with npl planes (2 when two buffers fit)
  __host__ __device__ static constexpr int ak_ring(int npl) {
    return AK_COLS / (npl * kPlaneCols) >= 2 ? 2 : 1;
  }
  static constexpr int NAK_SYM = ak_ring(NSYM + 1);
  static constexpr int COL_DS = AK_COLS;
  static constexpr int COL_DPV = COL_DS + 4 * NS;
  static constexpr int LBO_Q = (NS / 8) * 128;          // K-major stride of 16-byte K chunks
  static constexpr int BQ_PLANE = 128 * NS;             // u8/s8 [128 K] x [NS]
  static constexpr int BQ_BYTES = NPL * BQ_PLANE;
  static constexpr int QBLOCK = BQ_BYTES + kQConstBytes;
  static constexpr int REC = (MB + 1 + VB) * 16 + 20;
  static constexpr int TILE_BYTES = 128 * REC;
  static constexpr int OFF_SIGNS = MB * 2048;
  static constexpr int OFF_V = (MB + 1) * 2048;
  static constexpr int OFF_NORMS = (MB + 1 + VB) * 2048;
  static constexpr int OFF_VSZ = OFF_NORMS + 512;
  static constexpr bool PACKED_V = (VB == 2);
  static constexpr int AV_BYTES = 128 * 128;            // [128 channel slots] x [128 tokens]
  static constexpr int BP_BYTES = 128 * NPV;            // [128 tokens] x [NPV]
  static constexpr int SBO_V = 2048;                    // MN-major stride of 16-byte chunks
  static constexpr int MERGE_BYTES = (kWorkGroups - 1) * 128 * G * 4 + kWorkGroups * 4 * G * 4 * 5 + 1024;
  static constexpr int FIXED = NR * AV_BYTES + NR * BP_BYTES + QBLOCK + MERGE_BYTES + 2048;
  static constexpr int STAGES_FIT = (224 * 1024 - FIXED) / TILE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static_assert(NPL * kPlaneCols <= AK_COLS, "tensor memory budget");
  static_assert(STAGES >= 4, "shared memory budget");
  static_assert(TILE_BYTES % 16 == 0, "bulk copy size");
  static_assert(QBLOCK == (int)qblock_bytes_for(MB, G), "query block size");
};

template <class C>
struct TcSmem {
  alignas(128) uint8_t stage[C::STAGES][C::TILE_BYTES];
  alignas(128) uint8_t av[C::NR][C::AV_BYTES];
  alignas(128) uint8_t bp[C::NR][C::BP_BYTES];
  alignas(128) uint8_t bq[C::QBLOCK];  // B_q operand + score constants
  uint64_t full[C::STAGES];
  uint64_t empty[C::STAGES];
  uint64_t ak_ready[2], s_ready[2], s_free[2];
  uint64_t av_ready[C::NR], p_ready[C::NR], pv_done[C::NR], pv_free[C::NR];
  uint64_t red_bar[kWorkGroups];
  uint64_t q_full;
  uint32_t tmem_base;
  volatile int abort_flag;
  alignas(16) float red[kWorkGroups][2][C::G + 1][4];  // [group][slot][head | value scale][warp]
  float fin_m[kWorkGroups][C::G];
  float lsum[kWorkGroups][4][C::G];
  float zsum[kWorkGroups][4][C::G][4];
  float accx[kWorkGroups - 1][128][C::G];  // groups 1.. hand their accumulators to group 0
  float dal[kWorkGroups][4][C::G + 1];     // per warp: alpha of its last tile, fixed-point scale
};

// Bounded pipeline wait of one thread (limit a.wait_ns, 2 s by default) that
// also gives up when another role has aborted; a timeout raises the CTA's
// abort flag, the call's status word and the device's sticky error word.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         const DecodeArgs &a) {
  bool timed_out = false;
  if (pipe_wait(bar, parity, abort_flag, a.wait_ns, a.wait_hint_ns, &timed_out)) return true;
  if (timed_out) {
    atomicOr(a.status, 1);
    if (a.errors) atomicOr(a.errors, (unsigned int)TQ_ERRF_DECODE_WAIT);
  }
  return false;
}

// The wait of a converged worker warp.  Every input of the decision -- the
// barrier phase, the abort flag, the clock -- is read by one warp-wide
// instruction, so the lanes of a converged warp decide alike and leave
// together (no vote needed; a vote per wait measured 3.5% on decode).
__device__ __forceinline__ bool wait_warp(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          const DecodeArgs &a) {
  return wait_bar(bar, parity, abort_flag, a);
}

// The same with an explicit vote, for the MMA issuer warps (off the hot path).
__device__ __forceinline__ bool wait_vote(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          const DecodeArgs &a) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag, a));
}

// Spin word of code-bit subset S over 32 coordinates: bit set <=> the
// product of the spins 2 b_k - 1, k in S, is +1 (an even number of zero bits).
__device__ __forceinline__ uint32_t subset_word(int S, uint32_t b0, uint32_t b1, uint32_t b2) {
  uint32_t x = ((S & 1) ? b0 : 0u) ^ ((S & 2) ? b1 : 0u) ^ ((S & 4) ? b2 : 0u);
  return (__popc(S) & 1) ? x : ~x;
}

// The odd code-bit subsets in increasing order: the planes of a symmetric
// codebook (1 | 1, 2 | 1, 2, 4, 7 at m = 1, 2, 3).
__host__ __device__ constexpr int odd_subset(int p) { return p < 2 ? p + 1 : (p == 2 ? 4 : 7); }

// Eight u8 operand words of one 32-coordinate bit word w: word k, byte i is
// coordinate 8i + k with weight 2^(k mod 4) (bits 4..7 are taken from w >> 4
// so no operand byte exceeds 8).
__device__ __forceinline__ void plane_operands(uint32_t w, uint32_t *o) {
  const uint32_t w4 = w >> 4;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    o[k] = w & (0x01010101u << k);
    o[4 + k] = w4 & (0x01010101u << k);
  }
}

// Score MMAs of one tile with a compile-time plane count: planes 0..NPM-1
// accumulate the MSE term, plane NPM (the signs) the QJL term; four K = 32
// steps per plane.
template <int NPM, int LBO_Q, int BQ_PLANE>
__device__ __forceinline__ void issue_scores(bool leader, uint32_t a_base, uint64_t dbq, uint32_t d_mse,
                                             uint32_t d_qjl, uint32_t id_s) {
#pragma unroll
  for (int p = 0; p <= NPM; ++p)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t b_d = dbq + (uint64_t)((p * BQ_PLANE + kk * 2 * LBO_Q) >> 4);
      const uint32_t d = p < NPM ? d_mse : d_qjl;
      const uint32_t acc = (p < NPM) ? ((p | kk) ? 1u : 0u) : (kk ? 1u : 0u);
      if (leader) mma_i8_ts(d, a_base + p * kPlaneCols + 8 * kk, b_d, id_s, acc);
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
  // split-major grid: every unit's first splits are scheduled before any
  // last (ragged, shorter) split, so the short CTAs fill the tail
  // the query blocks, the status words and the work list come from the
  // preceding kernel
  pdl_wait();
  pdl_trigger();
  // this CTA's (split, KV head, sequence): work items largest first, so the
  // short ones fill the tail
  int split, h, b, len;
  {
    const int units = a.batch * a.h_kv;
    const int2 it = a.order ? a.order[blockIdx.x] : make_int2((int)blockIdx.x, -1);
    split = it.x / units;
    const int u = it.x - split * units;
    b = u / a.h_kv;
    h = u - b * a.h_kv;
    len = it.y;
  }
  // A codebook whose operand planes fit in tensor memory only once (the
  // query-block kernel decided it): this split runs the SIMT split-K body
  // on 128 threads instead.
  if (a.status[1] != 0) {
    if (tid < 128) splitk_simt_body<G>(a, split, h, b, tid, smem_raw, 1);
    return;
  }

  if (len < 0) {
    len = a.len[b] - a.len_sub;
    len = len < 0 ? 0 : (len > a.max_len ? a.max_len : len);
  }
  const int tile0 = split * a.tiles_per_split;
  const int t_begin = tile0 * kTile;
  const int t_end = min(len, (split + 1) * a.tiles_per_split * kTile);
  const int ntile = t_end > t_begin ? (t_end - t_begin + kTile - 1) / kTile : 0;
  auto part_row = [&](int g) {
    return a.part + (((size_t)b * a.h_q + (size_t)h * G + g) * a.part_stride + split) * (kD + 2);
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
      mbar_init(&S.empty[s], 4);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&S.ak_ready[i], 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_ready[i], 1);
      mbar_init(&S.s_free[i], 4);
    }
    for (int i = 0; i < kWorkGroups; ++i) mbar_init(&S.red_bar[i], 4);
    for (int i = 0; i < C::NR; ++i) {
      mbar_init(&S.av_ready[i], 4);
      mbar_init(&S.p_ready[i], 4);
      mbar_init(&S.pv_done[i], 1);
      mbar_init(&S.pv_free[i], 4);
    }
    mbar_init(&S.q_full, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&S.tmem_base, kTmemCols);

  const uint8_t *tiles = reinterpret_cast<const uint8_t *>(a.data) +
                         (((size_t)b * a.h_kv + h) * a.ntiles + tile0) * (size_t)C::TILE_BYTES;
  const QConst &Q = *reinterpret_cast<const QConst *>(S.bq + C::BQ_BYTES);

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;

  if (warp == 0) {
    // ---------------- producer --------------------------------------------
    if (lane == 0) {
      mbar_arrive_expect_tx(&S.q_full, C::QBLOCK);
      bulk_g2s(S.bq, a.qblocks + ((size_t)b * a.h_kv + h) * C::QBLOCK, C::QBLOCK, &S.q_full);
      int issued = 0;
      // (a test of the timeout path withholds every tile copy: the workers'
      // bounded waits on them then run out)
      for (int i = 0; i < (a.test_withhold ? 0 : ntile); ++i) {
        const int s = i % C::STAGES;
        if (i >= C::STAGES &&
            !wait_bar(&S.empty[s], ((i / C::STAGES) - 1) & 1, &S.abort_flag, a))
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
  } else if (warp == 1 || warp == kPvWarp) {
    // ---------------- MMA issuers -----------------------------------------
    // Warp 1 issues the score MMAs of tiles 0, 1, ..., warp kPvWarp the P.V
    // MMAs; each sleeps in blocking mbarrier waits for its own queue, so
    // neither spends issue slots of the sub-partitions it shares with the
    // worker groups, and neither waits behind the other.  The whole warp
    // runs the loop (descriptors stay warp-uniform); one elected lane issues.
    const bool leader = elect_one();
    auto wait_all = [&](uint64_t *bar, uint32_t parity) { return wait_vote(bar, parity, &S.abort_flag, a); };
    const bool qok = wait_all(&S.q_full, 0);
    int last = -1;  // last tile whose MMAs were committed
    if (warp == 1) {
      const uint32_t id_s = idesc_i8(128, C::NS, false, true, false, false);
      const int nm = qok ? Q.n_mse : 0, npl = nm + 1;
      const int akb = C::ak_ring(npl);
      const uint64_t dbq = smem_desc(S.bq, C::LBO_Q, 128);
      for (int is = 0; qok && is < ntile; ++is) {
        const int ab = akb == 2 ? (is & 1) : 0;
        // one hand-over barrier per tile parity, also with a single A_k
        // buffer (one barrier completing every tile stalled at GQA 8)
        if (!wait_all(&S.ak_ready[is & 1], (is >> 1) & 1)) break;
        if (is >= 2 && !wait_all(&S.s_free[is & 1], ((is - 2) >> 1) & 1)) break;
        tc_fence_after();
        const uint32_t d_mse = tbase + C::COL_DS + (is & 1) * 2 * C::NS;
        const uint32_t d_qjl = d_mse + C::NS;
        if (nm == C::NSYM) {
          // symmetric codebook: plane count and buffer offsets are
          // compile-time, so the descriptors stay in uniform registers
          issue_scores<C::NSYM, C::LBO_Q, C::BQ_PLANE>(
              leader, tbase + (C::NAK_SYM == 2 ? (is & 1) : 0) * (C::NSYM + 1) * kPlaneCols, dbq, d_mse,
              d_qjl, id_s);
        } else {
          const uint32_t a_base = tbase + ab * npl * kPlaneCols;
          for (int p = 0; p < npl; ++p) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t b_d = dbq + (uint64_t)((p * C::BQ_PLANE + kk * 2 * C::LBO_Q) >> 4);
              const uint32_t acc = (p < nm) ? ((p | kk) ? 1u : 0u) : (kk ? 1u : 0u);
              if (leader) mma_i8_ts(p < nm ? d_mse : d_qjl, a_base + p * kPlaneCols + 8 * kk, b_d, id_s, acc);
            }
          }
        }
        if (leader) mma_commit(&S.s_ready[is & 1]);
        __syncwarp();
        last = is;
      }
      // never leave with an MMA in flight
      if (last >= 0) mbar_wait(&S.s_ready[last & 1], (last >> 1) & 1);
    } else {
      const uint32_t id_p = idesc_i8(128, C::NPV, false, false, true, true);
      const uint64_t dav0 = smem_desc(S.av[0], 128, C::SBO_V), dbp0 = smem_desc(S.bp[0], 128, C::SBO_V);
      for (int ip = 0; qok && ip < ntile; ++ip) {
        const int pb = ip % C::NR;
        const uint32_t rph = (ip / C::NR) & 1;
        if (!wait_all(&S.p_ready[pb], rph)) break;
        if (!wait_all(&S.av_ready[pb], rph)) break;
        if (ip >= C::NR && !wait_all(&S.pv_free[pb], rph ^ 1)) break;
        tc_fence_after();
        const uint32_t d_pv = tbase + C::COL_DPV + pb * C::NPV;
        const uint64_t da = dav0 + (uint64_t)((pb * C::AV_BYTES) >> 4);
        const uint64_t db = dbp0 + (uint64_t)((pb * C::BP_BYTES) >> 4);
#pragma unroll
        for (int ins = 0; ins < 4; ++ins)
          if (leader) mma_i8_ss(d_pv, da + (uint64_t)(32 * ins), db + (uint64_t)(32 * ins), id_p, ins ? 1u : 0u);
        if (leader) mma_commit(&S.pv_done[pb]);
        __syncwarp();
        last = ip;
      }
      if (last >= 0) mbar_wait(&S.pv_done[last % C::NR], (last / C::NR) & 1);
    }
  } else {
    // ---------------- worker groups ----------------------------------------
    // Group grp (warps 2 + 4 grp .. 5 + 4 grp, one per TMEM lane quarter)
    // takes tiles grp, grp + 4, ... through every SIMT step: plane operands
    // to tensor memory, value operand, score epilogue, online softmax with
    // its own running max / sum, P' operand and the P.V read-back.  The four
    // groups' states are merged at the end like four splits.
    const int grp = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int t = 32 * q4 + lane;  // token slot (score, operands) == TMEM lane == M slot of P.V
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    // value channel of this M slot and the 4^m weight its operand bytes carry
    const int kk = C::PACKED_V ? 2 * ((t >> 2) & 3) : 0;
    const int chan = C::PACKED_V ? 16 * (t >> 4) + 4 * (t & 3) + ((t >> 2) & 3)
                                 : 32 * (t >> 5) + 8 * (t & 3) + 4 * ((t >> 4) & 1) + ((t >> 2) & 3);
    const float kappa = qjl_kappa();
    const float scale2 = a.softmax_scale * kLog2e;
    const bool qok = wait_warp(&S.q_full, 0, &S.abort_flag, a);
    const int nm = qok ? Q.n_mse : 0, npl = nm + 1;
    const int akb = C::ak_ring(npl);
    // symmetric codebook: the planes are the odd subsets, known at compile
    // time, so the spin words need no selects
    bool sym = nm == C::NSYM;
#pragma unroll
    for (int p = 0; p < C::NSYM; ++p) sym = sym && Q.subset[p] == odd_subset(p);

    const int qt1 = a.qt - 1, gshift = 31 - __clz(G / a.qt);
    // The running maxima start at -1e30, below any logit, not at -inf: a head
    // whose tiles so far masked every token (causal prefill rows) then keeps
    // the factor exp2(0) = 1 instead of exp2(-inf + inf) = NaN, with no
    // select in the loop, and its -1e30 drops out of every merge below
    // (exp2(-1e30 - m) = 0, or an all-empty state stays 0 / 0 -> 0).
    // zs: per head the zero-point sums of the four value groups, as pairs
    // (updated two groups per paired f32 instruction)
    float mrun[G], lsum[G], acc[G];
    float2 zs[G][2];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mrun[g] = -1e30f;
      lsum[g] = 0.f;
      acc[g] = 0.f;
#pragma unroll
      for (int gh = 0; gh < 2; ++gh) zs[g][gh] = make_float2(0.f, 0.f);
    }
    // P.V read-back of tile jt in slot rb: acc = acc * alpha + D * sc, with
    // alpha[0..G-1] and sc = alpha[G] as this warp left them in shared memory
    float *dal = S.dal[grp][q4];
    auto readback = [&](int jt, int rb) -> bool {
      if (!wait_warp(&S.pv_done[rb], (jt / C::NR) & 1, &S.abort_flag, a)) return false;
      tc_fence_after();
      constexpr int PB = C::PB;
      uint32_t d[PB * G];
      tmem_ld_cols<PB * G>(tbase + lane_off + C::COL_DPV + rb * C::NPV + q4 * PB * G, d);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.pv_free[rb]);
      const float sc = dal[G] * exp2i(-kk);  // this M slot carries code * 4^m
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float v = fmaf(65536.f, (float)d[PB * g + 2], fmaf(256.f, (float)d[PB * g + 1], (float)d[PB * g]));
        if constexpr (PB == 4) v = fmaf(16777216.f, (float)d[PB * g + 3], v);
        acc[g] = fmaf(acc[g], dal[g], v * sc);
      }
      return true;
    };
    // with its own P.V slot a group reads tile jt's result back at its next
    // tile (jt + 4), when the MMA has long finished
    int prev = -1;

    constexpr int NVW = C::PACKED_V ? 8 : 4 * VB;
    bool ok = qok;
    for (int i = grp; ok && i < ntile; i += kWorkGroups) {
      const int n = i / kWorkGroups, s = i % C::STAGES, rb = i % C::NR;
      ok = false;
      // 1. code / sign plane words of the tile
      if (!wait_warp(&S.full[s], (i / C::STAGES) & 1, &S.abort_flag, a)) break;
      const uint8_t *st = S.stage[s];
      uint32_t bw[3][4], sw[4];
      {
#pragma unroll
        for (int p = 0; p < 3; ++p) {
          if (p < MB) {
            const uint4 v = *reinterpret_cast<const uint4 *>(st + p * kPlaneBytes + t * kRowBytes);
            bw[p][0] = v.x; bw[p][1] = v.y; bw[p][2] = v.z; bw[p][3] = v.w;
          } else {
            bw[p][0] = bw[p][1] = bw[p][2] = bw[p][3] = 0u;
          }
        }
        const uint4 sv = *reinterpret_cast<const uint4 *>(st + C::OFF_SIGNS + t * kRowBytes);
        sw[0] = sv.x; sw[1] = sv.y; sw[2] = sv.z; sw[3] = sv.w;
      }

      // 2. plane operands -> A_k buffer of tile i, free once the score MMA
      //    of tile i - akb has finished
      if (i >= akb) {
        const int pt = i - akb;
        if (!wait_warp(&S.s_ready[pt & 1], (pt >> 1) & 1, &S.abort_flag, a)) break;
        // the stores below must follow the MMA's reads of the buffer
        tc_fence_after();
      }
      const int ab = akb == 2 ? (i & 1) : 0;
      {
        const uint32_t a_base = tbase + lane_off + ab * npl * kPlaneCols;
        if (sym) {
#pragma unroll
          for (int p = 0; p <= C::NSYM; ++p) {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              uint32_t r[16];
#pragma unroll
              for (int wd = 0; wd < 2; ++wd)
                plane_operands(p < C::NSYM ? subset_word(odd_subset(p), bw[0][2 * h2 + wd], bw[1][2 * h2 + wd],
                                                         bw[2][2 * h2 + wd])
                                           : sw[2 * h2 + wd],
                               r + 8 * wd);
              tmem_st16(a_base + p * kPlaneCols + 16 * h2, r);
            }
          }
        } else {
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            if (p > nm) break;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              uint32_t r[16];
#pragma unroll
              for (int wd = 0; wd < 2; ++wd)
                plane_operands((p < nm) ? subset_word(Q.subset[p < 7 ? p : 6], bw[0][2 * h2 + wd], bw[1][2 * h2 + wd],
                                                      bw[2][2 * h2 + wd])
                                        : sw[2 * h2 + wd],
                               r + 8 * wd);
              tmem_st16(a_base + p * kPlaneCols + 16 * h2, r);
            }
          }
        }
      }

      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.ak_ready[i & 1]);

      // 3. the P.V slot: its last tile's operands must have been consumed
      //    (after the planes are handed over, so the score MMA starts first)
      if constexpr (C::OWN_SLOT) {
        if (prev >= 0 && !readback(prev, rb)) break;
      } else {
        if (i >= C::NR && !wait_warp(&S.pv_done[rb], ((i - C::NR) / C::NR) & 1, &S.abort_flag, a)) break;
      }

      // 4. value codes, norms and value scales; the stage is then released
      uint32_t vw[NVW];
      uint32_t nrw;
      uint4 szr;
      {
        if constexpr (C::PACKED_V) {
          const uint4 v0 = *reinterpret_cast<const uint4 *>(st + C::OFF_V + t * kPackedRowBytes);
          const uint4 v1 = *reinterpret_cast<const uint4 *>(st + C::OFF_V + t * kPackedRowBytes + 16);
          vw[0] = v0.x; vw[1] = v0.y; vw[2] = v0.z; vw[3] = v0.w;
          vw[4] = v1.x; vw[5] = v1.y; vw[6] = v1.z; vw[7] = v1.w;
        } else {
#pragma unroll
          for (int p = 0; p < VB; ++p) {
            const uint4 v = *reinterpret_cast<const uint4 *>(st + C::OFF_V + p * kPlaneBytes + t * kRowBytes);
            vw[4 * p] = v.x; vw[4 * p + 1] = v.y; vw[4 * p + 2] = v.z; vw[4 * p + 3] = v.w;
          }
        }
        nrw = *reinterpret_cast<const uint32_t *>(st + C::OFF_NORMS + t * 4);
        szr = *reinterpret_cast<const uint4 *>(st + C::OFF_VSZ + t * 16);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[s]);
      // value codes -> A_v (MN-major, shared memory)
      {
        uint8_t *row = S.av[rb] + (t >> 3) * 128 + (t & 7) * 16;
        if constexpr (C::PACKED_V) {
          // packed row: word w holds channels 16w .. 16w+15; mask m keeps
          // channel 16w + 4i + m in byte i as code * 4^m (M slot 16w + 4m + i)
#pragma unroll
          for (int w = 0; w < 8; ++w)
            *reinterpret_cast<uint4 *>(row + w * C::SBO_V) =
                make_uint4(vw[w] & 0x03030303u, vw[w] & 0x0C0C0C0Cu, vw[w] & 0x30303030u,
                           vw[w] & 0xC0C0C0C0u);
        } else {
          // bit-planes: u32 x of chunk m16 holds, in byte i, the code of
          // channel 32 (m16 / 2) + 8 i + 4 (m16 % 2) + x (M slot 16 m16 + 4 x + i)
#pragma unroll
          for (int m16 = 0; m16 < 8; ++m16) {
            uint32_t o[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const int k = 4 * (m16 & 1) + x;
              uint32_t c = 0;
#pragma unroll
              for (int p = 0; p < VB; ++p) c |= ((vw[4 * p + (m16 >> 1)] >> k) & 0x01010101u) << p;
              o[x] = c;
            }
            *reinterpret_cast<uint4 *>(row + m16 * C::SBO_V) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.av_ready[rb]);

      // 5. score epilogue; limbs combine as (D0 + 128 D1) 2^-F + (D2 + 128 D3) 2^(14-F)
      if (!wait_warp(&S.s_ready[i & 1], (i >> 1) & 1, &S.abort_flag, a)) break;
      tc_fence_after();
      float mse[G], qjl[G];
      {
        const uint32_t base = tbase + lane_off + C::COL_DS + (i & 1) * 2 * C::NS;
        if constexpr (4 * G == C::NS && G <= 4) {
          // the MSE and QJL accumulators are adjacent: one load for both
          uint32_t d[8 * G];
          tmem_ld_cols<8 * G>(base, d);
          tmem_wait_ld();
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const int am = (int)d[4 * g] + 128 * (int)d[4 * g + 1];
            const int bm = (int)d[4 * g + 2] + 128 * (int)d[4 * g + 3];
            const float fm = Q.fm[g];
            mse[g] = fmaf(fm * 16384.f, (float)bm, fmaf(fm, (float)am, Q.cm[g]));
            const int as = (int)d[4 * G + 4 * g] + 128 * (int)d[4 * G + 4 * g + 1];
            const int bs = (int)d[4 * G + 4 * g + 2] + 128 * (int)d[4 * G + 4 * g + 3];
            const float fs = Q.fs[g];
            qjl[g] = fmaf(fs * 16384.f, (float)bs, fmaf(fs, (float)as, Q.ncsum[g]));
          }
        } else {
          uint32_t d[4 * G];
          tmem_ld_cols<4 * G>(base, d);
          tmem_wait_ld();
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const int am = (int)d[4 * g] + 128 * (int)d[4 * g + 1];
            const int bm = (int)d[4 * g + 2] + 128 * (int)d[4 * g + 3];
            const float fm = Q.fm[g];
            mse[g] = fmaf(fm * 16384.f, (float)bm, fmaf(fm, (float)am, Q.cm[g]));
          }
          tmem_ld_cols<4 * G>(base + C::NS, d);
          tmem_wait_ld();
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const int as = (int)d[4 * g] + 128 * (int)d[4 * g + 1];
            const int bs = (int)d[4 * g + 2] + 128 * (int)d[4 * g + 3];
            const float fs = Q.fs[g];
            qjl[g] = fmaf(fs * 16384.f, (float)bs, fmaf(fs, (float)as, Q.ncsum[g]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.s_free[i & 1]);

      // 6. logits, tile maxima over the group's 128 tokens, online softmax
      const int tpos = t_begin + i * kTile + t;
      const bool valid = tpos < t_end;
      const __half2 nr = *reinterpret_cast<const __half2 *>(&nrw);
      const float nk = __low2float(nr), rn = __high2float(nr);
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
        const float score = nk * fmaf(krn, qjl[g], mse[g]);
        // prefill: query token g >> gshift of the chunk sees len - (qt - 1 - that) tokens
        lg[g] = (valid && tpos + qt1 - (g >> gshift) < len) ? score * scale2 : -INFINITY;
      }
      float(&red)[G + 1][4] = S.red[grp][n & 1];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float u = redux_max_f32(lg[g]);
        if (lane == 0) red[g][q4] = u;
      }
      {
        const float u = redux_max_f32(msc);
        if (lane == 0) red[G][q4] = u;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.red_bar[grp]);
      if (!wait_warp(&S.red_bar[grp], n & 1, &S.abort_flag, a)) break;
      float alpha[G];
      bool changed = false;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float4 r4 = *reinterpret_cast<const float4 *>(red[g]);
        const float mnew = max3f(max3f(mrun[g], r4.x, r4.y), r4.z, r4.w);
        alpha[g] = ex2_approx(mrun[g] - mnew);
        changed |= (mnew != mrun[g]);
        mrun[g] = mnew;
      }
      const float4 rs = *reinterpret_cast<const float4 *>(red[G]);
      const float mscale = max3f(max3f(rs.x, rs.y, rs.z), rs.w, 0.f);
      if (changed) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          lsum[g] *= alpha[g];
#pragma unroll
          for (int gh = 0; gh < 2; ++gh) zs[g][gh] = __fmul2_rn(zs[g][gh], make_float2(alpha[g], alpha[g]));
        }
      }
      // p * scale <= mscale < 2^(e+1); fixed point with values < 2^21
      const int F = mscale > 0.f ? 20 - ilog2f(mscale) : 0;
      const float fscale = mscale > 0.f ? exp2i(F) : 0.f;
      float vscf[4];
#pragma unroll
      for (int gg = 0; gg < 4; ++gg) vscf[gg] = vsc[gg] * fscale;  // exact: power-of-two scale
      float p[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        p[g] = ex2_approx(lg[g] - mrun[g]);  // a masked token: 2^-inf = 0
        lsum[g] += p[g];
#pragma unroll
        for (int gh = 0; gh < 2; ++gh)
          zs[g][gh] = __ffma2_rn(make_float2(p[g], p[g]), make_float2(vze[2 * gh], vze[2 * gh + 1]), zs[g][gh]);
      }

      // 7. P' operand: column n = (group * G + head) * PB + byte, the PB
      //    low bytes of p * scale * 2^F as 22-bit fixed point
      {
        uint8_t *row = S.bp[rb] + (t >> 3) * 128 + (t & 7) * 16;
        if constexpr (C::PB == 4) {
#pragma unroll
          for (int c = 0; c < G; ++c) {
            uint32_t w4[4];
#pragma unroll
            for (int x = 0; x < 4; x += 2) {
              const int gg0 = (4 * c + x) / G, g0 = (4 * c + x) % G;
              const int gg1 = (4 * c + x + 1) / G, g1 = (4 * c + x + 1) % G;
              const float2 f = __ffma2_rn(make_float2(p[g0], p[g1]), make_float2(vscf[gg0], vscf[gg1]),
                                          make_float2(12582912.f, 12582912.f));
              w4[x] = __float_as_uint(f.x) & 0x3FFFFFu;
              w4[x + 1] = __float_as_uint(f.y) & 0x3FFFFFu;
            }
            *reinterpret_cast<uint4 *>(row + c * C::SBO_V) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        } else {
          // 3 bytes per value, packed back to back: 4G values -> 3G words
          uint32_t w[3 * G];
#pragma unroll
          for (int k = 0; k < 3 * G; ++k) w[k] = 0u;
#pragma unroll
          for (int j = 0; j < 4 * G; ++j) {
            const int gg = j / G, g = j % G;
            const uint32_t v = __float_as_uint(fmaf(p[g], vscf[gg], 12582912.f)) & 0x3FFFFFu;
            const int pos = 3 * j, wi = pos >> 2, off = pos & 3;
            w[wi] |= v << (8 * off);
            if (off > 1) w[wi + 1] |= v >> (8 * (4 - off));
          }
#pragma unroll
          for (int c = 0; c < 3 * G / 4; ++c)
            *reinterpret_cast<uint4 *>(row + c * C::SBO_V) =
                make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.p_ready[rb]);

      // 8. P.V read-back (now, or at this group's next tile)
      if (lane == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) dal[g] = alpha[g];
        dal[G] = mscale > 0.f ? exp2i(-F) : 0.f;
      }
      __syncwarp();
      if constexpr (C::OWN_SLOT) {
        prev = i;
      } else {
        if (!readback(i, rb)) break;
      }
      ok = true;
    }
    if constexpr (C::OWN_SLOT) {
      if (ok && prev >= 0) ok = readback(prev, prev % C::NR);
    }

    // merge the four groups' states; unnormalised partial output
    // sum_t p_t (code * scale + zero) of the split
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float l = warp_sum(lsum[g]);
      if (lane == 0) S.lsum[grp][q4][g] = l;
#pragma unroll
      for (int gg = 0; gg < 4; ++gg) {
        const float z = warp_sum((gg & 1) ? zs[g][gg >> 1].y : zs[g][gg >> 1].x);
        if (lane == 0) S.zsum[grp][q4][g][gg] = z;
      }
      if (t == 0) S.fin_m[grp][g] = mrun[g];
      if (grp > 0) S.accx[grp - 1][t][g] = acc[g];
    }
    named_bar_sync(1, 32 * 4 * kWorkGroups);
    if (grp == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float mm = -INFINITY;
#pragma unroll
        for (int k = 0; k < kWorkGroups; ++k) mm = fmaxf(mm, S.fin_m[k][g]);
        float o = 0.f, lt = 0.f;
#pragma unroll
        for (int k = 0; k < kWorkGroups; ++k) {
          const float mk = S.fin_m[k][g];
          const float f = (mk == -INFINITY) ? 0.f : exp2f(mk - mm);
          float z = 0.f, l = 0.f;
#pragma unroll
          for (int wq = 0; wq < 4; ++wq) {
            z += S.zsum[k][wq][g][q4];
            l += S.lsum[k][wq][g];
          }
          const float ak = k == 0 ? acc[g] : S.accx[k - 1][t][g];
          o = fmaf(ak + z, f, o);
          lt = fmaf(l, f, lt);
        }
        float *pr = part_row(g);
        pr[chan] = o;
        if (t == 0) {
          // m (log2 units, as the SIMT path) and l of the split
          pr[kD] = mm;
          pr[kD + 1] = lt;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
    tmem_relinquish();
  }
}


// ---------------------------------------------------------------------------
// Query blocks: for every (sequence, KV head) the score MMA's B operand
// (s8, in its shared-memory byte layout) and the score constants, built once
// per decode call.  A CTA copies Pi and S into shared memory (16-byte
// asynchronous copies, all in flight at once) and rotates the G query heads
// of each of its units, q~ = Pi q, s^ = S q (fp32): warp w takes rows
// 32 w .. 32 w + 31 of [Pi; S], reads each row once against all G queries
// and reduces the lanes' partial sums by recursive halving, so lane l ends
// with row 32 w + l.  Plane P < n_mse holds 2 a_S q~ for the P-th
// active code-bit subset S (Walsh coefficient a_S of the codebook), the last
// plane holds 2 s^.  K byte kappa of a plane is operand byte i of TMEM column
// c = kappa / 4, i.e. coordinate j = 32 (c / 8) + 8 i + (c % 8) with weight
// 2^((c % 8) mod 4), so it holds X = round(x_j 2^(F - weight exponent)) as
// four signed base-128 limbs; F per head keeps |X| < 2^26.
// ---------------------------------------------------------------------------
// The decode kernel's work list: items i = split * B * H_kv + b * H_kv + h
// ordered by their tile count, largest first, equal counts in item order, so
// the block scheduler hands the longest splits out first and the short ones
// fill the tail, and equal splits keep the split-major order.  A stable
// counting sort by one CTA of 256 threads: every item's count computed once
// (in parallel, into shared memory), a histogram over kOrderBins counts and
// its scan, then one warp places the items in item order.  Lists longer than
// kSortMax keep the item order.
constexpr int kOrderBins = 1024;
constexpr int kSortMax = 4096;
__device__ __forceinline__ void build_work_list(const DecodeArgs &a, int tid) {
  __shared__ int bins[kOrderBins];
  __shared__ unsigned short keys[kSortMax];
  __shared__ int lens[kSortMax];
  const int units = a.batch * a.h_kv, n = units * a.nsplit;
  auto clamped_len = [&](int i) {
    const int b = (i % units) / a.h_kv;
    const int len = a.len[b] - a.len_sub;
    return len < 0 ? 0 : (len > a.max_len ? a.max_len : len);
  };
  if (n > kSortMax) {
    for (int i = tid; i < n; i += 256) a.order[i] = make_int2(i, clamped_len(i));
    return;
  }
  for (int i = tid; i < kOrderBins; i += 256) bins[i] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += 256) {
    const int split = i / units;
    const int len = clamped_len(i);
    lens[i] = len;
    const int t_begin = split * a.tiles_per_split * kTile;
    const int t_end = min(len, (split + 1) * a.tiles_per_split * kTile);
    const int nt = t_end > t_begin ? (t_end - t_begin + kTile - 1) / kTile : 0;
    const int k = kOrderBins - 1 - min(nt, kOrderBins - 1);  // bin 0: the largest
    keys[i] = (unsigned short)k;
    atomicAdd(&bins[k], 1);
  }
  __syncthreads();
  if (tid < 32) {  // exclusive scan: lane l takes bins 32 l .. 32 l + 31
    int sum = 0;
    for (int j = 0; j < 32; ++j) sum += bins[32 * tid + j];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (tid >= o) incl += v;
    }
    int off = incl - sum;
    for (int j = 0; j < 32; ++j) {
      const int c = bins[32 * tid + j];
      bins[32 * tid + j] = off;
      off += c;
    }
    __syncwarp();
    // stable placement: 32 items at a time in item order, equal keys ranked
    // by lane
    for (int i0 = 0; i0 < n; i0 += 32) {
      const int i = i0 + tid;
      const int k = i < n ? (int)keys[i] : -1;  // past the end: a key of its own
      const unsigned same = __match_any_sync(0xffffffffu, k);
      const int leader = __ffs(same) - 1;
      const int rank = __popc(same & ((1u << tid) - 1u));
      int base = 0;
      if (tid == leader && k >= 0) base = atomicAdd(&bins[k], __popc(same));
      base = __shfl_sync(0xffffffffu, base, leader);
      if (k >= 0) a.order[base + rank] = make_int2(i, lens[i]);
    }
  }
  __syncthreads();
}

template <int MB, int VB, int G>
__global__ void __launch_bounds__(256, 1) qblock_kernel(const __grid_constant__ DecodeArgs a) {
  using C = Cfg<MB, VB, G>;
  constexpr int NC = 1 << MB;
  extern __shared__ __align__(16) float qsm[];
  float *mats = qsm;                        // [2][128][128]: Pi, S
  float *rot = mats + 2 * kD * kD;          // [G][2][128]
  float *red = rot + G * 2 * kD;            // [8 warps][G][2]: sum, max |.|
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // The decode kernel may launch now (it waits for this grid).  This grid
  // itself is launched as a dependent of the call's predecessor (typically
  // the quantize-append of the new token): it reads only the queries and the
  // layer constants, writes only the workspace, and waits for the
  // predecessor before it finishes, so the decode kernel's wait covers both.
  pdl_trigger();

  for (int i = tid; i < kD * kD / 4; i += 256) {
    cp_async16(mats + 4 * i, a.pi + 4 * i);
    cp_async16(mats + kD * kD + 4 * i, a.s + 4 * i);
  }
  // Walsh coefficients of the codebook, idx paired with its complement so
  // that a symmetric codebook gives exact zeros for the even subsets
  float cent[NC];
#pragma unroll
  for (int i = 0; i < NC; ++i) cent[i] = a.centroids[i];
  float wal[NC];
#pragma unroll
  for (int S = 0; S < NC; ++S) {
    float acc = 0.f;
    const bool even = (__popc(S) & 1) == 0;
#pragma unroll
    for (int idx = 0; idx < NC / 2; ++idx) {
      const float pr = (__popc(~idx & S) & 1) ? -1.f : 1.f;  // prod of spins over S
      const float pair = even ? cent[idx] + cent[NC - 1 - idx] : cent[idx] - cent[NC - 1 - idx];
      acc = fmaf(pr, pair, acc);
    }
    wal[S] = acc / (float)NC;
  }
  int nm = 0, subs[7];
  float wts[7];
  float wmax = 0.f, wsum = 0.f;
#pragma unroll
  for (int S = 1; S < NC; ++S) {
    if (wal[S] != 0.f) {
      subs[nm] = S;
      wts[nm] = wal[S];
      ++nm;
      wmax = fmaxf(wmax, fabsf(wal[S]));
      wsum += wal[S];
    }
  }
  if (nm == 0) {  // degenerate codebook: one all-zero plane
    subs[0] = 1;
    wts[0] = 0.f;
    nm = 1;
  }
  // A codebook whose planes fit in tensor memory only once (an asymmetric
  // codebook in a shape with little room) goes to the SIMT split-K body in
  // the decode kernel, which reads the rotated queries written below.  This kernel runs first
  // in every tensor-core call, so it also clears the call's status word.
  const bool fallback = C::ak_ring(nm + 1) < 2;
  if (blockIdx.x == 0 && tid == 0) {
    a.status[0] = 0;
    a.status[1] = fallback ? 1 : 0;
  }
  // (the last CTA has the fewest units)
  if (blockIdx.x == gridDim.x - 1 && a.order) build_work_list(a, tid);
  cp_async_wait_all();
  __syncthreads();

  const int units = a.batch * a.h_kv;
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int b = u / a.h_kv, h = u % a.h_kv;
    {  // warp w: rows 32 w .. 32 w + 31 of [Pi; S] against the G queries
      const float *mrows = mats + (warp < 4 ? 0 : kD * kD) + 32 * (warp & 3) * kD + 4 * lane;
      // heads per pass (register budget): a divisor of G, at most 4
      constexpr int GB = G <= 4 ? G : (G % 4 == 0 ? 4 : (G % 3 == 0 ? 3 : (G % 2 == 0 ? 2 : 1)));
      static_assert(G % GB == 0, "heads per pass must divide G");
#pragma unroll
      for (int g0 = 0; g0 < G; g0 += GB) {
        float qx[GB][4];
#pragma unroll
        for (int gi = 0; gi < GB; ++gi)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            qx[gi][e] = load_elem(a.q, a.q_dtype, qrow_offset(a, b, h * G + g0 + gi) + 4 * lane + e);
        float p[GB][32];
#pragma unroll
        for (int r0 = 0; r0 < 32; r0 += 8) {
          float4 w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = *reinterpret_cast<const float4 *>(mrows + (size_t)(r0 + e) * kD);
#pragma unroll
          for (int e = 0; e < 8; ++e)
#pragma unroll
            for (int gi = 0; gi < GB; ++gi)
              p[gi][r0 + e] = fmaf(w[e].w, qx[gi][3], fmaf(w[e].z, qx[gi][2],
                                   fmaf(w[e].y, qx[gi][1], w[e].x * qx[gi][0])));
        }
        // recursive halving: lane l ends with row 32 w + l
#pragma unroll
        for (int sft = 16; sft >= 1; sft >>= 1) {
          const bool upper = (lane & sft) != 0;
#pragma unroll
          for (int q = 0; q < sft; ++q)
#pragma unroll
            for (int gi = 0; gi < GB; ++gi) {
              const float send = upper ? p[gi][q] : p[gi][q + sft];
              const float keep = upper ? p[gi][q + sft] : p[gi][q];
              p[gi][q] = keep + __shfl_xor_sync(0xffffffffu, send, sft);
            }
        }
        const int o = 32 * warp + lane;  // row of [Pi; S]
#pragma unroll
        for (int gi = 0; gi < GB; ++gi) {
          rot[(g0 + gi) * 2 * kD + o] = p[gi][0];
          if (fallback) a.qrot[((size_t)b * a.h_q + h * G + g0 + gi) * 2 * kD + o] = p[gi][0];
          // per head: this warp's sum and max |.| of q~ (warps 0-3) or s^ (4-7)
          const float sm = warp_sum(p[gi][0]), mx = warp_max(fabsf(p[gi][0]));
          if (lane == 0) {
            red[(warp * G + g0 + gi) * 2 + 0] = sm;
            red[(warp * G + g0 + gi) * 2 + 1] = mx;
          }
        }
      }
    }
    __syncthreads();
    uint8_t *qb = a.qblocks + (size_t)u * C::QBLOCK;
    QConst *qc = reinterpret_cast<QConst *>(qb + C::BQ_BYTES);
    int fm[G], fs[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float sq = 0.f, mq = 0.f, ss = 0.f, ms = 0.f;
      for (int wq = 0; wq < 4; ++wq) {
        sq += red[(wq * G + g) * 2 + 0];
        mq = fmaxf(mq, red[(wq * G + g) * 2 + 1]);
        ss += red[((wq + 4) * G + g) * 2 + 0];
        ms = fmaxf(ms, red[((wq + 4) * G + g) * 2 + 1]);
      }
      const float bm = 2.f * wmax * mq, bs = 2.f * ms;
      fm[g] = bm > 0.f ? 25 - ilogbf(bm) : 0;
      fs[g] = bs > 0.f ? 25 - ilogbf(bs) : 0;
      if (tid == 0) {
        // spins are 2 bit - 1: the -1 halves are constants per head
        qc->cm[g] = (wal[0] - wsum) * sq;
        qc->ncsum[g] = -ss;
        qc->fm[g] = ldexpf(1.f, -fm[g]);
        qc->fs[g] = ldexpf(1.f, -fs[g]);
      }
    }
    if (tid == 0) {
      qc->n_mse = nm;
      for (int p = 0; p < 7; ++p) qc->subset[p] = p < nm ? subs[p] : 0;
    }
    // the B_q bytes, written straight to the unit's query block (columns
    // beyond the 4 G limbs are zero)
    for (int kappa = tid; kappa < (nm + 1) * 128; kappa += 256) {
      const int P = kappa >> 7, rem = kappa & 127;
      const int col = rem >> 2, bi = rem & 3;
      const int wd = col >> 3, k = col & 7, kw = k & 3;
      const int coord = 32 * wd + 8 * bi + k;
      uint8_t *dst0 = qb + P * C::BQ_PLANE + (rem >> 4) * C::LBO_Q + (rem & 15);
#pragma unroll
      for (int n = 4 * G; n < C::NS; ++n) dst0[(n >> 3) * 128 + (n & 7) * 16] = 0;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float x;
        int F;
        if (P < nm) {
          x = 2.f * wts[P] * rot[g * 2 * kD + coord];
          F = fm[g];
        } else {
          x = 2.f * rot[g * 2 * kD + kD + coord];
          F = fs[g];
        }
        int X = __float2int_rn(ldexpf(x, F - kw));
#pragma unroll
        for (int l = 0; l < 4; ++l) {
          const int dgt = (l < 3) ? (((X + 64) & 127) - 64) : X;
          X = (X - dgt) >> 7;
          const int n = g * 4 + l;
          dst0[(n >> 3) * 128 + (n & 7) * 16] = (uint8_t)(int8_t)dgt;
        }
      }
    }
    __syncthreads();  // rot and red are reused by the next unit
  }
  pdl_wait();
}

template <int MB, int VB, int G>
size_t qblock_smem_bytes() {
  using C = Cfg<MB, VB, G>;
  return sizeof(float) * (2 * kD * kD + G * 2 * kD + 8 * G * 2);
}

template <int MB, int VB, int G>
cudaError_t launch_tc(const DecodeArgs &a, cudaStream_t stream) {
  using C = Cfg<MB, VB, G>;
  const size_t smem = sizeof(TcSmem<C>);
  static_assert(sizeof(TcSmem<C>) <= 227 * 1024, "shared memory per CTA");
  static_assert(sizeof(TcSmem<C>) >= (size_t)SplitkSmem<G>::kBytes, "fallback body scratch");
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<MB, VB, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const size_t qsmem = qblock_smem_bytes<MB, VB, G>();
  e = cudaFuncSetAttribute(qblock_kernel<MB, VB, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)qsmem);
  if (e != cudaSuccess) return e;
  const int units = a.batch * a.h_kv;
  const int qgrid = units < a.num_sms ? units : a.num_sms;
  e = launch_pdl(qblock_kernel<MB, VB, G>, dim3(qgrid), dim3(256), qsmem, stream, a);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_tc_kernel<MB, VB, G>, dim3(a.h_kv * a.batch * a.nsplit), dim3(kTcThreads), smem,
                    stream, a);
}

}  // namespace

size_t decode_tc_qblock_bytes(int key_bits, int G) { return qblock_bytes_for(key_bits - 1, G); }

bool decode_tc_supported(int key_bits, int value_bits, int G, int value_mode, int d) {
  // MSE values and head dims other than 128: the SIMT split-K kernel
  if (value_mode != TQ_VALUES_GROUP || d != kD) return false;
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
