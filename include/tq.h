/*
 * tq.h -- C ABI of the TurboQuant-prod compressed KV-cache library for
 * NVIDIA B200 (sm_100a).
 *
 * What the library computes (the pages' statement of the method):
 *
 *  - Keys ("TurboQuant" explainer, troisinh.com, "Ý tưởng cốt lõi";
 *    "turboquant/audit_claims.py", AUDIT 1 and AUDIT 5): each key head
 *    vector k is normalised, u = k / ||k||, rotated by a fixed random
 *    orthogonal Pi, and every rotated coordinate is bucketized against a
 *    (key_bits - 1)-bit Lloyd-Max codebook fitted to N(0, 1/d).  The
 *    residual r = u - Pi^T c (c the centroids of the chosen cells) is kept
 *    as 1-bit QJL signs sign(S r) plus ||r||.  ||k|| and ||r|| are stored
 *    as fp16.
 *  - Values (AUDIT 1: value_bits, value_group_size): asymmetric min/max
 *    quantization per group of 32 channels with fp16 scale and zero.
 *  - Decode ("03. Results & Benchmarks", turboquant_cutile, "Latency
 *    Benchmarks"): one pass over the compressed cache with the query
 *    rotated once (Pi q, S q); each score is the centroid-lookup inner
 *    product scaled by ||k|| plus the unbiased QJL correction
 *    ||k|| * ||r|| * sqrt(pi/2)/d * <S q, 2 sign - 1>; then softmax and the
 *    group-dequantized value accumulation.  Split-K over the sequence with a
 *    separate combine step.
 *
 * Conventions for every call:
 *  - Ownership: the caller owns every buffer and the stream.  The library
 *    allocates no memory and never synchronises (except tq_device_errors);
 *    its state is a cached per-device SM count, the wait limit, one 4-byte
 *    error word and one 8-byte refinement counter per device (plus the
 *    no-allocation entry point's fixed scratch).
 *  - Pointers documented as "device" must be device (or managed) memory of
 *    the current CUDA device; "host" pointers are read before the call
 *    returns.
 *  - Errors: arguments are validated on the host before any launch; a bad
 *    argument returns a status and launches nothing.  A launch failure
 *    returns TQ_ERR_CUDA (from cudaGetLastError).  Kernels never trap; an
 *    asynchronous fault surfaces at the caller's next synchronisation.
 *  - Bounded waits: the pipelined tensor-core kernels hand work between warp
 *    roles through shared-memory barriers, and every such wait gives up after
 *    a time limit (2 s; tq_set_wait_limit_ns).  A kernel that gives up stops,
 *    lets its own copies and tensor-core operations finish, frees its tensor
 *    memory and returns, so the GPU stays usable; it records the failure in
 *    the device's sticky error word (tq_device_errors) and in the call's own
 *    result: decode calls write NaN output rows (and set the workspace status
 *    word, see tq_decode_attention), quantize-append writes NaN norms into
 *    the records it owns, so decode over them returns NaN.
 *  - Calls are asynchronous on `stream` and re-entrant.  Calls that write
 *    the same cache region (or the same workspace) must be ordered by the
 *    caller.
 *  - Head dims d = 64, 128 and 256 with group = 32 are built (the
 *    tensor-core kernels at d = 128, the SIMT kernels at all three); other
 *    values return TQ_ERR_UNSUPPORTED.  TurboQuant-MSE values (tq_value_mode) are encoded
 *    by the SIMT quantize-append kernel and decoded by the SIMT split-K
 *    kernel, accumulated in the rotated space and rotated back once per
 *    head in the combine step.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *tq_stream_t;

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative size, bad alignment */
  TQ_ERR_UNSUPPORTED = 2,      /* d, group, bit width or dtype not built */
  TQ_ERR_CAPACITY = 3,         /* len + n_new > capacity, batch too large */
  TQ_ERR_WORKSPACE = 4,        /* workspace missing or too small */
  TQ_ERR_CUDA = 5,             /* a CUDA runtime call or launch failed */
  TQ_ERR_INTERNAL = 6
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1 } tq_dtype;

/* How values are stored. */
typedef enum {
  TQ_VALUES_GROUP = 0, /* asymmetric min/max quantization per group of 32
                          channels, fp16 scale and zero ("turboquant/
                          audit_claims.py", AUDIT 1: value_bits,
                          value_group_size) */
  TQ_VALUES_MSE = 1    /* TurboQuant-MSE: Lloyd-Max cells of the rotated unit
                          value Pi v / ||v|| plus the fp16 norm ("03. Results &
                          Benchmarks", "At a Glance -> Compression": 3 bits
                          per coordinate for keys and values, 5.02x) */
} tq_value_mode;

/* Bits of the sticky per-device error word (tq_device_errors). */
#define TQ_ERRF_DECODE_WAIT 1u   /* a decode kernel gave up on a bounded wait */
#define TQ_ERRF_QUANTIZE_WAIT 2u /* a quantize-append kernel gave up on one */

/* Tokens per cache tile; capacity must be a multiple of it. */
#define TQ_TILE_TOKENS 128
/* Largest batch tq_quantize_append takes (its lengths travel as kernel
 * parameters). */
#define TQ_MAX_BATCH 1024

/* Human-readable name of a status code (static string). */
TQ_API const char *tq_status_string(tq_status s);

/*
 * tq_make_codebook -- host only, deterministic.
 *
 * Lloyd-Max scalar quantizer for N(0, 1/d) with 2^mse_bits levels: the
 * MSE-optimal codebook for a rotated coordinate (explainer, "Ý tưởng cốt
 * lõi" and "Tại sao nó hoạt động"; the audit's mse_quantizer keeps
 * centroids and decision boundaries, AUDIT 1).  Lloyd's iteration
 * (boundary = midpoint of neighbouring centroids, centroid = conditional
 * mean of its cell) in double precision until no centroid moves by more
 * than 1e-14 / sqrt(d).
 *
 *   mse_bits    1..4
 *   d           > 0
 *   centroids   host, [2^mse_bits] doubles, written ascending
 *   boundaries  host, [2^mse_bits - 1] doubles, written ascending
 * Returns TQ_ERR_INVALID_ARGUMENT for a null pointer, TQ_ERR_UNSUPPORTED
 * for mse_bits outside 1..4 or d < 1.
 */
TQ_API tq_status tq_make_codebook(int mse_bits, int d, double *centroids,
                           double *boundaries);

/* Constants of one layer.  All pointers: device, fp32, read-only, owned by
 * the caller, alive for the duration of every call that uses them. */
typedef struct {
  int d;          /* head dimension: 64, 128 or 256 */
  int key_bits;   /* 2..4 total key bits: key_bits - 1 Lloyd-Max bits + 1 QJL bit */
  int value_bits; /* 2..4 */
  int group;      /* value quantization group; 32 */
  const float *pi;         /* [d][d] row-major: Pi, y = Pi u; 16-byte aligned */
  const float *s;          /* [d][d] row-major: S, QJL sketch of r is S r; 16-byte aligned */
  const float *centroids;  /* [2^(key_bits-1)] ascending; any codebook works.
                              Decode expands it in the code bits (its Walsh
                              expansion): tq_make_codebook's symmetric
                              codebooks need only the odd terms; a caller-made
                              asymmetric one also needs the even terms, and in
                              the shapes where those planes fit in tensor
                              memory only once (3-bit keys at GQA 4 and 8 with
                              2-bit values, 4-bit keys at GQA 4, 3-bit keys and
                              values at GQA 6) decode runs the SIMT split-K
                              kernel for it (decided on the device per call) */
  const float *boundaries; /* [2^(key_bits-1) - 1] ascending decision boundaries */
  int value_mode;          /* tq_value_mode */
  const float *v_centroids;  /* TQ_VALUES_MSE: the values' codebook, [2^value_bits]
                                ascending (tq_make_codebook(value_bits, d));
                                NULL for TQ_VALUES_GROUP */
  const float *v_boundaries; /* TQ_VALUES_MSE: [2^value_bits - 1] ascending */
  const double *s_pit;       /* device, [d][d] row-major float64: W = S Pi^T,
                                W[j][m] = sum_i S[j][i] Pi[m][i], as
                                tq_sketch_product writes it from pi and s;
                                16-byte aligned.  tq_quantize_append re-decides
                                a QJL sign whose single-precision sketch
                                component is next to zero (|(S r)_j| < 1e-5) in
                                float64 as z_j = S_j . u - sum_m c_m W[j][m]
                                (= S_j . (u - Pi^T c)); required there, unused
                                by the other calls (may be NULL) */
  const void *tc_operands;   /* device, TQ_TC_OPERAND_BYTES bytes, 128-byte
                                aligned, or NULL: the tensor-core append's
                                shared-memory operand images of Pi (three
                                bf16 parts whose sum is Pi) and of W (fp16 hi
                                and lo parts of W x 2^8), as
                                tq_prepare_operands writes them from pi and
                                s_pit.  With NULL every CTA of every
                                tq_quantize_append builds them itself (same
                                bytes, ~10 us more a call); they must be
                                rewritten when pi or s_pit change.  d = 128
                                only (ignored otherwise) */
} tq_params;

/* Bytes of the tensor-core append's operand images (tq_prepare_operands). */
#define TQ_TC_OPERAND_BYTES (5 * 128 * 128 * 2)

/*
 * One layer's compressed cache: a single caller-owned device buffer.
 *
 * Layout (the pages fix none; this is the library's):
 *  - For every sequence b and KV head h (b-major, then h), capacity/128
 *    tiles of 128 tokens; tile (b, h, t) starts at byte
 *    ((b * h_kv + h) * (capacity / 128) + t) * tile_bytes.
 *  - A tile holds, in order, for its 128 token slots:
 *      1. key code bit-planes: (key_bits - 1) planes, each [128][d/8] bytes;
 *         plane p holds bit p of each coordinate's Lloyd-Max cell index;
 *      2. QJL sign plane [128][d/8]; bit 1 means sign +1 ((S r)_j >= 0);
 *      3. value codes: for value_bits = 2, packed codes [128][d/4] bytes,
 *         byte i holding channels 4i .. 4i+3 (channel 4i + m in bits 2m and
 *         2m+1); for value_bits = 3 or 4, value_bits bit-planes [128][d/8]
 *         each, plane p holding bit p of each code;
 *      4. norms [128] x {||k||, ||r||}, two little-endian fp16 per token;
 *      5. value groups [128][d/group] x {scale, zero}, two fp16 each.
 *    In a plane row, byte i bit k (LSB first) is coordinate 8 i + k.
 *  - With TQ_VALUES_MSE, section 3 holds value_bits bit-planes of the
 *    values' cell indices (at every value_bits, plane p = bit p) and section
 *    5 holds the value norms [128] x fp16; R = (key_bits + value_bits) d/8 +
 *    4 + 2 (102 bytes for 3-bit keys and values).
 *  - Record bytes per (token, KV head) R = (key_bits + value_bits) d/8 + 4
 *    + 4 d/group (100 bytes for 3-bit keys and 2-bit values at d = 128);
 *    tile_bytes = 128 R.
 *  - data must be 256-byte aligned.  Slots beyond a sequence's length may
 *    hold anything; they are never read by decode.
 */
typedef struct {
  int batch;    /* sequences */
  int h_kv;     /* KV heads */
  int capacity; /* token slots per sequence, multiple of 128 */
  void *data;   /* device, tq_cache_bytes() bytes */
} tq_cache;

/*
 * tq_sketch_product -- write W = S Pi^T in float64 (the d x d products of the
 * float32 Pi and S, each summed in float64 in index order) into s_pit,
 * device, d * d doubles, 16-byte aligned.  Only p->d, p->pi and p->s are
 * read.  Asynchronous on `stream`.  TQ_ERR_INVALID_ARGUMENT for null or
 * misaligned pointers, TQ_ERR_UNSUPPORTED for d.
 */
TQ_API tq_status tq_sketch_product(const tq_params *p, double *s_pit, tq_stream_t stream);

/*
 * tq_prepare_operands -- write the tensor-core append's operand images into
 * dst (device, TQ_TC_OPERAND_BYTES bytes, 128-byte aligned) from p->pi and
 * p->s_pit (which tq_sketch_product must have written, earlier on the same
 * stream), for p->tc_operands.  Once per layer.  Asynchronous on `stream`.
 * TQ_ERR_INVALID_ARGUMENT for null or misaligned pointers,
 * TQ_ERR_UNSUPPORTED for d != 128.
 */
TQ_API tq_status tq_prepare_operands(const tq_params *p, void *dst, tq_stream_t stream);

/* Bytes per (token, KV head) record R, or 0 for unsupported params. */
TQ_API size_t tq_record_bytes(const tq_params *p);

/* Bytes of a cache buffer for the given shape, or 0 for bad arguments. */
TQ_API size_t tq_cache_bytes(const tq_params *p, int batch, int h_kv, int capacity);

/*
 * tq_quantize_append -- compress T new tokens of every sequence and write
 * them at the end of the sequence (the store's append_chunk(k, v),
 * "turboquant/audit_claims.py", AUDIT 1).
 *
 *   k, v        device, [batch][T][h_kv][d] contiguous, `dtype` (F32 or
 *               BF16), 16-byte aligned
 *   T           tokens per sequence in k and v (>= 0; 0 is a no-op)
 *   len_host    host, [batch]: current length of each sequence; token t of
 *               sequence b is written at position len_host[b] + t
 *   n_new_host  host, [batch] or NULL: tokens of sequence b to take
 *               (<= T); NULL takes all T for every sequence
 * The caller advances its lengths afterwards; the library keeps none.
 * Errors: TQ_ERR_CAPACITY if len + n_new > capacity for any sequence or
 * batch > TQ_MAX_BATCH; TQ_ERR_INVALID_ARGUMENT for null pointers (p->s_pit
 * included), negative sizes or misalignment; TQ_ERR_UNSUPPORTED for params.
 * A zero key stores ||k|| = ||r|| = 0 with all-zero codes and signs.
 * Norms above the fp16 range (65504) are not representable (unsupported).
 */
TQ_API tq_status tq_quantize_append(const tq_params *p, const tq_cache *c,
                             const void *k, const void *v, tq_dtype dtype,
                             int T, const int32_t *len_host,
                             const int32_t *n_new_host, tq_stream_t stream);

/*
 * Workspace bytes tq_decode_attention needs for these shapes (the rotated
 * queries and the split-K partial softmax states).  0 for bad arguments.
 */
TQ_API size_t tq_decode_workspace_size(const tq_params *p, const tq_cache *c,
                                int h_q, int max_len);

/*
 * tq_decode_attention -- one decode step of attention over the compressed
 * cache, in one pass over the packed records, split over the sequence
 * (split-K) and merged by a log-sum-exp combine.
 *
 *   q              device, [batch][h_q][d], q_dtype (F32 or BF16)
 *   h_q            query heads; a multiple of h_kv; query head hq reads KV
 *                  head hq / (h_q / h_kv)
 *   len_dev        device, [batch] int32: cached tokens of each sequence;
 *                  a sequence with length 0 gets a zero output row
 *   max_len        host: an upper bound of every len_dev[b] (used to size
 *                  the split grid), 0 <= max_len <= capacity; tokens at or
 *                  beyond max_len are not read
 *   softmax_scale  logits = score * softmax_scale (1/sqrt(d) is the
 *                  standard choice); must be finite
 *   out            device, [batch][h_q][d] fp32
 *   workspace      device, >= tq_decode_workspace_size(p, c, h_q, max_len)
 *                  bytes, 256-byte aligned; contents need no initialisation.
 *                  Its first int32 is the call's status word once the call
 *                  has run: 0, or nonzero if a kernel of the call gave up on a
 *                  bounded wait, in which case every output row is NaN.
 * Errors: TQ_ERR_WORKSPACE if the workspace is missing or too small;
 * TQ_ERR_INVALID_ARGUMENT / TQ_ERR_UNSUPPORTED as for the other calls.
 */
TQ_API tq_status tq_decode_attention(const tq_params *p, const tq_cache *c,
                              const void *q, tq_dtype q_dtype, int h_q,
                              const int32_t *len_dev, int max_len,
                              float softmax_scale, float *out, void *workspace,
                              size_t workspace_bytes, tq_stream_t stream);

/*
 * tq_decode_attention_window -- tq_decode_attention over the compressed
 * cache plus a window of recent tokens kept exactly, merged into the same
 * softmax ("turboquant/audit_claims.py", AUDIT 1: the store keeps a ring
 * buffer of the 128 most recent tokens in bf16 next to the compressed
 * history).  Window tokens contribute exact scores q.k * softmax_scale and
 * exact values; the result equals one softmax over both sets.
 *
 *   win_k, win_v   device, [batch][h_kv][win_cap][d], win_dtype (F32 or
 *                  BF16), 16-byte aligned; slot order is free (attention
 *                  does not depend on it)
 *   win_len_dev    device, [batch] int32: valid window slots 0..win_cap of
 *                  each sequence (values outside are clamped)
 *   win_cap        host, 1 <= win_cap <= 128
 * The other arguments are tq_decode_attention's, with the same workspace
 * size.  A sequence with no compressed tokens and no window tokens gets a
 * zero output row.
 */
TQ_API tq_status tq_decode_attention_window(const tq_params *p, const tq_cache *c,
                                     const void *q, tq_dtype q_dtype, int h_q,
                                     const int32_t *len_dev, int max_len,
                                     const void *win_k, const void *win_v,
                                     tq_dtype win_dtype, const int32_t *win_len_dev,
                                     int win_cap, float softmax_scale, float *out,
                                     void *workspace, size_t workspace_bytes,
                                     tq_stream_t stream);

/*
 * Workspace bytes tq_prefill_attention needs for these shapes.  0 for bad
 * arguments.
 */
TQ_API size_t tq_prefill_workspace_size(const tq_params *p, const tq_cache *c,
                                 int h_q, int t_chunk, int max_len);

/*
 * Query tokens one pass of tq_prefill_attention takes together for these
 * shapes (each pass streams the compressed records once): a power of two,
 * 1 when no wider tensor-core shape is built.  0 for bad arguments.
 */
TQ_API int tq_prefill_tokens_per_pass(const tq_params *p, int h_q, int h_kv, int t_chunk);

/*
 * tq_prefill_attention -- causal attention of a chunk of t_chunk query
 * tokens per sequence over the compressed cache, after the chunk's own keys
 * and values were appended ("turboquant/audit_claims.py", AUDIT 7 and 8:
 * long-context prefill as scaled-dot-product attention with a causal mask
 * over the stored cache; here the stored cache is the compressed one, read
 * in place).  Query token t of the chunk (0-based) of sequence b attends to
 * the first len_dev[b] - (t_chunk - 1 - t) cached tokens, with the decode
 * estimator of tq_decode_attention.  Passes of up to 4 / (h_q / h_kv) query
 * tokens (a power of two the tensor-core kernel is built for; one token at
 * GQA 4 and above) share every streamed KV tile: the chunk's tokens join the
 * query heads of a KV head.
 *
 *   q              device, [batch][t_chunk][h_q][d], q_dtype (F32 or BF16)
 *   t_chunk        query tokens per sequence, 1 <= t_chunk <= max_len
 *   len_dev        device, [batch] int32: cached tokens of each sequence,
 *                  the chunk included (len_dev[b] >= t_chunk expected; a
 *                  query token that sees no token gets a zero row)
 *   max_len        host: an upper bound of every len_dev[b]
 *   out            device, [batch][t_chunk][h_q][d] fp32
 *   workspace      device, >= tq_prefill_workspace_size(p, c, h_q,
 *                  t_chunk, max_len) bytes, 256-byte aligned
 * The other arguments and the errors are tq_decode_attention's.
 */
TQ_API tq_status tq_prefill_attention(const tq_params *p, const tq_cache *c,
                               const void *q, tq_dtype q_dtype, int h_q, int t_chunk,
                               const int32_t *len_dev, int max_len, float softmax_scale,
                               float *out, void *workspace, size_t workspace_bytes,
                               tq_stream_t stream);

/* Size of the fixed device scratch tq_decode_attention_noalloc uses. */
#define TQ_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/*
 * tq_decode_attention_noalloc -- tq_decode_attention for callers that cannot
 * provide a workspace.  The pages have no counterpart of this call; it
 * exists for users of this library.
 *
 * Some callers cannot allocate device memory for the library: a plain C host
 * that links only libtq and owns no device allocator, a decode loop that must
 * not call cudaMalloc (it can synchronise the whole device and stall other
 * streams), or an engine that reserved all free device memory for its own
 * pool at start-up.  This entry point takes the same arguments as
 * tq_decode_attention minus the workspace and allocates nothing: its scratch
 * (rotated queries and split-K partial states) is one fixed array of
 * TQ_NOALLOC_SCRATCH_BYTES (8 MiB) in device memory, reserved in every GPU
 * that loads the library until the process exits.
 *
 *  - A call whose scratch need (tq_decode_workspace_size for the same
 *    shapes) exceeds TQ_NOALLOC_SCRATCH_BYTES returns TQ_ERR_WORKSPACE and
 *    launches nothing.
 *  - The first call on a device looks up the array's device address with
 *    that device current and caches it; make that first call before any
 *    stream capture.  The cached address does not survive a device reset
 *    (cudaDeviceReset): calling this entry point again after one is not
 *    supported.
 *  - All calls share the one array and it keeps the previous call's contents
 *    (nothing in it needs clearing: every byte the kernels read is written
 *    earlier in the same call).  Calls that overlap on the GPU -- on
 *    different streams, or from different host threads without ordering --
 *    race on the array and produce wrong results; order them.
 * Other errors as for tq_decode_attention.
 */
TQ_API tq_status tq_decode_attention_noalloc(const tq_params *p, const tq_cache *c,
                                             const void *q, tq_dtype q_dtype, int h_q,
                                             const int32_t *len_dev, int max_len,
                                             float softmax_scale, float *out,
                                             tq_stream_t stream);

/*
 * tq_set_wait_limit_ns -- set the time limit of the kernels' bounded waits
 * for calls made afterwards from any host thread (0 restores the default,
 * 2 s); the kernels' suspend hint per wait test is min(limit, 1 ms).  For
 * tests of the timeout path: a limit shorter than a call needs makes its
 * kernels give up (NaN results, the error word set) and return.  Always
 * TQ_OK.
 */
TQ_API tq_status tq_set_wait_limit_ns(unsigned long long ns);

/*
 * tq_test_withhold_handoffs -- for tests of the timeout path only: while on
 * (nonzero), the tensor-core kernels of later calls withhold one hand-off
 * that their other roles wait for (decode: the tile copies; quantize-append:
 * the loaded key operand), so those bounded waits run out after the wait
 * limit and the failure reporting above can be observed.  Nothing faults:
 * every wait is bounded and each kernel returns.  Off by default.  Always
 * TQ_OK.
 */
TQ_API tq_status tq_test_withhold_handoffs(int on);

/*
 * tq_test_sign_refine_threshold -- for tests of the float64 sign refinement
 * only: quantize-append calls made afterwards re-decide in float64 every QJL
 * sign whose single-precision sketch component has |(S r)_j| < z (0 restores
 * the default, 1e-5; negative: TQ_ERR_INVALID_ARGUMENT).  A larger z sends
 * many more keys through the refinement (slower, same stored bits outside
 * float64 rounding).
 */
TQ_API tq_status tq_test_sign_refine_threshold(double z);

/*
 * tq_test_refine_count -- synchronise the current device, then read (and, if
 * `clear` is nonzero, reset) the number of QJL sign bits that quantize-append
 * kernels on it have re-decided in float64 since the last reset.  count: host
 * pointer.  TQ_ERR_INVALID_ARGUMENT for a null pointer, TQ_ERR_CUDA if the
 * device reports an error.
 */
TQ_API tq_status tq_test_refine_count(unsigned long long *count, int clear);

/*
 * tq_device_errors -- synchronise the current device, then read (and, if
 * `clear` is nonzero, reset) its sticky error word: an OR of TQ_ERRF_* bits
 * set by kernels that gave up on a bounded wait since the last clear.
 *   flags  host, written.
 * The first call on a device looks the word's device address up (once per
 * device); launches made by the library's other calls do the same.
 * Errors: TQ_ERR_INVALID_ARGUMENT for a null pointer, TQ_ERR_CUDA if the
 * device reports an error.
 */
TQ_API tq_status tq_device_errors(uint32_t *flags, int clear);

/*
 * tq_dequantize -- explicit reconstruction of cached tokens [start,
 * start + count) of sequence b (the audit's quantizer.dequantize(prod_q),
 * AUDIT 2):  k_hat = ||k|| (Pi^T c + sqrt(pi/2)/d ||r|| S^T (2 sign - 1)),
 * v_hat = code * scale + zero.  Off the decode path; for tests and tools.
 *
 *   k_out, v_out  device, [count][h_kv][d] fp32 each
 */
TQ_API tq_status tq_dequantize(const tq_params *p, const tq_cache *c, int b,
                        int start, int count, float *k_out, float *v_out,
                        tq_stream_t stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* TQ_H_ */
