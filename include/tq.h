/*
 * tq.h -- C ABI of the compressed KV-cache library (B200, sm_100a).
 *
 * One hot path: TurboQuant-style compression of the KV cache (a seeded
 * randomized Hadamard rotation, 2-D polar quantization with an fp16 scale,
 * a 1-bit QJL sketch of the key residual) and single-token decode attention
 * computed straight from the packed cold cache next to a full-precision hot
 * ring of the most recent tokens (Monarch's hot/cold split).
 *
 * Sources (page title, section):
 *  [TQ-PL]   "TurboQuant: kompresja KV-cache w LLM 6 razy bez utraty
 *            dokładności" -- "Zasada działania PolarQuant" (rotate, then
 *            radius/angle, then quantize), "Kompensacja błędów przez QJL"
 *            (1-bit code of the residual that preserves inner products).
 *  [TQ-ES]   "TurboQuant: optimización de memoria para KV caches en
 *            inferencia de LLMs" -- "Flujo de Cuantificación de KV Cache con
 *            TurboQuant", steps 1-7 (step 6: attention logits computed from
 *            the compressed cache).
 *  [TQ-3B]   "Compresión del caché KV de los LLM a 3 bits: TurboQuant de
 *            Google Research" -- "Aplicaciones más allá de los LLMs"
 *            (vector search over the same codes).
 *  [MONARCH] "Monarch v3: Paginación KV Inspirada en NES para una Inferencia
 *            de LLM 78% Más Rápida" -- "Cómo funciona" (hot region at full
 *            precision, cold region compressed, sliding-window eviction),
 *            "Bucle de Decodificación Simplificado" (evict_oldest_to_cold;
 *            aggregate, softmax, apply).
 *  [TC]      "Tensor Cache: Eviction-conditioned Associative Memory for
 *            Transformers" -- "Metodología" (the first-level cache is a ring
 *            whose overwrite becomes a write into the second tier).
 *
 * Conventions for every call
 *  - Memory: the caller allocates every device buffer (sizes from
 *    tq_cache_bytes); the library never calls cudaMalloc.  The library owns
 *    only the host-side handle (freed by tq_cache_destroy).  Input buffers
 *    are borrowed until the stream-ordered work that reads them completes.
 *  - Streams: every device call is asynchronous on the given stream and
 *    never synchronizes, except tq_get_status and the tq_export_* helpers.
 *  - Errors: argument, shape and capacity errors are returned synchronously
 *    before any launch, and leave the handle unchanged.  Launch failures
 *    return TQ_ERR_CUDA.  Conditions detected on the device (an fp16 scale
 *    that overflows, a bounded wait that gave up) are latched into a device
 *    status word and returned (and cleared) by tq_get_status.  Nothing in
 *    the library traps or asserts on the device.
 *  - Layouts: fp16 buffers are IEEE binary16, passed as void*.  Shapes are
 *    row-major and contiguous.  B = batch, Hq / Hkv = query / KV heads,
 *    G = Hq / Hkv, d = head_dim, W = hot window, m = QJL bits.
 *  - Thread safety: a handle may be used from one host thread at a time.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TQ_ABI_VERSION 1

typedef enum tq_status {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,   /* null pointer, bad shape or value            */
  TQ_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim 96) */
  TQ_ERR_CAPACITY = 3,      /* the cold store would exceed its capacity    */
  TQ_ERR_RANGE = 4,         /* (device) an fp16 scale or norm overflowed   */
  TQ_ERR_TIMEOUT = 5,       /* (device) a bounded wait gave up             */
  TQ_ERR_CUDA = 6           /* a CUDA runtime call or launch failed        */
} tq_status;

/* One handle per attention layer. */
typedef struct tq_config {
  int32_t batch;            /* B >= 1                                        */
  int32_t num_q_heads;      /* Hq, a multiple of Hkv with G = Hq/Hkv <= 8    */
  int32_t num_kv_heads;     /* Hkv >= 1                                      */
  int32_t head_dim;         /* d: 64 or 128                                  */
  int32_t hot_window;       /* W >= 1: tokens kept at fp16 in the hot ring   */
  int64_t cold_capacity;    /* max compressed tokens per (row, kv head)      */
  int32_t b_r;              /* radius bits   >= 1                            */
  int32_t b_theta;          /* angle bits    >= 1, b_r + b_theta <= 8        */
  int32_t qjl_bits;         /* m: 64 or 128 sign bits per key                */
  uint64_t seed;            /* drives the rotation signs D and QJL matrix S  */
} tq_config;

typedef struct tq_cache tq_cache;

/* Human-readable name of a status code (static string). */
const char* tq_status_string(tq_status s);

/* TQ_ABI_VERSION of the loaded library. */
int32_t tq_abi_version(void);

/*
 * Device memory the caller must provide for a configuration.
 *   hot_bytes   fp16 hot ring, K then V, each [B, Hkv, W, d].
 *   cold_bytes  packed cold store: per (row, kv head) a run of 64-token
 *               blocks; inside a block, field planes (K codes, K sign bits,
 *               K scales, K residual norms, V codes, V scales), token-major
 *               and 16-byte aligned.  Bytes per cold token per kv head:
 *               K: d/2*(b_r+b_theta)/8 + m/8 + 4, V: d/2*(b_r+b_theta)/8 + 2.
 *   workspace_bytes  rotation signs, QJL matrix, per-call query transforms,
 *               split partials and the device status word.
 * Each buffer must be 256-byte aligned.  Any output pointer may be NULL.
 */
tq_status tq_cache_bytes(const tq_config* cfg, size_t* hot_bytes,
                         size_t* cold_bytes, size_t* workspace_bytes);

/*
 * Bind a handle to caller-owned device buffers and upload the seeded method
 * randomness (D and S, generated on the host by the library) into the
 * workspace with stream-ordered copies.  The cache starts empty.  *out is
 * valid until tq_cache_destroy.  The buffers' previous contents are ignored.
 */
tq_status tq_cache_create(const tq_config* cfg, void* hot_mem, void* cold_mem,
                          void* workspace_mem, cudaStream_t stream,
                          tq_cache** out);

/* Free the host handle (device buffers stay the caller's). NULL is a no-op. */
tq_status tq_cache_destroy(tq_cache* cache);

/* Host-side counters: compressed tokens, valid hot tokens, next ring slot.
 * For a ragged batch (rows with different counts): the largest n_cold and
 * n_hot over the rows and row 0's ring slot; tq_cache_row_counts gives
 * each row's own. */
tq_status tq_cache_counts(const tq_cache* cache, int64_t* n_cold,
                          int32_t* n_hot, int32_t* ring_pos);
tq_status tq_cache_row_counts(const tq_cache* cache, int32_t row, int64_t* n_cold,
                              int32_t* n_hot, int32_t* ring_pos);

/*
 * Compress n new tokens straight into the cold store (prefill path).
 * [TQ-PL] "Zasada działania PolarQuant" + "Kompensacja błędów przez QJL";
 * [TQ-ES] steps 1-5.  For every (row, kv head) and token, K and V are
 * rotated (y = H_d D x / sqrt(d)), split into d/2 pairs mapped to
 * (rho, theta), coded on an endpoint radius grid (b_r bits, scale
 * s16 = fp16(max rho)) and a periodic angle grid (b_theta bits); keys also
 * store fp16(||r||) and m bits [(S r)_i >= 0] of the residual r = y - y_hat.
 * The code decisions are computed in float64 on the device.
 *   k, v  device fp16 [B, Hkv, n, d] (contiguous)
 *   n     >= 0 (0 is a no-op)
 * Tokens land at cold indices n_cold .. n_cold+n-1 of every (row, kv head).
 * Returns TQ_ERR_CAPACITY (nothing launched) if n_cold + n > cold_capacity.
 */
tq_status tq_encode_append(tq_cache* cache, const void* k, const void* v,
                           int64_t n, cudaStream_t stream);

/*
 * Insert n new tokens into the hot ring (decode path).
 * [MONARCH] "Cómo funciona" (sliding-window eviction) and "Bucle de
 * Decodificación Simplificado" (evict_oldest_to_cold); [TC] "Metodología"
 * (ring overwrite feeds the second tier).  Equivalent to n single inserts in
 * order: when the ring already holds W tokens, the oldest one is encoded
 * exactly as tq_encode_append does and appended to the cold store, then the
 * new token takes its slot (pos mod W).
 *   k_new, v_new  device fp16 [B, Hkv, n, d];  n >= 1
 * Returns TQ_ERR_CAPACITY (nothing launched) if the evictions would overflow
 * the cold store.
 */
tq_status tq_evict_window(tq_cache* cache, const void* k_new,
                          const void* v_new, int32_t n, cudaStream_t stream);

/*
 * Per-row lengths (ragged batches): the rows of a batch -- sequences of
 * different lengths -- append and insert different numbers of tokens, and
 * every later call attends each row's own tokens (the per-row lengths of
 * the "TurboQuant: kompresja KV-cache ..." page's format; no row is padded
 * in the cold store).
 *   k, v / k_new, v_new  device fp16 [B, Hkv, n_max, d]; row b's first
 *               n_rows[b] tokens are used (0 <= n_rows[b] <= n_max)
 *   n_rows      HOST int32 [B]
 * tq_encode_append_rows appends row b's tokens at its own cold count;
 * tq_evict_window_rows inserts them into its own ring (a full ring evicts
 * its oldest tokens into the row's cold store, as tq_evict_window).
 * TQ_ERR_CAPACITY (nothing launched) if a row would exceed cold_capacity.
 * While the rows' counts differ, the batch may have at most 128 rows
 * (TQ_ERR_UNSUPPORTED otherwise), and the threshold-gated decode, the
 * Tensor Cache tier and promotion are unavailable (TQ_ERR_UNSUPPORTED);
 * tq_encode_append / tq_evict_window then act as the _rows calls with the
 * same n for every row.  Uniform inputs take the uniform paths.
 */
tq_status tq_encode_append_rows(tq_cache* cache, const void* k, const void* v, int64_t n_max,
                                const int32_t* n_rows, cudaStream_t stream);
tq_status tq_evict_window_rows(tq_cache* cache, const void* k_new, const void* v_new,
                               int32_t n_max, const int32_t* n_rows, cudaStream_t stream);

/*
 * Single-token decode attention over hot U cold tokens.
 * [TQ-ES] step 6 (logits from the compressed cache); [MONARCH] "Bucle de
 * Decodificación Simplificado" (aggregate, softmax, apply).  For query head
 * h (kv head h / G), with q' = R q and q'' = S q':
 *   hot token:  l = sigma <q, k>
 *   cold token: l = sigma ( s16/(2^b_r-1) <q', y_hat_unit>
 *                           + rn16 sqrt(pi/2)/m <q'', 2 bits - 1> )
 *   p = softmax(l) over every valid hot and cold token
 *   out = sum_hot p v + R^T sum_cold p s16_v/(2^b_r-1) v_hat_unit
 * Accumulation is fp32; the products run on tensor cores with fp16
 * operands.  Every valid token is attended (no mask; K is cached after any
 * positional encoding).
 *   q      device fp16 [B, Hq, d], 16-byte aligned (else TQ_ERR_INVALID_ARG)
 *   out    device fp32 [B, Hq, d]
 *   softmax_scale  sigma; 0 selects 1/sqrt(d)
 * With no valid token at all, out is zero.
 * Ordering: the call's first kernel (q-prep) is a programmatic dependent
 * launch of whatever the stream ran before it, and it reads q before it
 * waits for that kernel.  So the kernel that writes q must not signal its
 * dependents early (griddepcontrol.launch_dependents /
 * cudaTriggerProgrammaticLaunchCompletion before its writes of q): ordinary
 * kernels, PyTorch's included, never do, and the library's own kernels do
 * not write q.  Everything else the call reads is read after the wait.
 */
tq_status tq_decode_attention(tq_cache* cache, const void* q, float* out,
                              float softmax_scale, cudaStream_t stream);

/*
 * tq_decode_attention without caller-provided scratch (the pages have no
 * counterpart; this is an integration convenience).  For callers that may
 * not allocate device memory while they run -- an allocator-free serving
 * loop, a plugin whose host owns every allocation, a process whose memory
 * is reserved up front.  It computes exactly what tq_decode_attention does,
 * with the same kernels, but keeps the per-call scratch (rotated queries and
 * split partials) in a 4 MiB array compiled into the library: one copy per
 * GPU that loads the library, resident until the process exits.  The call
 * never allocates (no cudaMalloc / cudaFree, no allocating library call).
 *   - The first call on a device looks up that array's device address
 *     (cudaGetSymbolAddress) and remembers it; make that first call before
 *     any stream capture.  The handle's device must be current.
 *   - Calls whose GPU work overlaps (other streams, other handles on the
 *     same device) share the array and race; serialize them.
 *   - Returns TQ_ERR_CAPACITY, launching nothing, when this configuration's
 *     scratch (about units x (partials + 2) x G x (d + 2) x 4 bytes plus the
 *     query transforms) exceeds 4 MiB.
 */
tq_status tq_decode_attention_static(tq_cache* cache, const void* q, float* out,
                                     float softmax_scale, cudaStream_t stream);

/*
 * Decode attention with a threshold-gated cold tier.  This is the loop on
 * the Monarch v3 page ("Bucle de Decodificación Simplificado"): the hot
 * scores are computed first, and the cold pages are read only while the
 * largest hot score is below a threshold.  Per query head h:
 *   g_h = max over the hot window of q_h . k_t, the plain product without
 *         softmax_scale, in fp32 from the fp16 q and K;
 *   if the hot window is non-empty and g_h >= threshold, h attends to its
 *   hot window alone (one softmax over the hot tokens);
 *   otherwise h gets exactly tq_decode_attention's result (hot and cold).
 * A (row, kv head) whose query heads all skip has none of its cold records
 * read.  The remaining cold work is split again over all CTAs, so the time
 * saved scales with the skipped units.
 *   q, out, softmax_scale  as tq_decode_attention
 *   threshold  any non-NaN float (+inf: never skip; -inf: skip whenever
 *              the hot window is non-empty)
 *   head_skip  NULL, or device int32 [B, Hq]: written with 1 for the heads
 *              that skipped their cold tier, else 0
 * Scratch comes from the handle's workspace (as tq_decode_attention).
 * Returns TQ_ERR_INVALID_ARG for a NaN threshold or a NULL q / out.
 */
tq_status tq_decode_attention_gated(tq_cache* cache, const void* q, float* out,
                                    float softmax_scale, float threshold, int32_t* head_skip,
                                    cudaStream_t stream);

/*
 * Tensor Cache second tier ("Tensor Cache: Eviction-conditioned Associative
 * Memory for Transformers", section "Metodología"): an alternative to the
 * compressed cold store.  Once enabled on a handle:
 *   - every token the hot ring displaces in tq_evict_window is written into
 *     a d x d float32 matrix A of its (row, kv head) instead of the cold
 *     store: A <- lambda A + eta (k outer v), in eviction order (a run of E
 *     evictions is applied at once as lambda^E A + eta sum_e
 *     lambda^(E-1-e) k_e v_e^T, the same value);
 *   - every decode call adds sigmoid(g_h) (q_h A) to query head h's output
 *     (q_h the fp16 query, A that of its kv head), after the softmax over
 *     the ring and over any cold tokens appended before enabling.
 * lambda, eta and g are learned on the page; here they are given.
 *
 * tq_tc_bytes: device bytes of the tier's buffer for a configuration: A as
 *   [B, Hkv, d, d] float32 (256-byte aligned), then lambda [Hkv], eta [Hkv]
 *   and sigmoid(g) [Hq] as float32.
 * tq_tc_enable: binds the caller's buffer (256-byte aligned, at least
 *   tq_tc_bytes; owned by the caller, kept until tq_cache_destroy), sets A
 *   to zero and copies the parameters (host arrays lambda [Hkv], eta [Hkv],
 *   gate [Hq]); synchronizes `stream`.  TQ_ERR_INVALID_ARG for a NULL or
 *   misaligned pointer, a non-finite lambda or eta, a NaN gate, or a handle
 *   that already has the tier.
 */
tq_status tq_tc_bytes(const tq_config* cfg, size_t* bytes);
tq_status tq_tc_enable(tq_cache* cache, void* tc_mem, const float* lambda, const float* eta,
                       const float* gate, cudaStream_t stream);

/*
 * Attention-weighted promotion with sticky counters ("Monarch v3 ...",
 * section "Cómo funciona", item "Promoción Ponderada por Atención": cold
 * tokens that draw much attention return to the full-precision hot region,
 * with a persistence count against thrashing; the page's benchmark uses a
 * threshold of 0.15 and a sticky count of 3).  Once enabled on a handle:
 *   - every tq_decode_attention (and _static) call also finds, per (row, kv
 *     head), the cold tokens whose mass -- the mean over the kv head's query
 *     heads of the token's softmax weight in that call -- is >= threshold.
 *     A token's count rises by one at each call where it is such a hit and
 *     returns to 0 at any call where it is not; at `sticky` it is promoted
 *     and its count cleared.  Promotions are dropped while the hot window
 *     is not yet full.
 *   - the next tq_evict_window inserts, per (row, kv head), its promoted
 *     tokens first -- their K and V dequantized to fp16, R^T (s16/(2^b_r-1)
 *     c_r (cos, sin)), in ascending cold position -- and then the n new
 *     tokens.  Every insert evicts the ring's oldest token: the first ones
 *     take the promoted tokens' cold positions, the last n are appended, so
 *     every (row, kv head) keeps the same cold count.  Ring positions then
 *     differ per (row, kv head); decode attention is order-free in the ring.
 * tq_promotion_bytes: size of the caller's buffer (per-unit state, every
 *   cold token's logits [B*Hkv, cold_capacity, G] as float32, the heads'
 *   softmax normalisers, the promoted tokens' fp16 staging).
 * tq_promotion_enable: binds that buffer (256-byte aligned, kept until
 *   tq_cache_destroy), synchronizes `stream`.  TQ_ERR_INVALID_ARG for a NULL
 *   or misaligned buffer, a threshold outside [1/8, 1] (at most 8 tokens per
 *   (row, kv head) can then be hits, since their masses sum to at most 1),
 *   sticky < 1, a hot window of 8 tokens or fewer, a handle with the Tensor
 *   Cache tier, or promotion already on.  Afterwards tq_evict_window returns
 *   TQ_ERR_INVALID_ARG for n > hot_window - 8 once the window is full, and
 *   tq_decode_attention_gated returns TQ_ERR_UNSUPPORTED.
 * tq_promotion_state: copies the per-(row, kv head) state to a HOST array
 *   out[B*Hkv][28] (synchronizes `stream`): [0] tokens with a running count,
 *   [1] tokens promoted by the last decode and not yet moved, [2] the ring
 *   position, [3] 0, [4..11] the counted cold positions (ascending, -1 when
 *   unused), [12..19] their counts, [20..27] the promoted cold positions.
 */
tq_status tq_promotion_bytes(const tq_config* cfg, size_t* bytes);
tq_status tq_promotion_enable(tq_cache* cache, void* mem, float threshold, int32_t sticky,
                              cudaStream_t stream);
tq_status tq_promotion_state(tq_cache* cache, int32_t* out, cudaStream_t stream);

/*
 * Synchronize `stream`, then return and clear the latched device status
 * (TQ_OK, TQ_ERR_RANGE or TQ_ERR_TIMEOUT; TQ_ERR_UNSUPPORTED when the
 * attention kernel found its dynamic shared memory at a window address its
 * table layout does not fit), or TQ_ERR_CUDA if the stream itself reports
 * an error.  After a timeout or that layout error an attention launch has
 * written no partial results, so every decode call on the handle writes NaN
 * to all of `out` until this call has cleared the status.
 */
tq_status tq_get_status(tq_cache* cache, cudaStream_t stream);

/*
 * Copy cold records of one (row, kv head) to HOST buffers in canonical
 * form (synchronizes `stream`): pair j's word (c_r << b_theta) | c_theta
 * LSB-first at bit j*(b_r+b_theta); sign bit i at bit i; fp16 raw bits.
 *   k_codes [count, d/2*(b_r+b_theta)/8]  k_bits [count, m/8]
 *   k_s16 [count]  k_rn16 [count]  v_codes [count, ...]  v_s16 [count]
 * Requires start + count <= n_cold.  Any output pointer may be NULL.
 */
tq_status tq_export_cold(tq_cache* cache, int32_t row, int32_t kv_head,
                         int64_t start, int64_t count, uint8_t* k_codes,
                         uint8_t* k_bits, uint16_t* k_s16, uint16_t* k_rn16,
                         uint8_t* v_codes, uint16_t* v_s16,
                         cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Vector inner-product search over the same codes.
 * [TQ-3B] "Aplicaciones más allá de los LLMs": the compressed vectors serve
 * vector search / RAG ranking.  Database vectors (float32, dimension d_in,
 * zero-padded to d = the next power of two >= 64) are encoded exactly like
 * keys: rotation, polar codes, fp16 scale, m QJL sign bits of the residual
 * and its fp16 norm.  A query q is scored against vector i by the same
 * estimator as a cold attention logit, without the softmax scale:
 *   score = s16_i/(2^b_r-1) <q', x_hat_unit_i> + rn16_i sqrt(pi/2)/m <q'', 2 bits_i - 1>
 * and the k best scores per query are returned (descending; equal scores
 * in index order).
 * ---------------------------------------------------------------------- */
typedef struct tq_vec_config {
  int32_t dim;              /* d_in, 1..256                                  */
  int32_t b_r;              /* radius bits; b_r + b_theta must equal 8       */
  int32_t b_theta;          /* angle bits                                    */
  int32_t qjl_bits;         /* m: 8..256, a multiple of 8                    */
  uint64_t seed;            /* rotation signs D and QJL matrix S             */
} tq_vec_config;

typedef struct tq_vec_index tq_vec_index;

/*
 * Sizes for an index over n vectors:
 *   codes_bytes      the packed database (256-byte aligned): codes (one
 *                    byte per pair, d/2 per vector) and sign bits (m bits
 *                    zero-padded to 32 bytes per vector) in groups of 32
 *                    vectors, each vector's bytes in 16-byte chunks stored
 *                    chunk-major inside the group ([n/32][chunk][32][16]);
 *                    then s16 [n] and rn16 [n]; each section 256-byte
 *                    aligned.  tq_export_vectors returns the canonical form.
 *   workspace_bytes  D, S, query transforms for up to `max_queries` queries
 *                    and the per-split top-k partials of a search.
 */
tq_status tq_vec_bytes(const tq_vec_config* cfg, int64_t n, int32_t max_queries,
                       size_t* codes_bytes, size_t* workspace_bytes);

/* Bind a search handle to a caller-owned workspace (uploads D and S). */
tq_status tq_vec_create(const tq_vec_config* cfg, int64_t n, int32_t max_queries,
                        void* workspace_mem, cudaStream_t stream, tq_vec_index** out);
tq_status tq_vec_destroy(tq_vec_index* index);

/*
 * Encode database vectors [start, start + count) of x (device float32
 * [count, d_in], row-major) into `codes` (device, tq_vec_bytes layout).
 * Decisions in float64 as for tq_encode_append.
 */
tq_status tq_encode_vectors(tq_vec_index* index, const float* x, int64_t start,
                            int64_t count, void* codes, cudaStream_t stream);

/*
 * Top-k estimated inner products of nq queries (device float32 [nq, d_in])
 * against all n encoded vectors.  scores: device float32 [nq, k]; idx:
 * device int32 [nq, k].  1 <= k <= 16, nq <= max_queries.  The products
 * run on tensor cores (tcgen05, fp16 operands, fp32 accumulation), 128
 * queries per CTA.  The kernel's waits are bounded: one that gives up
 * latches TQ_ERR_TIMEOUT in the index's status word (tq_vec_get_status)
 * and that search's results are undefined.
 */
tq_status tq_ip_search(tq_vec_index* index, const void* codes, const float* q, int32_t nq,
                       int32_t k, float* scores, int32_t* idx, cudaStream_t stream);

/* The latched device status of an index's searches (synchronizes the
 * stream, then clears it): TQ_OK or TQ_ERR_TIMEOUT. */
tq_status tq_vec_get_status(tq_vec_index* index, cudaStream_t stream);

/*
 * Canonical records of database vectors [start, start + count) to HOST
 * buffers (synchronizes): codes [count][d/2*(b_r+b_theta)/8] in the
 * LSB-first stream form of tq_export_cold, bits [count][m/8], s16, rn16.
 */
tq_status tq_export_vectors(tq_vec_index* index, const void* codes, int64_t start,
                            int64_t count, uint8_t* codes_out, uint8_t* bits_out,
                            uint16_t* s16_out, uint16_t* rn16_out, cudaStream_t stream);

/*
 * Measurement hook: when `start` and `stop` are non-NULL, every following
 * tq_decode_attention call on this handle records `start` on its stream
 * right before the attention kernel and `stop` right after it, so that a
 * caller can time that kernel alone with cudaEventElapsedTime.  Pass NULLs
 * to stop recording.  The events are borrowed, not owned.
 */
tq_status tq_set_attend_events(tq_cache* cache, cudaEvent_t start, cudaEvent_t stop);

/*
 * Limit of each bounded wait in the attention kernel (the wait for a cold
 * tile's bulk copy; the pages have no counterpart: this serves failure
 * testing).  limit_ns < 0 restores the default of 2 s.  limit_ns = 0 makes
 * every such wait give up at once, without polling, which forces the
 * timeout path: the kernel latches TQ_ERR_TIMEOUT, waits (under the default
 * limit) for the copies it already issued, and returns without partials.
 * Applies to the following decode calls on this handle.
 */
tq_status tq_set_wait_limit(tq_cache* cache, int64_t limit_ns);

/*
 * The library's own seeded method randomness (host only, no GPU needed),
 * exactly as uploaded by tq_cache_create:
 *   signs[i] = +1 / -1  (i < d)         QJL matrix S [m, d] float32.
 * Generator: rand64(seed, stream, i) = mix64(mix64(seed + stream)
 * + (i + 1) * 0x9E3779B97F4A7C15) with the SplitMix64 finalizer mix64;
 * stream 0: sign = top bit clear ? +1 : -1; stream 1: Box-Muller (first
 * output) from draws 2k, 2k+1 for entry k = row * d + col, in float64 with
 * the C library's log/cos/sqrt, rounded to float32.
 */
tq_status tq_rotation_signs(uint64_t seed, int32_t d, int8_t* signs);
tq_status tq_qjl_matrix(uint64_t seed, int32_t m, int32_t d, float* S);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
