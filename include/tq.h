/*
 * tq.h -- C ABI of the TurboQuant KV-cache codec for NVIDIA B200 (sm_100a).
 *
 * Method source ("TQ" below): the web page "TurboQuant 설명: 무엇인지와 LLM
 * 메모리 6배 절약 구현 방법" (TurboQuant explained: what it is and how to
 * implement 6x LLM memory savings), a2a-mcp.org:
 *   TQ §Stage 1  random orthogonal rotation (QR of a Gaussian matrix), the
 *                Beta((d-1)/2,(d-1)/2) coordinate law, Lloyd-Max quantizer;
 *   TQ §Stage 2  1-bit QJL sign sketch of the residual (bias correction);
 *   TQ §How it works / §How to implement  logits straight from the indices
 *                with the query rotated once; quantize on every cache update.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers named "device" must point to memory of the current CUDA device;
 *    "host" pointers to ordinary host memory.  The library never allocates
 *    cache, input, output or workspace memory: the caller owns all of it.  The
 *    only library-owned memory is the small set of constant tables inside a
 *    tq_codebook (freed by tq_codebook_free).
 *  - Calls that take a stream are asynchronous on that stream (pass 0 for the
 *    legacy default stream); they return after the launches are queued.
 *  - Argument errors are detected on the host and returned synchronously
 *    (TQ_EINVAL / TQ_EUNSUPPORTED) with nothing launched; tq_last_error()
 *    then returns a message (thread-local, valid until the next call).
 *  - Errors found by the kernels (a block-table entry outside [0, n_pages), a
 *    norm too large for fp16, a bounded wait that gave up) are OR-ed into
 *    *error_word of the cache (TQ_DEV_ERR_* bits) when it is not NULL.  The
 *    kernels never trap; read the word after synchronizing the stream.  An
 *    out-of-range page is skipped (nothing read or written through it).
 *  - Shapes are row-major and contiguous unless a stride is given.
 *
 * Packed record layout (layout version 3)
 * ---------------------------------------
 * d_pad = 64 ceil(d/64), m_pad = 64 ceil(m/64), E = d_pad/4, F = m_pad/4.
 * A record is 4 chunks; chunk t holds coordinates [tE, tE+E) and QJL rows
 * [tF, tF+F) as 32-bit words: index words, then ceil(F/32) QJL words.  The
 * stored code of a coordinate is its level index for b <= 3 and the nibble
 * neg << 3 | mu for b = 4 (idx >= 8: neg 0, mu = idx - 8; else neg 1,
 * mu = 7 - idx).  Bit k of the code of local element l: b = 1: word l/32, bit
 * 4(l%8) + (l%32)/8; b = 2: word l/16, bit 4(l%8) + 2((l%16)/8) + k; b = 3:
 * groups of 32 elements in 3 words, element l' = l%32 of group g = l/32 at
 * word 3g + l'/8, bit 4(l'%8) + k when l' < 24, else word 3g + k, bit
 * 4(l' - 24) + 3 (a last group of 16 uses 2 words, word 3(E/32) + l'/8, bit
 * 4(l'%8) + k); b = 4: word l/8, bit 4((l%8)/2 + 4(l%2)) + k.  QJL row l:
 * QJL word l/32, bit 8(l%4) + (l%32)/4, set where (S r)_i < 0.
 * Padding coordinates store code 0.  A page holds page_tokens tokens of
 * every KV head; a head block is page_tokens records followed by
 * page_tokens norm slots (fp16 ||x||, then fp16 ||r|| when m > 0), padded to
 * 16 bytes.  Token `pos` of sequence b, head h lives in page
 * block_table[b * max_pages_per_seq + pos / page_tokens], slot
 * pos % page_tokens.  tq_layout() reports the sizes.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_EINVAL = 1,        /* bad argument (NULL pointer, bad size, misalignment) */
  TQ_EUNSUPPORTED = 2,  /* valid but not built (e.g. bits > 4 on the GPU path) */
  TQ_ERANGE = 3,        /* a value outside its representable range */
  TQ_ETIMEOUT = 4,      /* a bounded device wait gave up */
  TQ_ECUDA = 5,         /* a CUDA runtime call failed */
  TQ_ENOMEM = 6         /* the codebook's constant tables could not be allocated */
} tq_status;

typedef enum { TQ_BF16 = 0, TQ_F16 = 1, TQ_F32 = 2 } tq_dtype;

/* Bits OR-ed into tq_cache.error_word by the kernels. */
#define TQ_DEV_ERR_PAGE 1u     /* block-table entry outside [0, n_pages) */
#define TQ_DEV_ERR_RANGE 2u    /* a norm >= 65520 became +inf in fp16 */
#define TQ_DEV_ERR_TIMEOUT 4u  /* a bounded mbarrier wait gave up */
#define TQ_DEV_ERR_CONFIG 8u   /* a kernel found its shared memory misaligned and did nothing */

/* Codec parameters.  d: head dimension, a multiple of 8 with 8 <= d <= 256.
 * bits: Lloyd-Max bits per coordinate, 1..4 on the GPU path (TQ §Stage 1).
 * m: QJL rows (TQ §Stage 2), 0 (MSE-only, e.g. values) or m_pad == d_pad.
 * seed_pi / seed_s seed the Gaussian matrices of Pi and S (SplitMix64 used as
 * a counter-based generator, Box-Muller normals, row-major fill). */
typedef struct {
  int32_t d;
  int32_t bits;
  int32_t m;
  uint64_t seed_pi;
  uint64_t seed_s;
} tq_params;

typedef struct tq_codebook tq_codebook;

/* Sizes of the packed format for a codebook (see "Packed record layout"). */
typedef struct {
  int32_t d_pad;
  int32_t m_pad;
  int32_t words_per_chunk;   /* 32-bit words in each of the 4 chunks */
  int32_t code_bytes;        /* bytes of one record (16 * words_per_chunk) */
  int32_t norm_bytes;        /* bytes of one norm slot: 4 with QJL, else 2 */
  int32_t head_block_bytes;  /* page_tokens records + norm slots, 16-aligned */
  int64_t page_bytes;        /* n_kv_heads * head_block_bytes */
} tq_layout_info;

/* A paged cache of packed records, owned by the caller.  pages: device,
 * n_pages * page_bytes bytes, 16-byte aligned.  block_table: device int32
 * [batch, max_pages_per_seq].  page_tokens: a power of two, 16..256.
 * error_word: device uint32 or NULL.  Every int32 / uint32 / float array the
 * entry points take (block_table, error_word, start_pos, ctx_len, weights,
 * out) must be aligned to its element size; a misaligned one is TQ_EINVAL. */
typedef struct {
  void* pages;
  int64_t n_pages;
  int32_t page_tokens;
  int32_t n_kv_heads;
  const int32_t* block_table;
  int64_t max_pages_per_seq;
  uint32_t* error_word;
} tq_cache;

/* Builds the codebook on the host in float64 and uploads its constant tables
 * to the current device (synchronously): Pi = Q of the QR of the seeded
 * Gaussian d x d matrix with diag(R) > 0 (TQ §Stage 1); S, the seeded
 * Gaussian m x d matrix (TQ §Stage 2); the Lloyd-Max centroids and midpoint
 * boundaries of the Beta((d-1)/2,(d-1)/2) law by numerical integration
 * (TQ §Stage 1).  *out receives a handle owned by the caller. */
tq_status tq_codebook_build(const tq_params* params, tq_codebook** out);

/* Same as tq_codebook_build but builds only the float64 host tables (no
 * device is touched).  Such a codebook can be exported and inspected, and is
 * rejected with TQ_EINVAL by the calls that launch kernels. */
tq_status tq_codebook_build_host(const tq_params* params, tq_codebook** out);

/* Releases the handle and its device tables.  NULL is allowed. */
void tq_codebook_free(tq_codebook* cb);

/* Copies the float64 host tables of a codebook into caller arrays (each may
 * be NULL): pi [d*d] row-major (y = Pi x), s [m*d], centroids [2^bits]
 * ascending, boundaries [2^bits - 1]. */
tq_status tq_codebook_export(const tq_codebook* cb, double* pi, double* s,
                             double* centroids, double* boundaries);

/* Copies the reconstruction levels the library decodes with (host, 2^bits
 * doubles, ascending) into `levels`, and their scale exponent into
 * *scale_exp (may be NULL).  TQ §Stage 1 gives the Lloyd-Max centroids; how
 * they are stored is this library's choice: for bits <= 3 every level is an
 * 8-bit integer k times 2^-f (k = round(c 2^f), half to even, f the largest
 * integer with max|c| 2^f <= 127; *scale_exp = f), so that a decoded
 * coordinate is one signed byte; for bits = 4 the levels are the fp16
 * roundings of the centroids (*scale_exp = INT32_MIN).  The residual of the
 * QJL stage, the logits and the value path all use these levels.  Works on
 * host-only codebooks too. */
tq_status tq_codebook_levels(const tq_codebook* cb, double* levels, int32_t* scale_exp);

/* Fills *info with the packed-format sizes for this codebook. */
tq_status tq_layout(const tq_codebook* cb, int32_t page_tokens, int32_t n_kv_heads,
                    tq_layout_info* info);

/* Online quantize-and-append (TQ §Stage 1 + §Stage 2; TQ §How to implement:
 * quantization on every cache update).  x: device [batch, n_kv_heads, n_new,
 * d] of dtype.  start_pos: device int32 [batch], position of x[b, :, 0].
 * For every vector: ||x|| (fp32, stored fp16), y = Pi x / ||x||, indices
 * by threshold search over the Lloyd-Max boundaries, and when m > 0 the
 * residual r = y - c[idx] (rotated space; c = the reconstruction levels, see tq_codebook_levels), ||r|| (fp16) and the m signs of
 * S r; the packed record is written into its page slot.  Each token owns its
 * bytes, so appends that start inside a page are safe; calls on one stream
 * are ordered.  Returns TQ_EINVAL for bad shapes, dtype or pointers. */
tq_status tq_quantize_append(const tq_codebook* cb, const void* x, tq_dtype dtype,
                             int64_t batch, int32_t n_kv_heads, int64_t n_new,
                             const int32_t* start_pos, const tq_cache* cache,
                             void* stream);

/* The keys and the values of one cache update (TQ §How to implement:
 * quantize on every cache update), equivalent to tq_quantize_append(key_cb,
 * k, ...) followed by tq_quantize_append(value_cb, v, ...) with the same
 * dtype, shape and start_pos.  k, v: device [batch, n_kv_heads, n_new, d].
 * For d = 128 keys with a sketch (m_pad = 128), values without one, and at
 * most 256 vectors of each (decode steps), both are coded by one kernel
 * launch (a cluster of 8 CTAs per vector); other shapes take the two calls. */
tq_status tq_quantize_append_kv(const tq_codebook* key_cb, const void* k, const tq_codebook* value_cb,
                                const void* v, tq_dtype dtype, int64_t batch, int32_t n_kv_heads, int64_t n_new,
                                const int32_t* start_pos, const tq_cache* key_cache, const tq_cache* value_cache,
                                void* stream);

/* Workspace (device bytes) that tq_logits needs for these sizes. */
size_t tq_logits_workspace_bytes(const tq_codebook* cb, int64_t batch, int32_t n_kv_heads,
                                 int32_t n_q_heads);

/* Fused logits from the packed keys (TQ §Stage 2 and §How it works): for
 * query head hq of sequence b (KV head hq / (n_q_heads / n_kv_heads)) and
 * every key position t < ctx_len[b],
 *   out[(b * n_q_heads + hq) * out_stride + t] = ||k|| ( <Pi q, c[idx]>
 *        + sqrt(pi/2)/m ||r|| <S q, sign> )   (sign_i = -1 where the bit is 1)
 * with the query rotated once.  No 1/sqrt(d) scale, no softmax.  Positions
 * t >= ctx_len[b] are not written.  q: device [batch, n_q_heads, d] of dtype.
 * ctx_len: device int32 [batch], each <= max_ctx <= out_stride.  workspace:
 * device, at least tq_logits_workspace_bytes(), 16-byte aligned (the rotated,
 * sketched queries as tensor-core fragments; every call rewrites what it
 * reads, so it needs no clearing).  Two kernel launches: the query
 * preparation, then the logits kernel by programmatic dependent launch (it
 * streams the cache while the queries are prepared). */
tq_status tq_logits(const tq_codebook* cb, const tq_cache* cache, const void* q,
                    tq_dtype dtype, int64_t batch, int32_t n_q_heads,
                    const int32_t* ctx_len, int64_t max_ctx, float* out,
                    int64_t out_stride, void* workspace, size_t workspace_bytes,
                    void* stream);

/* Workspace (device bytes) that tq_logits_topk needs for these sizes (0 for
 * bad arguments, k outside [1, 32]). */
size_t tq_logits_topk_workspace_bytes(const tq_codebook* cb, int64_t batch, int32_t n_kv_heads,
                                      int32_t n_q_heads, int64_t max_ctx, int32_t k);

/* The k best logits per query head (TQ §Benchmarks: nearest-neighbour search
 * scored from the codes, top-k recall; the estimate is tq_logits'): for query
 * head hq of sequence b, the k largest L[b, hq, t] over t < ctx_len[b], best
 * first, equal scores in increasing t:
 *   top_scores[(b * n_q_heads + hq) * k + j], top_idx[...] = t
 * (score -inf and index -1 past the ctx_len[b] found).  Meant for many query
 * heads per KV head (queries are taken 64 at a time): the codes of 128 keys
 * are decoded once per 64 queries into tensor memory and scored against them
 * on the tcgen05 tensor cores, and the epilogue keeps each query's best k.
 * The scores equal tq_logits' estimate up to fp32 rounding (the query enters
 * as fp16 hi + lo for the codebook term and fp16 for the sketch term); ties
 * between scores that differ by rounding may rank either way.  q: device
 * [batch, n_q_heads, d] of dtype; ctx_len: device int32 [batch]; top_scores /
 * top_idx: device [batch, n_q_heads, k]; k in [1, 32]; pages of at least 16
 * tokens (TQ_EUNSUPPORTED otherwise).  workspace: device, at least
 * tq_logits_topk_workspace_bytes(), 256-byte aligned.  Three kernel launches
 * (query operands, scoring, merge of the CTAs' lists); a bad page is
 * reported in the cache's error word and its keys are not ranked. */
tq_status tq_logits_topk(const tq_codebook* cb, const tq_cache* cache, const void* q, tq_dtype dtype,
                         int64_t batch, int32_t n_q_heads, const int32_t* ctx_len, int64_t max_ctx, int32_t k,
                         float* top_scores, int32_t* top_idx, void* workspace, size_t workspace_bytes,
                         void* stream);

/* tq_logits for callers that cannot allocate device memory where they call
 * it (a serving loop whose memory is an arena carved up at start-up, a host
 * framework or plugin interface that hands an operator no workspace, code
 * that must not call cudaMalloc/cudaFree on its hot path because those can
 * block or synchronize the device).  The method has no counterpart: this is
 * an interface variant, not a step of the method.  Arguments and results are
 * those of tq_logits; the workspace comes from a file-scope device array of
 * tq_logits_noalloc_scratch_bytes() = 1 MiB that every device loading the
 * library holds until exit.  A request needing more than that
 * (tq_logits_workspace_bytes() > 1 MiB) returns TQ_EINVAL with nothing
 * launched.  Every call on a device shares the array, so calls that overlap
 * on the GPU race; order them on one stream (or with events).  Each call
 * rewrites all of the scratch it reads, so nothing needs clearing.  The first
 * call on a device looks up the array's address (cudaGetSymbolAddress, with
 * that device current) and keeps it for the life of the process, so a device
 * reset (cudaDeviceReset, or destroying and re-creating the primary context)
 * while the library is loaded is not supported: the kept address would be
 * stale.  Allocates nothing. */
tq_status tq_logits_noalloc(const tq_codebook* cb, const tq_cache* cache, const void* q,
                            tq_dtype dtype, int64_t batch, int32_t n_q_heads,
                            const int32_t* ctx_len, int64_t max_ctx, float* out,
                            int64_t out_stride, void* stream);

/* Size in bytes of the static scratch behind tq_logits_noalloc. */
size_t tq_logits_noalloc_scratch_bytes(void);

/* Workspace (device bytes) that tq_dequant_values needs for these sizes. */
size_t tq_values_workspace_bytes(const tq_codebook* cb, int64_t batch, int32_t n_kv_heads,
                                 int32_t n_q_heads, int64_t max_ctx);

/* Value path from packed records ("TurboQuant explained", §Stage 1: the
 * values are coded by the MSE stage alone -- no QJL sketch -- and read back
 * as the rotated-back centroid vector, v_hat = ||v|| Pi^T c[idx], c the
 * reconstruction levels).  Mode A (weights == NULL): out device [batch, n_kv_heads,
 * out_stride, d] of out_dtype receives v_hat for t < ctx_len[b].  Mode B
 * (weights != NULL, device fp32 [batch, n_q_heads, w_stride]): out device
 * fp32 [batch, n_q_heads, d] receives sum_{t < ctx_len[b]} weights[b,hq,t]
 * v_hat_t, accumulated in the rotated space and rotated back once.  For mode B
 * out_dtype must be TQ_F32 and out_stride is ignored; with max_ctx = 0 out is
 * cleared (every context is empty).  workspace: device, at least
 * tq_values_workspace_bytes() (0 is enough for mode A).  out, weights and
 * workspace must be aligned to their element size (TQ_EINVAL otherwise). */
tq_status tq_dequant_values(const tq_codebook* cb, const tq_cache* cache,
                            const float* weights, int64_t w_stride, int64_t batch,
                            int32_t n_q_heads, const int32_t* ctx_len, int64_t max_ctx,
                            void* out, tq_dtype out_dtype, int64_t out_stride,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Workspace (device bytes) that tq_attend needs for these sizes (either of
 * its two forms; the page sizes, which choose the form, are not arguments). */
size_t tq_attend_workspace_bytes(const tq_codebook* key_cb, const tq_codebook* value_cb, int64_t batch,
                                 int32_t n_kv_heads, int32_t n_q_heads, int64_t max_ctx);

/* Decode attention from the packed caches (TQ §How it works: logits from the
 * compressed keys, values from their codes): for query head hq of sequence b
 * (KV head hq / (n_q_heads / n_kv_heads)),
 *   out[b, hq, :] = sum_{t < ctx_len[b]} softmax_t(scale * L[b, hq, t]) v_hat_t
 * with L the tq_logits estimate and v_hat_t = ||v_t|| Pi_v^T c[idx_t] (the
 * value codebook's reconstruction); a row with ctx_len[b] = 0 is all zeros
 * (with max_ctx = 0 the whole of out is cleared and nothing else runs).
 * key_cb / key_cache and value_cb / value_cache as for tq_logits and
 * tq_dequant_values (same d and n_kv_heads; value_cb has m = 0).  q: device
 * [batch, n_q_heads, d] of dtype; out: device fp32 [batch, n_q_heads, d];
 * scale: usually 1/sqrt(d).  workspace: device, at least
 * tq_attend_workspace_bytes(), 256-byte aligned.  A token whose key or value
 * page is out of range is left out of the softmax (and reported in that
 * cache's error word).  Kernels on the stream: for d <= 128 and caches with
 * equal page sizes, the fused split-K form (query preparation, one pass over
 * both caches with an online softmax writing per-CTA partials, a merge that
 * applies Pi_v^T); otherwise query preparation, logits, row softmax, value
 * accumulation and its finish. */
tq_status tq_attend(const tq_codebook* key_cb, const tq_cache* key_cache, const tq_codebook* value_cb,
                    const tq_cache* value_cache, const void* q, tq_dtype dtype, int64_t batch,
                    int32_t n_q_heads, const int32_t* ctx_len, int64_t max_ctx, float scale, float* out,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Self-test of the device-side failure path: one small kernel waits on an
 * mbarrier that nothing completes, with the bounded wait every streaming
 * kernel uses; after about a second the wait gives up and the kernel ORs
 * TQ_DEV_ERR_TIMEOUT into *error_word (device, uint32) and returns.  No
 * fault, trap or hang; asynchronous on the stream.  TQ_EINVAL for a NULL
 * error_word.  The method has no counterpart: this checks the library. */
tq_status tq_selftest_wait_timeout(uint32_t* error_word, void* stream);

/* Host-side tables of the recursive polar form of stage 1 ("TurboQuant
 * explained", §Stage 1, PolarQuant paragraph): the rotated unit vector's
 * coordinates are paired recursively into polar form, level 1 giving angles
 * atan2(u[2i+1], u[2i]) in [-pi, pi] and level l > 1 angles atan2(rho[2i+1],
 * rho[2i]) in [0, pi/2] of the previous level's radii.  For a uniform unit
 * vector level-1 angles are uniform and a level-l angle has sin^2 phi ~
 * Beta(k/2, k/2), k = 2^(l-1).  Writes the Lloyd-Max quantizer of that law
 * with 2^bits levels: centroids (host, 2^bits doubles, ascending, symmetric
 * about the middle of the support), boundaries (host, 2^bits - 1 midpoints,
 * or NULL) and the mean squared angle error (or NULL).  level in [1, 8],
 * bits in [1, 8] (TQ_EINVAL / TQ_EUNSUPPORTED otherwise).  No GPU needed. */
tq_status tq_polar_angle_codebook(int32_t level, int32_t bits, double* centroids, double* boundaries,
                                  double* distortion);

/* ---- the recursive polar form of stage 1 ("TurboQuant explained", §Stage 1,
 * PolarQuant paragraph; §Stage 2 on top) ------------------------------------
 * The rotated unit vector u = Pi x / ||x|| is paired recursively into polar
 * form: level 1 angles atan2(u[2i+1], u[2i]) in [-pi, pi], level l > 1 angles
 * atan2(rho[2i+1], rho[2i]) in [0, pi/2] of the previous level's radii, d - 1
 * angles in all (d a power of two).  Each angle is coded with `bits` bits by
 * the Lloyd-Max quantizer of its level's law (tq_polar_angle_codebook; a tie
 * goes to the upper cell); ||x|| is kept in fp16.  With m > 0 the residual
 * r = u - Pi^T u_hat (original space, u_hat the inverse recursion over the
 * centroids) keeps the m signs of S r and fp16 ||r||.  Pi and S come from the
 * same seeds and generators as tq_codebook_build's.  The records are a plain
 * array (no pages):
 *   words [0, CW): angle codes, CW = ceil((d - 1) bits / 32), angle a (level 1
 *                  first, then by index) at bits a bits .. of the little-endian
 *                  word stream;
 *   words [CW, CW + m/32): sign bits, bit i set where (S r)_i < 0;
 *   word CW + m/32: fp16 ||x|| (low half), fp16 ||r|| (high half, 0 when m = 0);
 *   padded to tq_polar_record_bytes() (a multiple of 16). */
typedef struct tq_polar tq_polar;

/* Builds the polar codec (host float64 tables, device fp32 copies).  d in {64,
 * 128, 256}, bits in [1, 4], m a multiple of 32 in [0, d] (TQ_EUNSUPPORTED
 * otherwise); needs a CUDA device.  Free with tq_polar_free. */
tq_status tq_polar_build(int32_t d, int32_t bits, int32_t m, uint64_t seed_pi, uint64_t seed_s, tq_polar** out);
void tq_polar_free(tq_polar* p);
/* Bytes of one record (0 for NULL). */
int32_t tq_polar_record_bytes(const tq_polar* p);

/* Encodes x (device [n, d] of dtype) into records (device [n] records,
 * 16-byte aligned).  A norm that overflows fp16 sets TQ_DEV_ERR_RANGE in
 * *error_word (device uint32, may be NULL).  One kernel launch. */
tq_status tq_polar_encode(const tq_polar* p, const void* x, tq_dtype dtype, int64_t n, void* records,
                          uint32_t* error_word, void* stream);

/* Workspace (device bytes) of tq_polar_logits for nq queries. */
size_t tq_polar_logits_workspace_bytes(const tq_polar* p, int32_t nq);

/* Logits from the polar records without reconstructing the keys:
 *   out[j * out_stride + t] = ||x_t|| ( <Pi q_j, u_hat_t> + sqrt(pi/2)/m ||r_t|| <S q_j, sign_t> )
 * for every query j < nq (device [nq, d] of dtype) and record t < n; the first
 * term folds the rotated query bottom-up through the angle tree (2 (d - 1)
 * FMAs per key and query).  workspace: device, at least
 * tq_polar_logits_workspace_bytes(), 16-byte aligned.  Two kernel launches. */
tq_status tq_polar_logits(const tq_polar* p, const void* records, int64_t n, const void* q, tq_dtype dtype,
                          int32_t nq, float* out, int64_t out_stride, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Message for the last failed call on this thread ("" if none). */
const char* tq_last_error(void);

/* Layout version of the packed records this library writes and reads. */
int32_t tq_layout_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TQ_H_ */
