/*
 * li.h -- C ABI of libli, the B200 (sm_100a) LatentIndex decode indexer.
 *
 * What it computes.  LatentIndex (paperlayer summary of arXiv 2610.04635,
 * "LatentIndex: Cross-Layer Sharing with Layer-Specific Selection for Sparse
 * Attention") keeps ONE indexer cache per group of G layers: a latent c_s
 * built by the group's first ("anchor") layer from its hidden state (Sec. 3.1).
 * Every layer l of the group owns a decoder W_K^l; at inference the decoder is
 * absorbed into the layer's query, qt_{t,h} = W_K^{l T} q_{t,h}, so the layer
 * scores the shared latent directly (Sec. 3.1, Sec. B.2).  The score is the
 * DSA-style head-weighted ReLU form
 *
 *     score(t, s) = sum_h w_{t,h} * max(0, qt_{t,h} . c_s + beta_{t,h})
 *
 * (beta = q . b_K for decoders with an output bias, Sec. A.3; NULL otherwise),
 * and each layer keeps its own top-k tokens (Sec. 3.1, up to 2048 per query,
 * Sec. 4.1).  In hierarchical selection (HS) the anchor proposes its top-B
 * candidates and each follower rescores only those (Sec. 3.2, Sec. C.4).  A
 * DSA-style comparison path scores per-layer key caches with the raw query.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.  Every pointer argument is a DEVICE pointer unless marked "host".
 *   The caller owns all memory, including the workspace; the library never
 *   allocates device memory.  A workspace must be at least
 *   li_workspace_bytes(...) bytes, 256-byte aligned, and zero-filled once
 *   before its first use; after that the library keeps it consistent.  Its
 *   first 4 bytes are the device status word (see li_device_status).
 * Streams.  `stream` is a cudaStream_t (NULL = legacy default stream).  Every
 *   call only enqueues work on that stream and returns; none synchronises,
 *   except li_device_status.  A li_ctx must not be used by two host threads
 *   at once.  Two calls that share a workspace must be ordered on the GPU.
 * Errors.  Host-detected errors (bad arguments, shapes, dtypes, alignment, a
 *   short workspace) return before anything is enqueued and leave every
 *   output untouched; li_last_error(ctx) then describes the problem.  A
 *   failing CUDA call returns LI_ERR_CUDA.  Errors found on the device (an
 *   append past capacity, a candidate index outside the valid prefix, a
 *   bounded wait that ran out) are recorded in the workspace's status word
 *   and reported by li_device_status.  No C++ exception crosses this ABI.
 * Selections.  A selection of budget k over n valid positions returns the
 *   k_eff = min(k, n) positions with the largest scores, ordered by (score
 *   descending, position ascending) to decide who is in, and written in
 *   ascending position order; slots k_eff..k-1 hold -1 (indices) and -inf
 *   (scores).  -0.0 ranks equal to +0.0, and a selected -0.0 score may be
 *   returned as +0.0.  NaN scores are invalid input.
 * Valid prefix.  In decode (q_pos == NULL) the query of sequence b sees
 *   positions [0, lengths[b]) -- the current token is appended before it
 *   scores.  With q_pos, query (b, t) sees [0, min(lengths[b], q_pos[b][t]+1)).
 */
#ifndef LI_H
#define LI_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LI_API __attribute__((visibility("default")))
#else
#define LI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LI_OK = 0,
  LI_ERR_ARG = 1,              /* null pointer or out-of-range scalar          */
  LI_ERR_SHAPE = 2,            /* unsupported or inconsistent sizes            */
  LI_ERR_DTYPE = 3,            /* dtype not supported for this operand         */
  LI_ERR_ALIGN = 4,            /* pointer or row not 16-byte aligned           */
  LI_ERR_WORKSPACE = 5,        /* workspace missing, short or misaligned       */
  LI_ERR_CAPACITY = 6,         /* (device) append past the cache capacity      */
  LI_ERR_CUDA = 7,             /* a CUDA runtime / driver call failed          */
  LI_ERR_DEVICE_TIMEOUT = 8,   /* (device) a bounded wait ran out              */
  LI_ERR_UNSUPPORTED = 9,      /* valid request this build does not implement  */
  LI_ERR_INDEX = 10            /* (device) candidate index outside the prefix  */
} li_status;

typedef enum { LI_F32 = 0, LI_BF16 = 1, LI_E4M3 = 2 } li_dtype;

/* Opaque host-side context: device properties, cached driver entry points,
 * the last error message, the wait limit and the optional launch profile.
 * It owns no device memory. */
typedef struct li_ctx li_ctx;

/* A per-group latent cache (LatentIndex) or a per-layer key cache (DSA path).
 * data    [batch][capacity][dim] elements of `dtype`, row-major; each row must
 *         be a multiple of 16 bytes and `data` 16-byte aligned.
 * scale   [batch][capacity] fp32 per-token dequantisation scale (LI_E4M3
 *         only, NULL otherwise): element value = scale[b][s] * e4m3 code.
 *         Every scale of a valid row must be finite and >= 0: the scan takes
 *         it outside the ReLU (max(0, a x) = a max(0, x) only for a >= 0).
 *         The library's own appends write amax / 448, or 1 for a zero row.
 * lengths [batch] int32 valid rows per sequence (read and advanced on the
 *         device by li_append_latent).
 * dim: multiple of 8 (F32), 16 (BF16) or 32 (E4M3), at most 256.  Scanning
 * an E4M3 cache (li_score_topk, li_hs_anchor_candidates, li_dsa_score_topk)
 * needs capacity % 4 == 0 and a 16-byte aligned scale array.
 * scale_split: 0 for one scale per row.  For E4M3 caches, a value in
 *         (0, dim) that is a multiple of 32 selects segmented fp8 (Sec. B.2,
 *         Sec. C.1): two scales per row, scale [batch][capacity][2], the
 *         first for elements [0, scale_split) (the rotary branch) and the
 *         second for [scale_split, dim) (the NoPE branch).  Must be 0 for
 *         F32 and BF16 caches.                                            */
typedef struct {
  void* data;
  float* scale;
  int32_t* lengths;
  int32_t batch;
  int32_t capacity;
  int32_t dim;
  li_dtype dtype;
  int32_t scale_split;
} li_cache;

/* The queries of one layer for every sequence of the batch.
 * q       [batch][T][H][dim] of `dtype`: the absorbed query qt for LatentIndex
 *         (li_absorb_query output) or the raw query for the DSA path.  dtype
 *         must match the cache: F32 with F32 (tf32 tensor cores), BF16 with
 *         BF16, E4M3 with E4M3.  16-byte aligned.
 * q_scale [batch][T][H] fp32 per-(token, head) dequantisation scale of an
 *         E4M3 query; NULL otherwise.  Finite and >= 0 (without beta it is
 *         folded into the head weight, outside the ReLU).
 * beta    [batch][T][H] fp32 decoder-bias term added before the ReLU, or NULL.
 * w       [batch][T][H] fp32 head weights.
 * T       query tokens per sequence (1 = decode).  H heads, 1..256.
 * q_pos   [batch][T] int32 causal positions, or NULL for decode.           */
typedef struct {
  const void* q;
  li_dtype dtype;
  const float* q_scale;
  const float* beta;
  const float* w;
  int32_t T;
  int32_t H;
  const int32_t* q_pos;
} li_query;

/* ------------------------------------------------------------------ setup */

/* Create a context bound to CUDA device `device` (host-side state only).
 * Fails with LI_ERR_UNSUPPORTED unless the device is compute capability 10.0. */
LI_API li_status li_create(li_ctx** ctx, int device);
LI_API li_status li_destroy(li_ctx* ctx);
/* Message of the last host-detected error on this context ("" if none).
 * The string is owned by the context and valid until its next call. */
LI_API const char* li_last_error(const li_ctx* ctx);
LI_API const char* li_status_string(li_status s);

/* Bytes of workspace any call on caches of `batch` sequences with `T` query
 * tokens each, `capacity` rows, budget k and HS budget B (0 if unused) needs.
 * A workspace of this size serves every entry point for those sizes. */
LI_API size_t li_workspace_bytes(const li_ctx* ctx, int batch, int T, int capacity, int H, int k, int B);

/* Reads the device status word of `ws` after synchronising `stream`, stores
 * it in *out (host) and clears it.  Returns LI_OK or LI_ERR_CUDA. */
LI_API li_status li_device_status(li_ctx* ctx, const void* ws, void* stream, li_status* out);

/* Upper bound, in nanoseconds, of every wait inside the library's kernels
 * (default 2e9 = 2 s).  When a wait runs out the kernel records
 * LI_ERR_DEVICE_TIMEOUT, drains its own copies in flight, frees its tensor
 * memory and returns.  0 makes every wait that is not already satisfied
 * when it starts give up at once (a way to exercise that path).  The
 * outputs of a call whose wait ran out are undefined; read the status with
 * li_device_status before the workspace's next use. */
LI_API li_status li_set_wait_limit(li_ctx* ctx, uint64_t ns);

/* ------------------------------------------------------------- a1: append */

/* Latent (or key) construction and append (LatentIndex summary, Sec. 3.1:
 * the anchor's hidden states build the shared latent once per token; the
 * DSA path builds one key per layer the same way).  For every sequence b and
 * new token t < T: c = W_down h[b][t] (fp32 accumulation), stored as the
 * cache dtype (F32 as is; BF16 round-to-nearest-even; E4M3 with
 * scale = amax|c| / 448 in fp32 division (1 if amax = 0) and codes
 * e4m3_satfinite(c_i / scale)), into row lengths[b] + t; then
 * lengths[b] += T.
 * h       [batch][T][d_model] of h_dtype (F32 or BF16).
 * W_down  [cache->dim][d_model] of h_dtype, row-major; or NULL, in which case
 *         h is already [batch][T][cache->dim] fp32 and is stored as is.
 * If lengths[b] + T > capacity nothing is written for b, lengths[b] is left
 * unchanged and the status word records LI_ERR_CAPACITY. */
LI_API li_status li_append_latent(li_ctx* ctx, const li_cache* cache, const void* h, li_dtype h_dtype,
                           int d_model, const void* W_down, int T, void* ws, size_t ws_bytes,
                           void* stream);

/* The two-branch latent (Sec. 3.1: RoPE and NoPE branches concatenated and
 * cached once per group; Sec. A.2: the rotary branch is rotated before
 * caching; Sec. A.4: one or more complex sources per rotary frequency;
 * Sec. D.2: LayerNorm on the NoPE branch only).  li_append_latent_ex applies
 * these to each new row after c = W_down h and before quantisation.
 * Rotary branch: elements [rope_offset, rope_offset + rope_dim) hold
 *   rope_dim / 2 complex slots, slot p = (x[2p], x[2p+1]) counted from
 *   rope_offset, of frequency f = p / rope_sources.  The row written at
 *   cache row s (its sequence position) has slot p multiplied by
 *   exp(i s inv_freq[f]): x' = x cos - y sin, y' = x sin + y cos, with the
 *   angle formed exactly and its cosine and sine taken in double precision,
 *   rounded to fp32.  rope_dim = 0 disables it; otherwise rope_offset and
 *   rope_dim are even, rope_dim is a multiple of 2 * rope_sources and
 *   inv_freq is a device array of rope_dim / (2 rope_sources) fp32.
 *   Decoders must be frequency-wise complex on this branch (each layer's
 *   rotary key slot f a complex combination of the sources of frequency f),
 *   so that absorbing them into post-RoPE queries scores the rotated latent
 *   exactly; the native key layout they target is the caller's choice.
 * NoPE branch: elements [norm_offset, norm_offset + norm_dim) are replaced
 *   by (x - mean) / sqrt(var + norm_eps) * gamma + beta (biased variance,
 *   fp32, correctly rounded division and square root); gamma and beta are
 *   device arrays of norm_dim fp32, or NULL for 1 and 0.  norm_dim = 0
 *   disables it.
 * The two ranges must lie inside the row and must not overlap.            */
typedef struct {
  int32_t rope_offset;
  int32_t rope_dim;
  int32_t rope_sources;
  const float* inv_freq;
  int32_t norm_offset;
  int32_t norm_dim;
  const float* norm_gamma;
  const float* norm_beta;
  float norm_eps;
} li_latent_transform;

/* li_append_latent with the two-branch transforms; tf NULL is
 * li_append_latent.  Errors: LI_ERR_ARG / LI_ERR_SHAPE for an invalid
 * transform (checked on the host before anything is enqueued).           */
LI_API li_status li_append_latent_ex(li_ctx* ctx, const li_cache* cache, const void* h, li_dtype h_dtype,
                              int d_model, const void* W_down, int T, const li_latent_transform* tf,
                              void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------- a2: absorb */

/* Query-side decoder absorption (LatentIndex summary, Sec. 3.1, Sec. A.2,
 * Sec. B.2): for each of n_tok query tokens and H heads,
 * qt[t][h][i] = sum_j W_K[h][j][i] * q[t][h][j]  (fp32 accumulation) and, if
 * b_K is given, beta[t][h] = sum_j q[t][h][j] * b_K[h][j].
 * q       [n_tok][H][d_k] of q_dtype (F32 or BF16).
 * W_K     decoder of layer l, [d_k][d_c] of q_dtype, row-major (key = W_K c),
 *         head h at W_K + h * W_K_head_stride elements (0 = shared by all
 *         heads); or NULL for the identity (d_c == d_k: plain conversion).
 * b_K     [d_k] fp32 per head at b_K + h * b_K_head_stride, or NULL.
 * out_dtype F32, BF16 (round-to-nearest-even) or E4M3: then q_abs_scale
 *         [n_tok][H] receives scale = amax_i |qt| / 448 (1 if 0) and q_abs the
 *         codes e4m3_satfinite(qt_i / scale).
 * q_abs   [n_tok][H][d_c] of out_dtype.  beta [n_tok][H] fp32 or NULL.     */
LI_API li_status li_absorb_query(li_ctx* ctx, const void* q, li_dtype q_dtype, int n_tok, int H, int d_k,
                          const void* W_K, int64_t W_K_head_stride, const float* b_K,
                          int64_t b_K_head_stride, int d_c, li_dtype out_dtype, void* q_abs,
                          float* q_abs_scale, float* beta, void* stream);

/* Absorption for a whole group at once (training-aware instantiation,
 * Sec. D.2: every layer's query comes from the anchor's hidden state, so the
 * G layers' queries exist together).  For sequence b, layer l < G and head
 * h: q_abs[b][l][h] = W_K[l]^T q[b][l][h], with the arithmetic and rounding
 * of li_absorb_query with a shared decoder, written stacked so that the G
 * layers are the T = G query rows of one li_score_topk call (one pass over
 * the latent for the group).  One launch for all layers.
 * q       [batch][G][H][d_k] of q_dtype (F32 or BF16).
 * W_K     host array of G device pointers, each a decoder [d_k][d_c] of
 *         q_dtype, 16-byte aligned (d_k * d_c * element size a multiple of
 *         16); shared by the heads of its layer; no decoder bias.
 * q_abs   [batch][G][H][d_c] of out_dtype; q_abs_scale [batch][G][H] fp32
 *         for E4M3 output (as li_absorb_query).
 * Needs 1 <= G <= 8, d_c even, batch * H <= 65535 * 2.                      */
LI_API li_status li_absorb_query_group(li_ctx* ctx, const void* q, li_dtype q_dtype, int batch, int G, int H,
                                int d_k, const void* const* W_K, int d_c, li_dtype out_dtype,
                                void* q_abs, float* q_abs_scale, void* stream);

/* ------------------------------------------------ a3 + a4: scan and select */

/* Full-prefix LatentIndex scoring and per-layer selection (Sec. 3.1): scores
 * every valid position of every query with the head-weighted ReLU form, on
 * tensor cores, without per-head scores leaving the chip, then selects the
 * top-k per query row.
 * out_idx   [batch][T][k] int32 (see "Selections").
 * out_score [batch][T][k] fp32 selected scores, or NULL.
 * scores_dump [batch][T][capacity] fp32, or NULL: receives every valid score
 *           (positions past the valid prefix are not written).
 * The T query rows of a sequence share every read of the cache: up to
 * 256 / H of them go into one MMA.  Stacking the G layers' absorbed decode
 * queries of a group as T = G rows (possible when all of them exist at
 * once, as in the training-aware instantiation of Sec. D.2, where every
 * layer's query comes from the anchor's hidden state) scores the whole
 * group with one pass over the latent; each row's scores and selection are
 * the same as with that row alone.                                        */
LI_API li_status li_score_topk(li_ctx* ctx, const li_cache* cache, const li_query* q, int k,
                        int32_t* out_idx, float* out_score, float* scores_dump, void* ws,
                        size_t ws_bytes, void* stream);

/* --------------------------------------------------------- a5: HS anchor */

/* HS step 1 (Sec. 3.2, Sec. C.4): the anchor scores its full prefix and
 * proposes cand = its top-B_eff positions, B_eff = min(B, valid length),
 * ascending, -1 padded, with cand_n = B_eff; anchor_idx = its own top-k of
 * the same scores (a subset of cand).  Requires B >= k.
 * cand [batch][T][B], cand_n [batch][T], anchor_idx [batch][T][k] int32;
 * anchor_score [batch][T][k] fp32 or NULL; scores_dump as li_score_topk. */
LI_API li_status li_hs_anchor_candidates(li_ctx* ctx, const li_cache* cache, const li_query* q, int B,
                                  int k, int32_t* cand, int32_t* cand_n, int32_t* anchor_idx,
                                  float* anchor_score, float* scores_dump, void* ws,
                                  size_t ws_bytes, void* stream);

/* ------------------------------------------------------- a6: HS follower */

/* HS step 2 (Sec. 3.2, Sec. C.4): a follower layer gathers only the latent
 * rows cand[b][t][0 .. cand_n[b][t]) (ascending token positions from
 * li_hs_anchor_candidates of the same step), scores them with its own
 * absorbed query and selects its own top-min(k, cand_n) by (score desc,
 * token position asc), written as token positions ascending, -1 padded.
 * A candidate outside [0, lengths[b]) records LI_ERR_INDEX on the device
 * and is scored -inf.
 * scores_dump [batch][T][B] fp32 or NULL: score of candidate j at [..][j]. */
LI_API li_status li_hs_follower_refine(li_ctx* ctx, const li_cache* cache, const li_query* q,
                                const int32_t* cand, const int32_t* cand_n, int B, int k,
                                int32_t* out_idx, float* out_score, float* scores_dump, void* ws,
                                size_t ws_bytes, void* stream);

/* ------------------------------------------------------ a7: DSA-style path */

/* DSA-style per-layer comparison path (Sec. 1 and Sec. B.3: native DSA keeps a
 * key cache per layer and scans the full prefix at every layer): scores the
 * layer's own key cache (dim = d_k) with the raw query and selects top-k.
 * Arguments as li_score_topk; key caches are filled with li_append_latent
 * (W_down = the layer's key projection). */
LI_API li_status li_dsa_score_topk(li_ctx* ctx, const li_cache* key_cache, const li_query* q, int k,
                            int32_t* out_idx, float* out_score, float* scores_dump, void* ws,
                            size_t ws_bytes, void* stream);

/* ------------------------------------------- scan and select without workspace */

/* li_score_topk for callers that cannot hand the library any device memory
 * of their own.  This entry point has no counterpart in the LatentIndex
 * summary; it exists for the library's users.  Typical such callers: a
 * plugin or foreign-function boundary that receives only a stream and its
 * input and output buffers and has no allocator to draw a workspace from,
 * and latency-critical code that must not call an allocator (an allocation
 * can synchronise the device or fail under memory pressure at the worst
 * moment).
 *
 * Computes exactly what li_score_topk computes (same kernels, same results)
 * with out_idx [batch][T][k] and out_score [batch][T][k] (or NULL) as there,
 * but its scratch -- the device status word and the fp32 scores of every
 * query row -- is a fixed 8 MiB array inside the library image, not a
 * workspace: nothing is allocated, ever.
 * Limits: batch * T * capacity * 4 + 256 <= 8 MiB (e.g. 4 x 131072, 16 x
 *   32768), capacity <= 131072 and batch * T <= 65535; larger requests are
 *   refused with LI_ERR_WORKSPACE / LI_ERR_UNSUPPORTED before anything is
 *   enqueued (use li_score_topk with a workspace).
 * Setup: the first call on a device looks up the scratch's device address
 *   (once per device, with the context's device current; a failure returns
 *   LI_ERR_CUDA).  Make that first call before any stream capture begins.
 *   The address belongs to the device's current CUDA context: when that
 *   context changes (after cudaDeviceReset, say), the next call looks it up
 *   again, and that call too must come before any capture.
 * Zeroing: the scratch starts zeroed when the library is loaded; the status
 *   word is cleared by every call itself; the scores need no clearing.
 * Status: device-detected errors (a bounded wait that ran out) are written to
 *   device_status ([1] int32, device pointer) at the end of the call when it
 *   is not NULL; li_device_status does not see them.
 * Concurrency: every call on a device shares the one scratch array, so two
 *   calls whose work overlaps on the GPU (different streams, or different
 *   host threads without ordering) race and corrupt each other's results.
 *   Order them on one stream. */
LI_API li_status li_score_topk_static(li_ctx* ctx, const li_cache* cache, const li_query* q, int k,
                               int32_t* out_idx, float* out_score, int32_t* device_status, void* stream);

/* ----------------------------------------------------- a4: plain selection */

/* Top-k of `rows` fp32 rows (LatentIndex summary, Sec. 3.1: every layer
 * keeps its own top-k tokens; Sec. C.4: the budget is capped by the valid
 * prefix), by the rule under "Selections" above: row r is
 * scores[r * row_stride + 0 .. n_r), n_r = lengths ? lengths[r] : n
 * (lengths[r] is clamped to [0, n]; lengths is [rows] int32 or NULL).
 * out_idx [rows][k] int32, out_score [rows][k] fp32 or NULL.
 * ws: li_workspace_bytes(ctx, rows, 1, n, 1, k, 0) bytes.  Needs
 * rows <= 65535; rows longer than 131072 positions take a multi-kernel path.
 * Rows of up to 131072 positions are selected by one cluster of CTAs per
 * row that exchange digit counts through each other's shared memory; those
 * waits are bounded like every other.  A row whose wait ran out records
 * LI_ERR_DEVICE_TIMEOUT in the status word and leaves slots 0..k_eff-1
 * unwritten (the padding after them is written first). */
LI_API li_status li_topk(li_ctx* ctx, const float* scores, int rows, int n, int64_t row_stride,
                  const int32_t* lengths, int k, int32_t* out_idx, float* out_score, void* ws,
                  size_t ws_bytes, void* stream);

/* ------------------------------------------------------ selection quality */

/* Attention-mass recall of a selection (Sec. 4.1 and Table 1; Sec. D.3:
 * the mass a selection captures relative to each head's own top-K set, from
 * each layer's dense attention; Sec. C.2: averaged over heads; Sec. C.3:
 * mean-attention recall against the best shared size-K set of the head
 * average).  For query row r with valid prefix n_r (lengths[r], or N when
 * lengths is NULL) and head h:
 *   recall[r][h] = (sum of probs[r][h][s] over selected s = sel[r][j] with
 *                   0 <= s < n_r) / (sum of the min(K, n_r) largest
 *                   probs[r][h][s], s < n_r), or 0 when that sum is 0;
 *   mean_recall[r] = the same for pbar[r][s] = (sum_h probs[r][h][s]) / H.
 * The best sets are exact (the library's top-k); masses are summed in fp32.
 * probs [rows][H][N] fp32 device (entries at s >= n_r are ignored);
 * sel [rows][k] int32 device, -1 padded (a selection output);
 * recall [rows][H] fp32 device; mean_recall [rows] fp32 device or NULL.
 * ws: li_recall_workspace_bytes(ctx, rows, H, N, K) bytes, 256-byte
 * aligned, zero-filled before first use (status word at offset 0).
 * Needs rows * H <= 65535.  An IndexCache follower (Sec. 1, Sec. 2) reuses
 * the anchor's selection unchanged: pass the anchor's out_idx as sel.
 * Evaluation tooling: no counterpart on the decode path.                  */
LI_API size_t li_recall_workspace_bytes(const li_ctx* ctx, int rows, int H, int N, int K);
LI_API li_status li_attention_recall(li_ctx* ctx, const float* probs, int rows, int H, int N,
                              const int32_t* lengths, const int32_t* sel, int k, int K,
                              float* recall, float* mean_recall, void* ws, size_t ws_bytes,
                              void* stream);

/* ------------------------------------------------------------- profiling */

/* Launch profile: when enabled, every kernel launch (and workspace clear) of
 * the library is bracketed by CUDA events on the launching stream.
 * li_profile_read synchronises the recorded events and copies up to `max`
 * records into the host array `out` (in launch order), returning the number
 * of records in *count; li_profile_reset clears them.  Profiling adds two
 * event records per launch and is off by default; leave it off while a
 * stream is being captured into a CUDA graph. */
typedef struct {
  char kernel[48];       /* "scan", "gather", "topk_cluster", "append", ...    */
  float ms;              /* event-timed duration of the launch                   */
  int32_t grid;          /* CTAs launched (0 when not tracked)                   */
  int32_t block;         /* threads per CTA                                      */
  int32_t smem;          /* dynamic shared memory bytes per CTA                  */
} li_profile_record;

/* Diagnostic tile trace of the scoring kernels: when `buf` (device, at least
 * 8 * 64 * 8 * 8 = 32768 bytes) is set, every later scan / gather launch
 * writes, for each of its first 8 CTAs and their first 64 tiles, 8 uint64
 * SM clock-cycle stamps [cta][tile][event] (comparable within one CTA): 0 the loader got the tile's first
 * stage, 1 it issued the last one, 2 the MMA issuer saw the first stage
 * full, 3 it committed the tile, 4 the epilogue saw the accumulator full, 5
 * the epilogue released it.  NULL turns tracing off. */
LI_API li_status li_set_trace(li_ctx* ctx, void* buf, size_t bytes);

LI_API li_status li_profile_enable(li_ctx* ctx, int enable);
LI_API li_status li_profile_read(li_ctx* ctx, li_profile_record* out, int max, int* count);
LI_API li_status li_profile_reset(li_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* LI_H */
