/*
 * fh.h -- C ABI of the B200 FlashHead retrieval head.
 *
 * FlashHead replaces the dense LM classification head z = E h (FlashHead
 * write-up, www.framerc.cn/news/2430929, section 1.1) by a two-stage
 * retrieval (section 2.2.2: h -> centroid_scores -> top_p_clusters ->
 * token_scores):
 *
 *   1. centroid scores  s = C h over c balanced clusters (section 1.2.2),
 *      C in bf16, or in INT4 or INT8 with one bf16 scale per 32 elements
 *      (selective quantisation, section 1.2.4);
 *   2. probe selection: the p best clusters (multi-probe retrieval,
 *      section 1.2.2), or p clusters drawn by multinomial sampling at
 *      temperature T (section 1.2.3), realised as the top p of
 *      s/T + g with Gumbel noise g = -ln(-ln u) from caller uniforms u;
 *   3. gather of the b = v/c tokens of every chosen cluster through the
 *      dense cluster-to-token map C2T (balanced clustering, section 1.2.1);
 *   4. candidate logits z_t = E_t h for those p*b tokens (section 1.2.4,
 *      stage 2 in full precision);
 *   5. argmax, or a token drawn from softmax(z/T) over the candidates by
 *      inverse CDF with a caller uniform (section 1.2.3).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named as device pointers must be CUDA device memory of the
 *   current device; the caller owns them. E, C / C_q / C_scales and C2T are
 *   borrowed by fh_create and must outlive the handle.
 * - bf16 data is passed as `const void*` (IEEE bfloat16, row-major).
 * - Every call is asynchronous on `stream` (a cudaStream_t) unless stated
 *   otherwise. Argument errors are detected on the host and returned at
 *   once, before anything is enqueued. Errors found by a kernel (an
 *   out-of-range cluster id, a bounded wait that ran out) are recorded in a
 *   device status word and reported by fh_get_device_status().
 * - Ties: a ranking of clusters breaks equal keys by the lower cluster id,
 *   an argmax of logits by the lower token id.
 * - The library allocates device memory only in fh_create (one workspace
 *   sized by max_batch and max_probes) and frees it in fh_destroy.
 *   Calls on one handle must be stream-ordered (they share the workspace).
 * - Accumulation is fp32; results match an fp64 evaluation of the same
 *   steps within 2e-3 * |row| * |h| (row = the centroid or token row).
 */
#ifndef FH_H_
#define FH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* fh_stream_t;

typedef enum {
  FH_OK = 0,
  FH_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, size out of range, bad mode or T */
  FH_ERR_INVALID_C2T = 2,   /* C2T is not a permutation of 0..v-1 */
  FH_ERR_UNSUPPORTED = 3,   /* device is not sm_100, or a shape this build does not handle */
  FH_ERR_OOM = 4,           /* workspace allocation failed */
  FH_ERR_CUDA = 5,          /* a CUDA runtime call failed */
  FH_ERR_OUT_OF_RANGE = 6,  /* (device) a cluster id outside [0, c) or repeated in a row */
  FH_ERR_TIMEOUT = 7        /* (device) a bounded wait inside a kernel ran out */
} fh_status;

typedef enum {
  FH_CENTROID_BF16 = 0,     /* C: bf16 [c, d] */
  FH_CENTROID_INT4_G32 = 1, /* C_q: uint8 [c, d/2], C_scales: bf16 [c, d/32] */
  FH_CENTROID_INT8_G32 = 2  /* C_q: int8 [c, d], C_scales: bf16 [c, d/32] (W8A16) */
} fh_centroid_format;

typedef enum {
  FH_C2T_INT32 = 0,         /* C2T: int32 [c, b] */
  FH_C2T_UINT16 = 1         /* C2T: uint16 [c, b], v <= 65536 */
} fh_c2t_format;

typedef enum {
  FH_GREEDY = 0,            /* top-p clusters by score, argmax token */
  FH_SAMPLE_GUMBEL = 1      /* Gumbel-top-p clusters at T, softmax(z/T) token */
} fh_mode;

/*
 * Head description (balanced clustering, write-up section 1.2.1: every one of
 * the c clusters holds exactly b = v/c tokens; C2T[k][j] is the j-th token of
 * cluster k, so slot k*b + j of the flattened map names one token).
 *
 *  v, d, c, b   vocabulary, hidden size, clusters, tokens per cluster;
 *               v == c*b, d % 8 == 0 (d % 32 == 0 for INT4 / INT8), 1 <= c.
 *  E            device bf16 [v, d], 16-byte aligned.
 *  C            device bf16 [c, d], 16-byte aligned (BF16 format, else NULL).
 *  C_q          device uint8 [c, d/2] (INT4 format): element 2i in the low
 *               nibble of byte i, 2i+1 in the high nibble, two's complement;
 *               or device int8 [c, d] (INT8 format): one two's-complement
 *               byte per element (the W8A16 row of the write-up's parameter
 *               table, section 5.2).
 *  C_scales     device bf16 [c, d/32] (INT4 and INT8 formats): value = code * scale.
 *  C2T          device int32 [c, b] (4-byte aligned), or, with c2t_format
 *               FH_C2T_UINT16 and v <= 65536, device uint16 [c, b] (2-byte
 *               aligned): the compact map of the write-up's section 2.2.1,
 *               half the bytes; every token id is read through it as is.
 *  fmt          fh_centroid_format.
 *  max_batch    largest B any call will pass (>= 1).
 *  max_probes   largest p any call will pass (1 <= max_probes <= c).
 *  c2t_format   fh_c2t_format (0, the int32 map, when the field is left zero).
 */
typedef struct {
  int32_t v, d, c, b;
  const void* E;
  const void* C;
  const uint8_t* C_q;
  const void* C_scales;
  const void* C2T;
  int32_t fmt;
  int32_t max_batch;
  int32_t max_probes;
  int32_t c2t_format;
} fh_head_desc;

typedef struct fh_head fh_head;

/*
 * Create a head. Validates the description, checks on the device that C2T
 * is a permutation of 0..v-1 (FH_ERR_INVALID_C2T otherwise), allocates the
 * workspace, and fills two library-owned copies inside it: the token rows of
 * E in cluster-major order (row k*b + j = E[C2T[k][j]], v*d*2 bytes; a
 * cluster's b rows are one contiguous block, read without a C2T lookup), and,
 * for INT4 / INT8, each centroid row packed with its scales (row = d/2 or
 * d code bytes, then d/16 scale bytes, padded to 16 bytes) so that one bulk
 * copy moves a row. Synchronises `stream`. On success *out owns the workspace; release it
 * with fh_destroy. E itself is still read by the dense head.
 */
fh_status fh_create(const fh_head_desc* desc, fh_stream_t stream, fh_head** out);

/* Free the workspace and the handle. Waits for the device first. NULL is a no-op. */
void fh_destroy(fh_head* head);

/*
 * Stage 1 (write-up section 1.2.2): scores[r][k] = sum_i C[k][i] * hidden[r][i]
 * for r < B, k < c (INT4 / INT8: C dequantised exactly, code * scale).
 *  hidden  device bf16 [B, d], 16-byte aligned.
 *  scores  device fp32 [B, c].
 */
fh_status fh_centroid_scores(fh_head* head, const void* hidden, int32_t B, float* scores,
                             fh_stream_t stream);

/*
 * Probe selection (sections 1.2.2 and 1.2.3). For each row r the p clusters
 * with the largest key, key = scores (FH_GREEDY) or scores/T - ln(-ln u)
 * with u = u_clusters[r][k] clamped to [2^-126, 1 - 2^-24] (FH_SAMPLE_GUMBEL).
 *  scores       device fp32 [B, c].
 *  u_clusters   device fp32 [B, c]; only read in FH_SAMPLE_GUMBEL (else may be NULL).
 *  cluster_ids  device int32 [B, p], written in ascending cluster-id order.
 * T must be finite and > 0 in FH_SAMPLE_GUMBEL; 1 <= p <= max_probes.
 */
fh_status fh_select_clusters(fh_head* head, const float* scores, int32_t B, int32_t p,
                             int32_t mode, float T, const float* u_clusters,
                             int32_t* cluster_ids, fh_stream_t stream);

/*
 * Gather + stage 2 (sections 1.2.1 and 1.2.4). For row r, the candidates
 * are the tokens of the clusters in cluster_ids[r] taken in canonical order
 * (cluster id ascending, slot j ascending): for the q-th smallest chosen
 * cluster k, position q*b + j holds token C2T[k][j] and its logit
 * E[token] . hidden[r].
 *  cluster_ids  device int32 [B, p], any order, distinct within a row.
 *  token_ids    device int32 [B, p*b].
 *  logits       device fp32  [B, p*b].
 * A row with an id outside [0, c) or a repeated id is skipped (its outputs
 * are left untouched) and FH_ERR_OUT_OF_RANGE is recorded on the device.
 */
fh_status fh_candidate_logits(fh_head* head, const void* hidden, int32_t B, int32_t p,
                              const int32_t* cluster_ids, int32_t* token_ids, float* logits,
                              fh_stream_t stream);

/*
 * The whole head (section 2.2.2): scores, selection, gather, candidate
 * logits and the output token, fused so that intermediates stay on chip or
 * in the workspace.
 *  hidden           device bf16 [B, d], 16-byte aligned.
 *  u_clusters       device fp32 [B, c]  (FH_SAMPLE_GUMBEL only, else NULL).
 *  u_token          device fp32 [B]     (FH_SAMPLE_GUMBEL only, else NULL);
 *                   clamped to [0, 1 - 2^-24]; the token is the first
 *                   candidate, in canonical order, whose running sum of
 *                   exp(z/T - max z/T) exceeds u_token * total.
 *  out_tokens       device int32 [B].
 *  out_cluster_ids  device int32 [B, p] ascending, or NULL.
 *  out_max_logit    device fp32 [B] (largest candidate logit), or NULL.
 */
fh_status fh_decode(fh_head* head, const void* hidden, int32_t B, int32_t p, int32_t mode,
                    float T, const float* u_clusters, const float* u_token,
                    int32_t* out_tokens, int32_t* out_cluster_ids, float* out_max_logit,
                    fh_stream_t stream);

/*
 * Dense comparison head (write-up section 1.1): z = E h over the whole
 * vocabulary and its argmax.
 *  logits      device fp32 [B, v], or NULL to skip writing them.
 *  out_argmax  device int32 [B].
 */
fh_status fh_dense_head(fh_head* head, const void* hidden, int32_t B, float* logits,
                        int32_t* out_argmax, fh_stream_t stream);

/*
 * Allocation-free dense head: the same z = E h and argmax as fh_dense_head
 * (write-up section 1.1), with no handle. The write-up has no counterpart to
 * this entry point; it serves callers that must not allocate device memory
 * while they run (a serving process whose allocator already holds the free
 * HBM; a latency-critical loop, where cudaMalloc / cudaFree may synchronise
 * the device). It allocates nothing: the kernel's scratch (one word per hidden
 * row plus an exit ticket) is a fixed 1 KB device array inside this library,
 * zero between calls.
 *  E           device bf16 [v, d] row-major, 16-byte aligned; read only.
 *  v, d        vocabulary size >= 1; hidden size, a multiple of 8, <= 2560.
 *  hidden      device bf16 [B, d] row-major, 16-byte aligned.
 *  B           1 .. FH_NOALLOC_MAX_ROWS; a larger B returns FH_ERR_INVALID_ARG
 *              (the fixed scratch holds FH_NOALLOC_MAX_ROWS rows).
 *  logits      device fp32 [B, v], or NULL to skip writing them.
 *  out_argmax  device int32 [B] (lowest token id among equal maxima).
 * Errors: FH_ERR_INVALID_ARG (null / misaligned pointer, size out of range),
 * FH_ERR_UNSUPPORTED (d > 2560, or not an sm_100 device), FH_ERR_CUDA.
 * The first call on each device resolves the scratch's address
 * (cudaGetSymbolAddress, which may load the module) and sets kernel
 * attributes: make it before any stream capture begins. All calls on a
 * device share the scratch: launches that can overlap in time (unordered
 * streams, concurrent host threads) race and corrupt each other's results.
 * Cost: every group of up to 8 hidden rows is one pass over E, so a call with
 * B > 8 reads E about ceil(B / 8) times (fh_dense_head reads it once from
 * B = 64 on, on the tensor cores).
 */
#define FH_NOALLOC_MAX_ROWS 64
fh_status fh_dense_head_noalloc(const void* E, int32_t v, int32_t d, const void* hidden, int32_t B,
                                float* logits, int32_t* out_argmax, fh_stream_t stream);

/*
 * Synchronise `stream`, then return and clear the device status word
 * (FH_OK if no kernel recorded an error since the last read).
 */
fh_status fh_get_device_status(fh_head* head, fh_stream_t stream);

/* Static description of a status code. */
const char* fh_status_string(fh_status status);

/*
 * Clock-cycle budget of the device-wide waits inside fused kernels (default
 * about one second). A wait that runs out records FH_ERR_TIMEOUT and its
 * kernel returns early; 0 makes every such wait give up at once (used to
 * exercise that path).
 */
fh_status fh_set_spin_budget(fh_head* head, int64_t cycles);


/*
 * Introspection: FH_QUERY_WORKSPACE_BYTES, FH_QUERY_LAST_UNION (number of
 * distinct clusters gathered by the last batched fh_decode, after
 * fh_get_device_status or a stream sync), FH_QUERY_NUM_SMS,
 * FH_QUERY_FUSED_B1 (1 if B = 1 decodes run the single fused kernel),
 * FH_QUERY_LAST_LIST / FH_QUERY_LAST_FULL (last fused B = 1 decode: keys
 * that fell in its histogram of the predicted boundary region, and 1 if its
 * selection fell back to a histogram of all c keys). Queries that read device
 * counters synchronise the device.
 */
typedef enum {
  FH_QUERY_WORKSPACE_BYTES = 0,
  FH_QUERY_LAST_UNION = 1,
  FH_QUERY_NUM_SMS = 2,
  FH_QUERY_FUSED_B1 = 3,
  FH_QUERY_LAST_LIST = 4,
  FH_QUERY_LAST_FULL = 5
} fh_query_key;
fh_status fh_query(fh_head* head, int32_t key, int64_t* value);

/*
 * Speculative drafting (write-up section 4.2): check FlashHead draft tokens
 * against the dense head. For row r, p = softmax(z/T) over the vocabulary
 * (z = logits[r], the dense head's logits) and q = softmax(z/T) over the
 * draft's candidate tokens cand_tokens[r][0..n) (the tokens of the clusters
 * it was drawn from, e.g. fh_candidate_logits' token ids). The draft x =
 * draft[r] is kept when u_accept[r] < p(x) / q(x); otherwise the token is the
 * inverse-CDF draw (token id order) at u_resample[r] from max(0, p - q). For
 * every cluster set the result follows p exactly (standard speculative
 * sampling with the draft law taken given the chosen clusters).
 *  logits       device fp32 [B, v].
 *  cand_tokens  device int32 [B, n], distinct ids in [0, v) per row.
 *  draft        device int32 [B], one of the row's candidates.
 *  u_accept, u_resample  device fp32 [B], uniforms in [0, 1).
 *  out_tokens   device int32 [B]; -1 and FH_ERR_OUT_OF_RANGE in the device
 *               status when a candidate or the draft is out of range or the
 *               draft is not a candidate.
 * FH_ERR_UNSUPPORTED when the candidate bitmap (v bits) exceeds shared memory.
 */
fh_status fh_speculative_verify(fh_head* head, const float* logits, const int32_t* cand_tokens, int32_t n,
                                int32_t B, const int32_t* draft, float T, const float* u_accept,
                                const float* u_resample, int32_t* out_tokens, fh_stream_t stream);

/*
 * Adaptive probe count (write-up section 1.2.2, "dynamic adjustment"; section
 * 4.2: fewer probes for frequent tokens). For each row r of scores, out_p[r]
 * = the smallest p in [p_min, p_max] whose top-p clusters hold at least a
 * fraction tau of softmax(scores[r] / T) over all c clusters (the mass of the
 * top p depends only on the p largest scores, not on the order of ties).
 * Use it with fh_decode / fh_select_clusters row by row.
 *  scores  device fp32 [B, c] (fh_centroid_scores' output).
 *  out_p   device int32 [B].
 * 0 < tau <= 1, 1 <= p_min <= p_max <= c, T finite and > 0.
 * FH_ERR_UNSUPPORTED when a row's scores (next power of two of c, fp32) exceed shared memory.
 */
fh_status fh_adaptive_probes(fh_head* head, const float* scores, int32_t B, float tau, int32_t p_min,
                             int32_t p_max, float T, int32_t* out_p, fh_stream_t stream);

/*
 * Hot-cluster residency (write-up section 2.2.1: the token rows of frequently
 * used clusters kept in fast on-chip memory). Requests into L2 the token rows
 * of the given clusters (their b x d bf16 block in the head's cluster-major
 * copy of E) and their C2T rows, on `stream`, and returns without waiting: a
 * serving loop passes the clusters it expects the next decode to choose. It
 * only warms a cache; no result of any call depends on it.
 *  cluster_ids  device int32 [n], each in [0, c); an id out of range is skipped
 *               and FH_ERR_OUT_OF_RANGE is recorded in the device status.
 * n >= 0 (0: nothing is launched). FH_ERR_INVALID_ARG for a null head, n < 0,
 * or a null cluster_ids with n > 0.
 */
fh_status fh_prefetch_clusters(fh_head* head, const int32_t* cluster_ids, int32_t n, fh_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FH_H_ */
