/*
 * fh_cluster.h -- C ABI of the offline balanced clustering that produces a
 * FlashHead head (centres C and the cluster-to-token map C2T).
 *
 * What it computes (FlashHead write-up, www.framerc.cn/news/2430929,
 * section 2.1 "offline clustering", with the balance rule of section 1.2.1):
 *
 *   1. every token embedding is L2-normalised (spherical k-means);
 *   2. c starting centres are picked by k-means++ seeding, or given;
 *   3. each step scores every token against every centre (cosine
 *      similarity of unit vectors, a v x c product), assigns the tokens so
 *      that every cluster holds exactly b = v/c of them, and moves each
 *      centre to the normalised mean of its tokens;
 *   4. the steps repeat until an assignment repeats the previous one, or
 *      max_iter times (the write-up's loop runs 1000).
 *
 * Readings of what the write-up leaves open (they fix every result):
 *   - the balanced assignment is the global greedy over (token, cluster)
 *     pairs by similarity descending, ties to the lower token id, then the
 *     lower cluster id; a pair is taken while its token is unassigned and its
 *     cluster has room. It is computed here by rounds of proposals (every
 *     unassigned token proposes to its best cluster among those that would
 *     not reject it; every cluster keeps its best b), which reaches the same
 *     assignment because, under one strict order of all pairs, the balanced
 *     assignment with no token preferring a cluster that holds a worse pair
 *     is unique and is the greedy one;
 *   - k-means++: first centre token floor(u[0]*v); centre j is the first
 *     token (in id order) whose running sum of squared Euclidean distances to
 *     the nearest chosen centre exceeds u[j] times the total; the lowest
 *     unchosen token if every distance is 0;
 *   - a zero embedding stays zero; a cluster whose mean is zero keeps its
 *     previous centre; C2T lists a cluster's tokens in ascending id.
 *
 * Precision: the normalised embeddings and the centres are stored as bf16
 * (the operands of the similarity product), similarities and sums are
 * accumulated in fp32, the seeding's running sums in fp64. An assignment
 * is decided exactly on the fp32 similarities it is given.
 *
 * Conventions as in fh.h: caller-owned device pointers, asynchronous on
 * `stream` unless stated, argument errors returned before anything is
 * enqueued, one workspace allocated in fh_cluster_create. Limits: v == c*b,
 * 1 <= b <= 32, d % 8 == 0, d <= 8192, 16-byte aligned bf16 pointers.
 */
#ifndef FH_CLUSTER_H_
#define FH_CLUSTER_H_

#include "fh.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct fh_cluster fh_cluster;

/*
 * Allocate the builder's workspace for v tokens of size d in c clusters:
 * the normalised embeddings (bf16 [v, d]), the similarity matrix (fp32
 * [c, v], 4*c*v bytes), working centres and the assignment state.
 * Synchronises `stream`. FH_ERR_UNSUPPORTED off sm_100 or outside the
 * limits above, FH_ERR_OOM if the allocation fails.
 */
fh_status fh_cluster_create(int32_t v, int32_t d, int32_t c, fh_stream_t stream, fh_cluster** out);

/* Free the workspace and the handle. Waits for the device first. NULL is a no-op. */
void fh_cluster_destroy(fh_cluster* cl);

/*
 * Step 1: En[t] = bf16(E[t] / |E[t]|), norm in fp32; a zero row stays zero.
 *  E, En  device bf16 [v, d] (may not overlap).
 */
fh_status fh_cluster_normalize(fh_cluster* cl, const void* E, void* En, fh_stream_t stream);

/*
 * Step 2: k-means++ seeds over the rows of En.
 *  En        device bf16 [v, d] (unit rows, as written by fh_cluster_normalize).
 *  u         device fp32 [c], uniforms in [0, 1).
 *  seed_ids  device int32 [c], the chosen tokens in draw order.
 */
fh_status fh_cluster_seed(fh_cluster* cl, const void* En, const float* u, int32_t* seed_ids,
                          fh_stream_t stream);

/*
 * Centres from tokens: C[k] = En[ids[k]].
 *  ids  device int32 [c], each in [0, v) (FH_ERR_OUT_OF_RANGE in the device
 *       status otherwise; the row is then left unwritten).
 *  C    device bf16 [c, d].
 */
fh_status fh_cluster_gather(fh_cluster* cl, const void* En, const int32_t* ids, void* C,
                            fh_stream_t stream);

/*
 * Step 3a: S[k][t] = sum_i C[k][i] * En[t][i] (fp32), on the tensor cores.
 *  En  device bf16 [v, d]; C device bf16 [c, d]; S device fp32 [c, v].
 */
fh_status fh_cluster_similarities(fh_cluster* cl, const void* En, const void* C, float* S,
                                  fh_stream_t stream);

/*
 * Step 3b: the balanced assignment of S (every cluster exactly b tokens).
 *  S       device fp32 [c, v] (finite values).
 *  assign  device int32 [v]: cluster of every token.
 *  C2T     device int32 [c, b]: tokens of every cluster, ascending.
 *  rounds  host int32, nullable: proposal rounds it took.
 * Synchronous: the host waits for each round's count of unassigned tokens.
 */
fh_status fh_cluster_assign(fh_cluster* cl, const float* S, int32_t* assign, int32_t* C2T,
                            int32_t* rounds, fh_stream_t stream);

/*
 * Step 3c: C[k] = bf16(m / |m|), m = sum of En over the tokens C2T[k][0..b);
 * a cluster with m = 0 keeps C[k] as given.
 *  C2T  device int32 [c, b], entries in [0, v).
 *  C    device bf16 [c, d], read (previous centres) and written.
 */
fh_status fh_cluster_update(fh_cluster* cl, const void* En, const int32_t* C2T, void* C,
                            fh_stream_t stream);

/*
 * The whole loop: normalise E, start from the tokens init_ids (if not NULL)
 * or from k-means++ seeds drawn with u_init, then steps 3a-3c until an
 * assignment repeats the previous one or max_iter steps have run.
 *  E           device bf16 [v, d].
 *  init_ids    device int32 [c] or NULL.
 *  u_init      device fp32 [c] (read when init_ids is NULL).
 *  C_out       device bf16 [c, d]: final centres.
 *  C2T_out     device int32 [c, b]: final map (tokens ascending per cluster).
 *  iterations  host int32, nullable: steps run.
 * Synchronous (the host checks convergence after every step).
 */
fh_status fh_cluster_build(fh_cluster* cl, const void* E, const int32_t* init_ids, const float* u_init,
                           int32_t max_iter, void* C_out, int32_t* C2T_out, int32_t* iterations,
                           fh_stream_t stream);

/* Read and clear the builder's device status word (synchronises `stream`). */
fh_status fh_cluster_get_device_status(fh_cluster* cl, fh_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif  /* FH_CLUSTER_H_ */
