/*
 * ckv.h -- C ABI of libckv.so: B200 (sm_100a) kernels for ClusterKV-style
 * semantic cluster recall of the KV cache.
 *
 * Method: "ClusterKV: Manipulating LLM KV Cache in Semantic Space for
 * Recallable Compression" (Liu, Li, Zhao, Zhang, Guo; arXiv 2412.03213v2),
 * as summarised section by section on its paperlayer.ai page. After prefill,
 * each KV head's keys are grouped by cosine k-means ("III.B Clustering in the
 * Semantic Space"); the centroids, cluster sizes, their prefix sums and the
 * token indices sorted by cluster are kept ("IV.C Selection and Indexing");
 * at each decode step the query ranks the clusters by attention weight and
 * whole clusters are recalled until a token budget is met, the last one
 * trimmed ("IV.C Selection and Indexing", "III.C Selection at the Granularity
 * of Semantic Clusters"); attention then runs over the recalled tokens plus
 * the attention-sink and recent tokens ("II.A LLM Inference and KV Cache").
 *
 * Conventions shared by every call
 * --------------------------------
 * - A "problem" is one (layer, batch, KV head). P problems are processed per
 *   call; problem p's data sits at base + p * stride.
 * - d (head dimension) must be 128.
 * - dtype: CKV_BF16 (bf16 storage, fp32 accumulation; the clustering
 *   similarity runs on tcgen05 tensor cores) or CKV_F32 (fp32 storage and
 *   arithmetic on CUDA cores).
 * - All pointers are device memory owned by the caller. The library allocates
 *   nothing, keeps no state between calls other than a device error word (see
 *   ckv_device_error) and cached per-device attributes, and never
 *   synchronises except in ckv_device_error.
 * - Every call is asynchronous and ordered on `stream` (a cudaStream_t passed
 *   as void*; NULL is the legacy default stream).
 * - Arguments are validated on the host before anything is launched; a bad
 *   argument returns CKV_ERR_INVALID and launches nothing. A launch failure
 *   returns CKV_ERR_CUDA. ckv_last_error() gives a one-line reason for the
 *   calling thread's last failure.
 * - Device-side checks: an out-of-range label, perm entry, selected index or
 *   tail position is skipped (never dereferenced) and sets a bit in the
 *   device error word instead of faulting.
 *
 * Region layout inside each problem
 * ---------------------------------
 *   positions [0, sink)                attention sinks, always attended
 *   positions [tok_begin, tok_end)     clustered tokens (prefill: [sink, L-W))
 *   positions [tail_begin, tail_end)   recent tokens, attended densely
 * Cluster metadata arrays are sized by capacities so that clusters of
 * generated tokens can be appended later ("III.B": every so many decode steps
 * the generated tokens alone are clustered into a few new centroids):
 *   centroids      float [P][C_cap][d]   mu: the mean of the raw member keys
 *   centroids_hat  dtype [P][C_cap][d]   mu / ||mu|| rounded to dtype: the
 *                                        copy the assignment step uses
 *   centroids_lp   dtype [P][C_cap][d]   mu rounded to dtype: the copy the
 *                                        decode-time scoring uses
 *   sizes          int32 [P][C_cap]      members per cluster
 *   offsets        int32 [P][C_cap + 1]  start of cluster c in perm (absolute
 *                                        slot); cluster c owns slots
 *                                        [offsets[c], offsets[c+1])
 *   labels         int32 [P][perm_cap]   slot perm_base + i holds the cluster
 *                                        id (cluster_base + local id) of token
 *                                        tok_begin + i
 *   perm           int32 [P][perm_cap]   token positions grouped by cluster,
 *                                        ascending within each cluster
 * A clustering call writes clusters [cluster_base, cluster_base + C) and perm
 * slots [perm_base, perm_base + tok_end - tok_begin); the prefill call uses
 * (0, 0) and an appended call continues where the previous one ended.
 */
#ifndef CKV_H
#define CKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CKV_OK = 0,
    CKV_ERR_INVALID = 1,     /* bad argument; nothing was launched */
    CKV_ERR_CUDA = 2,        /* a CUDA launch or runtime call failed */
    CKV_ERR_TIMEOUT = 3,     /* a bounded device wait gave up */
    CKV_ERR_UNSUPPORTED = 4  /* valid but not implemented (dtype/shape) */
} ckv_status;

typedef enum { CKV_F32 = 0, CKV_BF16 = 1 } ckv_dtype;

/* Device error bits (see ckv_device_error). */
#define CKV_DEVERR_LABEL 0x1u   /* a label outside [cluster_base, cluster_base+C) */
#define CKV_DEVERR_PERM 0x2u    /* a perm entry outside [tok_begin, tok_end) */
#define CKV_DEVERR_INDEX 0x4u   /* a selected / tail position outside the K/V rows */
#define CKV_DEVERR_OFFSETS 0x8u /* offsets not monotone or outside [0, perm_cap] */
#define CKV_DEVERR_TIMEOUT 0x10u /* a bounded device wait gave up (the kernel stopped early) */

/* Similarity that clustering assigns keys by ("III.B Clustering in the
 * Semantic Space": cosine; the paper's ablation compares L2 and inner
 * product). Inner product and L2 assign against the raw mean rounded to the
 * storage type (centroids_hat holds that copy); L2 ranks by
 * k . m - |m|^2 / 2 (the same argmin as |k - m|^2), with |m|^2 / 2 kept in
 * an fp32 bias array. A zero mean is a valid centroid for both. */
typedef enum { CKV_COSINE = 0, CKV_INNER = 1, CKV_L2 = 2 } ckv_metric;

/* Largest supported number of clusters per problem (C_cap). */
#define CKV_MAX_CLUSTERS 4096

const char *ckv_status_string(int status);
/* One-line reason for the calling thread's last non-OK status ("" if none). */
const char *ckv_last_error(void);
int ckv_version(void);

/* Read (and optionally clear) the device error word of the current device.
 * Synchronises `stream`. *flags receives the CKV_DEVERR_* bits. Returns
 * CKV_ERR_TIMEOUT if CKV_DEVERR_TIMEOUT is set (the outputs of the call that
 * set it are incomplete), else CKV_OK. */
ckv_status ckv_device_error(unsigned int *flags, int clear, void *stream);

/* ---- clustering --------------------------------------------------------- */

/* Workspace for ckv_cluster / ckv_index: per-chunk cluster histograms.
 * n_tok = tok_end - tok_begin. */
size_t ckv_index_workspace_bytes(int P, int n_tok, int C);
size_t ckv_cluster_workspace_bytes(int P, int n_tok, int C);
/* Workspace for ckv_cluster_ex: ckv_cluster_workspace_bytes plus, for L2, the
 * bias of the clusters being built. 0 for an unknown metric. */
size_t ckv_cluster_ex_workspace_bytes(int P, int n_tok, int C, int metric);

/* Cosine k-means over the keys of [tok_begin, tok_end) of every problem
 * ("III.B Clustering in the Semantic Space": assign each key to the centroid
 * of highest cosine similarity, move each centroid to the mean of its keys).
 * Seeding: centroid c starts at the key of position tok_begin + c * floor(n/C)
 * (the paper does not say how it seeds). Exactly `iters` rounds of (assign,
 * update) run; there is no early exit. On return: labels are the last round's
 * assignment, centroids the means of exactly those clusters (a cluster that
 * ended empty keeps its previous centroid), and sizes/offsets/perm the index
 * of those labels ("IV.C Selection and Indexing").
 *   keys            dtype, problem p's row t at keys + p*problem_stride + t*d
 *   problem_stride  elements between problems (>= tok_end * d)
 *   C, iters        1 <= C <= n_tok, C <= C_cap - cluster_base; iters >= 1
 *   workspace       >= ckv_cluster_workspace_bytes(P, n_tok, C) bytes, any
 *                   contents, 256-byte aligned
 * Errors: CKV_ERR_INVALID for null pointers, d != 128, C < 1, n_tok < C,
 * iters < 1, capacities exceeded, a small or misaligned workspace. */
ckv_status ckv_cluster(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                       int tok_begin, int tok_end, int C, int iters, int cluster_base,
                       int perm_base, int C_cap, int perm_cap, float *centroids,
                       void *centroids_hat, void *centroids_lp, int32_t *labels,
                       int32_t *sizes, int32_t *offsets, int32_t *perm, void *workspace,
                       size_t ws_bytes, void *stream);

/* ckv_cluster with a choice of similarity and for background use beside
 * other GPU work ("IV.B Semantic Clustering": clustering is launched
 * asynchronously and overlaps other inference kernels). Arguments as
 * ckv_cluster, plus
 *   metric    a ckv_metric (CKV_COSINE gives exactly ckv_cluster's results);
 *             workspace >= ckv_cluster_ex_workspace_bytes(P, n_tok, C, metric)
 *   max_sms   upper bound on the SMs the persistent tensor-core assignment
 *             kernel occupies (0 = all); the other clustering kernels are
 *             short-lived CTAs that interleave with other streams' work, so
 *             running this on a low-priority stream leaves the remaining SMs
 *             to the caller's high-priority kernels.
 * Clustering into cluster slots [cluster_base, cluster_base + C) and perm
 * slots [perm_base, perm_base + n_tok) beyond a problem's n_clusters does not
 * disturb a concurrent ckv_select / ckv_select_decode of those problems: they
 * read clusters [0, n_clusters) only, and the one shared entry,
 * offsets[cluster_base], is rewritten with the value it holds
 * (perm_base). Publishing the new clusters (raising n_clusters, moving
 * tail_begin) is the caller's, after this call's work has completed.
 * Errors as ckv_cluster, and CKV_ERR_INVALID for an unknown metric or
 * max_sms < 0. */
ckv_status ckv_cluster_ex(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                          int tok_begin, int tok_end, int C, int iters, int cluster_base,
                          int perm_base, int C_cap, int perm_cap, float *centroids,
                          void *centroids_hat, void *centroids_lp, int32_t *labels,
                          int32_t *sizes, int32_t *offsets, int32_t *perm, void *workspace,
                          size_t ws_bytes, int metric, int max_sms, void *stream);

/* Stage: strided seeding only (mu, mu-hat and the scoring copy of clusters
 * [cluster_base, cluster_base + C)). Arguments as in ckv_cluster. */
ckv_status ckv_init_centroids(const void *keys, ckv_dtype dt, int P, int64_t problem_stride,
                              int d, int tok_begin, int tok_end, int C, int cluster_base,
                              int C_cap, float *centroids, void *centroids_hat,
                              void *centroids_lp, void *stream);
/* Seeding under a ckv_metric: centroids_hat = the seed key itself for
 * CKV_INNER and CKV_L2; for CKV_L2 bias[p][cluster_base + c] (fp32, [P][C_cap],
 * caller-owned) receives half its squared norm. bias may be null otherwise. */
ckv_status ckv_init_centroids_ex(const void *keys, ckv_dtype dt, int P, int64_t problem_stride,
                                 int d, int tok_begin, int tok_end, int C, int cluster_base,
                                 int C_cap, float *centroids, void *centroids_hat,
                                 void *centroids_lp, int metric, float *bias, void *stream);

/* Stage: assignment. labels[p][perm_base + i] = cluster_base + argmax_c
 * (k_i . centroids_hat[c]) over c in [0, C), ties to the lowest c. For bf16
 * this is a bf16 x bf16 -> fp32 tensor-core contraction with the argmax fused
 * into its epilogue; for fp32 an FFMA contraction. */
ckv_status ckv_assign(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                      int tok_begin, int tok_end, const void *centroids_hat, int C,
                      int cluster_base, int C_cap, int32_t *labels, int perm_base, int perm_cap,
                      void *stream);
/* Assignment with a per-centroid bias: argmax_c (k_i . centroids_hat[c] -
 * bias[p][cluster_base + c]) ([P][C_cap] fp32, as written by the _ex seeding
 * and update for CKV_L2). A null bias is ckv_assign. */
ckv_status ckv_assign_ex(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                         int tok_begin, int tok_end, const void *centroids_hat, int C,
                         int cluster_base, int C_cap, int32_t *labels, int perm_base,
                         int perm_cap, const float *bias, void *stream);

/* Stage: cluster index of the labels of slots [perm_base, perm_base + n_tok):
 * offsets[cluster_base + c] for c in [0, C] (the last one is
 * perm_base + n_tok) and perm, a stable bucket sort (ascending position within
 * each cluster). Labels must lie in [cluster_base, cluster_base + C). */
ckv_status ckv_index(const int32_t *labels, int P, int tok_begin, int tok_end, int C,
                     int cluster_base, int C_cap, int perm_base, int perm_cap,
                     int32_t *offsets, int32_t *perm, void *workspace, size_t ws_bytes,
                     void *stream);

/* Stage: centroid update from an index: for each cluster c in
 * [cluster_base, cluster_base + C), mu_c = mean of the keys at
 * perm[offsets[c] .. offsets[c+1]) (summed in double in perm order),
 * sizes[c] = its member count, centroids_hat = mu/||mu|| and centroids_lp =
 * mu, both rounded to dtype once from double. A cluster with no members or a
 * zero mean keeps its previous centroids. tok_begin/tok_end bound the valid
 * perm entries. */
ckv_status ckv_update(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                      int tok_begin, int tok_end, int C, int cluster_base, int C_cap,
                      const int32_t *offsets, const int32_t *perm, int perm_cap,
                      float *centroids, void *centroids_hat, void *centroids_lp,
                      int32_t *sizes, void *stream);
/* Update under a ckv_metric: for CKV_INNER and CKV_L2 centroids_hat = mu
 * rounded to dtype, a zero mean is kept as the centroid, and for CKV_L2
 * bias[p][cluster_base + c] receives half the squared norm of that rounded
 * copy (bias may be null otherwise). Clusters with no members keep their
 * previous values, bias included. */
ckv_status ckv_update_ex(const void *keys, ckv_dtype dt, int P, int64_t problem_stride, int d,
                         int tok_begin, int tok_end, int C, int cluster_base, int C_cap,
                         const int32_t *offsets, const int32_t *perm, int perm_cap,
                         float *centroids, void *centroids_hat, void *centroids_lp,
                         int32_t *sizes, int metric, float *bias, void *stream);

/* ---- decode-time selection ---------------------------------------------- */

size_t ckv_select_workspace_bytes(int P, int C_cap);

/* Cluster-granularity recall ("IV.C Selection and Indexing"). For problem p
 * with n_clusters[p] clusters:
 *   score s_c = sum over the G query heads of q_g . centroids_lp[c], computed
 *     in fp32 in a fixed order (channels split in 32 groups of 4, each summed
 *     with fmaf from 0 in channel order, the groups combined by an xor
 *     butterfly over 16, 8, 4, 2, 1, then heads added in order). The softmax
 *     is monotone, so ranking by this logit ranks by attention weight.
 *   rank: clusters by descending score, ties to the lower cluster id;
 *   fill: clusters are taken whole while they fit in the budget; the first
 *     that does not fit contributes its first (lowest-position) tokens up to
 *     the budget and the walk stops.
 * Output: sel_idx[p][0 .. sel_cnt[p]) token positions in rank order, then perm
 * order; sel_cnt[p] = min(budget, total clustered tokens).
 *   q             dtype [P][G][d]
 *   n_clusters    int32 [P] (device), each in [0, C_cap]
 *   budget        >= 0; sel_idx has row stride `budget`
 *   G             1..8 */
ckv_status ckv_select(const void *q, ckv_dtype dt, int P, int G, int d,
                      const void *centroids_lp, const int32_t *n_clusters, int C_cap,
                      const int32_t *offsets, const int32_t *perm, int perm_cap, int budget,
                      int32_t *sel_idx, int32_t *sel_cnt, void *workspace, size_t ws_bytes,
                      void *stream);

/* ---- fused decode step -------------------------------------------------- */

/* One decode step in one launch: ckv_select followed by ckv_sparse_decode,
 * with the same arguments, outputs and results (sel_idx / sel_cnt
 * bit-identical to ckv_select; out equal to ckv_sparse_decode up to fp32
 * summation order). One thread-block cluster of up to 8 CTAs per problem
 * (as many as keep every problem resident in one wave; one when even that
 * needs several waves) shares the cluster scores and the partial attention
 * results through distributed shared memory; each CTA finds the selection
 * on its own copy of the scores (a weighted radix select for the cluster
 * where the budget is reached), so no workspace and no second kernel are
 * needed. Supports G in {1, 2, 4} and up to 32768 attended rows per problem
 * (sink + budget + max_tail); other shapes return CKV_ERR_UNSUPPORTED (use
 * the two separate calls). */
ckv_status ckv_select_decode(const void *q, ckv_dtype dt, int P, int G, int d,
                             const void *centroids_lp, const int32_t *n_clusters, int C_cap,
                             const int32_t *offsets, const int32_t *perm, int perm_cap,
                             int budget, int32_t *sel_idx, int32_t *sel_cnt, const void *K,
                             const void *V, int64_t kv_problem_stride, int kv_rows, int sink,
                             const int32_t *tail_begin, const int32_t *tail_end, int max_tail,
                             float scale, float *out, void *stream);

/* ckv_select_decode with the accounting of a cache that keeps the KV of the
 * clusters selected in the last R decode steps ("D. Caching KV of Selected
 * Tokens": the GPU cache retains the KV and cluster labels of the last R
 * steps and loads only clusters absent from it; the paper settles on R = 1).
 * Same selection and output, plus, per problem p:
 *   last_sel     int32 [P][C_cap], caller-owned: the last step that selected
 *                each cluster; initialise to a value far below any step (for
 *                example -2^30); updated with this step's selection
 *   step         this step's number (increasing from call to call)
 *   R            steps the cache keeps (>= 0; 0 caches nothing)
 *   cache_stats  int32 [P][4]: selected clusters that were cached (hits), the
 *                selected (non-empty) clusters, recalled tokens of the hits,
 *                recalled tokens (sel_cnt)
 *   miss_list    int32 [P][C_cap] or null: the selected clusters that were not
 *                cached (the ones to load), in rank order; its length is
 *                cache_stats[1] - cache_stats[0]
 * A null last_sel is ckv_select_decode. Errors as ckv_select_decode, and
 * CKV_ERR_INVALID for a cache without cache_stats or with R < 0. */
ckv_status ckv_select_decode_cached(const void *q, ckv_dtype dt, int P, int G, int d,
                                    const void *centroids_lp, const int32_t *n_clusters,
                                    int C_cap, const int32_t *offsets, const int32_t *perm,
                                    int perm_cap, int budget, int32_t *sel_idx, int32_t *sel_cnt,
                                    const void *K, const void *V, int64_t kv_problem_stride,
                                    int kv_rows, int sink, const int32_t *tail_begin,
                                    const int32_t *tail_end, int max_tail, float scale,
                                    float *out, int32_t *last_sel, int step, int R,
                                    int32_t *cache_stats, int32_t *miss_list, void *stream);

/* ---- sparse decode attention -------------------------------------------- */

/* max_rows bounds sink + budget + (tail_end - tail_begin) over all problems. */
size_t ckv_decode_workspace_bytes(int P, int G, int d, int max_rows);

/* out[p][g] = sum_{j in A} softmax_j(scale * q_g . k_j) v_j with
 * A = [0, sink) + sel_idx[p][0..sel_cnt[p]) + [tail_begin[p], tail_end[p])
 * ("II.A LLM Inference and KV Cache"; the attended set is the paper's
 * selected tokens plus sinks and recent tokens). Split-K over A with an
 * fp32 online softmax; partial results are merged by a second kernel.
 *   q            dtype [P][G][d];  K, V dtype, row t of problem p at
 *                base + p*kv_problem_stride + t*d; kv_rows rows per problem
 *   tail_begin/tail_end  int32 [P] (device)
 *   max_tail     upper bound of tail_end - tail_begin (grid sizing)
 *   out          float [P][G][d]
 *   workspace    >= ckv_decode_workspace_bytes(P, G, d, sink + budget +
 *                max_tail) bytes, 256-byte aligned */
ckv_status ckv_sparse_decode(const void *q, const void *K, const void *V, ckv_dtype dt, int P,
                             int G, int d, int64_t kv_problem_stride, int kv_rows, int sink,
                             const int32_t *tail_begin, const int32_t *tail_end, int max_tail,
                             const int32_t *sel_idx, const int32_t *sel_cnt, int budget,
                             float scale, float *out, void *workspace, size_t ws_bytes,
                             void *stream);

/* Allocation-free variant of ckv_sparse_decode. The paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory --
 * a plugin or operator hook that is handed its tensors by a host framework
 * but no allocator (the framework's pool owns the device memory, so a private
 * cudaMalloc would bypass its accounting or fail once the pool has reserved
 * the device), and decode loops that must not call cudaMalloc/cudaFree at all
 * because those calls can synchronise the device and stall other streams.
 * Such a caller still passes q, K, V, the selection and `out` exactly as for
 * ckv_sparse_decode, but no workspace: the split-K partials live in a fixed
 * file-scope device array of CKV_NOALLOC_SCRATCH_BYTES inside the library
 * (one per GPU that loads the library, held until the process exits).
 *   - A call whose partials would not fit returns CKV_ERR_INVALID with a
 *     clear message and launches nothing; ckv_sparse_decode_noalloc_scratch_bytes
 *     gives the bytes a shape needs on the current device.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - Every call on a device shares the one array, which keeps the last
 *     call's contents (nothing in it needs to start at zero: each call writes
 *     every partial it reads). Calls that overlap on the GPU (other streams,
 *     other host threads) race on it: serialise them.
 *   - It calls no cudaMalloc, cudaFree or allocating library routine.
 * Arguments, layout, results and errors are otherwise those of
 * ckv_sparse_decode. */
#define CKV_NOALLOC_SCRATCH_BYTES (8u << 20)
size_t ckv_sparse_decode_noalloc_scratch_bytes(int P, int G, int d, int max_rows);
ckv_status ckv_sparse_decode_noalloc(const void *q, const void *K, const void *V, ckv_dtype dt,
                                     int P, int G, int d, int64_t kv_problem_stride,
                                     int kv_rows, int sink, const int32_t *tail_begin,
                                     const int32_t *tail_end, int max_tail,
                                     const int32_t *sel_idx, const int32_t *sel_cnt,
                                     int budget, float scale, float *out, void *stream);

/* Append one generated token per problem: K/V row tail_end[p] <- new_k[p] /
 * new_v[p] (dtype [P][d]); then tail_end[p] += 1. A full cache (tail_end[p]
 * >= kv_rows) writes nothing and sets CKV_DEVERR_INDEX. */
ckv_status ckv_append(void *K, void *V, ckv_dtype dt, int P, int d, int64_t kv_problem_stride,
                      int kv_rows, const void *new_k, const void *new_v, int32_t *tail_end,
                      void *stream);

/* Self-test of the device timeout reporting (no counterpart in the paper):
 * one thread waits, up to limit_us microseconds of the GPU's global timer, for
 * a device flag that nothing sets, then records CKV_DEVERR_TIMEOUT in the
 * device error word, exactly as a bounded wait inside a kernel does when it
 * gives up. ckv_device_error then returns CKV_ERR_TIMEOUT; the context stays
 * usable. limit_us in [0, 1000000]; CKV_ERR_INVALID otherwise. */
ckv_status ckv_selftest_timeout(unsigned int limit_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* CKV_H */
