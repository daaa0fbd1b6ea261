/*
 * dsa.h -- C ABI of libdsa.so: dynamic sparse attention for NVIDIA B200 (sm_100a).
 *
 * The operations follow two pages on dynamic sparse attention:
 *  - MInference 1.0 ("MInference 1.0: Accelerating Pre-filling for Long-Context
 *    LLMs via Dynamic Sparse Attention"), section "方法介紹" (method): the
 *    block-sparse index from mean-pooled Q and K (pooling commutes with MatMul),
 *    the vertical-slash index from the last queries against all keys, and a
 *    block-sparse FlashAttention kernel; Fig. 4: slash lines as 64x64 blocks,
 *    vertical lines as 1x64 column tiles.
 *  - Squeezed Attention ("Squeezed Attention：基于语义聚类的长上下文LLM推理加速"),
 *    section "技术方案" (technical approach, online stage): compare the query with
 *    every centroid, keep the top clusters, attend over their keys and values only.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller.  Tensors are
 *    dense, row-major, bf16 (IEEE bfloat16 bits) unless stated otherwise.
 *    Prefill: Q [Hq][n][d], K and V [Hkv][n][d], O [Hq][n][d].  q-head h reads
 *    KV head h / (Hq/Hkv) (grouped-query attention).
 *  - The block is 64 tokens; n must be a multiple of 64; d is 64 or 128.
 *  - Index outputs are int32, ascending within each list, padded with -1 after
 *    the count.  Ties in every top-k go to the lower index.
 *  - Every call is asynchronous on `stream` (0 = legacy default stream); it
 *    returns after launching.  The library allocates no device memory: scratch
 *    lives in the caller's workspace `ws`.
 *  - Workspace protocol: call with ws == NULL to get the required size in
 *    *ws_bytes (nothing is launched, return 0).  Then call again with a buffer
 *    of at least that size (256-byte aligned).  The first 256 bytes of any
 *    workspace hold a sticky device status word: zero them once before first
 *    use; dsa_get_status() reads and clears it.
 *  - Return codes: DSA_OK; DSA_ERR_INVALID_ARG (null pointer, bad size or
 *    shape, ws too small); DSA_ERR_UNSUPPORTED (d not in {64,128}, n % 64,
 *    block != 64, sizes beyond the limits below); DSA_ERR_CAPACITY (an output
 *    list capacity is too small for the requested budget); DSA_ERR_CUDA (a
 *    launch or runtime error; the CUDA error is left for cudaGetLastError);
 *    DSA_ERR_TIMEOUT (reported by dsa_get_status: a bounded device-side wait
 *    expired and the kernel returned early).
 *  - Limits: n <= 2^21 tokens per head; Hq*n and Hkv*n < 2^31 rows.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dsa_stream_t; /* same type as cudaStream_t */

enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = -1,
  DSA_ERR_UNSUPPORTED = -2,
  DSA_ERR_CAPACITY = -3,
  DSA_ERR_CUDA = -4,
  DSA_ERR_TIMEOUT = -5
};

/*
 * sparse_index_estimate -- block-sparse index (MInference 1.0, method section:
 * mean pooling of Q and K over 64-token blocks; the pooled score Q̄_i·K̄_j
 * equals the mean of the block's raw scores because pooling commutes with
 * MatMul).  Also the decode centroid build (Squeezed Attention, technical
 * approach: per-cluster centroids, here per 64-token block means).
 *
 *  q          [Hq][n][d] bf16, or NULL for pool-only mode (then only pooled_k
 *             is produced and the index arguments are ignored).
 *  k          [Hkv][n][d] bf16.  For a decode cache [B][Hkv][S][d] pass
 *             Hkv = B*Hkv and n = S.
 *  block      must be 64.
 *  k_fixed    > 0: keep min(i+1, k_fixed) blocks in total for query block i,
 *             counting the forced sink (block 0) and diagonal (block i).
 *  keep_ratio > 0: keep the forced blocks plus ceil(rho*(i+1)) more (at most
 *             i-1), rho taken in parts per million: floor(keep_ratio*1e6+0.5).
 *             Exactly one of k_fixed and keep_ratio must be positive.
 *  block_idx  [Hq][n/64][kcap] int32 out; block_cnt [Hq][n/64] int32 out.
 *             kcap must be >= the largest count the budget gives (else
 *             DSA_ERR_CAPACITY).
 *  pooled_k   optional [Hkv][n/64][d] fp32 out: the per-block mean keys.
 *             Required in pool-only mode.
 *  Ranking uses fp32-accurate scores (three FP16 tensor-core products of the
 *  means split into hi + lo after a power-of-two scale per query block and per
 *  KV head, |error| ~ 2^-21 of |Q̄||K̄|); the remaining candidates of query
 *  block i are blocks 1..i-1.  A bounded wait that expires sets the workspace
 *  status word (DSA_ERR_TIMEOUT through dsa_get_status).
 */
int sparse_index_estimate(const void* q, const void* k, int Hq, int Hkv, int n, int d, int block,
                          int k_fixed, float keep_ratio, int32_t* block_idx, int32_t* block_cnt,
                          int kcap, float* pooled_k, void* ws, size_t* ws_bytes, dsa_stream_t stream);

/*
 * vertical_slash_index -- vertical-slash index and its execution plan
 * (MInference 1.0, method section: the attention of the last queries against
 * all keys scores vertical lines and slash lines; Fig. 4: slash lines run as
 * 64x64 blocks, vertical lines as 1x64 column tiles).
 *
 *  Rows i_r = n - last_q + r (r < last_q), causal softmax of q_i·k_j*scale
 *  over j <= i_r.  vert[j] = sum_r P[r,j];  slash[o] = sum_r P[r, i_r - o].
 *  Keeps n_vert columns (columns 0..63 always among them) and n_slash offsets
 *  (offset 0 always among them).
 *  last_q     must be 64.   64 <= n_vert <= n;  1 <= n_slash <= n.
 *  vert_idx   optional [Hq][n_vert] int32 out (ascending kept columns).
 *  slash_off  optional [Hq][n_slash] int32 out (ascending kept offsets).
 *  Plan for each (h, qb), ascending, -1 padded:
 *   block_idx [Hq][n/64][kcap], block_cnt [Hq][n/64]: the aligned key blocks
 *             qb - floor(o/64) and qb - ceil(o/64) (if >= 0) of every kept
 *             offset o <= 64*qb + 63.  kcap >= min(n/64, 2*n_slash).
 *   col_idx   [Hq][n/64][ccap], col_cnt [Hq][n/64]: kept columns
 *             j <= 64*qb + 63 whose block is not selected.  ccap >= n_vert.
 */
int vertical_slash_index(const void* q, const void* k, int Hq, int Hkv, int n, int d, int last_q,
                         int n_vert, int n_slash, float scale, int32_t* vert_idx, int32_t* slash_off,
                         int32_t* block_idx, int32_t* block_cnt, int kcap, int32_t* col_idx,
                         int32_t* col_cnt, int ccap, void* ws, size_t* ws_bytes, dsa_stream_t stream);

/*
 * block_sparse_attn_fwd -- causal softmax attention over the chosen key
 * blocks and columns only (MInference 1.0, method section: block-sparse
 * FlashAttention; Fig. 4).
 *
 *  For query row i of q-head h in query block qb: the attended set is
 *  (union of blocks block_idx[h][qb][0..cnt) and columns col_idx[h][qb][0..cnt))
 *  intersected with keys j <= i.  O_i = sum softmax(q_i·k_j*scale) v_j.
 *  Lists must be ascending, in range, duplicate-free, blocks <= qb and
 *  columns < 64*qb with their block not in the block list (the library trusts
 *  them; set DSA_VALIDATE=1 in the environment to have them checked on the
 *  device first: a bad list then returns DSA_ERR_INVALID_ARG).
 *  col_idx/col_cnt may be NULL (blocks only).
 *  lse        optional [Hq][n] fp32 out: natural-log sum of exp of the scaled
 *             scores (-inf for an empty set, whose O row is 0).
 */
int block_sparse_attn_fwd(const void* q, const void* k, const void* v, void* o, int Hq, int Hkv, int n,
                          int d, float scale, const int32_t* block_idx, const int32_t* block_cnt, int kcap,
                          const int32_t* col_idx, const int32_t* col_cnt, int ccap, float* lse, void* ws,
                          size_t* ws_bytes, dsa_stream_t stream);

/*
 * a_shape_index -- static A-shape block index (MInference 1.0, method
 * section: the A-shape pattern keeps the first tokens, an attention sink, and
 * a local window of recent tokens).  Query block qb keeps key blocks
 * [0, min(n_sink, qb+1)) and [max(0, qb-n_local+1), qb], ascending, -1 padded;
 * the lists feed block_sparse_attn_fwd unchanged.
 *  block_idx [Hq][n/64][kcap], block_cnt [Hq][n/64] int32 out;
 *  kcap >= min(n/64, n_sink + n_local).  n_sink >= 0, n_local >= 1.
 */
int a_shape_index(int Hq, int n, int n_sink, int n_local, int32_t* block_idx, int32_t* block_cnt, int kcap,
                  dsa_stream_t stream);

/*
 * sparse_decode_attn -- one query token per sequence over a fixed KV cache,
 * attending only over the best-ranked 64-token blocks (Squeezed Attention,
 * technical approach, online stage: score the query against every centroid,
 * keep the top clusters, attend only over their keys and values).
 *
 *  q          [B][Hq][d] bf16.   k_cache, v_cache [B][Hkv][S][d] bf16.
 *  centroids  [B][Hkv][S/64][d] fp32 block means of k_cache (build them with
 *             sparse_index_estimate in pool-only mode).
 *  keep       blocks kept among 0..S/64-2 (or 0..S/64-1 when force_last == 0)
 *             by the raw score q·c, ties to the lower block; force_last adds
 *             the last block (it holds the newest tokens).
 *  o          [B][Hq][d] bf16 out.
 *  sel_idx    optional [B][Hq][kcap] int32 out (ascending kept blocks),
 *             sel_cnt optional [B][Hq]; kcap >= keep + force_last when given.
 *  Sizes: d in {64, 128}; Hq / Hkv in {1, 2, 4, 8}; S % 64 == 0 and S <= 1,600,000
 *  or so (one q-head's block scores, ids and bitmap, 8.125 B per 64-token
 *  block, stay under 200 KB of shared memory); larger S returns
 *  DSA_ERR_UNSUPPORTED.
 */
int sparse_decode_attn(const void* q, const void* k_cache, const void* v_cache, const float* centroids,
                       int B, int Hq, int Hkv, int S, int d, int keep, int force_last, float scale, void* o,
                       int32_t* sel_idx, int32_t* sel_cnt, int kcap, void* ws, size_t* ws_bytes,
                       dsa_stream_t stream);

/*
 * sparse_decode_attn_static -- sparse_decode_attn without a workspace: the
 * same computation and arguments (minus ws / ws_bytes), its scratch held in a
 * fixed 32 MiB array inside the library's device memory.  The pages have no
 * counterpart of this entry point; it exists for callers that cannot allocate
 * device memory: a plugin or serving engine whose allocator owns the whole GPU
 * budget and offers no allocation hook, or a decode loop that must never call
 * cudaMalloc (it may synchronize the device and can fail once memory is
 * fragmented).  The caller still passes inputs and outputs.
 *
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *    Every GPU that loads the library holds the 32 MiB array until exit.
 *  - Sizes whose scratch exceeds 32 MiB are rejected with DSA_ERR_CAPACITY
 *    before any launch.  The scratch is 256 B + B·Hq·ceil(nb/32)·4 B (kept
 *    bitmaps) + B·Hkv·nb·5 B (union lists and masks) + B·Hkv·4 B +
 *    B·Hq·nc·(d+2)·4 B (chunk partials, nc = ceil(nb/64)) + B·Hq·nb·4 B (block
 *    scores), nb = S/64, each part rounded up to 256 B: B=16, Hq=32, Hkv=8,
 *    S=131072, d=128 needs 14.2 MB.
 *  - The first call on a device looks up the array's device address on that
 *    device (make the device current first); make that first call before any
 *    stream capture.  The address is kept per device context: after a device
 *    reset (a new primary context) the next call looks it up again.
 *  - All calls share the one array, which keeps the previous call's contents;
 *    each call clears the status word it needs zeroed.  Calls that overlap on
 *    the GPU (different streams, or other host threads, without ordering
 *    between them) race on the array.
 *  - Device-side timeouts are not reported by this entry point (there is no
 *    workspace to pass to dsa_get_status); launch errors are returned.
 */
int sparse_decode_attn_static(const void* q, const void* k_cache, const void* v_cache, const float* centroids,
                              int B, int Hq, int Hkv, int S, int d, int keep, int force_last, float scale,
                              void* o, int32_t* sel_idx, int32_t* sel_cnt, int kcap, dsa_stream_t stream);

/*
 * kmeans_clusters -- the offline stage of cluster-ranked decode (Squeezed
 * Attention, technical approach: the fixed context's keys are clustered with
 * K-means; each cluster gets a centroid and each key an index to its cluster).
 * Lloyd's algorithm over the first n_ctx keys of every (batch, KV head):
 * centroids start at the means of C equal contiguous segments
 * (segment c = keys floor(c n_ctx / C) .. floor((c+1) n_ctx / C) - 1); each of
 * `iters` rounds assigns every key to its nearest centroid (squared Euclidean
 * distance in fp32, ties to the lower cluster) and moves every non-empty
 * cluster's centroid to the mean of its keys (an empty cluster keeps its
 * centroid).  The outputs are the last round's assignment and the centroids
 * computed from it.
 *
 *  k_cache    [B][Hkv][S][d] bf16 (d in {64, 128}); 1 <= C <= n_ctx <= S, C <= 4096.
 *  centroids  [B][Hkv][C][d] fp32 out.   assign [B][Hkv][n_ctx] int32 out.
 *  offsets    [B][Hkv][C+1] int32 out, tokens [B][Hkv][n_ctx] int32 out: the
 *             keys of cluster c, ascending, are tokens[offsets[c] .. offsets[c+1]).
 *  iters      >= 1 rounds.
 * Deterministic: the centroid sums run in token order.
 */
int kmeans_clusters(const void* k_cache, int B, int Hkv, int S, int d, int n_ctx, int C, int iters,
                    float* centroids, int32_t* assign, int32_t* offsets, int32_t* tokens, void* ws,
                    size_t* ws_bytes, dsa_stream_t stream);

/*
 * cluster_pack_kv -- a copy of the fixed context's K and V rows in cluster
 * order, made once after kmeans_clusters (Squeezed Attention, technical
 * approach: the context is fixed, so what is computed offline is reused by
 * every decode step): k_packed[b][g][p] = k_cache[b][g][tokens[b][g][p]] for
 * p < n_ctx, and the same for V, so cluster c occupies positions
 * offsets[c] .. offsets[c+1] - 1.
 *
 *  k_cache, v_cache  [B][Hkv][S][d] bf16.   tokens: kmeans_clusters' output.
 *  k_packed, v_packed  [B][Hkv][n_ctx][d] bf16 out (caller-owned, 16-byte aligned).
 * Launches one kernel on `stream`; no workspace.
 */
int cluster_pack_kv(const void* k_cache, const void* v_cache, const int32_t* tokens, int B, int Hkv, int S, int d,
                    int n_ctx, void* k_packed, void* v_packed, dsa_stream_t stream);

/*
 * cluster_decode_attn -- the online stage over K-means clusters (Squeezed
 * Attention, technical approach: compare the query with every centroid, keep
 * the top clusters, attend only over the keys and values of those clusters).
 * Each q-head ranks the non-empty clusters of its KV head by the raw score
 * q.c, keeps the best min(keep, non-empty) (ties to the lower cluster), and
 * attends over the keys of the kept clusters plus the unclustered tail
 * [n_ctx, S) (the newest tokens, the current one included).
 *
 *  q          [B][Hq][d] bf16.   k_cache, v_cache [B][Hkv][S][d] bf16.
 *  centroids, offsets, tokens: kmeans_clusters' outputs for the same cache.
 *  o          [B][Hq][d] bf16 out.
 *  k_packed, v_packed  optional (both or neither) [B][Hkv][n_ctx][d] bf16:
 *             cluster_pack_kv's cluster-ordered copy of the context.  With
 *             it, a kept cluster is read as one contiguous range; without,
 *             its K and V rows are gathered from the caches by token id.
 *  sel_idx    optional [B][Hq][kcap] int32 out (ascending kept clusters, -1
 *             padded), sel_cnt optional [B][Hq]; kcap >= min(keep, C).
 * The union of a GQA group's kept clusters is read once for the group.  The
 * result does not depend on the copy (same rows, same order).
 */
int cluster_decode_attn(const void* q, const void* k_cache, const void* v_cache, const float* centroids,
                        const int32_t* offsets, const int32_t* tokens, const void* k_packed, const void* v_packed,
                        int B, int Hq, int Hkv, int S, int d, int n_ctx, int C, int keep, float scale, void* o,
                        int32_t* sel_idx, int32_t* sel_cnt, int kcap, void* ws, size_t* ws_bytes,
                        dsa_stream_t stream);

/*
 * dsa_get_status -- synchronize `stream`, read the workspace's device status
 * word, clear it, and return DSA_OK or the first error recorded on the device
 * (DSA_ERR_TIMEOUT for an expired bounded wait, DSA_ERR_INVALID_ARG for a list
 * rejected in validation mode).  Returns DSA_ERR_CUDA if the stream itself
 * reports an error.
 */
int dsa_get_status(const void* ws, dsa_stream_t stream);

/*
 * dsa_block_index_capacity -- the list capacity `kcap` sparse_index_estimate
 * needs for this budget: the largest per-query-block count (sink + diagonal +
 * extra blocks) over all n/64 query blocks.  Same budget rules and argument
 * checks as sparse_index_estimate; returns a negative DSA_ERR_* code on bad
 * arguments.  Host-only, launches nothing.
 */
int dsa_block_index_capacity(int n, int block, int k_fixed, float keep_ratio);

/* Library version string, e.g. "dsa 0.1 sm_100a". */
const char* dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
