/*
 * lsa.h - C ABI of the Latent Sparse Attention (LSA) hot path on NVIDIA B200.
 *
 * LSA replaces the full key scan of a sparse-attention indexer by a search
 * through a hierarchy of key clusters built in a low-rank latent space, and
 * then runs exact softmax attention over the keys it picked.
 *
 * Sources (web pages on LSA), cited below by key and section:
 *  [p1] "The 10M-token attention layer spends 98% of its time finding tokens"
 *  [p2] "Latent Sparse Attention speeds up the search for useful tokens in very
 *       long contexts", "Reduce the cost of finding the tokens to attend to"
 *  [p3] "Latent Sparse Attention: tree search over keys for 10M-token context",
 *       TL;DR and flowchart
 *  [p4] "Researchers report 72.4x faster attention-layer prefill at 10 million
 *       tokens", "Search the clusters, not every key", "Prompt processing is
 *       not response generation"
 *  [p5] "Latent Sparse Attention (LSA): The 72.4x and 22.7x Speedups, and What
 *       They Compare Against", "How does LSA work?" steps 1-3, "Prefill,
 *       decode and training", "Can I run LSA?"
 *
 * Conventions for every call:
 *  - Pointers named "device" must be CUDA device memory of the current device
 *    (or managed memory); "host" pointers are ordinary host memory.
 *  - Tensors are dense, row-major, with the layouts stated per argument.
 *    Head-of-sequence layouts: K and V are [batch][ld_tokens][hkv][d];
 *    Q is [batch][nq][hq][d].  dtype is LSA_F32 or LSA_BF16 (IEEE bf16).
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and is asynchronous unless stated otherwise.  Argument errors are
 *    detected on the host and returned before anything is enqueued.
 *  - Errors found by a kernel (an index out of range, a broken exactness
 *    precondition, a full leaf) are latched in a device word of the index or
 *    of the library and reported by lsa_check(), which synchronises.
 *  - The caller owns every buffer it passes.  An lsa_index owns the device
 *    memory of the latent keys, centroids and bucket lists; it keeps no
 *    pointer to the caller's K, Q, V or W after a call returns.
 *  - No call aborts or throws.  Every int-returning call returns an
 *    lsa_status code.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct lsa_index lsa_index;

typedef enum {
    LSA_OK = 0,
    LSA_ERR_INVALID_ARG = 1,   /* bad pointer, size, layout or parameter */
    LSA_ERR_CUDA = 2,          /* a CUDA runtime call failed */
    LSA_ERR_OOM = 3,           /* device allocation failed; nothing leaked */
    LSA_ERR_INEXACT = 4,       /* integer-grid mode met a value off its exact range */
    LSA_ERR_TIMEOUT = 5,       /* reserved: a bounded device wait gave up */
    LSA_ERR_DEVICE = 6,        /* a kernel met an out-of-range index and skipped it */
    LSA_ERR_CAPACITY = 7       /* lsa_append found a leaf with no free slot */
} lsa_status;

typedef enum { LSA_F32 = 0, LSA_BF16 = 1 } lsa_dtype;

#define LSA_MAX_LEVELS 4

/* Index construction parameters.  [p5 "How does LSA work?" step 1: blocks of
 * keys are averaged, mapped to a low-rank latent space and grouped into
 * buckets that form a tree; p2: the hierarchical tree variant.] */
typedef struct {
    int64_t batch;          /* sequences (>= 1) */
    int64_t n_tokens;       /* tokens per sequence to index (>= 1) */
    int64_t ld_tokens;      /* token capacity per sequence of the K buffer (>= n_tokens) */
    int32_t hkv;            /* KV heads; every (sequence, KV head) is one unit with its own tree */
    int32_t d;              /* head dimension: 64 or 128 */
    int32_t r;              /* latent rank: 16, 32, 64 or 128 */
    int32_t pool;           /* P keys per pooled block, 1..16 */
    int32_t dtype;          /* lsa_dtype of K */
    int32_t levels;         /* tree depth 1..LSA_MAX_LEVELS (1 = flat buckets) */
    int32_t level_sizes[LSA_MAX_LEVELS]; /* nodes per level, top first, leaves last, non-decreasing */
    int32_t lloyd_iters;    /* Lloyd rounds per level (>= 1) */
    int32_t grid_log2;      /* 0: float centroids; g in 1..8: centroids rounded half-to-even
                               onto multiples of 2^-g (exact integer workloads) */
    int32_t sink;           /* S: blocks that start before token S are never candidates */
    int64_t append_capacity;/* tokens per sequence lsa_append may add after the build (>= 0) */
} lsa_build_params;

/* Selection parameters.  [p5 "How does LSA work?" steps 2-3; p3 TL;DR] */
typedef struct {
    int32_t hq;             /* query heads; a multiple of hkv; each KV head's group of
                               hq/hkv query heads shares one selection (mean latent query) */
    int32_t beam;           /* B: nodes kept per tree level (1..1024) */
    int32_t topk;           /* K: long-range budget in tokens; ceil(K/P) blocks are taken */
    int32_t sink;           /* S: must equal the build's sink */
    int32_t window;         /* W: causal local window in tokens (>= 1) */
} lsa_select_params;

/* Host-side description of an index (lsa_index_info). */
typedef struct {
    int64_t units;          /* batch * hkv */
    int64_t n_tokens;       /* tokens indexed so far, per sequence */
    int64_t n_blocks;       /* complete blocks indexed so far, per unit */
    int64_t block_capacity; /* blocks per unit the slot arrays can hold */
    int64_t device_bytes;   /* device memory held by the index */
    int32_t levels;
    int32_t level_sizes[LSA_MAX_LEVELS];
    int32_t r, pool, sink, grid_log2;
} lsa_index_info_t;

/* What lsa_index_get copies out. */
typedef enum {
    LSA_GET_CENTROIDS = 0,     /* float  [units][level_sizes[level]][r] */
    LSA_GET_PARENT = 1,        /* int32  [units][level_sizes[level]]  (level >= 1) */
    LSA_GET_LEAF_OF_BLOCK = 2, /* int32  [units][n_blocks] */
    LSA_GET_MINPOS = 3,        /* int64  [units][level_sizes[level]]  (INT64_MAX = none) */
    LSA_GET_OBJECTIVE = 4,     /* double [lloyd_iters][units] of that level's k-means */
    LSA_GET_LATENT = 5,        /* float  [units][n_blocks][r] latent keys in block order */
    LSA_GET_LEAF_COUNT = 6     /* int32  [units][leaves] blocks per leaf */
} lsa_get_what;

/* ----------------------------------------------------------------- calls */

/* Build the bucket hierarchy of every (sequence, KV head).
 *  K: device, [batch][ld_tokens][hkv][d] of dtype; tokens [0, n_tokens) are read.
 *  W: device, float [d][r], the latent map (row = input dimension).
 * Steps: latent keys Kl[b] = W^T * mean(K[bP .. bP+P-1]) for every complete
 * block; Lloyd k-means of the latent keys into level_sizes[levels-1] leaves
 * (centroid j starts at point floor(j*n/k); ties to the lower id; an empty
 * cluster keeps its centroid); then k-means of each level's centroids into
 * the level above.  [p1: keys are clustered before any query is scored; p5 step 1; p2]
 * On success *out receives a new index owned by the caller (lsa_free_index).
 * On failure *out is set to NULL and no device memory is left allocated.
 * The build is enqueued on `stream`; lsa_check() reports device-side errors. */
int lsa_build_index(const lsa_build_params* params, const void* K, const float* W,
                    void* stream, lsa_index** out);

/* Same index, but with the clustering given instead of computed (for
 * decoupled checks and for trees made elsewhere).
 *  leaf_of_block: device int32 [units][n_blocks], leaf id of every block.
 *  parents[l] for l = 1..levels-1: device int32 [units][level_sizes[l]],
 *      parent (at level l-1) of every level-l node; parents[0] is ignored.
 *  centroids[l] for l = 0..levels-1: device float [units][level_sizes[l]][r].
 * Latent keys are still computed from K and W. */
int lsa_build_index_from_tree(const lsa_build_params* params, const void* K, const float* W,
                              const int32_t* leaf_of_block, const int32_t* const* parents,
                              const float* const* centroids, void* stream, lsa_index** out);

/* Tree-search selection for nq queries per sequence.
 *  Q: device [batch][nq][hq][d] of the index's dtype.
 *  q_pos: device int64 [batch][nq] query positions, or NULL for
 *      position(query j) = q_pos0 + j in every sequence.
 *  idx: device int32 [batch][nq][hkv][max_sel]; cnt: device int32 [batch][nq][hkv].
 * For the query at position i and KV head h: latent query = mean over the
 * group's heads of W^T q; at each level score the eligible nodes (all top
 * nodes, then the children of the kept ones) by latent dot product and keep the
 * best `beam`; score the candidate blocks of the kept leaves and keep the best
 * ceil(K/P).  A block is a candidate iff it starts at or after S and ends at or
 * before i - W; a node is eligible iff it holds a candidate.  Ties go to the
 * lower id.  The row of idx lists, ascending, the sink [0, min(S, i+1)), the
 * tokens of the chosen blocks and the window [max(0, i-W+1), i]; cnt holds its
 * length and the rest of the row is -1.  max_sel must be at least
 * ceil(K/P)*P + S + W.  Calls of 4,096 or more (query, KV head) pairs score
 * the dense upper levels (and, when the leaf level is the only one below
 * them, the kept nodes' leaves) for tiles of queries first, with the same
 * arithmetic, so the rows are the same bits; that takes stream-ordered
 * scratch (pool memory) of at most 1 GiB, or 2 GiB with the leaf scores, per
 * call, the queries running in chunks that fit.  [p3 TL;DR: the query is
 * compared with centroids first and only a few buckets are searched; p1;
 * p5 steps 2-3] */
int lsa_select(const lsa_index* index, const lsa_select_params* params, const void* Q,
               int64_t nq, const int64_t* q_pos, int64_t q_pos0,
               int32_t* idx, int32_t* cnt, int32_t max_sel, void* stream);

/* Allocation-free form of lsa_select.  The pages have no counterpart: this
 * is a deployment aid.  lsa_select takes its scratch (the latent queries,
 * batch*nq*hkv*r floats) from the device's stream-ordered pool.  Some callers
 * cannot allocate device memory while they serve: a framework whose caching
 * allocator already owns the device's memory, a decode loop that must never
 * stall on an allocation or trigger a pool trim, a process that fixes its
 * memory budget before it starts serving.  This call instead uses one fixed
 * buffer of LSA_SELECT_NOALLOC_MAX_FLOATS floats (4 MiB), declared by the
 * library as a device variable; every GPU that loads the library holds those
 * 4 MiB until the process exits.
 *  - Arguments, results and errors are those of lsa_select.
 *  - batch*nq*hkv*r above LSA_SELECT_NOALLOC_MAX_FLOATS returns
 *    LSA_ERR_INVALID_ARG before anything is enqueued (split the queries into
 *    chunks and pass q_pos0 per chunk).
 *  - It calls no cudaMalloc, cudaFree or other allocating routine.
 *  - Its first call on a device looks up the buffer's device address, once
 *    per device, with that device current; make that first call before any
 *    stream capture.
 *  - Every call shares the one buffer and it keeps the last call's contents.
 *    Each call rewrites all of the part it reads, so nothing needs clearing,
 *    but calls whose GPU work can overlap (e.g. two streams with no ordering
 *    between them) race on the buffer and must not be issued that way. */
#define LSA_SELECT_NOALLOC_MAX_FLOATS 1048576
int lsa_select_noalloc(const lsa_index* index, const lsa_select_params* params, const void* Q,
                       int64_t nq, const int64_t* q_pos, int64_t q_pos0,
                       int32_t* idx, int32_t* cnt, int32_t max_sel, void* stream);

/* lsa_select that also counts the latent rows it scored, summed over all
 * (query, KV head) pairs: scored is a device uint64[2] the caller zeroes;
 * scored[0] += eligible tree nodes scored (centroid rows), scored[1] +=
 * candidate blocks scored (latent key rows).  These are the work counts behind
 * a bytes-moved figure (each scored row is r values).  Same results as
 * lsa_select; costs two atomic adds per warp.  The pages give no
 * counterpart: it exists for measurement. */
int lsa_select_work(const lsa_index* index, const lsa_select_params* params, const void* Q,
                    int64_t nq, const int64_t* q_pos, int64_t q_pos0,
                    int32_t* idx, int32_t* cnt, int32_t max_sel, unsigned long long* scored,
                    void* stream);

/* Training-free latent map: W = the r leading principal directions of the
 * pooled keys ([p5] "How does LSA work?", the D-LSA options, one of which
 * needs no training and takes a PCA map).  Every (sequence, KV head)'s keys are pooled as
 * in the build (mean of `pool` consecutive keys, complete blocks only) and all
 * pooled keys form one sample; their covariance (centred, divided by the
 * count, accumulated in fp64) is diagonalised on the device (parallel cyclic
 * Jacobi).
 *  K: device [batch][ld_tokens][hkv][d] (bf16 or f32), tokens [0, n_tokens).
 *  W: device float [d][r] out: eigenvectors of the r largest eigenvalues in
 *     descending order, each signed so that its entry of largest magnitude
 *     (lowest index among equal magnitudes) is positive; usable directly as
 *     the W of lsa_build_index / lsa_select.
 *  eigvals: device double [r] out (the r largest eigenvalues), or NULL.
 *  d in {64, 128}; 1 <= r <= d; at least one complete block.
 *  Errors: LSA_ERR_INVALID_ARG before anything is enqueued; LSA_ERR_OOM for
 *  its stream-ordered scratch (2 d^2 + d doubles). */
int lsa_pca_map(const void* K, int64_t batch, int64_t n_tokens, int64_t ld_tokens, int32_t hkv,
                int32_t d, int32_t pool, int32_t dtype, int32_t r, float* W, double* eigvals,
                void* stream);

/* The quadratic baseline indexer: every candidate block is scored, no tree.
 * Same arguments and output format as lsa_select (beam is ignored).
 * Calls of 64 or more (query, KV head) pairs with r <= 64 first filter on the
 * tensor cores (fp16 scores of 128 queries x 256 blocks per tile; a per-query
 * histogram gives a threshold that provably keeps every block of the exact
 * top ceil(K/P)), then rank the survivors with the exact fp32 arithmetic of
 * the per-query kernel, so the selected blocks are the same bits as scoring
 * every block exactly.  Stream-ordered scratch: the fp16 keys (2 B x 64 per
 * block), and for each chunk of up to ~2 GiB/(16 KB x KV heads) queries,
 * 16 KB of candidate lists per (query, KV head).
 * [p3 flowchart, red path: the full key scan] */
int lsa_fullscan_select(const lsa_index* index, const lsa_select_params* params, const void* Q,
                        int64_t nq, const int64_t* q_pos, int64_t q_pos0,
                        int32_t* idx, int32_t* cnt, int32_t max_sel, void* stream);

/* ---------------------------------------------------------------------
 * Context parallelism: one sequence's context split over shards (GPUs).
 * The pages say only that the 10M-token runs split one sequence over several
 * GPUs ([p5] "What do 22.7x and 72.4x actually compare?", "Can I run
 * LSA?").  Reading used here: shard s holds the block-aligned token range
 * [t0_s, t1_s) of K and V and its own index over it (built with
 * sink = max(0, S - t0_s), so the sink rule stays the global one); every
 * shard picks its local top ceil(K/P) blocks with their scores
 * (lsa_select_blocks); the picks of all shards are merged into the global top
 * ceil(K/P) by (score desc, block asc), and the selection row is written as
 * lsa_select writes it (lsa_merge_selection); each shard attends the rows of
 * that selection it holds (lsa_localize_rows + lsa_sparse_attn, with lse) and
 * the parts are combined by their log-sum-exps (lsa_merge_attn).  The
 * collectives between the steps (an all-gather of the picks, an all-gather of
 * the attention parts) are the caller's (NCCL through torch.distributed in
 * the Python package). */

/* The tree search of lsa_select on one shard, returning the chosen blocks
 * with their scores instead of a selection row.
 *  index: the shard's index (tokens of the shard in its own positions 0..).
 *  Q, nq, q_pos, q_pos0: as lsa_select, positions in the WHOLE sequence.
 *  token_offset: the shard's first token t0 (a multiple of the pool size); a
 *      query at position i is searched at index position i - token_offset
 *      (negative: nothing is chosen).
 *  scores: device float [batch][nq][hkv][kb_cap], blocks: device int32
 *      [batch][nq][hkv][kb_cap] (block ids in the whole sequence, i.e. index
 *      block + t0/P), count: device int32 [batch][nq][hkv]: entries
 *      [0, count) hold the chosen blocks in no particular order; the rest
 *      are -inf / -1.  kb_cap >= ceil(K/P).
 * Same rules, arithmetic and ties as lsa_select.  Stream-ordered scratch as
 * lsa_select. */
int lsa_select_blocks(const lsa_index* index, const lsa_select_params* params, const void* Q, int64_t nq,
                      const int64_t* q_pos, int64_t q_pos0, int64_t token_offset, float* scores, int32_t* blocks,
                      int32_t* count, int32_t kb_cap, void* stream);

/* Merge of the shards' picks into selection rows.
 *  scores, blocks, count: device, parts x the layouts of lsa_select_blocks
 *      (part p at offset p * batch * nq * hkv rows); 1 <= parts <= 64,
 *      parts * kb_cap <= 16384.  Block ids must be distinct within a row.
 *  q_pos / q_pos0: positions of the queries in the whole sequence.
 *  idx, cnt, max_sel: as lsa_select (max_sel >= ceil(K/P)*P + S + W).
 * Per (query, KV head): the top ceil(K/P) of the union of the parts by
 * (score desc, block asc), then the row sink | tokens of the chosen blocks |
 * window, ascending, -1 after, as lsa_select. */
int lsa_merge_selection(int32_t parts, const float* scores, const int32_t* blocks, const int32_t* count,
                        int32_t kb_cap, int64_t batch, int64_t nq, int32_t hkv, const int64_t* q_pos, int64_t q_pos0,
                        int32_t pool, int32_t topk, int32_t sink, int32_t window, int32_t* idx, int32_t* cnt,
                        int32_t max_sel, void* stream);

/* The entries of selection rows that fall in [lo, hi), shifted by -lo, in
 * order: rows of the caller's shard in the shard's own token positions.
 *  idx, cnt: device [rows][max_sel] and [rows] (entries past cnt ignored);
 *  idx_out, cnt_out: device, same shapes; idx_out may be idx itself, or must
 *  not overlap it.  Rows left without entries get cnt_out = 0 (lsa_sparse_attn
 *  then gives O = 0 and lse = -inf for them). */
int lsa_localize_rows(const int32_t* idx, const int32_t* cnt, int64_t rows, int32_t max_sel, int64_t lo, int64_t hi,
                      int32_t* idx_out, int32_t* cnt_out, void* stream);

/* Attention over a union of disjoint row sets from its parts:
 *  O_parts: device [parts][rows][hq][d] of dtype (each part normalised over
 *  its own rows), lse_parts: device float [parts][rows][hq] (natural log of
 *  the part's softmax denominator, -inf for an empty part).
 *  O: device [rows][hq][d]; lse: device float [rows][hq] or NULL.
 * O = sum_s e^(lse_s - m) O_s / sum_s e^(lse_s - m), lse = m + log(sum_s
 * e^(lse_s - m)), m = max_s lse_s (parts in order, fp32); all parts empty ->
 * O = 0, lse = -inf.  rows = batch * nq of the attention calls. */
int lsa_merge_attn(int32_t parts, const void* O_parts, const float* lse_parts, int64_t rows, int32_t hq, int32_t d,
                   int32_t dtype, void* O, float* lse, void* stream);

/* Exact softmax attention over selected tokens.
 *  Q: device [batch][nq][hq][d]; K, V: device [batch][ld_tokens][hkv][d];
 *  idx/cnt as written by lsa_select (entries past cnt are ignored).
 *  O: device [batch][nq][hq][d] of dtype; lse: device float [batch][nq][hq]
 *  or NULL (natural log of the softmax denominator of the scaled scores).
 * O[q,h] = sum_j softmax_j(q_h . k_j / sqrt(d)) v_j over the row of KV head
 * h / (hq/hkv); fp32 accumulation.  A row with cnt = 0 yields O = 0 and
 * lse = -inf.  An index outside [0, ld_tokens) is skipped and latched as
 * LSA_ERR_DEVICE.  For bf16, Q, K, V and O must be 16-byte aligned (else
 * LSA_ERR_INVALID_ARG).  [p5 step 3: LSA leaves the attention itself as it
 * was; p3 flowchart: exact attention over the subset] */
int lsa_sparse_attn(const void* Q, const void* K, const void* V, const int32_t* idx,
                    const int32_t* cnt, int64_t batch, int64_t nq, int32_t hq, int32_t hkv,
                    int32_t d, int32_t dtype, int32_t max_sel, int64_t ld_tokens,
                    void* O, float* lse, void* stream);

/* The same attention for a run of consecutive query positions, faster when
 * each row list is a selection as lsa_select writes it: query qi sits at
 * position i = q_pos0 + qi and its row is the sink [0, min(sink, i+1)), then
 * long-range tokens in [sink, i-window], then the window
 * [max(sink, i-window+1), i], ascending without repeats.  The sink and window
 * rows are read once per tile of consecutive queries (a dense band, masked per
 * query) and only the long-range entries are gathered per query; the two
 * softmax parts are merged by their maxima, so the result is the attention of
 * lsa_sparse_attn over the same row up to fp32 rounding order.
 *  - Arguments as lsa_sparse_attn, plus q_pos0 (>= 0, q_pos0 + nq <=
 *    ld_tokens), sink (>= 0) and window (>= 1), the values lsa_select used.
 *  - A row that is ascending but not of that form is attended whole from the
 *    list, with the same result; rows must be ascending without repeats.
 *  - bf16 with hq/hkv in {1, 2, 4, 8, 16} takes the band path; other cases
 *    run the lsa_sparse_attn kernels.
 *  - Needs batch*nq*hq*(d+2) floats of stream-ordered scratch (pool memory).
 * [p5 step 3: attention covers the chosen distant keys, the first S tokens
 * and the last W; the attention kernel itself is unchanged] */
int lsa_sparse_attn_banded(const void* Q, const void* K, const void* V, const int32_t* idx,
                           const int32_t* cnt, int64_t batch, int64_t nq, int64_t q_pos0,
                           int32_t hq, int32_t hkv, int32_t d, int32_t dtype, int32_t max_sel,
                           int64_t ld_tokens, int32_t sink, int32_t window,
                           void* O, float* lse, void* stream);

/* Decode: index tokens [n_tokens, n_tokens + n_new) that the caller has
 * already written into K (same layout and ld_tokens as the build).  Every
 * block this completes is pooled, mapped, and placed in its nearest leaf
 * (squared distance over all leaves, frozen centroids, ties to the lower id)
 * after that leaf's older blocks; node eligibility is updated.  A leaf with
 * no free slot latches LSA_ERR_CAPACITY: the block keeps its leaf label
 * (LSA_GET_LEAF_OF_BLOCK) but is not selectable until lsa_relayout.
 * [p5 "Prefill, decode and training"; p4 "Prompt processing is not response
 * generation"] */
int lsa_append(lsa_index* index, const void* K, int64_t n_new, void* stream);

/* Decode maintenance, part 1 (the pages say nothing about keeping the index
 * up during decode, only that every generated token looks at all earlier
 * tokens, p5 "Prefill, decode and training"; this is the plainest
 * upkeep that leaves the selection rule unchanged).  Lays the leaf buckets of
 * every unit out again from the current leaf labels: each leaf's blocks in
 * ascending order, the blocks that lsa_append gave to a full leaf
 * (LSA_ERR_CAPACITY) included, then fresh free slots for the append capacity
 * that is left, shared among the leaves in proportion to their sizes as at
 * the build; minpos of every node is recomputed.  Labels and centroids do not
 * change, so lsa_select afterwards sees every block exactly where lsa_append
 * put it.  Clears a latched LSA_ERR_CAPACITY (other latched bits stay).
 *  - Stream-ordered, no host synchronisation; stream-ordered scratch of about
 *    5 x 4 B per indexed block.
 *  - Returns LSA_ERR_CAPACITY, with nothing changed, if the index's slot
 *    arrays could not hold the layout (cannot happen within the build's
 *    append_capacity); LSA_ERR_INVALID_ARG for a dead handle. */
int lsa_relayout(lsa_index* index, void* stream);

/* Decode maintenance, part 2 (a reading like part 1): recompute every
 * centroid from its current members, memberships fixed, bottom-up: a leaf's
 * centroid is the mean of the latent keys of its blocks (appended blocks
 * included, those waiting for lsa_relayout too), an upper node's the mean of
 * its children's refreshed centroids; the rules of the build's update step
 * (fp64 sums in ascending member order, an empty node keeps its centroid,
 * rounding onto the grid when grid_log2 > 0).  Right after a build it changes
 * nothing.  Later appends use the refreshed leaf centroids.
 *  - Stream-ordered; scratch as lsa_relayout.  LSA_ERR_INVALID_ARG for a
 *    dead handle; a broken grid precondition latches LSA_ERR_INEXACT.
 * [p5 step 1: keys clustered into buckets organised as a hierarchy] */
int lsa_refresh_centroids(lsa_index* index, void* stream);

/* Stage calls, exposed for checks and for callers that compose the path. */

/* Kl[u][b][:] = W^T * mean of the P keys of block b, for every complete block
 * of tokens [0, n_tokens).  Kl: device float [batch*hkv][n_tokens/P][r]. */
int lsa_project_pool(const void* K, const float* W, int64_t batch, int64_t n_tokens,
                     int64_t ld_tokens, int32_t hkv, int32_t d, int32_t r, int32_t pool,
                     int32_t dtype, float* Kl, void* stream);

/* qbar[b][j][h][:] = mean over the group of KV head h of W^T Q[b][j][g][:].
 * qbar: device float [batch][nq][hkv][r]. */
int lsa_query_latent(const void* Q, const float* W, int64_t batch, int64_t nq, int32_t hq,
                     int32_t hkv, int32_t d, int32_t r, int32_t dtype, float* qbar, void* stream);

/* Lloyd k-means of `units` independent point sets.
 *  X: device float [units][n][r]; labels: device int32 [units][n];
 *  C: device float [units][k][r] (output); objective: device double
 *  [iters][units] (sum of squared distances after each assign) or NULL.
 *  C_init: device float [units][k][r], the centroids the first round assigns
 *  against, or NULL for the build's stride init (centroid j = point
 *  floor(j*n/k)); it may not overlap C.  Starting from given centroids lets a
 *  caller run any single Lloyd round of a longer run.
 * Same rules as the build (ties low, empty keeps, grid). */
int lsa_kmeans(const float* X, int64_t units, int64_t n, int32_t r, int32_t k, int32_t iters,
               int32_t grid_log2, int32_t* labels, float* C, const float* C_init, double* objective,
               void* stream);

/* Copy one array of the index to `dst` (device or host memory, dst_bytes
 * large enough; see lsa_get_what for shapes).  Synchronises `stream`.
 * Index statistics are read through this call and lsa_index_info: the
 * objective after every Lloyd round of every level (LSA_GET_OBJECTIVE), the
 * bucket sizes (LSA_GET_LEAF_COUNT), the device bytes held
 * (lsa_index_info_t.device_bytes), and every array of the tree. */
int lsa_index_get(const lsa_index* index, int32_t what, int32_t level, void* dst,
                  int64_t dst_bytes, void* stream);

/* Host-side description; does not touch the device. */
int lsa_index_info(const lsa_index* index, lsa_index_info_t* out);

/* Synchronise `stream`, then return and clear the first error latched by a
 * kernel of this index (or of index-free calls when index is NULL). */
int lsa_check(lsa_index* index, void* stream);

/* Free an index (NULL is a no-op).  A pointer that is not a live index is
 * detected by its magic word and ignored. */
void lsa_free_index(lsa_index* index);

/* Static text for a status code. */
const char* lsa_strerror(int status);

/* Test hook: make the n-th next device allocation of the library fail
 * (n >= 1), to exercise the LSA_ERR_OOM path; n = 0 disarms it. */
void lsa_debug_fail_alloc_after(int32_t n);

/* Test hook for the dense-level scoring of large selections (the scores of
 * the upper tree levels whose parents all fit in the beam, computed for a
 * tile of queries at a time before the per-query search; the selection is
 * bit-identical either way): min_pairs < 0 turns it off, 0 restores the
 * default threshold of (query, KV head) pairs per call, > 0 sets it;
 * chunk_bytes > 0 bounds the score buffer (queries run in chunks that fit),
 * 0 restores the default of 1 GiB. */
void lsa_debug_dense_config(int64_t min_pairs, int64_t chunk_bytes);

/* Test hook for the leaf tiles of large selections (when the leaf level is the
 * only level below the dense ones: the kept nodes of the last dense level and
 * the kept leaves are chosen for all queries by exact warp-wide selections,
 * and the leaves' scores computed per node for many queries at a time; the
 * selection is bit-identical either way): on = 0 turns them off, 1 on (the
 * default). */
void lsa_debug_leaf_tiles(int32_t on);

/* One prefill layer from host memory: build the index of K, select for every
 * query position 0 .. nq-1, and attend (banded form), with the host-device
 * copies overlapped with the kernels.  [p5 "How does LSA work?" steps 1-3:
 * the keys are bucketed, each query searches the buckets, attention covers
 * the chosen keys, the sink and the window; p4 "Prompt processing is not
 * response generation": prefill selects for every position at once]
 * A context holds the device copies of Q, K, V, W, O and lse, the selection
 * rows of one chunk, three streams and their events:
 *  - lsa_prefill_create: params->batch must be 1; 1 <= nq <= n_tokens; the
 *    queries are split into min(chunks, nq) chunks of consecutive positions
 *    (chunks >= 1).  Allocates with cudaMalloc (synchronous).  On failure
 *    *out is NULL and nothing is left allocated.
 *  - lsa_prefill_run enqueues one layer after the work already on `stream`
 *    and makes `stream` wait for all of it:
 *      hK, hV: host [1][ld_tokens][hkv][d] of dtype (all ld_tokens rows are
 *        copied); hW: host float [d][r]; hQ: host [1][nq][hq][d] of dtype;
 *      hO: host [1][nq][hq][d] of dtype, written; hlse: host float [1][nq][hq]
 *        or NULL (then the lse is not copied back).
 *    K and W go up first and the index is built while V and then the queries
 *    go up chunk by chunk; each chunk is selected and attended as soon as its
 *    queries are up, and its output comes down while the next chunk
 *    computes.  Results are those of lsa_build_index, lsa_select and
 *    lsa_sparse_attn_banded called per chunk (q_pos0 = the chunk's first
 *    position) with the same parameters.  Host buffers must stay valid until
 *    `stream` passes the run; pinned (page-locked) memory lets the copies
 *    overlap, pageable memory works but serialises them.  Runs on one
 *    context are ordered among themselves whatever streams they are given.
 *    On success *index_out receives the layer's index, owned by the caller
 *    (lsa_free_index once `stream` has passed the run); on an error it is
 *    NULL, the work already enqueued still completes before `stream` goes on,
 *    and the context stays usable.  The current device must be the one the
 *    context was created on.
 *  - lsa_prefill_free synchronises the context's streams and frees it. */
typedef struct lsa_prefill lsa_prefill;
int lsa_prefill_create(const lsa_build_params* params, const lsa_select_params* sp, int64_t nq,
                       int32_t chunks, lsa_prefill** out);
int lsa_prefill_run(lsa_prefill* prefill, const void* hQ, const void* hK, const void* hV, const float* hW,
                    void* hO, float* hlse, void* stream, lsa_index** index_out);
void lsa_prefill_free(lsa_prefill* prefill);

/* Number of kernels the library has launched in this process (a host-side
 * counter, incremented at every launch; for accounting in benchmarks). */
int64_t lsa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H_ */
