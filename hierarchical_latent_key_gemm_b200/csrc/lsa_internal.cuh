// Internal declarations shared by the LSA CUDA translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <vector>

#include "lsa.h"

namespace lsa {

constexpr uint32_t kIndexMagic = 0x4C534131u;   // "LSA1"
constexpr uint32_t kFreedMagic = 0xDEADBEEFu;
constexpr int64_t kNoPos = INT64_MAX;           // minpos of a node with no candidate block

// Error bits latched by kernels into a device word.
enum : int32_t {
    kErrDevice = 1,     // out-of-range index met and skipped
    kErrInexact = 2,    // integer-grid precondition broken
    kErrCapacity = 4,   // a leaf had no free slot on append
    kErrTimeout = 8,    // reserved for bounded waits
};

__device__ __forceinline__ void latch(int32_t* err, int32_t bit) {
    if (err) atomicOr(err, bit);
}

// ----------------------------------------------------------- allocation
// Every device allocation of the library goes through Arena, so a failed
// build frees all it took and the test hook can force a failure.
struct Arena {
    std::vector<void*> ptrs;
    int64_t bytes = 0;
    cudaStream_t stream = nullptr;
    bool async = false;    // stream-ordered scratch (cudaMallocAsync) vs persistent
    int status = LSA_OK;

    template <typename T>
    T* alloc(int64_t count) {
        if (status != LSA_OK) return nullptr;
        void* p = nullptr;
        int64_t nbytes = count * (int64_t)sizeof(T);
        if (nbytes <= 0) nbytes = 256;
        nbytes = (nbytes + 255) & ~int64_t(255);
        if (!alloc_raw(&p, nbytes)) {
            status = LSA_ERR_OOM;
            return nullptr;
        }
        ptrs.push_back(p);
        bytes += nbytes;
        return static_cast<T*>(p);
    }
    bool alloc_raw(void** p, int64_t nbytes);
    void release();
    ~Arena() { release(); }
};

// Counts down the OOM test hook; true = this allocation must fail.
bool debug_alloc_should_fail();

// Host-side count of kernel launches issued by the library (diagnostics).
void note_launch();

}  // namespace lsa

struct lsa_index {
    uint32_t magic;
    lsa_build_params p;
    int device;
    int64_t units;         // batch * hkv
    int64_t nb;            // complete blocks indexed per unit
    int64_t nb_cap;        // block capacity per unit (row stride of Kl)
    int64_t n_tokens;      // tokens indexed per sequence
    int64_t slots;         // total bucket slots over all units
    int32_t L;             // leaves
    float* W;              // [d][r]
    float* Kl;             // [units][nb_cap][r] latent keys, block order
    float* Klp;            // [slots][r] latent keys, bucket order
    int32_t* blk;          // [slots] block id (within its unit) of every slot
    int32_t* leaf_start;   // [units*L] first slot of each leaf (global slot index)
    int32_t* leaf_cnt;     // [units*L] blocks in each leaf
    int32_t* leaf_cap;     // [units*L] slots reserved for each leaf
    int32_t* leaf_of_block;// [units][nb_cap]
    float* cent[LSA_MAX_LEVELS];      // [units*n_l][r]
    int64_t* minpos[LSA_MAX_LEVELS];  // [units*n_l]
    int32_t* parent[LSA_MAX_LEVELS];  // [units*n_l] node id at level l-1 (l >= 1)
    int32_t* child_off[LSA_MAX_LEVELS];  // [units*n_l + 1] into child_ids (l < levels-1)
    int32_t* child_ids[LSA_MAX_LEVELS];  // [units*n_{l+1}] child id within the unit
    double* objective[LSA_MAX_LEVELS];   // [iters][units]
    // The same levels in tree order (children of a node contiguous), the
    // layout the selection reads.  Position q of level l holds node ord_id[q].
    int32_t* ord_id[LSA_MAX_LEVELS];     // [units*n_l] node id at each position
    int32_t* ord_pos[LSA_MAX_LEVELS];    // [units*n_l] position of each node id
    float* ord_cent[LSA_MAX_LEVELS];     // [units*n_l][r]
    int64_t* ord_mp[LSA_MAX_LEVELS];     // [units*n_l] minpos by position
    int32_t* ord_coff[LSA_MAX_LEVELS];   // [units*n_l + 1] global child positions (l < levels-1)
    int32_t* err;          // latched kernel error bits
    lsa::Arena* mem;       // owns every device allocation above
};

namespace lsa {

int cuda_status(cudaError_t e);
int err_bits_to_status(int32_t bits);

// Library-wide error word for calls that have no index (attention, stages).
int32_t* global_err_word();

// ---------------------------------------------------------------- sort/scan
// Exclusive prefix sum of n int32 values; out[n] receives the total when
// out_len > n.  scratch: see scan_scratch_elems.
int64_t scan_scratch_elems(int64_t n);
void scan_exclusive(const int32_t* in, int32_t* out, int64_t n, int32_t* scratch, cudaStream_t s);

// Stable LSD radix sort of (key, value) pairs by the low `bits` bits of key.
// Buffers: k0/v0 hold the input; the sorted result lands in *kout/*vout
// (one of the two buffer pairs).
int64_t radix_scratch_elems(int64_t n);
void radix_sort(uint32_t* k0, int32_t* v0, uint32_t* k1, int32_t* v1, int64_t n, int bits,
                int32_t* scratch, cudaStream_t s, uint32_t** kout, int32_t** vout);

// ---------------------------------------------------------------- k-means
struct KmeansOut {
    int32_t* labels;    // [units*n] local labels (last assign)
    float* C;           // [units*k][r] last update
    int32_t* perm;      // [units*n] global point ids (u*n+i) sorted by (u, label), stable
    int32_t* off;       // [units*k + 1] global offsets into perm
    double* objective;  // [iters][units] or null
};
// X: [units][ldx][r] (rows 0..n-1 of each unit are the points); labels are
// written at out.labels[u*ldl + i].
int run_kmeans(const float* X, int64_t ldx, int64_t units, int64_t n, int r, int k, int iters,
               int grid_log2, KmeansOut out, int64_t ldl, int32_t* err, cudaStream_t s, Arena& scratch,
               const float* C_init = nullptr);

// Stable grouping of points by label (see run_kmeans); workspace sized for
// (units, n, k) by alloc_group_work.
struct GroupWork {
    int64_t total = 0, nc = 0;
    uint32_t *k0 = nullptr, *k1 = nullptr;
    int32_t *v0 = nullptr, *v1 = nullptr, *counts = nullptr, *scratch = nullptr;
};
GroupWork alloc_group_work(int64_t units, int64_t n, int k, Arena& A);
int group_by_label(const int32_t* labels, int64_t ldl, int64_t units, int64_t n, int k, int32_t* perm,
                   int32_t* off, int32_t* err, cudaStream_t s, const GroupWork& w);

// Tensor-core assign (kmeans_tc.cu): prepare the split points once per run,
// then one call per Lloyd round.
bool assign_tc_supported(int r, int grid_log2);
int assign_tc_prepare_points(const float* X, int64_t ldx, int64_t units, int64_t n, int r, int k, const float* C0,
                             Arena& A, cudaStream_t s, void** work_out);
int assign_tc_run(void* work, const float* C, const float* cc, int64_t units, int64_t n, int r, int k,
                  int32_t* labels, int64_t ldl, int32_t* err, cudaStream_t s);
void assign_tc_release(void* work);

// ---------------------------------------------------------------- latents
int launch_project_pool(const void* K, const float* W, int64_t batch, int64_t n_blocks,
                        int64_t ld_tokens, int hkv, int d, int r, int pool, int dtype,
                        float* Kl, int64_t kl_unit_stride, cudaStream_t s);
int launch_query_latent(const void* Q, const float* W, int64_t batch, int64_t nq, int hq, int hkv,
                        int d, int r, int dtype, float* qbar, cudaStream_t s);

// ---------------------------------------------------------------- select
// Scored-blocks output of the tree search (context-parallel shards): per
// (query, KV head) row the kept blocks (index block id + blk_shift) and their
// scores in [row][kb_cap], any order, -1 / -inf after *n; query positions are
// index positions + pos_shift.
struct ScoredOut {
    int64_t pos_shift;
    int32_t blk_shift;
    int kb_cap;
    float* score;
    int32_t* block;
    int32_t* n;
};
int launch_select(const lsa_index* ix, const lsa_select_params* sp, const float* qbar, int64_t nq,
                  const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int max_sel,
                  bool fullscan, cudaStream_t s, unsigned long long* work = nullptr,
                  const ScoredOut* scored = nullptr);
// Dense upper levels scored ahead of the search (node_scores.cu): the
// leading `levels` levels' scores for every node, row-major per (query, KV
// head) row, level l from column off[l]; launch_select_rows runs the search
// over nq rows whose queries, positions and outputs start at the given
// pointers (sequence stride nq_stride) and takes those levels' scores from S.
struct PreScores {
    const float* S;
    int64_t ld;
    int levels;
    int off[LSA_MAX_LEVELS];
    // optional (leaf tiles): per row the kept nodes of the last dense level
    // [row][beam] and their count (-1: the row runs the whole search), and the
    // scores of their children, row-major [row][s2_ld] in kept-node order
    const int32_t* b1;
    const int32_t* nb1;
    const float* S2;
    int64_t s2_ld;
};
int launch_select_rows(const lsa_index* ix, const lsa_select_params* sp, const float* qbar, int64_t nq_stride,
                       int64_t nq, const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int max_sel,
                       bool fullscan, cudaStream_t s, unsigned long long* work, const ScoredOut* scored,
                       const PreScores* pre);
int dense_levels(const lsa_index* ix, int beam, int max_cols, int* col_off);
int launch_node_scores(const lsa_index* ix, const float* qbar, int64_t nq_stride, int64_t nqc, int levels,
                       const int* col_off, float* S, int64_t ld, cudaStream_t s);
// The tree search of nq queries: dense levels first when the call is large
// enough, in chunks of queries whose scores fit a bounded buffer.
int launch_select_tree(const lsa_index* ix, const lsa_select_params* sp, const float* qbar, int64_t nq,
                       const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int max_sel,
                       cudaStream_t s, unsigned long long* work, const ScoredOut* scored, Arena& A);
// Full scan on the tensor cores (fullscan_tc.cu): candidate lists from a
// filtering GEMM, ranked exactly by the per-query kernel (select.cu).
struct ListIn {
    const int32_t* cand;
    const int32_t* count;
    int64_t npad;
    int cap;
};
bool fullscan_tc_applies(const lsa_index* ix, const lsa_select_params* sp);
int launch_fullscan_tc(const lsa_index* ix, const lsa_select_params* sp, const float* qbar, int64_t nq,
                       const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int max_sel,
                       cudaStream_t s, Arena& A);
int launch_select_lists(const lsa_index* ix, const lsa_select_params* sp, const float* qbar, int64_t nq_stride,
                        int64_t nq_grid, const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt,
                        int max_sel, const ListIn& li, cudaStream_t s);
// Merge of per-shard scored blocks into selection rows (select.cu).
int launch_merge_selection(int parts, const float* score, const int32_t* block, const int32_t* count, int kb_cap,
                           int64_t batch, int64_t nq, int hkv, const int64_t* q_pos, int64_t q_pos0, int pool,
                           int kb, int sink, int window, int32_t* idx, int32_t* cnt, int max_sel, cudaStream_t s);
// Rows of a selection inside [lo, hi), shifted by -lo (cp.cu); LSE merge of
// attention parts (cp.cu).
int launch_localize_rows(const int32_t* idx, const int32_t* cnt, int64_t rows, int max_sel, int64_t lo, int64_t hi,
                         int32_t* idx_out, int32_t* cnt_out, cudaStream_t s);
int launch_merge_attn(int parts, const void* O_parts, const float* lse_parts, int64_t rows, int hq, int d, int dtype,
                      void* O, float* lse, cudaStream_t s);

// ---------------------------------------------------------------- attention
int launch_sparse_attn(const void* Q, const void* K, const void* V, const int32_t* idx,
                       const int32_t* cnt, int64_t batch, int64_t nq, int hq, int hkv, int d,
                       int dtype, int max_sel, int64_t ld_tokens, void* O, float* lse,
                       int32_t* err, cudaStream_t s);
int launch_banded_attn(const void* Q, const void* K, const void* V, const int32_t* idx, const int32_t* cnt,
                       int64_t batch, int64_t nq, int64_t q_pos0, int hq, int hkv, int d, int max_sel,
                       int64_t ld_tokens, int sink, int window, void* O, float* lse, int32_t* err, cudaStream_t s);
// training-free latent map (pca.cu)
int launch_pca_map(const void* K, int64_t batch, int64_t n_tokens, int64_t ld_tokens, int hkv, int d, int pool,
                   int dtype, int r, float* W, double* evals, cudaStream_t s);
// tensor-core band of the banded attention (attn_band_tc.cu): partials as the mma.sync band kernel writes them
int launch_band_tc(const void* Q, const void* K, const void* V, int64_t batch, int64_t nq, int64_t q_pos0, int hq,
                   int hkv, int d, int64_t ld_tokens, int sink, int window, float* part_o, float2* part_ml,
                   int32_t* err, cudaStream_t s);

// ---------------------------------------------------------------- append
int launch_append(lsa_index* ix, const void* K, int64_t first_block, int64_t n_new_blocks,
                  cudaStream_t s);

// ---------------------------------------------------------------- tree finish
// Given leaf labels with their stable order, the upper-level parents with
// theirs, and the centroids, lay out the buckets, child lists and minpos.
int finish_tree(lsa_index* ix, const int32_t* leaf_perm, const int32_t* leaf_off,
                const int32_t* const* up_perm, const int32_t* const* up_off, cudaStream_t s,
                Arena& scratch);

// Decode maintenance: lay the leaves out again from the block labels
// (tree.cu), recompute every centroid from its members (kmeans.cu), and the
// tree-order copies of centroids and minpos that the selection reads.
int relayout_leaves(lsa_index* ix, cudaStream_t s, Arena& scratch);
int refresh_centroids(lsa_index* ix, cudaStream_t s, Arena& scratch);
void gather_tree_order(lsa_index* ix, cudaStream_t s);

}  // namespace lsa
