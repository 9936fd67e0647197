// Scores of the dense upper tree levels for a tile of queries at a time.
//
// The tree search (tree-search wiki note, TL;DR; LSA explainer, "How does LSA
// work?" step 2) keeps, level by level, the best `beam` of the eligible nodes.
// While the levels above a level hold no more nodes than the beam, every
// eligible node of it is a candidate for every query: that level is scored
// densely, the same rows for all queries of a KV head.  This kernel computes
// q̄ · c for all of those (query, node) pairs as a register-tiled fp32 product
// (64 queries x 64 nodes per pass of a CTA, 4 x 4 per thread, both operands in
// shared memory), so the per-query search reads one float per node instead of
// a centroid row.
//
// The scores are bit-identical to the per-query kernel's dot products: that
// kernel splits a row of r floats into 2 r / 8 runs of 8, lane g of a group
// of r / 16 lanes accumulates run g and run r/16 + g in two fused multiply-add
// chains from zero, adds them, and the group sums its lanes by a butterfly of
// xor-shuffles (strides r/32, ..., 1).  The same runs, chains and additions
// are taken here in the same order (tree<g, o> below), so the selection does
// not depend on which kernel scored a node.
#include <atomic>

#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kNsThreads = 256;
constexpr int kNsTq = 64;   // queries per CTA tile
constexpr int kNsTn = 64;   // nodes per pass
constexpr int kNsPad = 4;   // shared row padding (keeps 16-byte alignment)

struct NsArgs {
    const float* qbar;       // rows (bseq * nq_stride + qi) * hkv + h, qi in [0, nqc)
    int64_t nq_stride, nqc;
    int hkv;
    const float* cent[LSA_MAX_LEVELS];   // [units * n_l][r], tree order
    int n_l[LSA_MAX_LEVELS];
    int col_off[LSA_MAX_LEVELS + 1];     // first column of each scored level
    int levels;                          // scored levels (leading ones)
    int ncols;                           // col_off[levels]
    float* S;                            // rows (bseq * nqc + qi) * hkv + h
    int64_t ld;                          // floats per row of S (multiple of 4)
};

// acc[i][j] (queries 4 tq + i, nodes 4 tn + j) = the fused multiply-add chain
// over dims 8 c .. 8 c + 7, from zero
template <int R>
__device__ __forceinline__ void chain(const float* qs, const float* cs, int tq, int tn, int c, float (&acc)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int d = 8 * c + j;
        const float4 a = *reinterpret_cast<const float4*>(qs + d * (kNsTq + kNsPad) + 4 * tq);
        const float4 b = *reinterpret_cast<const float4*>(cs + d * (kNsTn + kNsPad) + 4 * tn);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[i * 4 + k] = __fmaf_rn(av[i], bv[k], acc[i * 4 + k]);
    }
}

// value of lane g of a group of LPC lanes after the xor-shuffle steps of
// stride LPC/2 .. O have been applied (O == LPC: before any, the lane's own
// sum of its two chains)
template <int R, int G, int O>
__device__ __forceinline__ void tree(const float* qs, const float* cs, int tq, int tn, float (&out)[16]) {
    constexpr int LPC = R / 16;
    if constexpr (O == LPC) {
        float t[16];
        chain<R>(qs, cs, tq, tn, G, out);
        chain<R>(qs, cs, tq, tn, LPC + G, t);
#pragma unroll
        for (int e = 0; e < 16; ++e) out[e] = __fadd_rn(out[e], t[e]);
    } else {
        float t[16];
        tree<R, G, 2 * O>(qs, cs, tq, tn, out);
        tree<R, (G ^ O), 2 * O>(qs, cs, tq, tn, t);
#pragma unroll
        for (int e = 0; e < 16; ++e) out[e] = __fadd_rn(out[e], t[e]);
    }
}

template <int R>
__global__ __launch_bounds__(kNsThreads) void node_scores_kernel(const NsArgs a) {
    __shared__ __align__(16) float qs[R * (kNsTq + kNsPad)];
    __shared__ __align__(16) float cs[R * (kNsTn + kNsPad)];
    const int tid = threadIdx.x;
    const int tn = tid % 16, tq = tid / 16;
    const int u = blockIdx.y;
    const int64_t bseq = u / a.hkv;
    const int h = u % a.hkv;
    const int64_t q0 = (int64_t)blockIdx.x * kNsTq;
    const int nqt = (int)min((int64_t)kNsTq, a.nqc - q0);

    // query tile, transposed: qs[d][i] (rows past the end are zero)
    for (int e = tid; e < kNsTq * (R / 4); e += kNsThreads) {
        const int i = e / (R / 4), d4 = e % (R / 4);
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < nqt)
            v = *reinterpret_cast<const float4*>(a.qbar + ((bseq * a.nq_stride + q0 + i) * a.hkv + h) * R + 4 * d4);
        qs[(4 * d4 + 0) * (kNsTq + kNsPad) + i] = v.x;
        qs[(4 * d4 + 1) * (kNsTq + kNsPad) + i] = v.y;
        qs[(4 * d4 + 2) * (kNsTq + kNsPad) + i] = v.z;
        qs[(4 * d4 + 3) * (kNsTq + kNsPad) + i] = v.w;
    }
    const int ncols = a.ncols;
    for (int c0 = 0; c0 < ncols; c0 += kNsTn) {
        __syncthreads();   // the previous pass is done with cs (and qs is written)
        for (int e = tid; e < kNsTn * (R / 4); e += kNsThreads) {
            const int j = e / (R / 4), d4 = e % (R / 4);
            const int col = c0 + j;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (col < ncols) {
                // the column's level (constant indices only: no local copy of the arguments)
                const float* base = a.cent[0];
                int nl = a.n_l[0], off = 0;
#pragma unroll
                for (int k = 1; k < LSA_MAX_LEVELS; ++k) {
                    if (k < a.levels && col >= a.col_off[k]) {
                        base = a.cent[k];
                        nl = a.n_l[k];
                        off = a.col_off[k];
                    }
                }
                v = *reinterpret_cast<const float4*>(base + ((int64_t)u * nl + (col - off)) * R + 4 * d4);
            }
            cs[(4 * d4 + 0) * (kNsTn + kNsPad) + j] = v.x;
            cs[(4 * d4 + 1) * (kNsTn + kNsPad) + j] = v.y;
            cs[(4 * d4 + 2) * (kNsTn + kNsPad) + j] = v.z;
            cs[(4 * d4 + 3) * (kNsTn + kNsPad) + j] = v.w;
        }
        __syncthreads();
        float sc[16];
        tree<R, 0, 1>(qs, cs, tq, tn, sc);
        const int col = c0 + 4 * tn;
        if (col < ncols) {
            // ld is a multiple of 4 and col of 4: the 4 columns are in the row
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (4 * tq + i < nqt) {
                    float* o = a.S + ((bseq * a.nqc + q0 + 4 * tq + i) * a.hkv + h) * a.ld + col;
                    *reinterpret_cast<float4*>(o) = make_float4(sc[i * 4], sc[i * 4 + 1], sc[i * 4 + 2], sc[i * 4 + 3]);
                }
            }
        }
    }
}

}  // namespace

int dense_levels(const lsa_index* ix, int beam, int max_cols, int* col_off) {
    // level 0 is scored for every query; level l >= 1 is when all of level
    // l - 1 fits in the beam (then every eligible node of level l - 1 is kept,
    // and every eligible node of level l is a candidate)
    const lsa_build_params& p = ix->p;
    int lv = 0, cols = 0;
    col_off[0] = 0;
    while (lv < p.levels && (lv == 0 || p.level_sizes[lv - 1] <= beam) && cols + p.level_sizes[lv] <= max_cols) {
        cols += p.level_sizes[lv];
        col_off[lv + 1] = cols;
        ++lv;
    }
    return lv;
}

int launch_node_scores(const lsa_index* ix, const float* qbar, int64_t nq_stride, int64_t nqc, int levels,
                       const int* col_off, float* S, int64_t ld, cudaStream_t s) {
    const lsa_build_params& p = ix->p;
    if (nqc <= 0 || levels <= 0) return LSA_OK;
    NsArgs a{};
    a.qbar = qbar;
    a.nq_stride = nq_stride;
    a.nqc = nqc;
    a.hkv = p.hkv;
    for (int l = 0; l < levels; ++l) {
        a.cent[l] = ix->ord_cent[l];
        a.n_l[l] = p.level_sizes[l];
    }
    for (int l = 0; l <= levels; ++l) a.col_off[l] = col_off[l];
    a.levels = levels;
    a.ncols = col_off[levels];
    a.S = S;
    a.ld = ld;
    dim3 grid((unsigned)((nqc + kNsTq - 1) / kNsTq), (unsigned)ix->units);
    note_launch();
    switch (p.r) {
        case 16: node_scores_kernel<16><<<grid, kNsThreads, 0, s>>>(a); break;
        case 32: node_scores_kernel<32><<<grid, kNsThreads, 0, s>>>(a); break;
        case 64: node_scores_kernel<64><<<grid, kNsThreads, 0, s>>>(a); break;
        default: return LSA_ERR_INVALID_ARG;
    }
    return cuda_status(cudaGetLastError());
}

// Calls of this many (query, KV head) pairs or more score the dense levels
// first; the buffer of scores holds at most kDenseChunkBytes, so longer calls
// run in chunks of queries (each chunk: scores, then the search).
constexpr int64_t kDenseMinPairs = 4096;
constexpr int kDenseMaxCols = 4096;
constexpr int64_t kDenseChunkBytes = int64_t(1) << 30;
// test hook (lsa_debug_dense_config): -1 = off, else the pair threshold; chunk bytes
std::atomic<int64_t> g_dense_min_pairs{kDenseMinPairs};
std::atomic<int64_t> g_dense_chunk_bytes{kDenseChunkBytes};

int launch_select_tree(const lsa_index* ix, const lsa_select_params* sp, const float* qbar, int64_t nq,
                       const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int max_sel,
                       cudaStream_t s, unsigned long long* work, const ScoredOut* scored, Arena& A) {
    const lsa_build_params& p = ix->p;
    PreScores pre{};
    int col_off[LSA_MAX_LEVELS + 1] = {0};
    const int64_t min_pairs = g_dense_min_pairs.load();
    const bool dense = (p.r == 16 || p.r == 32 || p.r == 64) && min_pairs >= 0 && nq * ix->units >= min_pairs &&
                       sp->beam >= 1 && sp->beam <= 1024;
    pre.levels = dense ? dense_levels(ix, sp->beam, kDenseMaxCols, col_off) : 0;
    if (pre.levels == 0)
        return launch_select(ix, sp, qbar, nq, q_pos, q_pos0, idx, cnt, max_sel, false, s, work, scored);
    pre.ld = (col_off[pre.levels] + 3) / 4 * 4;
    for (int l = 0; l < pre.levels; ++l) pre.off[l] = col_off[l];
    const int64_t row_bytes = (int64_t)p.batch * p.hkv * pre.ld * 4;   // one query of every sequence
    int64_t chunk = g_dense_chunk_bytes.load() / row_bytes;
    if (chunk < 1) chunk = 1;
    if (chunk > nq) chunk = nq;
    float* S = A.alloc<float>(chunk * p.batch * p.hkv * pre.ld);
    if (A.status != LSA_OK) return A.status;
    pre.S = S;
    const int64_t hkv = p.hkv;
    for (int64_t q0 = 0; q0 < nq; q0 += chunk) {
        const int64_t nqc = (nq - q0) < chunk ? (nq - q0) : chunk;
        int st = launch_node_scores(ix, qbar + q0 * hkv * p.r, nq, nqc, pre.levels, col_off, S, pre.ld, s);
        if (st != LSA_OK) return st;
        ScoredOut so{};
        if (scored) {
            so = *scored;
            so.score += q0 * hkv * scored->kb_cap;
            so.block += q0 * hkv * scored->kb_cap;
            so.n += q0 * hkv;
        }
        st = launch_select_rows(ix, sp, qbar + q0 * hkv * p.r, nq, nqc, q_pos ? q_pos + q0 : nullptr, q_pos0 + q0,
                                idx ? idx + q0 * hkv * max_sel : nullptr, cnt ? cnt + q0 * hkv : nullptr, max_sel,
                                false, s, work, scored ? &so : nullptr, &pre);
        if (st != LSA_OK) return st;
    }
    return LSA_OK;
}

}  // namespace lsa

extern "C" void lsa_debug_dense_config(int64_t min_pairs, int64_t chunk_bytes) {
    lsa::g_dense_min_pairs.store(min_pairs == 0 ? lsa::kDenseMinPairs : (min_pairs < 0 ? -1 : min_pairs));
    lsa::g_dense_chunk_bytes.store(chunk_bytes > 0 ? chunk_bytes : lsa::kDenseChunkBytes);
}
