// Scores of the dense upper tree levels for a tile of queries at a time, and
// (leaf tiles, below) of the leaves of each query's kept nodes.
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

#include "select_common.cuh"

namespace lsa {
namespace {

constexpr int kNsThreads = 256;
constexpr int kNsTq = 64;   // queries per CTA tile
constexpr int kNsTn = 64;   // nodes per pass
constexpr int kNsPad = 4;   // shared row padding (keeps 16-byte alignment)

// Rows 0 .. N-1 of R floats each, row i's float4 d4 given by src(i, d4), into
// shared memory transposed: dst[d * P + i].  Two neighbouring lanes take the
// two float4 of one 32-byte sector of a row and a warp takes 16 rows, so a
// warp's loads use whole sectors and, with P = 4 (mod 32), each of its four
// stores hits 32 distinct banks (16 * d4 + i covers them all).
template <int N, int R, int P, class Src>
__device__ __forceinline__ void stage_transposed(float* dst, int tid, Src&& src) {
    static_assert(N % 16 == 0 && (R / 4) % 2 == 0 && P % 32 == 4, "conflict-free layout");
    for (int e = tid; e < N * (R / 4); e += kNsThreads) {
        const int p = e >> 1;
        const int i = p % N, d4 = 2 * (p / N) + (e & 1);
        const float4 v = src(i, d4);
        dst[(4 * d4 + 0) * P + i] = v.x;
        dst[(4 * d4 + 1) * P + i] = v.y;
        dst[(4 * d4 + 2) * P + i] = v.z;
        dst[(4 * d4 + 3) * P + i] = v.w;
    }
}

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
    stage_transposed<kNsTq, R, kNsTq + kNsPad>(qs, tid, [&](int i, int d4) {
        if (i >= nqt) return make_float4(0.f, 0.f, 0.f, 0.f);
        return *reinterpret_cast<const float4*>(a.qbar + ((bseq * a.nq_stride + q0 + i) * a.hkv + h) * R + 4 * d4);
    });
    const int ncols = a.ncols;
    for (int c0 = 0; c0 < ncols; c0 += kNsTn) {
        __syncthreads();   // the previous pass is done with cs (and qs is written)
        stage_transposed<kNsTn, R, kNsTn + kNsPad>(cs, tid, [&](int j, int d4) {
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
            return v;
        });
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

// ------------------------------------------------------------ leaf tiles
// When the tree's only sparse level is its leaf level, the leaves are scored
// for many queries at a time as well:
//   1. beam_dense_kernel (one warp per (query, KV head) row): the kept nodes of
//      the last dense level, i.e. the best `beam` of all its eligible nodes by
//      (score desc, id asc), from the dense scores; and for each kept node the
//      first slot of its children in the row's leaf-score buffer;
//   2. the (row, kept node) pairs grouped by node (the library's radix sort
//      on the node), every node's first pair and its tiles of 128 pairs;
//   3. leaf_scores_kernel: per tile, its 128 pairs x 32 of the node's children
//      at a time, the register-tiled fp32 product in the per-query kernel's
//      order, each score written to its row's slot;
//   4. the per-query kernel starts from those kept nodes and reads each leaf
//      candidate's score from its slot (one lane per candidate) instead of
//      scoring its row.
// The selection of step 1 is exact (radix select on the order-preserving
// key, ties by id), so the kept set equals the per-query search's.  A row
// whose kept nodes have more than kLtCap children falls back to the
// per-query search.
constexpr int kLtCap = 3072;    // leaf slots per row
constexpr int kLtPairs = 128;   // (row, kept node) pairs per leaf_scores CTA
constexpr int kLtKids = 32;     // children per pass of a leaf_scores CTA
constexpr int kLtWarps = 8;     // rows per beam kernel CTA
constexpr int kLtMaxBeam = 128;    // leaf tiles for beams up to this

struct LtArgs {
    int64_t rows, nqc, nq_stride, units;
    int hkv, beam, window, pool;
    const int64_t* q_pos;       // the chunk's positions (sequence stride nq_stride), or null
    int64_t q_pos0;
    int64_t pos_shift;
    const float* qbar;          // the chunk's latent queries (sequence stride nq_stride)
    const float* S;             // dense scores, rows (bseq * nqc + qi) * hkv + h
    int64_t ld;
    int off1, n1;               // last dense level: its column in S and its size
    const int64_t* mp1;         // its minpos [units * n1] (tree order)
    const int32_t* id1;         // its ids
    const int32_t* coff1;       // [units * n1 + 1] global child positions in the leaf level
    int n2;                     // leaves per unit
    const float* cent2;         // leaf centroids [units * n2][r], tree order
    const int64_t* mp2;
    const int32_t* id2;
    int32_t* b1;                // [rows][beam] kept positions of the last dense level
    int32_t* nb1;               // [rows] their count; -1: the row falls back
    int32_t* sb;                // [rows][beam + 1] first leaf slot of each kept node; [n] = total
    float* S2;                  // [rows][kLtCap] leaf scores
    int32_t* ncnt;              // [units * n1] pairs per node (zero on entry, zero on exit)
    int32_t* noff;              // [units * n1 + 1]
    int32_t* list;              // [rows * beam] pairs row * beam + e, grouped by node
    int32_t* toff;              // [units * n1 + 1] first tile of each node
    int32_t* tnode;             // [max tiles] node of each tile
};

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// The k-th largest of the values v (v != 0 only) the enumerator visits, by
// 8-bit radix passes over a 256-bin histogram of this warp.  Returns the
// value and in *need how many items equal to it belong to the k largest.
template <class Enum>
__device__ uint32_t warp_kth(int k, int* hist, Enum&& each, int* need) {
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, mask = 0;
    int kk = k;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = lane; b < 256; b += 32) hist[b] = 0;
        __syncwarp();
        // lanes that hit the same bin add once for all of them (the scores of a
        // row share their leading bits, so most lanes hit one bin)
        each([&](bool valid, uint32_t v) {
            const bool in = valid && v != 0u && (v & mask) == prefix;
            const int bin = in ? (int)((v >> shift) & 255u) : -1;
            const unsigned grp = __match_any_sync(0xffffffffu, bin);
            if (in && (threadIdx.x & 31) == __ffs(grp) - 1) atomicAdd(&hist[bin], __popc(grp));
        });
        __syncwarp();
        int c[8], sum = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            c[q] = hist[255 - lane * 8 - q];
            sum += c[q];
        }
        const int incl = warp_incl_scan(sum);
        const int excl = incl - sum;
        int dsel = -1, above = 0;
        if (excl < kk && kk <= incl) {
            int run = excl;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (dsel < 0 && run + c[q] >= kk) {
                    dsel = 255 - lane * 8 - q;
                    above = run;
                }
                run += c[q];
            }
        }
        const unsigned bal = __ballot_sync(0xffffffffu, dsel >= 0);
        const int src = __ffs(bal) - 1;
        dsel = __shfl_sync(0xffffffffu, dsel, src);
        above = __shfl_sync(0xffffffffu, above, src);
        prefix |= (uint32_t)dsel << shift;
        mask |= 255u << shift;
        kk -= above;
        __syncwarp();
    }
    *need = kk;
    return prefix;
}

// Exact top k by (key desc, id asc) of the candidates the enumerator visits
// (key 0: not eligible), one warp.  each(f) calls f(valid, key, id, t) for
// every candidate, 32 at a time with the warp converged; emit(slot, t) is
// called once per chosen candidate (slots 0 .. count-1, in visiting order).
// Returns the count, min(k, eligible).
template <class Each, class Emit>
__device__ int warp_topk(int k, int* hist, Each&& each, Emit&& emit) {
    const unsigned lt = (1u << (threadIdx.x & 31)) - 1u;
    int nel = 0;
    each([&](bool valid, uint32_t key, int, int) { nel += valid && key != 0u; });
    nel = warp_sum(nel);
    uint32_t T = 1u, I = 0xFFFFFFFFu;
    bool all_eq = true;
    if (nel > k) {
        int need;
        T = warp_kth(k, hist, [&](auto&& f) { each([&](bool valid, uint32_t key, int, int) { f(valid, key); }); },
                     &need);
        int neq = 0;
        each([&](bool valid, uint32_t key, int, int) { neq += valid && key == T; });
        neq = warp_sum(neq);
        all_eq = neq == need;
        if (!all_eq) {
            // the need smallest ids among the keys equal to T: the need largest of ~id
            int need2;
            const uint32_t P = warp_kth(need, hist, [&](auto&& f) {
                each([&](bool valid, uint32_t key, int id, int) { f(valid && key == T, ~(uint32_t)id); });
            }, &need2);
            I = ~P;
        }
    }
    int base = 0;
    each([&](bool valid, uint32_t key, int id, int t) {
        const bool take = valid && key != 0u &&
                          (nel <= k || key > T || (key == T && (all_eq || (uint32_t)id <= I)));
        const unsigned bal = __ballot_sync(0xffffffffu, take);
        if (take) emit(base + __popc(bal & lt), t);
        base += __popc(bal);
    });
    return base;
}

__device__ __forceinline__ void lt_row(const LtArgs& a, int64_t row, int64_t* u, int64_t* bound) {
    const int h = (int)(row % a.hkv);
    const int64_t bq = row / a.hkv;
    const int64_t qi = bq % a.nqc, bseq = bq / a.nqc;
    *u = bseq * a.hkv + h;
    const int64_t pos = (a.q_pos ? a.q_pos[bseq * a.nq_stride + qi] : a.q_pos0 + qi) - a.pos_shift;
    *bound = pos - a.window - a.pool + 1;
}

// the row's eligible level-1 scores as order-preserving keys (0: not
// eligible), kept in registers (KPL per lane, node t = 32 j + lane) when the
// level has at most 32 KPL nodes, else in this warp's shared row (KPL = 0);
// 32 keys a lane run at two CTAs per SM (128 registers), the others at four
template <int KPL>
__global__ __launch_bounds__(kLtWarps * 32, KPL == 32 ? 2 : 4) void beam_dense_kernel(const LtArgs a) {
    extern __shared__ uint32_t lt_smem[];
    __shared__ int hist_all[kLtWarps][256];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * kLtWarps + w;
    if (row >= a.rows) return;   // warp-uniform; no CTA barrier below
    int64_t u, bound;
    lt_row(a, row, &u, &bound);
    const float* sr = a.S + row * a.ld + a.off1;
    const int64_t* mp = a.mp1 + u * a.n1;
    const int32_t* id = a.id1 + u * a.n1;
    int32_t* out = a.b1 + row * a.beam;
    uint32_t kr[KPL > 0 ? KPL : 1];
    uint32_t* keyc = lt_smem + (size_t)w * a.n1;
    if constexpr (KPL > 0) {
        int64_t mpv[KPL];
        float sv[KPL];
#pragma unroll
        for (int j = 0; j < KPL; ++j) {
            const int t = j * 32 + lane;
            mpv[j] = INT64_MAX;
            sv[j] = 0.f;
            if (t < a.n1) {
                mpv[j] = __ldg(mp + t);
                sv[j] = __ldg(sr + t);
            }
        }
#pragma unroll
        for (int j = 0; j < KPL; ++j) kr[j] = mpv[j] <= bound ? fkey(sv[j]) : 0u;
    } else {
        for (int t0 = 0; t0 < a.n1; t0 += 128) {
            int64_t mpv[4];
            float sv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = t0 + j * 32 + lane;
                mpv[j] = INT64_MAX;
                sv[j] = 0.f;
                if (t < a.n1) {
                    mpv[j] = __ldg(mp + t);
                    sv[j] = __ldg(sr + t);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = t0 + j * 32 + lane;
                if (t < a.n1) keyc[t] = mpv[j] <= bound ? fkey(sv[j]) : 0u;
            }
        }
        __syncwarp();
    }
    // ids matter only for ties at the threshold and are read then
    auto each = [&](auto&& f) {
        if constexpr (KPL > 0) {
#pragma unroll
            for (int j = 0; j < KPL; ++j) {
                const int t = j * 32 + lane;
                f(t < a.n1, kr[j], kr[j] != 0u ? __ldg(id + t) : 0, t);
            }
        } else {
            for (int t0 = 0; t0 < a.n1; t0 += 32) {
                const int t = t0 + lane;
                const bool valid = t < a.n1;
                const uint32_t key = valid ? keyc[t] : 0u;
                f(valid, key, key != 0u ? __ldg(id + t) : 0, t);
            }
        }
    };
    const int n = warp_topk(a.beam, hist_all[w], each, [&](int slot, int t) { out[slot] = t; });
    __syncwarp();
    // first leaf slot of each kept node's children, in kept order
    const int32_t* co = a.coff1 + u * a.n1;
    int32_t* sbr = a.sb + row * (a.beam + 1);
    int carry = 0;
    for (int e0 = 0; e0 < n; e0 += 32) {
        const int e = e0 + lane;
        int c = 0;
        if (e < n) {
            const int q = out[e];
            c = __ldg(co + q + 1) - __ldg(co + q);
        }
        const int incl = warp_incl_scan(c);
        if (e < n) sbr[e] = carry + incl - c;
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
        sbr[n] = carry;
        a.nb1[row] = carry <= kLtCap ? n : -1;
    }
}

// sort key of every (row, kept node) pair: the node (units * n1 for a pair
// that does not exist, which sorts last); value: row * beam + e
__global__ void lt_keys_kernel(const LtArgs a, uint32_t* __restrict__ keys, int32_t* __restrict__ vals) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= a.rows * a.beam) return;
    const int64_t row = e / a.beam;
    const int k = (int)(e % a.beam);
    const int n = a.nb1[row];
    uint32_t key = (uint32_t)(a.units * a.n1);
    if (k < n) {   // (n < 0: the row falls back)
        const int64_t u = (row / a.hkv / a.nqc) * a.hkv + row % a.hkv;
        key = (uint32_t)(u * a.n1 + a.b1[row * a.beam + k]);
    }
    keys[e] = key;
    vals[e] = (int32_t)e;
}

// first pair of every node in the sorted keys (noff[g] = lower bound of g),
// and the node's tile count
__global__ void lt_bounds_kernel(const LtArgs a, const uint32_t* __restrict__ skeys, int64_t npairs) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nodes = a.units * a.n1;
    if (g > nodes) return;
    int64_t lo = 0, hi = npairs;   // first index with key >= g
    while (lo < hi) {
        const int64_t mid = (lo + hi) >> 1;
        if (skeys[mid] < (uint32_t)g) lo = mid + 1; else hi = mid;
    }
    a.noff[g] = (int32_t)lo;
}

// node of every tile (each node's thread writes its run of tiles)
__global__ void lt_tile_nodes_kernel(const LtArgs a) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= a.units * a.n1) return;
    for (int t = a.toff[g]; t < a.toff[g + 1]; ++t) a.tnode[t] = (int32_t)g;
}

__global__ void lt_tiles_kernel(const LtArgs a) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= a.units * a.n1) return;
    a.ncnt[g] = (a.noff[g + 1] - a.noff[g] + kLtPairs - 1) / kLtPairs;
}

// out[i][j] (pairs 4 tq + i, children 4 tn + j) = what lane g of a group of
// r/16 lanes holds before the butterfly (see chain/tree above), with the pair
// and child operands transposed in shared memory at strides PQ and PC
template <int R, int PQ, int PC>
__device__ __forceinline__ void lt_chain(const float* qs, const float* cs, int tq, int tn, int c,
                                         float (&acc)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int d = 8 * c + j;
        const float4 x = *reinterpret_cast<const float4*>(qs + d * PQ + 4 * tq);
        const float4 y = *reinterpret_cast<const float4*>(cs + d * PC + 4 * tn);
        const float av[4] = {x.x, x.y, x.z, x.w}, bv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[i * 4 + k] = __fmaf_rn(av[i], bv[k], acc[i * 4 + k]);
    }
}
template <int R, int PQ, int PC, int G, int O>
__device__ __forceinline__ void lt_tree(const float* qs, const float* cs, int tq, int tn, float (&out)[16]) {
    constexpr int LPC = R / 16;
    if constexpr (O == LPC) {
        float t[16];
        lt_chain<R, PQ, PC>(qs, cs, tq, tn, G, out);
        lt_chain<R, PQ, PC>(qs, cs, tq, tn, LPC + G, t);
#pragma unroll
        for (int e = 0; e < 16; ++e) out[e] = __fadd_rn(out[e], t[e]);
    } else {
        float t[16];
        lt_tree<R, PQ, PC, G, 2 * O>(qs, cs, tq, tn, out);
        lt_tree<R, PQ, PC, (G ^ O), 2 * O>(qs, cs, tq, tn, t);
#pragma unroll
        for (int e = 0; e < 16; ++e) out[e] = __fadd_rn(out[e], t[e]);
    }
}

// One CTA per tile of up to 128 pairs of one node: the pairs' latent queries
// and the node's children (32 at a time) transposed into shared memory, the
// 128 x 32 scores in the per-query kernel's order, each into its row's slot.
template <int R>
__global__ __launch_bounds__(kNsThreads, 3) void leaf_scores_kernel(const LtArgs a) {
    constexpr int PQ = kLtPairs + 4, PC = kLtKids + 4;
    __shared__ __align__(16) float qs[R * PQ];
    __shared__ __align__(16) float cs[R * PC];
    __shared__ int64_t prow[kLtPairs];
    __shared__ int pslot[kLtPairs];
    const int64_t nodes = a.units * a.n1;
    const int64_t t = blockIdx.x;
    if (t >= a.toff[nodes]) return;   // CTA-uniform
    const int64_t g = a.tnode[t];     // toff[g] <= t < toff[g + 1]
    const int64_t j0 = a.noff[g] + (t - a.toff[g]) * kLtPairs;
    const int np = (int)min((int64_t)kLtPairs, (int64_t)a.noff[g + 1] - j0);
    const int tid = threadIdx.x;
    // 8 x 32 threads, 4 children x 4 pairs each; a warp takes 16 children x
    // 32 pairs, so in a pass over at most 16 children the warps of the upper
    // half have nothing to score and skip it
    const int wq = (tid >> 5) & 3, wc = tid >> 7;
    const int tn = (tid & 3) + 4 * wc, tq = ((tid & 31) >> 2) + 8 * wq;
    if (tid < kLtPairs) {
        int64_t r = -1;
        int sl = 0;
        if (tid < np) {
            const int64_t e = a.list[j0 + tid];
            r = e / a.beam;
            sl = a.sb[r * (a.beam + 1) + (int)(e % a.beam)];
        }
        prow[tid] = r;
        pslot[tid] = sl;
    }
    __syncthreads();
    // the pairs' latent queries, transposed (pairs past np are zero)
    stage_transposed<kLtPairs, R, PQ>(qs, tid, [&](int i, int d4) {
        if (i >= np) return make_float4(0.f, 0.f, 0.f, 0.f);
        const int64_t r = prow[i];
        const int h = (int)(r % a.hkv);
        const int64_t bq = r / a.hkv;
        const int64_t qrow = ((bq / a.nqc) * a.nq_stride + bq % a.nqc) * a.hkv + h;
        return *reinterpret_cast<const float4*>(a.qbar + qrow * R + 4 * d4);
    });
    const int c_beg = a.coff1[g], nc = a.coff1[g + 1] - c_beg;   // global leaf positions
    for (int c0 = 0; c0 < nc; c0 += kLtKids) {
        __syncthreads();   // qs written; the previous pass is done with cs
        stage_transposed<kLtKids, R, PC>(cs, tid, [&](int j, int d4) {
            if (c0 + j >= nc) return make_float4(0.f, 0.f, 0.f, 0.f);
            return *reinterpret_cast<const float4*>(a.cent2 + ((int64_t)c_beg + c0 + j) * R + 4 * d4);
        });
        __syncthreads();
        if (4 * tq < np && 16 * wc < nc - c0) {
            float sc[16];
            lt_tree<R, PQ, PC, 0, 1>(qs, cs, tq, tn, sc);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int pi = 4 * tq + i;
                if (pi < np) {
                    float* o = a.S2 + prow[pi] * kLtCap + pslot[pi] + c0;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (c0 + 4 * tn + k < nc) o[4 * tn + k] = sc[i * 4 + k];
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
// test hook (lsa_debug_dense_config): -1 = off, else the pair threshold; chunk bytes;
// leaf tiles on or off
std::atomic<int64_t> g_dense_min_pairs{kDenseMinPairs};
std::atomic<int64_t> g_dense_chunk_bytes{kDenseChunkBytes};
std::atomic<int> g_leaf_tiles{1};
// the leaf-tile path runs in chunks whose buffers stay under this
constexpr int64_t kLtChunkBytes = int64_t(2) << 30;

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
    const int64_t hkv = p.hkv;
    // leaf tiles: the leaf level is the only sparse one (not for the scored-row counter,
    // which counts the per-query search's own candidates)
    const bool lt = g_leaf_tiles.load() != 0 && work == nullptr && pre.levels == p.levels - 1 &&
                    sp->beam <= kLtMaxBeam;
    const int beam = sp->beam;
    const int l1 = pre.levels - 1, n1 = p.level_sizes[l1];
    const int64_t per_row = (int64_t)pre.ld * 4 + (lt ? (int64_t)kLtCap * 4 + (int64_t)(4 * beam + 3) * 4 : 0);
    const int64_t row_bytes = (int64_t)p.batch * p.hkv * per_row;   // one query of every sequence
    int64_t chunk = (lt ? kLtChunkBytes : g_dense_chunk_bytes.load()) / row_bytes;
    if (lt && g_dense_chunk_bytes.load() != kDenseChunkBytes) chunk = g_dense_chunk_bytes.load() / row_bytes;
    if (chunk < 1) chunk = 1;
    if (chunk > nq) chunk = nq;
    const int64_t crow = chunk * p.batch * p.hkv;
    float* S = A.alloc<float>(crow * pre.ld);
    LtArgs la{};
    int32_t* scan_scr = nullptr;
    uint32_t* lt_k0 = nullptr;
    int32_t* lt_v0 = nullptr;
    uint32_t* lt_k1 = nullptr;
    int32_t* lt_v1 = nullptr;
    int32_t* lt_rs = nullptr;
    if (lt) {
        const int64_t nodes = ix->units * n1;
        la.S2 = A.alloc<float>(crow * kLtCap);
        la.b1 = A.alloc<int32_t>(crow * beam);
        la.nb1 = A.alloc<int32_t>(crow);
        la.sb = A.alloc<int32_t>(crow * (beam + 1));
        lt_v0 = A.alloc<int32_t>(crow * beam);
        la.ncnt = A.alloc<int32_t>(nodes);
        la.noff = A.alloc<int32_t>(nodes + 1);
        la.toff = A.alloc<int32_t>(nodes + 1);
        la.tnode = A.alloc<int32_t>((crow * beam + kLtPairs - 1) / kLtPairs + nodes);
        lt_k0 = A.alloc<uint32_t>(crow * beam);
        lt_k1 = A.alloc<uint32_t>(crow * beam);
        lt_v1 = A.alloc<int32_t>(crow * beam);
        lt_rs = A.alloc<int32_t>(radix_scratch_elems(crow * beam));
        scan_scr = A.alloc<int32_t>(scan_scratch_elems(nodes) + 1);
    }
    if (A.status != LSA_OK) return A.status;
    pre.S = S;
    if (lt) {
        la.units = ix->units;
        la.hkv = p.hkv;
        la.beam = beam;
        la.window = sp->window;
        la.pool = p.pool;
        la.pos_shift = scored ? scored->pos_shift : 0;
        la.S = S;
        la.ld = pre.ld;
        la.off1 = col_off[l1];
        la.n1 = n1;
        la.mp1 = ix->ord_mp[l1];
        la.id1 = ix->ord_id[l1];
        la.coff1 = ix->ord_coff[l1];
        la.n2 = p.level_sizes[l1 + 1];
        la.cent2 = ix->ord_cent[l1 + 1];
        la.mp2 = ix->ord_mp[l1 + 1];
        la.id2 = ix->ord_id[l1 + 1];
        la.nq_stride = nq;
    }
    for (int64_t q0 = 0; q0 < nq; q0 += chunk) {
        const int64_t nqc = (nq - q0) < chunk ? (nq - q0) : chunk;
        const float* qb = qbar + q0 * hkv * p.r;
        int st = launch_node_scores(ix, qb, nq, nqc, pre.levels, col_off, S, pre.ld, s);
        if (st != LSA_OK) return st;
        if (lt) {
            la.rows = nqc * p.batch * p.hkv;
            la.nqc = nqc;
            la.q_pos = q_pos ? q_pos + q0 : nullptr;
            la.q_pos0 = q_pos0 + q0;
            la.qbar = qb;
            const int64_t nodes = ix->units * n1;
            const int64_t pairs = la.rows * beam;
            const unsigned bd_grid = (unsigned)((la.rows + kLtWarps - 1) / kLtWarps);
            note_launch();
            if (n1 <= 16 * 32) {
                beam_dense_kernel<16><<<bd_grid, kLtWarps * 32, 0, s>>>(la);
            } else if (n1 <= 32 * 32) {
                beam_dense_kernel<32><<<bd_grid, kLtWarps * 32, 0, s>>>(la);
            } else {
                const size_t dense_smem = (size_t)kLtWarps * n1 * sizeof(uint32_t);
                cudaError_t e0 = cudaFuncSetAttribute(beam_dense_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      (int)dense_smem);
                if (e0 != cudaSuccess) return cuda_status(e0);
                beam_dense_kernel<0><<<bd_grid, kLtWarps * 32, dense_smem, s>>>(la);
            }
            // the pairs grouped by node: a stable radix sort on the node
            note_launch();
            lt_keys_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, s>>>(la, lt_k0, lt_v0);
            int kbits = 8;
            while (kbits < 32 && ((int64_t)1 << kbits) <= nodes) kbits += 8;
            uint32_t* skeys;
            int32_t* svals;
            radix_sort(lt_k0, lt_v0, lt_k1, lt_v1, pairs, kbits, lt_rs, s, &skeys, &svals);
            la.list = svals;
            note_launch();
            lt_bounds_kernel<<<(unsigned)((nodes + 1 + 255) / 256), 256, 0, s>>>(la, skeys, pairs);
            note_launch();
            lt_tiles_kernel<<<(unsigned)((nodes + 255) / 256), 256, 0, s>>>(la);
            scan_exclusive(la.ncnt, la.toff, nodes, scan_scr, s);
            note_launch();
            lt_tile_nodes_kernel<<<(unsigned)((nodes + 255) / 256), 256, 0, s>>>(la);
            // tiles: at most one partial tile per node beyond the full ones
            const int64_t max_tiles = (pairs + kLtPairs - 1) / kLtPairs + nodes;
            note_launch();
            switch (p.r) {
                case 16: leaf_scores_kernel<16><<<(unsigned)max_tiles, kNsThreads, 0, s>>>(la); break;
                case 32: leaf_scores_kernel<32><<<(unsigned)max_tiles, kNsThreads, 0, s>>>(la); break;
                default: leaf_scores_kernel<64><<<(unsigned)max_tiles, kNsThreads, 0, s>>>(la); break;
            }
            st = cuda_status(cudaGetLastError());
            if (st != LSA_OK) return st;
            pre.b1 = la.b1;
            pre.nb1 = la.nb1;
            pre.S2 = la.S2;
            pre.s2_ld = kLtCap;
        }
        ScoredOut so{};
        if (scored) {
            so = *scored;
            so.score += q0 * hkv * scored->kb_cap;
            so.block += q0 * hkv * scored->kb_cap;
            so.n += q0 * hkv;
        }
        st = launch_select_rows(ix, sp, qb, nq, nqc, q_pos ? q_pos + q0 : nullptr, q_pos0 + q0,
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

extern "C" void lsa_debug_leaf_tiles(int32_t on) { lsa::g_leaf_tiles.store(on ? 1 : 0); }
