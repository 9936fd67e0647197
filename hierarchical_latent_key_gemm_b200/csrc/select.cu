// Key selection: tree search and the full-scan baseline.
//
// Tree search (tree-search wiki note, TL;DR: the query compares itself with
// the cluster centroids and goes down into a few of the best buckets;
// 10M-token attention post: clusters are scored first, then the keys inside
// the chosen ones; LSA explainer, "How does LSA work?" steps 2-3): per (query, KV head), level
// by level, score the eligible nodes (all top nodes, then the children of the
// kept ones) and keep the best `beam`; score the candidate blocks inside the
// kept leaves and keep the best ceil(K/P); emit sink + blocks + window.
//
// Full scan (the previous indexer, the wiki note's flowchart, red path): the same top-K
// over every candidate block, no tree.
//
// One CTA per (query, KV head).  Every tree level is stored in tree order
// (children of a node are contiguous), so a candidate's minpos, original id
// and centroid row are independent loads; each sub-warp group of r/16 lanes
// (16 floats of the row per lane) walks a contiguous run of candidates.
// Scores stream through one shared-memory buffer; when it runs low, a
// block-wide select (on the order-preserving bit pattern of the fp32 score,
// then on the original id for ties) compacts it in place to the top k.  The
// order is total, (score desc, id asc), so the result does not depend on the
// order in which warps append.  One buffer instead of two halves the shared
// memory of a CTA, which leaves more of each SM's L1 for the centroid rows
// that every query of a unit reads.
#include <type_traits>

#include "select_common.cuh"

namespace lsa {
namespace {

// One candidate in flight per group at 8 CTAs (32 warps) per SM measured
// fastest on the 1M-token workload (194 ms; 2 in flight at 6 CTAs: 209 ms,
// at 4 CTAs: 249 ms).
#ifndef LSA_SELECT_UNROLL
#define LSA_SELECT_UNROLL 1
#endif
#ifndef LSA_SELECT_MIN_BLOCKS
#define LSA_SELECT_MIN_BLOCKS 8
#endif
constexpr int kSelThreads = 128;
constexpr int kUnroll = LSA_SELECT_UNROLL;  // candidates in flight per group

struct SelArgs {
    const float* ocent[LSA_MAX_LEVELS];     // [units*n_l][r], tree order
    const int64_t* omp[LSA_MAX_LEVELS];     // [units*n_l] minpos, tree order
    const int32_t* oid[LSA_MAX_LEVELS];     // [units*n_l] original id of each position
    const int32_t* ocoff[LSA_MAX_LEVELS];   // [units*n_l + 1] child position ranges (global)
    int n_l[LSA_MAX_LEVELS];
    int levels;
    const float* Klp;
    const int32_t* blk;
    const int32_t* leaf_start;
    const int32_t* leaf_cnt;
    const float* Kl;
    int64_t nb_cap, nb;
    int pool, sink, window, beam, kb, hkv;
    int64_t nq;
    const float* qbar;
    const int64_t* q_pos;
    int64_t q_pos0;
    int32_t* idx;
    int32_t* cnt;
    int max_sel;
    int cap;
    unsigned long long* work;   // optional: [0] += eligible nodes scored, [1] += candidate blocks scored
    // scored-blocks output (SCORED): the kept blocks and their scores, [row][kb_cap]
    int64_t pos_shift;          // query positions are given in the caller's numbering; index position = pos - shift
    int32_t blk_shift;          // block id written = index block id + blk_shift
    int kb_cap;
    float* out_score;
    int32_t* out_block;
    int32_t* out_n;
    // full scan over candidate lists (fullscan_tc.cu): for query qi of unit u,
    // two lists at l_cand + ((u * l_npad + qi) * 2 + half) * l_cap with
    // l_cnt entries each; a list longer than l_cap means "scan every block"
    const int32_t* l_cand;
    const int32_t* l_cnt;
    int64_t l_npad;
    int l_cap;
    // scores of the leading pre_levels tree levels, computed for all of their
    // nodes by the dense-level kernel (node_scores.cu) with this kernel's own
    // arithmetic: row (bseq * pre_nq + qi) * hkv + h, level l's node at
    // position q in column pre_off[l] + q
    const float* pre;
    int64_t pre_nq, pre_ld;
    int pre_levels;
    int pre_off[LSA_MAX_LEVELS];
    // leaf tiles (node_scores.cu): per row of the dense-score numbering the
    // kept nodes of the last dense level [row][beam] and their count (-1: the
    // row searches every level here), and their children's scores [row][s2_ld]
    // in kept-node order
    const int32_t* lt_b1;
    const int32_t* lt_nb1;
    const float* lt_s2;
    int64_t lt_ld;
};

// THREADS = kSelThreads for large grids; small grids (decode: a few queries)
// give each (query, KV head) kWideThreads so the few CTAs use more of the SM.
constexpr int kWideThreads = 1024;
constexpr int kWideCap = 8192;

// COUNT: also add the number of eligible rows scored to *a.work (a separate
// instantiation, so the counting costs the timed path nothing)
template <int R, bool FULL, int THREADS, bool COUNT, bool SCORED = false>
__global__ __launch_bounds__(THREADS, THREADS == kSelThreads ? LSA_SELECT_MIN_BLOCKS : 1) void select_kernel(
    const SelArgs a) {
    extern __shared__ float4 dyn4[];
    __shared__ SelShared sh;
    // one buffer of (score, id, position) x cap, compacted in place
    float* const bs = reinterpret_cast<float*>(dyn4);
    int* const bi = reinterpret_cast<int*>(bs + a.cap);
    int* const bp = reinterpret_cast<int*>(bs + 2 * a.cap);
    int* kk = reinterpret_cast<int*>(bs + 3 * a.cap);   // kept positions [beam]
    int* pre = kk + a.beam;          // [beam + 1]
    int* lo = pre + a.beam + 1;      // [beam]

    constexpr int LPC = R / 16;             // lanes per candidate row (16 floats each)
    constexpr int CPW = 32 / LPC;           // candidates per warp
    constexpr int NG = (THREADS / 32) * CPW;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane / LPC, gl = lane % LPC, gid = warp * CPW + g;
    const unsigned gmask = (LPC == 32) ? 0xffffffffu : (((1u << LPC) - 1u) << (g * LPC));

    const int64_t qi = blockIdx.x;
    const int u = blockIdx.y;
    const int64_t bseq = u / a.hkv;
    const int h = u % a.hkv;
    const int64_t row = (bseq * a.nq + qi) * a.hkv + h;
    const int64_t pos = (a.q_pos ? a.q_pos[bseq * a.nq + qi] : a.q_pos0 + qi) - a.pos_shift;
    const int64_t bound = pos - a.window - a.pool + 1;
    const int64_t b_lo = (a.sink + a.pool - 1) / a.pool;
    const int64_t b_hi = bound >= 0 ? bound / a.pool : -1;

    // lane gl of a group holds 32-byte pieces gl and gl + LPC of a row: each
    // 256-bit load instruction reads LPC * 32 contiguous bytes (whole 128-byte
    // lines) of every row it touches
    float qv[16];
    {
        const float* qp = a.qbar + row * R + gl * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            qv[j] = qp[j];
            qv[8 + j] = qp[LPC * 8 + j];
        }
    }
    auto dot = [&](const float* y) -> float {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            s0 = __fmaf_rn(qv[j], y[j], s0);
            s1 = __fmaf_rn(qv[8 + j], y[8 + j], s1);
        }
        float s = __fadd_rn(s0, s1);
#pragma unroll
        for (int o = LPC / 2; o >= 1; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(gmask, s, o));
        return s;
    };
    auto load_row = [&](const float* rowp, float* y) {
        ldg256(rowp + gl * 8, y);
        ldg256(rowp + (LPC + gl) * 8, y + 8);
    };

    for (int e = threadIdx.x; e < 256; e += blockDim.x) sh.hist[e] = 0;
    if (threadIdx.x == 0) { sh.count = 0; sh.nkept = 0; sh.thr = 0u; }
    __syncthreads();

    // eligible candidates this thread's group scored (leader lanes): tree nodes
    // while phase is 0, candidate blocks once it is 1
    unsigned nsc_node = 0, nsc_blk = 0;
    int phase = FULL ? 1 : 0;
    uint32_t lt_mask;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt_mask));
    // Push candidates t in [0, total) through the buffer, keeping the top k.
    // Each group walks a contiguous run of candidates, kUnroll at a time:
    // fetch(t, &state, &elig, &id, &p, y) issues the loads of candidate t
    // (state carries the owning node across consecutive t), and the results
    // are used only after every load of the batch is in flight.  Once the
    // buffer has been compacted, a candidate whose key is below the k-th kept
    // key cannot enter the top k and is not appended.  The buffer is compacted
    // only when the next chunk might not fit, and at the end.  Appends are
    // aggregated per warp: one shared-memory atomic per batch.  With LANE
    // (scores given, no rows to load), every lane is a group of its own and
    // fetch puts the candidate's score in y[0].
    auto stream_topk = [&](int total, int k, auto lane_mode, auto&& fetch) {
        constexpr bool LANE = decltype(lane_mode)::value;
        constexpr int NGx = LANE ? THREADS : NG;
        const int gidx = LANE ? (int)threadIdx.x : gid;
        const bool lead = LANE || gl == 0;
        if (k <= 0) return;  // nothing is kept; the buffer stays empty
        // entered with an empty buffer; nbuf mirrors sh.count between chunks
        if (threadIdx.x == 0) sh.thr = 0u;
        __syncthreads();
        int t0 = 0, nbuf = 0;
        while (t0 < total) {
            const uint32_t thr = sh.thr;
            const int t1 = min(total, t0 + (a.cap - nbuf));
            const int span = (t1 - t0 + NGx - 1) / NGx;
            const int tb = t0 + gidx * span;
            const int te = min(t1, tb + span);
            OwnerState state{-1, 0, 0};
            for (int s0 = 0; s0 < span; s0 += kUnroll) {
                float y[kUnroll][16];
                int idv[kUnroll], pv[kUnroll];
                bool ok[kUnroll];
#pragma unroll
                for (int v = 0; v < kUnroll; ++v) {
                    const int tt = tb + s0 + v;
                    ok[v] = tt < te;
                    if (ok[v]) fetch(tt, &state, &ok[v], &idv[v], &pv[v], y[v]);
                }
                float sc[kUnroll];
                uint32_t bal[kUnroll];
                int nb_warp = 0;
#pragma unroll
                for (int v = 0; v < kUnroll; ++v) {
                    if (ok[v]) {
                        if constexpr (LANE) sc[v] = y[v][0];
                        else sc[v] = dot(y[v]);
                        if (COUNT) {
                            if (phase) nsc_blk += lead;
                            else nsc_node += lead;
                        }
                        ok[v] = fkey(sc[v]) >= thr;
                    }
                    bal[v] = __ballot_sync(0xffffffffu, ok[v] && lead);
                    nb_warp += __popc(bal[v]);
                }
                int base = 0;
                if (lane == 0 && nb_warp) base = atomicAdd(&sh.count, nb_warp);
                base = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
                for (int v = 0; v < kUnroll; ++v) {
                    if (ok[v] && lead) {
                        const int p = base + __popc(bal[v] & lt_mask);
                        bs[p] = sc[v];
                        bi[p] = idv[v];
                        bp[p] = pv[v];
                    }
                    base += __popc(bal[v]);
                }
            }
            t0 = t1;
            __syncthreads();
            const int n = sh.count;
            // compact when done, or when less than a quarter of the buffer is free
            if (n > k && (t0 >= total || a.cap - n < a.cap / 4)) {
                topk_compact(bs, bi, bp, n, k, sh);
                if (threadIdx.x == 0) sh.count = k;
                nbuf = k;
            } else {
                nbuf = n;
            }
            __syncthreads();
        }
    };

    // owner of candidate t among the nk kept nodes (ranges pre[o]..pre[o+1]),
    // advanced from the previous candidate's owner
    // slot (or child position) of candidate t: the owner's run starts at
    // lo[o] for t = pre[o]; the owner, its run's end and base stay in registers
    auto slot_of = [&](int t, int nk, OwnerState* st) -> int {
        if (st->o < 0) {
            const int o = find_owner(pre, nk, t);
            st->o = o;
            st->next = pre[o + 1];
            st->base = lo[o] - pre[o];
        }
        while (t >= st->next) {
            const int o = ++st->o;
            st->next = pre[o + 1];
            st->base = lo[o] - pre[o];
        }
        return st->base + t;
    };

    if (!FULL) {
        int l_first = 0;
        const float* s2 = nullptr;
        if (a.lt_b1) {
            const int64_t srow = (bseq * a.pre_nq + qi) * a.hkv + h;
            const int n1 = a.lt_nb1[srow];
            if (n1 >= 0) {
                // the dense levels' kept nodes come from the leaf tiles, in the
                // order of their children's score slots: the search starts at
                // the leaf level and reads those scores
                const int lb = a.pre_levels;   // the leaf level
                const int32_t* co = a.ocoff[lb - 1] + (int64_t)u * a.n_l[lb - 1];
                const int child_base = u * a.n_l[lb];
                for (int e = threadIdx.x; e < n1; e += blockDim.x) {
                    const int q = a.lt_b1[srow * a.beam + e];
                    kk[e] = q;
                    lo[e] = co[q] - child_base;
                    pre[e] = co[q + 1] - co[q];
                }
                scan_pre(pre, n1);
                if (threadIdx.x == 0) sh.nkept = n1;
                __syncthreads();
                l_first = lb;
                s2 = a.lt_s2 + srow * a.lt_ld;
            }
        }
        for (int l = l_first; l < a.levels; ++l) {
            const int nl = a.n_l[l];
            const float* cent = a.ocent[l] + (int64_t)u * nl * R;
            const int64_t* mp = a.omp[l] + (int64_t)u * nl;
            const int32_t* oid = a.oid[l] + (int64_t)u * nl;
            const int nk = sh.nkept;
            const int total = (l == 0) ? nl : pre[nk];
            if (threadIdx.x == 0) sh.count = 0;
            __syncthreads();
            if (s2 && l == l_first) {
                // leaf scores from the leaf tiles: candidate t's score is in slot t
                stream_topk(total, a.beam, std::true_type{},
                            [&](int t, OwnerState* state, bool* el, int* id, int* p, float* y) {
                                const int q = slot_of(t, nk, state);
                                y[0] = __ldg(s2 + t);
                                *id = __ldg(oid + q);
                                *p = q;
                                *el = __ldg(mp + q) <= bound;
                            });
            } else if (l < a.pre_levels) {
                const float* ps = a.pre + ((bseq * a.pre_nq + qi) * a.hkv + h) * a.pre_ld + a.pre_off[l];
                stream_topk(total, a.beam, std::true_type{},
                            [&](int t, OwnerState* state, bool* el, int* id, int* p, float* y) {
                                const int q = (l == 0) ? t : slot_of(t, nk, state);
                                y[0] = __ldg(ps + q);
                                *id = __ldg(oid + q);
                                *p = q;
                                *el = __ldg(mp + q) <= bound;
                            });
            } else {
                stream_topk(total, a.beam, std::false_type{},
                            [&](int t, OwnerState* state, bool* el, int* id, int* p, float* y) {
                                const int q = (l == 0) ? t : slot_of(t, nk, state);
                                load_row(cent + (int64_t)q * R, y);
                                *id = __ldg(oid + q);
                                *p = q;
                                *el = __ldg(mp + q) <= bound;
                            });
            }
            const int n = sh.count;
            for (int e = threadIdx.x; e < n; e += blockDim.x) kk[e] = bp[e];
            __syncthreads();
            if (threadIdx.x == 0) sh.nkept = n;
            if (l + 1 < a.levels) {
                // child positions of kept node q: [co[q], co[q+1]) minus the unit's base
                const int32_t* co = a.ocoff[l] + (int64_t)u * nl;
                const int child_base = u * a.n_l[l + 1];
                for (int e = threadIdx.x; e < n; e += blockDim.x) {
                    const int q = kk[e];
                    lo[e] = co[q] - child_base;
                    pre[e] = co[q + 1] - co[q];
                }
                scan_pre(pre, n);
            }
            __syncthreads();
        }
        // candidate slot range of every kept leaf
        // (the kept leaves' original ids are still in the buffer; a leaf's
        // block ids ascend, so its candidates are the run between the counts
        // of ids below b_lo and of ids up to b_hi, read 16 at a time so the
        // loads of a leaf are in flight together)
        const int nk = sh.nkept;
        const int L = a.n_l[a.levels - 1];
        const int* kept_id = bi;
        for (int e = threadIdx.x; e < nk; e += blockDim.x) {
            const int64_t c = (int64_t)u * L + kept_id[e];
            const int st = a.leaf_start[c];
            const int cntl = a.leaf_cnt[c];
            const int32_t* bl = a.blk + st;
            int nlo = 0, nle = 0;
            for (int j0 = 0; j0 < cntl; j0 += 16) {
                int v[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = j0 + j < cntl ? __ldg(bl + j0 + j) : INT32_MAX;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    nlo += v[j] < b_lo;
                    nle += v[j] <= b_hi;
                }
            }
            lo[e] = st + nlo;
            pre[e] = max(0, nle - nlo);
        }
        scan_pre(pre, nk);
        if (threadIdx.x == 0) sh.count = 0;
        __syncthreads();
        phase = 1;
        stream_topk(pre[nk], a.kb, std::false_type{}, [&](int t, OwnerState* state, bool* el, int* id, int* p, float* y) {
            const int64_t slot = slot_of(t, nk, state);
            load_row(a.Klp + slot * R, y);
            *id = __ldg(a.blk + slot);
            *p = 0;
            *el = true;
        });
    } else {
        const int64_t hi = min(a.nb - 1, b_hi);
        const int total = hi >= b_lo ? (int)(hi - b_lo + 1) : 0;
        const float* kl = a.Kl + (int64_t)u * a.nb_cap * R;
        bool listed = false;
        if (a.l_cand) {
            const int64_t gr = (int64_t)u * a.l_npad + qi;
            const int n0 = a.l_cnt[gr * 2], n1 = a.l_cnt[gr * 2 + 1];
            if (n0 <= a.l_cap && n1 <= a.l_cap) {
                // every block that can be in the top K is in the two lists
                listed = true;
                const int32_t* L0 = a.l_cand + gr * 2 * a.l_cap;
                const int32_t* L1 = L0 + a.l_cap;
                stream_topk(n0 + n1, a.kb, std::false_type{}, [&](int t, OwnerState* state, bool* el, int* id, int* p, float* y) {
                    (void)state;
                    const int64_t b = t < n0 ? __ldg(L0 + t) : __ldg(L1 + (t - n0));
                    load_row(kl + b * R, y);
                    *id = (int)b;
                    *p = 0;
                    *el = true;
                });
            }
        }
        if (!listed) {
            stream_topk(total, a.kb, std::false_type{}, [&](int t, OwnerState* state, bool* el, int* id, int* p, float* y) {
                (void)state;
                const int64_t b = b_lo + t;
                load_row(kl + b * R, y);
                *id = (int)b;
                *p = 0;
                *el = true;
            });
        }
    }
    const int nsel = sh.count;
    if (SCORED) {
        // the chosen blocks with their scores, block ids shifted to the caller's numbering
        float* os = a.out_score + row * a.kb_cap;
        int32_t* ob = a.out_block + row * a.kb_cap;
        for (int e = threadIdx.x; e < a.kb_cap; e += blockDim.x) {
            os[e] = e < nsel ? bs[e] : -INFINITY;
            ob[e] = e < nsel ? bi[e] + a.blk_shift : -1;
        }
        if (threadIdx.x == 0) a.out_n[row] = nsel;
        return;
    }
    emit_row<THREADS>(bi, bp, nsel, pos, a.sink, a.window, a.pool, a.max_sel, a.idx + row * a.max_sel,
                      a.cnt + row);
    if (COUNT) {
        unsigned long long wn = nsc_node, wb = nsc_blk;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            wn += __shfl_xor_sync(0xffffffffu, wn, o);
            wb += __shfl_xor_sync(0xffffffffu, wb, o);
        }
        if (lane == 0) {
            atomicAdd(a.work, wn);
            atomicAdd(a.work + 1, wb);
        }
    }
}

template <int R, int THREADS>
int launch_select_t(const SelArgs& a, int64_t nq, int64_t units, bool fullscan, cudaStream_t s) {
    const size_t smem = (size_t)a.cap * 12 + (size_t)(3 * a.beam + 1) * 4;
    auto kern = fullscan ? select_kernel<R, true, THREADS, false>
                         : (a.work ? select_kernel<R, false, THREADS, true>
                                   : (a.out_score ? select_kernel<R, false, THREADS, false, true>
                                                  : select_kernel<R, false, THREADS, false>));
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_status(e);
    if (THREADS == kSelThreads) {
        // ask for no more shared memory than the resident CTAs need (each also
        // holds 1 KB for the system): the rest of the SM's 256 KB stays L1,
        // which keeps the upper tree levels that every query scores
        // (a hint: the percentage is clamped to 100, and a refusal leaves the
        // driver's own choice, which is correct, only slower)
        const int per = (int)(smem + sizeof(SelShared) + 1024);
        const int pct = min(100, (LSA_SELECT_MIN_BLOCKS * per * 100 + 233471) / 233472);
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, pct);
        if (e != cudaSuccess) return cuda_status(e);
    }
    dim3 grid((unsigned)nq, (unsigned)units);
    note_launch();
    kern<<<grid, THREADS, smem, s>>>(a);
    return cuda_status(cudaGetLastError());
}

template <int R>
int launch_select_r(const SelArgs& a, int64_t nq, int64_t units, bool fullscan, cudaStream_t s) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (nq * units < 2 * (int64_t)sms) {
        // one CTA per SM at most: a buffer that holds a whole level (fewer
        // compaction rounds), within the 227 KB a CTA may use
        SelArgs w = a;
        while (w.cap < kWideCap && (size_t)(2 * w.cap) * 12 + (size_t)(3 * w.beam + 1) * 4 <= 200 * 1024) w.cap *= 2;
        return launch_select_t<R, kWideThreads>(w, nq, units, fullscan, s);
    }
    return launch_select_t<R, kSelThreads>(a, nq, units, fullscan, s);
}

// ------------------------------------------------------------ shard merge
// Selection rows from per-shard picks (context parallelism): per (query, KV
// head) row, the union of every part's scored blocks, its top kb by (score
// desc, block asc) with the same compaction as the tree search, then the row
// of emit_row.  One CTA per row.
constexpr int kMergeThreads = 256;

struct MergeArgs {
    int parts, kb_cap, kb, hkv, pool, sink, window, max_sel, cap;
    int64_t rows, nq, q_pos0;
    const float* score;
    const int32_t* block;
    const int32_t* count;
    const int64_t* q_pos;
    int32_t* idx;
    int32_t* cnt;
};

__global__ __launch_bounds__(kMergeThreads) void merge_select_kernel(const MergeArgs m) {
    extern __shared__ float4 dyn4[];
    __shared__ SelShared sh;
    __shared__ int part_off[65];
    float* const bs = reinterpret_cast<float*>(dyn4);
    int* const bi = reinterpret_cast<int*>(bs + m.cap);
    int* const bp = reinterpret_cast<int*>(bs + 2 * m.cap);
    const int64_t row = blockIdx.x;
    const int64_t bseq = row / ((int64_t)m.nq * m.hkv);
    const int64_t qi = (row / m.hkv) % m.nq;
    const int64_t pos = m.q_pos ? m.q_pos[bseq * m.nq + qi] : m.q_pos0 + qi;
    for (int e = threadIdx.x; e < 256; e += blockDim.x) sh.hist[e] = 0;
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int p = 0; p < m.parts; ++p) {
            part_off[p] = acc;
            const int c = m.count[(int64_t)p * m.rows + row];
            acc += c < 0 ? 0 : (c > m.kb_cap ? m.kb_cap : c);
        }
        part_off[m.parts] = acc;
    }
    __syncthreads();
    const int n = part_off[m.parts];
    for (int t = threadIdx.x; t < m.parts * m.kb_cap; t += blockDim.x) {
        const int p = t / m.kb_cap, e = t % m.kb_cap;
        if (part_off[p] + e < part_off[p + 1]) {
            const int64_t src = ((int64_t)p * m.rows + row) * m.kb_cap + e;
            bs[part_off[p] + e] = m.score[src];
            bi[part_off[p] + e] = m.block[src];
            bp[part_off[p] + e] = 0;
        }
    }
    __syncthreads();
    int nsel = n;
    if (n > m.kb) {
        topk_compact(bs, bi, bp, n, m.kb, sh);
        nsel = m.kb;
    }
    __syncthreads();
    emit_row<kMergeThreads>(bi, bp, nsel, pos, m.sink, m.window, m.pool, m.max_sel, m.idx + row * m.max_sel,
                            m.cnt + row);
}

}  // namespace

int launch_select_rows(const lsa_index* ix, const lsa_select_params* sp, const float* qbar, int64_t nq_stride,
                       int64_t nq, const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int max_sel,
                       bool fullscan, cudaStream_t s, unsigned long long* work, const ScoredOut* scored,
                       const PreScores* pre) {
    const lsa_build_params& p = ix->p;
    if (sp->beam > 1024) return LSA_ERR_INVALID_ARG;
    SelArgs a{};
    for (int l = 0; l < p.levels; ++l) {
        a.ocent[l] = ix->ord_cent[l];
        a.omp[l] = ix->ord_mp[l];
        a.oid[l] = ix->ord_id[l];
        a.ocoff[l] = ix->ord_coff[l];
        a.n_l[l] = p.level_sizes[l];
    }
    a.levels = p.levels;
    a.Klp = ix->Klp;
    a.blk = ix->blk;
    a.leaf_start = ix->leaf_start;
    a.leaf_cnt = ix->leaf_cnt;
    a.Kl = ix->Kl;
    a.nb_cap = ix->nb_cap;
    a.nb = ix->nb;
    a.pool = p.pool;
    a.sink = p.sink;
    a.window = sp->window;
    a.beam = sp->beam;
    a.kb = (sp->topk + p.pool - 1) / p.pool;
    a.hkv = p.hkv;
    a.nq = nq_stride;
    a.qbar = qbar;
    a.q_pos = q_pos;
    a.q_pos0 = q_pos0;
    a.idx = idx;
    a.cnt = cnt;
    a.max_sel = max_sel;
    a.work = work;
    if (pre && !fullscan) {
        a.pre = pre->S;
        a.pre_nq = nq;
        a.pre_ld = pre->ld;
        a.pre_levels = pre->levels;
        for (int l = 0; l < pre->levels; ++l) a.pre_off[l] = pre->off[l];
        a.lt_b1 = pre->b1;
        a.lt_nb1 = pre->nb1;
        a.lt_s2 = pre->S2;
        a.lt_ld = pre->s2_ld;
    }
    if (scored) {
        a.pos_shift = scored->pos_shift;
        a.blk_shift = scored->blk_shift;
        a.kb_cap = scored->kb_cap;
        a.out_score = scored->score;
        a.out_block = scored->block;
        a.out_n = scored->n;
    }
    const int kmax = a.kb > a.beam ? a.kb : a.beam;
    int cap = 1024;
    while (cap < 2 * kmax) cap <<= 1;
    a.cap = cap;
    if (nq <= 0) return LSA_OK;
    switch (p.r) {
        case 16: return launch_select_r<16>(a, nq, ix->units, fullscan, s);
        case 32: return launch_select_r<32>(a, nq, ix->units, fullscan, s);
        case 64: return launch_select_r<64>(a, nq, ix->units, fullscan, s);
        case 128: return launch_select_r<128>(a, nq, ix->units, fullscan, s);
        default: return LSA_ERR_INVALID_ARG;
    }
}

int launch_select(const lsa_index* ix, const lsa_select_params* sp, const float* qbar, int64_t nq,
                  const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int max_sel, bool fullscan,
                  cudaStream_t s, unsigned long long* work, const ScoredOut* scored) {
    return launch_select_rows(ix, sp, qbar, nq, nq, q_pos, q_pos0, idx, cnt, max_sel, fullscan, s, work, scored,
                              nullptr);
}

}  // namespace lsa

namespace lsa {

int launch_merge_selection(int parts, const float* score, const int32_t* block, const int32_t* count, int kb_cap,
                           int64_t batch, int64_t nq, int hkv, const int64_t* q_pos, int64_t q_pos0, int pool,
                           int kb, int sink, int window, int32_t* idx, int32_t* cnt, int max_sel, cudaStream_t s) {
    MergeArgs m{};
    m.parts = parts;
    m.kb_cap = kb_cap;
    m.kb = kb;
    m.hkv = hkv;
    m.pool = pool;
    m.sink = sink;
    m.window = window;
    m.max_sel = max_sel;
    int cap = 1024;
    while (cap < parts * kb_cap) cap <<= 1;
    m.cap = cap;
    m.rows = batch * nq * hkv;
    m.nq = nq;
    m.q_pos0 = q_pos0;
    m.score = score;
    m.block = block;
    m.count = count;
    m.q_pos = q_pos;
    m.idx = idx;
    m.cnt = cnt;
    if (m.rows <= 0) return LSA_OK;
    const size_t smem = (size_t)cap * 12;
    cudaError_t e = cudaFuncSetAttribute(merge_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_status(e);
    note_launch();
    merge_select_kernel<<<(unsigned)m.rows, kMergeThreads, smem, s>>>(m);
    return cuda_status(cudaGetLastError());
}

}  // namespace lsa

namespace lsa {

int launch_select_lists(const lsa_index* ix, const lsa_select_params* sp, const float* qbar, int64_t nq_stride,
                        int64_t nq_grid, const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt,
                        int max_sel, const ListIn& li, cudaStream_t s) {
    const lsa_build_params& p = ix->p;
    SelArgs a{};
    a.levels = p.levels;
    a.Kl = ix->Kl;
    a.nb_cap = ix->nb_cap;
    a.nb = ix->nb;
    a.pool = p.pool;
    a.sink = p.sink;
    a.window = sp->window;
    a.beam = sp->beam;
    a.kb = (sp->topk + p.pool - 1) / p.pool;
    a.hkv = p.hkv;
    a.nq = nq_stride;
    a.qbar = qbar;
    a.q_pos = q_pos;
    a.q_pos0 = q_pos0;
    a.idx = idx;
    a.cnt = cnt;
    a.max_sel = max_sel;
    a.l_cand = li.cand;
    a.l_cnt = li.count;
    a.l_npad = li.npad;
    a.l_cap = li.cap;
    const int kmax = a.kb > a.beam ? a.kb : a.beam;
    int cap = 1024;
    while (cap < 2 * kmax) cap <<= 1;
    a.cap = cap;
    if (nq_grid <= 0) return LSA_OK;
    switch (p.r) {
        case 16: return launch_select_t<16, kSelThreads>(a, nq_grid, ix->units, true, s);
        case 32: return launch_select_t<32, kSelThreads>(a, nq_grid, ix->units, true, s);
        default: return launch_select_t<64, kSelThreads>(a, nq_grid, ix->units, true, s);
    }
}

}  // namespace lsa
