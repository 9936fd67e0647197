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
#include "lsa_internal.cuh"

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
    unsigned long long* work;   // optional: += eligible nodes and blocks scored
};

constexpr int kResolveCap = 128;

// a candidate group's current owner among the kept nodes: its index, the first
// candidate past its run, and (its run's first slot - its first candidate)
struct OwnerState {
    int o, next, base;
};   // most items of the threshold bin ranked pairwise

struct SelShared {
    int hist[256];
    int bc[4];
    int count;
    int count2;
    int nkept;
    uint32_t thr;   // no item below this key can be in the current top k (0: none yet)
    uint32_t wmin[32], wmax[32];
    int nres;
};

// 32 bytes from global memory in one 256-bit read-only load (32-byte aligned).
__device__ __forceinline__ void ldg256(const float* p, float* v) {
    asm volatile("ld.global.nc.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                 : "l"(p));
}

// Order-preserving map of a float onto uint32 (-0 and +0 map together).
__device__ __forceinline__ uint32_t fkey(float f) {
    const uint32_t u = __float_as_uint(__fadd_rn(f, 0.0f));
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// k-th largest key among n items (1 <= k <= n).  mode 0: key = fkey(score);
// mode 1: key = ~id, restricted to items with fkey(score) == tkey.
// Precondition: sh.hist is all zero; it is left all zero.  Two barriers per
// 8-bit pass.  Returns the key; *need = how many items equal to it belong to
// the top k, *eq = how many items equal it.  Also clears sh.count2.
__device__ uint32_t block_kth(const float* s, const int* id, int n, int k, int mode, uint32_t tkey,
                              SelShared& sh, int* need, int* eq) {
    uint32_t prefix = 0, pmask = 0;
    int kk = k, eqc = 0;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            uint32_t key;
            bool act;
            if (mode == 0) {
                key = fkey(s[i]);
                act = true;
            } else {
                act = fkey(s[i]) == tkey;
                key = ~(uint32_t)id[i];
            }
            if (act && (key & pmask) == prefix) atomicAdd(&sh.hist[(key >> shift) & 255u], 1);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            int c[8], sum = 0;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                c[t] = sh.hist[255 - lane * 8 - t];
                sh.hist[255 - lane * 8 - t] = 0;
                sum += c[t];
            }
            const int incl = warp_incl_scan(sum);
            const int excl = incl - sum;
            if (excl < kk && kk <= incl) {
                int run = excl;
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    if (run + c[t] >= kk) {
                        sh.bc[0] = 255 - lane * 8 - t;
                        sh.bc[1] = kk - run;
                        sh.bc[2] = c[t];
                        break;
                    }
                    run += c[t];
                }
            }
            if (lane == 0 && shift == 0) sh.count2 = 0;
        }
        __syncthreads();
        prefix |= (uint32_t)sh.bc[0] << shift;
        pmask |= 255u << shift;
        kk = sh.bc[1];
        eqc = sh.bc[2];
    }
    *need = kk;
    *eq = eqc;
    return prefix;
}

// Keep, in place, the items of (s, id, ps)[0, n) whose (key, id) pass `take`;
// they end up in [0, sh.count2) in no particular order.  Items move in rounds
// of kRound per thread: every thread holds its items of a round in registers
// before any thread writes, and since no more items are kept than were read,
// a kept item never lands past the round it came from.
constexpr int kRound = 4;

template <typename Take>
__device__ void filter_in_place(float* s, int* id, int* ps, int n, SelShared& sh, Take&& take) {
    if (threadIdx.x == 0) sh.count2 = 0;
    __syncthreads();
    const int T = blockDim.x;
    for (int r0 = 0; r0 < n; r0 += kRound * T) {
        float vs[kRound];
        int vi[kRound], vp[kRound];
        bool tk[kRound];
#pragma unroll
        for (int j = 0; j < kRound; ++j) {
            const int i = r0 + j * T + (int)threadIdx.x;
            tk[j] = false;
            vs[j] = 0.f;
            vi[j] = vp[j] = 0;
            if (i < n) {
                vs[j] = s[i];
                vi[j] = id[i];
                vp[j] = ps[i];
                tk[j] = take(fkey(vs[j]), vi[j]);
            }
        }
        __syncthreads();   // the whole round is in registers
#pragma unroll
        for (int j = 0; j < kRound; ++j) {
            if (tk[j]) {
                const int p = atomicAdd(&sh.count2, 1);
                s[p] = vs[j];
                id[p] = vi[j];
                ps[p] = vp[j];
            }
        }
        __syncthreads();
    }
}

// General form: exact k-th key by 8-bit radix passes, then ties by id.
__device__ void topk_compact_radix(float* s, int* id, int* ps, int n, int k, SelShared& sh) {
    int need, eq;
    const uint32_t T = block_kth(s, id, n, k, 0, 0u, sh, &need, &eq);
    const bool split = need < eq;
    uint32_t T2 = 0;
    if (split) {
        int need2, eq2;
        T2 = block_kth(s, id, n, need, 1, T, sh, &need2, &eq2);
    }
    if (threadIdx.x == 0) sh.thr = T;
    filter_in_place(s, id, ps, n, sh, [&](uint32_t key, int xi) {
        return key > T || (key == T && (!split || ~(uint32_t)xi >= T2));
    });
}

// Keep, in place, the top k of the n items in (s, id, ps) by (score desc, id
// asc), k < n; the result is (s, id, ps)[0..k) in no particular order.  The
// keys are binned by their offset from the smallest key, shifted so that at
// most 256 bins are used (monotone in the key); bins above the one that holds
// the k-th item are taken whole, and that bin's items are ranked exactly by
// (key, id).  If that bin holds more than kResolveCap items (or all keys are
// equal), the general radix select runs instead.
__device__ void topk_compact(float* s, int* id, int* ps, int n, int k, SelShared& sh) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    uint32_t kmn = 0xffffffffu, kmx = 0u;
    for (int i = tid; i < n; i += blockDim.x) {
        const uint32_t key = fkey(s[i]);
        kmn = min(kmn, key);
        kmx = max(kmx, key);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        kmn = min(kmn, __shfl_xor_sync(0xffffffffu, kmn, o));
        kmx = max(kmx, __shfl_xor_sync(0xffffffffu, kmx, o));
    }
    if (lane == 0) { sh.wmin[warp] = kmn; sh.wmax[warp] = kmx; }
    if (tid == 0) sh.nres = 0;
    __syncthreads();
    kmn = sh.wmin[0];
    kmx = sh.wmax[0];
    for (int w = 1; w < nw; ++w) {
        kmn = min(kmn, sh.wmin[w]);
        kmx = max(kmx, sh.wmax[w]);
    }
    if (kmn == kmx) {
        topk_compact_radix(s, id, ps, n, k, sh);
        return;
    }
    const int shift = max(0, 24 - __clz(kmx - kmn));   // (kmx - kmn) >> shift <= 255
    for (int i = tid; i < n; i += blockDim.x) atomicAdd(&sh.hist[(fkey(s[i]) - kmn) >> shift], 1);
    __syncthreads();
    if (warp == 0) {
        int c[8], sum = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            c[t] = sh.hist[255 - lane * 8 - t];
            sh.hist[255 - lane * 8 - t] = 0;
            sum += c[t];
        }
        const int incl = warp_incl_scan(sum);
        const int excl = incl - sum;
        if (excl < k && k <= incl) {
            int run = excl;
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                if (run + c[t] >= k) {
                    sh.bc[0] = 255 - lane * 8 - t;   // bin B of the k-th item
                    sh.bc[1] = k - run;              // items of B in the top k
                    sh.bc[2] = c[t];                 // items in B
                    break;
                }
                run += c[t];
            }
        }
    }
    __syncthreads();
    const uint32_t B = (uint32_t)sh.bc[0];
    const int need = sh.bc[1], cntB = sh.bc[2];
    const bool all_b = need == cntB;
    if (!all_b && cntB > min(kResolveCap, k)) {
        topk_compact_radix(s, id, ps, n, k, sh);
        return;
    }
    // bin B's items, to be ranked among themselves (keys are distinct: ids
    // are), listed in the histogram's storage (all zero again afterwards)
    uint32_t* const rkey = reinterpret_cast<uint32_t*>(sh.hist);
    int* const rid = sh.hist + kResolveCap;
    if (!all_b) {
        for (int i = tid; i < n; i += blockDim.x) {
            const uint32_t key = fkey(s[i]);
            if (((key - kmn) >> shift) == B) {
                const int r = atomicAdd(&sh.nres, 1);
                rkey[r] = key;
                rid[r] = id[i];
            }
        }
    }
    if (tid == 0) sh.thr = kmn + (B << shift);   // smallest key that falls in bin B
    // (filter_in_place's first barrier publishes the bin-B list and thr)
    filter_in_place(s, id, ps, n, sh, [&](uint32_t key, int xi) {
        const uint32_t b = (key - kmn) >> shift;
        if (b != B) return b > B;
        if (all_b) return true;
        int rank = 0;
        for (int j = 0; j < cntB; ++j) {
            const uint32_t yk = rkey[j];
            rank += yk > key || (yk == key && rid[j] < xi);
        }
        return rank < need;
    });
    if (!all_b) {
        // (filter_in_place ended with a barrier: nobody reads the list any more;
        // the next user of the histogram is behind further barriers)
        for (int e = tid; e < 2 * kResolveCap; e += blockDim.x) sh.hist[e] = 0;
    }
}

// Exclusive scan of pre[0..n) in place (values are counts), pre[n] = total.
__device__ void scan_pre(int* pre, int n) {
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int carry = 0;
        for (int base = 0; base < n; base += 32) {
            const int v = (base + lane < n) ? pre[base + lane] : 0;
            const int incl = warp_incl_scan(v);
            if (base + lane < n) pre[base + lane] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) pre[n] = carry;
    }
    __syncthreads();
}

__device__ __forceinline__ int find_owner(const int* pre, int nk, int t) {
    int lo = 0, hi = nk;  // pre[lo] <= t < pre[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] <= t) lo = mid; else hi = mid;
    }
    return lo;
}

// THREADS = kSelThreads for large grids; small grids (decode: a few queries)
// give each (query, KV head) kWideThreads so the few CTAs use more of the SM.
constexpr int kWideThreads = 1024;
constexpr int kWideCap = 8192;

// COUNT: also add the number of eligible rows scored to *a.work (a separate
// instantiation, so the counting costs the timed path nothing)
template <int R, bool FULL, int THREADS, bool COUNT>
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
    // ids sorted in registers: 512 for the narrow CTAs
    constexpr int kSortIpt = THREADS >= 512 ? 1 : (512 / THREADS > 4 ? 512 / THREADS : 4);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane / LPC, gl = lane % LPC, gid = warp * CPW + g;
    const unsigned gmask = (LPC == 32) ? 0xffffffffu : (((1u << LPC) - 1u) << (g * LPC));

    const int64_t qi = blockIdx.x;
    const int u = blockIdx.y;
    const int64_t bseq = u / a.hkv;
    const int h = u % a.hkv;
    const int64_t row = (bseq * a.nq + qi) * a.hkv + h;
    const int64_t pos = a.q_pos ? a.q_pos[bseq * a.nq + qi] : a.q_pos0 + qi;
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

    unsigned nscored = 0;   // eligible candidates this thread's group scored (leader lanes)
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
    // aggregated per warp: one shared-memory atomic per batch.
    auto stream_topk = [&](int total, int k, auto&& fetch) {
        if (k <= 0) return;  // nothing is kept; the buffer stays empty
        // entered with an empty buffer; nbuf mirrors sh.count between chunks
        if (threadIdx.x == 0) sh.thr = 0u;
        __syncthreads();
        int t0 = 0, nbuf = 0;
        while (t0 < total) {
            const uint32_t thr = sh.thr;
            const int t1 = min(total, t0 + (a.cap - nbuf));
            const int span = (t1 - t0 + NG - 1) / NG;
            const int tb = t0 + gid * span;
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
                        sc[v] = dot(y[v]);
                        if (COUNT) nscored += (gl == 0);
                        ok[v] = fkey(sc[v]) >= thr;
                    }
                    bal[v] = __ballot_sync(0xffffffffu, ok[v] && gl == 0);
                    nb_warp += __popc(bal[v]);
                }
                int base = 0;
                if (lane == 0 && nb_warp) base = atomicAdd(&sh.count, nb_warp);
                base = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
                for (int v = 0; v < kUnroll; ++v) {
                    if (ok[v] && gl == 0) {
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
        for (int l = 0; l < a.levels; ++l) {
            const int nl = a.n_l[l];
            const float* cent = a.ocent[l] + (int64_t)u * nl * R;
            const int64_t* mp = a.omp[l] + (int64_t)u * nl;
            const int32_t* oid = a.oid[l] + (int64_t)u * nl;
            const int nk = sh.nkept;
            const int total = (l == 0) ? nl : pre[nk];
            if (threadIdx.x == 0) sh.count = 0;
            __syncthreads();
            stream_topk(total, a.beam, [&](int t, OwnerState* state, bool* el, int* id, int* p, float* y) {
                int q;
                if (l == 0) {
                    q = t;
                } else {
                    q = slot_of(t, nk, state);
                }
                load_row(cent + (int64_t)q * R, y);
                *id = __ldg(oid + q);
                *p = q;
                *el = __ldg(mp + q) <= bound;
            });
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
        stream_topk(pre[nk], a.kb, [&](int t, OwnerState* state, bool* el, int* id, int* p, float* y) {
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
        stream_topk(total, a.kb, [&](int t, OwnerState* state, bool* el, int* id, int* p, float* y) {
            (void)state;
            const int64_t b = b_lo + t;
            load_row(kl + b * R, y);
            *id = (int)b;
            *p = 0;
            *el = true;
        });
    }
    const int nsel = sh.count;

    // ascending block ids
    int* arr = bp;   // the positions are no longer needed
    if (THREADS >= 512) {
        // wide CTAs: rank sort (each id counts the smaller ones), one barrier
        const int* src = bi;
        for (int e = threadIdx.x; e < nsel; e += THREADS) {
            const int x = src[e];
            int rank = 0;
            for (int j = 0; j < nsel; ++j) rank += src[j] < x;
            arr[rank] = x;
        }
        __syncthreads();
    } else if (nsel <= kSortIpt * THREADS) {
        // bitonic sort of IPT * THREADS items (padded with INT32_MAX), IPT per
        // thread in registers: item i = IPT tid + k; strides below IPT inside
        // a thread, up to 16 IPT across lanes by shuffles, 32 IPT and up
        // through shared memory
        constexpr int IPT = kSortIpt;
        constexpr int M = IPT * THREADS;
        int v[IPT];
        const int* src = bi;
#pragma unroll
        for (int k = 0; k < IPT; ++k) {
            const int i = IPT * threadIdx.x + k;
            v[k] = i < nsel ? src[i] : INT32_MAX;
        }
        __syncthreads();   // src and arr may be read and written below
        for (int size = 2; size <= M; size <<= 1) {
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                if (stride >= 32 * IPT) {
#pragma unroll
                    for (int k = 0; k < IPT; ++k) arr[IPT * threadIdx.x + k] = v[k];
                    __syncthreads();
#pragma unroll
                    for (int k = 0; k < IPT; ++k) {
                        const int i = IPT * threadIdx.x + k;
                        const int y = arr[i ^ stride];
                        const bool asc = (i & size) == 0;
                        const bool lower = (i & stride) == 0;
                        v[k] = (lower == asc) ? min(v[k], y) : max(v[k], y);
                    }
                    __syncthreads();
                } else if (stride >= IPT) {
#pragma unroll
                    for (int k = 0; k < IPT; ++k) {
                        const int i = IPT * threadIdx.x + k;
                        const int y = __shfl_xor_sync(0xffffffffu, v[k], stride / IPT);
                        const bool asc = (i & size) == 0;
                        const bool lower = (i & stride) == 0;
                        v[k] = (lower == asc) ? min(v[k], y) : max(v[k], y);
                    }
                } else {
                    // pairs (k, k + stride) inside the thread; every stride is
                    // unrolled so every register index is a constant
#pragma unroll
                    for (int st = IPT / 2; st >= 1; st >>= 1) {
                        if (st != stride) continue;
#pragma unroll
                        for (int k = 0; k < IPT; ++k) {
                            if (k & st) continue;
                            const bool asc = ((IPT * (int)threadIdx.x + k) & size) == 0;
                            const int lo = min(v[k], v[k + st]), hi = max(v[k], v[k + st]);
                            v[k] = asc ? lo : hi;
                            v[k + st] = asc ? hi : lo;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int k = 0; k < IPT; ++k) arr[IPT * threadIdx.x + k] = v[k];
        __syncthreads();
    } else {
        // bitonic sort, padded to a power of two
        int M = 1;
        while (M < nsel) M <<= 1;
        for (int e = threadIdx.x; e < M; e += blockDim.x) arr[e] = e < nsel ? bi[e] : INT32_MAX;
        __syncthreads();
        for (int size = 2; size <= M; size <<= 1) {
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                for (int t = threadIdx.x; t < (M >> 1); t += blockDim.x) {
                    const int i = 2 * stride * (t / stride) + (t % stride);
                    const int j = i + stride;
                    const bool asc = (i & size) == 0;
                    const int x = arr[i], y = arr[j];
                    if ((x > y) == asc) { arr[i] = y; arr[j] = x; }
                }
                __syncthreads();
            }
        }
    }

    // row = sink [0, ns) | blocks (P tokens each, ascending) | window [lo_w, pos] | -1 padding;
    // positions fit in int32 (checked by the caller), so no 64-bit division here
    const int lo_w = (int)max((int64_t)0, pos - a.window + 1);
    const int ns = min(a.sink, lo_w);
    const int nblk_tok = nsel * a.pool;
    const int total = ns + nblk_tok + ((int)pos - lo_w + 1);
    int32_t* out = a.idx + row * a.max_sel;
    // (consecutive threads write consecutive entries: the row is written coalesced)
    const unsigned P = (unsigned)a.pool;
    for (int e = threadIdx.x; e < a.max_sel; e += blockDim.x) {
        int v;
        if (e < ns) {
            v = e;
        } else if (e < ns + nblk_tok) {
            const unsigned t = (unsigned)(e - ns);
            const unsigned j = t / P;
            v = arr[j] * a.pool + (int)(t - j * P);
        } else if (e < total) {
            v = lo_w + (e - ns - nblk_tok);
        } else {
            v = -1;
        }
        out[e] = v;
    }
    if (threadIdx.x == 0) a.cnt[row] = (int32_t)total;
    if (COUNT) {
        unsigned long long w = nscored;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
        if (lane == 0) atomicAdd(a.work, w);
    }
}

template <int R, int THREADS>
int launch_select_t(const SelArgs& a, int64_t nq, int64_t units, bool fullscan, cudaStream_t s) {
    const size_t smem = (size_t)a.cap * 12 + (size_t)(3 * a.beam + 1) * 4;
    auto kern = fullscan ? select_kernel<R, true, THREADS, false>
                         : (a.work ? select_kernel<R, false, THREADS, true> : select_kernel<R, false, THREADS, false>);
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

}  // namespace

int launch_select(const lsa_index* ix, const lsa_select_params* sp, const float* qbar, int64_t nq,
                  const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int max_sel, bool fullscan,
                  cudaStream_t s, unsigned long long* work) {
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
    a.nq = nq;
    a.qbar = qbar;
    a.q_pos = q_pos;
    a.q_pos0 = q_pos0;
    a.idx = idx;
    a.cnt = cnt;
    a.max_sel = max_sel;
    a.work = work;
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

}  // namespace lsa
