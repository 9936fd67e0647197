// Block-wide selection helpers of the key-selection kernels (select.cu:
// per-query tree search, full scan, shard merge): the order-preserving score
// key, exact top-k compaction of (score, id) items by (score desc, id asc),
// and the selection row writer.  Everything here is in an anonymous
// namespace: each translation unit that includes it gets its own copy.
#pragma once

#include "lsa_internal.cuh"

namespace lsa {
namespace {

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

// Bitonic sort of IPT * THREADS ids (ids[0, nsel) padded with INT32_MAX), IPT
// per thread in registers: item i = IPT tid + k; strides below IPT inside a
// thread, up to 16 IPT across lanes by shuffles, 32 IPT and up through shared
// memory.  Leaves the sorted items in arr (which may alias ids), then a barrier.
template <int IPT, int THREADS>
__device__ void bitonic_ids(const int* ids, int nsel, int* arr) {
    constexpr int M = IPT * THREADS;
    int v[IPT];
#pragma unroll
    for (int k = 0; k < IPT; ++k) {
        const int i = IPT * threadIdx.x + k;
        v[k] = i < nsel ? ids[i] : INT32_MAX;
    }
    __syncthreads();   // ids and arr may be read and written below
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
}

// The selection row of the query at position pos: the nsel chosen block ids
// (ids[0, nsel), any order) sorted ascending (in `work`, which needs room for
// max(nsel, THREADS * kSortIpt) ints and may alias nothing else), then sink
// [0, min(S, pos+1)), the blocks' tokens and the window [max(0, pos-W+1), pos],
// -1 after; *cnt_out = the row's length.  Ends with the row written (no
// barrier after the last write).
template <int THREADS>
__device__ void emit_row(const int* ids, int* work, int nsel, int64_t pos, int sink, int window, int pool,
                         int max_sel, int32_t* out, int32_t* cnt_out) {
    constexpr int kSortIpt = THREADS >= 512 ? 1 : (512 / THREADS > 4 ? 512 / THREADS : 4);
    // ascending block ids
    int* arr = work;
    if (THREADS >= 512) {
        // wide CTAs: rank sort (each id counts the smaller ones), one barrier
        const int* src = ids;
        for (int e = threadIdx.x; e < nsel; e += THREADS) {
            const int x = src[e];
            int rank = 0;
            for (int j = 0; j < nsel; ++j) rank += src[j] < x;
            arr[rank] = x;
        }
        __syncthreads();
    } else if (nsel <= kSortIpt * THREADS) {
        // the smallest network that holds nsel (nsel is the same in every thread)
        if (kSortIpt >= 1 && nsel <= THREADS) bitonic_ids<1, THREADS>(ids, nsel, arr);
        else if (kSortIpt >= 2 && nsel <= 2 * THREADS) bitonic_ids<(kSortIpt >= 2 ? 2 : 1), THREADS>(ids, nsel, arr);
        else bitonic_ids<kSortIpt, THREADS>(ids, nsel, arr);
    } else {
        // bitonic sort, padded to a power of two
        int M = 1;
        while (M < nsel) M <<= 1;
        for (int e = threadIdx.x; e < M; e += blockDim.x) arr[e] = e < nsel ? ids[e] : INT32_MAX;
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
    const int lo_w = (int)max((int64_t)0, pos - window + 1);
    const int ns = min(sink, lo_w);
    const int nblk_tok = nsel * pool;
    const int total = ns + nblk_tok + ((int)pos - lo_w + 1);
    // (consecutive threads write consecutive entries: the row is written coalesced)
    const unsigned P = (unsigned)pool;
    for (int e = threadIdx.x; e < max_sel; e += blockDim.x) {
        int v;
        if (e < ns) {
            v = e;
        } else if (e < ns + nblk_tok) {
            const unsigned t = (unsigned)(e - ns);
            const unsigned j = t / P;
            v = arr[j] * pool + (int)(t - j * P);
        } else if (e < total) {
            v = lo_w + (e - ns - nblk_tok);
        } else {
            v = -1;
        }
        out[e] = v;
    }
    if (threadIdx.x == 0) *cnt_out = (int32_t)total;
}

}  // namespace
}  // namespace lsa
