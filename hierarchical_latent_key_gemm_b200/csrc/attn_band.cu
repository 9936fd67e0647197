// Exact softmax attention over the selection, split by where the rows come
// from.  The selection of query i is the union of the attention sink
// [0, min(S, i+1)), the chosen long-range blocks, and the local window
// [max(0, i-W+1), i] (LSA explainer, "How does LSA work?" step 3: the kept
// long-range keys plus the sink and a local window; the attention kernel itself
// is unchanged).  Sink and window rows are the same for neighbouring queries,
// so they are read once per tile of consecutive queries instead of once per
// query:
//
//   attn_band_tc_kernel (attn_band_tc.cu) dense tcgen05 tiles: 128 (query,
//                       head) rows per CTA against the contiguous key band
//                       [0, S) and [i0-W+1, i1], with the per-row mask
//                       j <= i && (j < S || j >= i-W+1); writes an unnormalised
//                       partial (acc, running max, sum of weights).
//   attn_gather_kernel  one warp per (query, KV head): the long-range entries of
//                       the row list only, starting from the band partial, and
//                       writes the normalised output.
//
// Both parts are the same softmax over disjoint key sets, merged by their
// maxima, so the result equals attention over the whole list up to rounding.
// A row list that does not have the selection form (checked in O(1) per row:
// rows are ascending without repeats, the first min(S, i+1) entries are the
// sink, the last ones the window) is processed whole by the gather kernel
// with the band partial ignored, so any ascending list gives exact attention.
//
// Gather kernel tensor-core layout: keys on the M side (16 per slice), the G
// heads of the group on N (n8 tiles), so no head padding to 16 rows:
// S^T = K_slice Q^T, then O^T += V^T P^T with P^T moved into B-operand order by
// movmatrix.  P is split into two bf16 terms (hi + lo) as in the other paths.
#include <algorithm>

#include "lsa_internal.cuh"
#include "tma_util.cuh"
#include "warp_mma.cuh"

namespace lsa {
namespace {


#ifndef LSA_GAT_WARPS
#define LSA_GAT_WARPS 1
#endif
#ifndef LSA_GAT_STAGES
#define LSA_GAT_STAGES 2
#endif
constexpr int kGatWarps = LSA_GAT_WARPS;    // queries per CTA (one warp each)
constexpr int kGatSlice = 16;               // keys per slice
constexpr int kGatStages = LSA_GAT_STAGES;  // slices in each warp's ring
constexpr int kGatTQ = 1;                   // slices of token ids read ahead of their copies
#ifndef LSA_GAT_ORDER_MIN
#define LSA_GAT_ORDER_MIN 65536
#endif
constexpr int64_t kGatOrderMinPairs = LSA_GAT_ORDER_MIN;   // fewer row lists run in row order

struct BandArgs {
    const __nv_bfloat16* Q;
    const __nv_bfloat16* K;
    const __nv_bfloat16* V;
    int64_t nq, q_pos0, ld_tokens;
    int hq, hkv, sink, window;
    float scale_log2;
    float* part_o;    // [batch*nq*hq][D] unnormalised sum of p * v
    float2* part_ml;  // [batch*nq*hq] (running max in log2 units, sum of weights)
};

struct GatherArgs {
    const __nv_bfloat16* Q;
    const __nv_bfloat16* K;
    const __nv_bfloat16* V;
    const int32_t* idx;
    const int32_t* cnt;
    int64_t nq, q_pos0, ld_tokens;
    int hq, hkv, max_sel, sink, window;
    float scale_log2;
    const float* part_o;
    const float2* part_ml;
    __nv_bfloat16* O;
    float* lse;
    int32_t* err;
    const int32_t* order;   // optional: pair (row list) processed by warp w of the grid, else w itself
    int64_t pairs;          // batch * nq * hkv
};

// NT = n8 tiles of heads (G <= 8 * NT; heads past G are zero and dropped)
template <int D, int NT>
__global__ __launch_bounds__(kGatWarps * 32) void attn_gather_kernel(const GatherArgs a) {
    constexpr int CH = D / 8;
    constexpr int SLICE_BYTES = kGatSlice * D * 2;
    constexpr int RPL = kGatSlice * CH / 32;   // rows of a slice each lane copies
    constexpr int RSTEP = 32 / CH;
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char* Ks = smem + warp * (2 * kGatStages * SLICE_BYTES);   // [stages][16][D]
    unsigned char* Vs = Ks + kGatStages * SLICE_BYTES;
    // per stage: bit k set when key k of the slice is a real token
    uint32_t* vmask = reinterpret_cast<uint32_t*>(smem + kGatWarps * 2 * kGatStages * SLICE_BYTES) + warp * kGatStages;
    const int G = a.hq / a.hkv;
    const int64_t wg = (int64_t)blockIdx.x * kGatWarps + warp;
    if (wg >= a.pairs) return;   // warp-uniform; the kernel has no CTA barrier
    // row list (b, query, KV head) of this warp: pairs run in the given order
    // (similar selections next to each other share rows in L2), else in row order
    const int64_t pr = a.order ? (int64_t)a.order[wg] : wg;
    const int h = (int)(pr % a.hkv);
    const int64_t bq = pr / a.hkv;
    const int64_t qi = bq % a.nq;
    const int64_t b = bq / a.nq;
    const int64_t i = a.q_pos0 + qi;
    const int64_t row = (b * a.nq + qi) * a.hkv + h;
    int n = a.cnt[row];
    if (n < 0 || n > a.max_sel) {
        if (lane == 0) latch(a.err, kErrDevice);
        n = n < 0 ? 0 : a.max_sel;
    }
    const int32_t* ir = a.idx + row * a.max_sel;

    // does the row have the selection form?
    const int ns = (int)min((int64_t)a.sink, i + 1);
    const int nw = i >= a.sink ? (int)min(i - a.sink + 1, (int64_t)a.window) : 0;
    bool form = n >= ns + nw;
    if (form && ns > 0) form = __ldg(ir) == 0 && __ldg(ir + ns - 1) == ns - 1;
    if (form && nw > 0) form = __ldg(ir + n - 1) == i && __ldg(ir + n - nw) == i - nw + 1;
    if (form && n - nw > ns) form = __ldg(ir + ns) >= a.sink && __ldg(ir + n - nw - 1) <= i - a.window;
    const int pbeg = form ? ns : 0, pend = form ? n - nw : n;

    // Q^T as B fragments: head = 8 nt + lane/4, dims 16 kt + 2 (lane%4) (+8)
    const int64_t qrow0 = (b * a.nq + qi) * a.hq + (int64_t)h * G;
    uint32_t qb[D / 16][NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int hh = nt * 8 + (lane >> 2);
        const uint32_t* qp = reinterpret_cast<const uint32_t*>(a.Q + (qrow0 + (hh < G ? hh : 0)) * D);
#pragma unroll
        for (int kt = 0; kt < D / 16; ++kt) {
            const int dd = 16 * kt + 2 * (lane & 3);
            qb[kt][nt][0] = hh < G ? __ldg(qp + dd / 2) : 0u;
            qb[kt][nt][1] = hh < G ? __ldg(qp + dd / 2 + 4) : 0u;
        }
    }

    // state: this thread's heads hA = 8 nt + 2 (lane%4), hB = hA + 1; O^T rows
    // (dims) 16 mt + lane/4 and + 8
    float m[NT][2], l[NT][2], ot[D / 16][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int hh = nt * 8 + 2 * (lane & 3) + c;
            float mm = -INFINITY, ll = 0.f;
            if (form && hh < G) {
                const float2 ml = a.part_ml[qrow0 + hh];
                mm = ml.x;
                ll = lane < 4 ? ml.y : 0.f;   // summed over the 8 key lanes at the end
            }
            m[nt][c] = mm;
            l[nt][c] = ll;
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) {
                float v0 = 0.f, v1 = 0.f;
                if (form && hh < G) {
                    const float* po = a.part_o + (qrow0 + hh) * D + 16 * mt + (lane >> 2);
                    v0 = po[0];
                    v1 = po[8];
                }
                ot[mt][nt][c] = v0;
                ot[mt][nt][2 + c] = v1;
            }
        }
    }

    const int nslice = (pend - pbeg + kGatSlice - 1) / kGatSlice;
    const __nv_bfloat16* kbase = a.K + (b * a.ld_tokens * a.hkv + h) * D;
    const __nv_bfloat16* vbase = a.V + (b * a.ld_tokens * a.hkv + h) * D;
    // token of key `lane` of slice s (lanes < 16); a bad index is latched and skipped
    auto fetch_tok = [&](int s) -> int {
        const int p = pbeg + s * kGatSlice + lane;
        int t = (lane < kGatSlice && s < nslice && p < pend) ? __ldg(ir + p) : -1;
        if (t >= a.ld_tokens || t < -1) {
            latch(a.err, kErrDevice);
            t = -1;
        }
        return t;
    };
    // each lane copies 16-byte column c of rows lane/CH + RSTEP*k; the shared
    // offsets of those rows and the column's source offset are fixed
    const int c_col = lane % CH;
    uint32_t dsto[RPL];
#pragma unroll
    for (int k = 0; k < RPL; ++k) dsto[k] = swz<D>(lane / CH + RSTEP * k, c_col);
    const char* ksrc = reinterpret_cast<const char*>(kbase + c_col * 8);
    const int64_t vk = reinterpret_cast<const char*>(vbase) - reinterpret_cast<const char*>(kbase);
    const int64_t rs = (int64_t)a.hkv * D * 2;
    auto load_slice = [&](int s, int tok_l) {
        const int st = s % kGatStages;
        const uint32_t kb = smem_u32(Ks + st * SLICE_BYTES), vb = smem_u32(Vs + st * SLICE_BYTES);
        const uint32_t live = __ballot_sync(0xffffffffu, tok_l >= 0);
        if (lane == 0) vmask[st] = live & 0xffffu;
#pragma unroll
        for (int k = 0; k < RPL; ++k) {
            const int tok = __shfl_sync(0xffffffffu, tok_l, lane / CH + RSTEP * k);
            const char* src = ksrc + (tok >= 0 ? (int64_t)tok * rs : 0);
            const int nbytes = tok >= 0 ? 16 : 0;
            cp_async16(kb + dsto[k], src, nbytes);
            cp_async16(vb + dsto[k], src + vk, nbytes);
        }
    };
    // token ids of the next TQ slices to load, oldest first (loads issued TQ
    // slices before the rows they address are copied)
    int tokq[kGatTQ];
#pragma unroll
    for (int j = 0; j < kGatTQ; ++j) tokq[j] = fetch_tok(j);
    auto pop_tok = [&](int s_next) -> int {
        const int t0 = tokq[0];
#pragma unroll
        for (int j = 0; j + 1 < kGatTQ; ++j) tokq[j] = tokq[j + 1];
        tokq[kGatTQ - 1] = fetch_tok(s_next);
        return t0;
    };
#pragma unroll
    for (int s = 0; s < kGatStages - 1; ++s) {
        const int tk = pop_tok(s + kGatTQ);
        if (s < nslice) load_slice(s, tk);
        cp_async_commit();
    }

    for (int s = 0; s < nslice; ++s) {
        cp_async_wait<kGatStages - 2>();
        __syncwarp();
        {
            const int tk = pop_tok(s + kGatStages - 1 + kGatTQ);
            if (s + kGatStages - 1 < nslice) load_slice(s + kGatStages - 1, tk);
        }
        cp_async_commit();
        const int st = s % kGatStages;
        const uint32_t kb = smem_u32(Ks + st * SLICE_BYTES), vb = smem_u32(Vs + st * SLICE_BYTES);
        // S^T = K_slice Q^T: rows = 16 keys, cols = heads
        // (all fragments first, then two independent accumulation chains)
        float sc[NT][4], sc2[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
            sc2[nt][0] = sc2[nt][1] = sc2[nt][2] = sc2[nt][3] = 0.f;
        }
        {
            const int kr = (lane & 7) + 8 * ((lane >> 3) & 1);
            uint32_t ka[D / 16][4];
#pragma unroll
            for (int kt = 0; kt < D / 16; ++kt)
                ldsm_x4(kb + swz<D>(kr, 2 * kt + (lane >> 4)), ka[kt][0], ka[kt][1], ka[kt][2], ka[kt][3]);
#pragma unroll
            for (int kt = 0; kt < D / 16; kt += 2) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma_bf16(sc[nt], ka[kt], qb[kt][nt][0], qb[kt][nt][1]);
                    mma_bf16(sc2[nt], ka[kt + 1], qb[kt + 1][nt][0], qb[kt + 1][nt][1]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[nt][e] += sc2[nt][e];
        }
        // keys lane/4 and lane/4 + 8 of the slice
        const uint32_t vm = vmask[st];
        const bool k0 = (vm >> (lane >> 2)) & 1u, k1 = (vm >> ((lane >> 2) + 8)) & 1u;
        uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float x0 = k0 ? sc[nt][0] * a.scale_log2 : -INFINITY;   // (key, hA)
            const float x1 = k0 ? sc[nt][1] * a.scale_log2 : -INFINITY;   // (key, hB)
            const float x2 = k1 ? sc[nt][2] * a.scale_log2 : -INFINITY;   // (key+8, hA)
            const float x3 = k1 ? sc[nt][3] * a.scale_log2 : -INFINITY;   // (key+8, hB)
            float mA = fmaxf(x0, x2), mB = fmaxf(x1, x3);
#pragma unroll
            for (int o = 4; o <= 16; o <<= 1) {
                mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, o));
                mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, o));
            }
            const float nA = fmaxf(m[nt][0], mA), nB = fmaxf(m[nt][1], mB);
            const float aA = (nA == -INFINITY) ? 1.f : exp2f(m[nt][0] - nA);
            const float aB = (nB == -INFINITY) ? 1.f : exp2f(m[nt][1] - nB);
            const float p0 = (nA == -INFINITY) ? 0.f : exp2f(x0 - nA);
            const float p2 = (nA == -INFINITY) ? 0.f : exp2f(x2 - nA);
            const float p1 = (nB == -INFINITY) ? 0.f : exp2f(x1 - nB);
            const float p3 = (nB == -INFINITY) ? 0.f : exp2f(x3 - nB);
            l[nt][0] = l[nt][0] * aA + (p0 + p2);
            l[nt][1] = l[nt][1] * aB + (p1 + p3);
            m[nt][0] = nA;
            m[nt][1] = nB;
            uint32_t h01, l01, h23, l23;
            split_pack(p0, p1, h01, l01);   // row = key lane/4, cols = (hA, hB)
            split_pack(p2, p3, h23, l23);   // row = key lane/4 + 8
            bh[nt][0] = movmatrix_t(h01);
            bh[nt][1] = movmatrix_t(h23);
            bl[nt][0] = movmatrix_t(l01);
            bl[nt][1] = movmatrix_t(l23);
            if (__any_sync(0xffffffffu, aA != 1.f || aB != 1.f)) {
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    ot[mt][nt][0] *= aA; ot[mt][nt][1] *= aB;
                    ot[mt][nt][2] *= aA; ot[mt][nt][3] *= aB;
                }
            }
        }
        // O^T += V^T P^T: rows = dims (16 per m tile), k = 16 keys
        // (all fragments first; the hi pass over every m tile, then the lo pass,
        // so no two consecutive MMAs share an accumulator)
        {
            const int vr = (lane & 7) + 8 * (lane >> 4);
            uint32_t va[D / 16][4];
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt)
                ldsm_x4_t(vb + swz<D>(vr, 2 * mt + ((lane >> 3) & 1)), va[mt][0], va[mt][1], va[mt][2], va[mt][3]);
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16(ot[mt][nt], va[mt], bh[nt][0], bh[nt][1]);
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16(ot[mt][nt], va[mt], bl[nt][0], bl[nt][1]);
        }
    }
    cp_async_wait<0>();
    __syncwarp();

    // normalise and write: stage [G][D] bf16 in this warp's ring, then 16-byte stores
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(Ks);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float ll = l[nt][c];
#pragma unroll
            for (int o = 4; o <= 16; o <<= 1) ll += __shfl_xor_sync(0xffffffffu, ll, o);
            const int hh = nt * 8 + 2 * (lane & 3) + c;
            const float inv = ll > 0.f ? 1.f / ll : 0.f;
            if (hh < G) {
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    const int dd = 16 * mt + (lane >> 2);
                    stage[hh * D + dd] = __float2bfloat16_rn(ot[mt][nt][c] * inv);
                    stage[hh * D + dd + 8] = __float2bfloat16_rn(ot[mt][nt][2 + c] * inv);
                }
                if (lane < 4 && a.lse)
                    a.lse[qrow0 + hh] = ll > 0.f ? (m[nt][c] + log2f(ll)) * 0.69314718055994531f : -INFINITY;
            }
        }
    }
    __syncwarp();
    uint4* dst = reinterpret_cast<uint4*>(a.O + qrow0 * D);
    const uint4* srcv = reinterpret_cast<const uint4*>(stage);
    for (int e = lane; e < G * D / 8; e += 32) dst[e] = srcv[e];
}

// Sort key of a row list for the gather order: its first entry after the sink
// (the smallest long-range token when the row is a selection).  Rows whose
// long-range sets overlap mostly share that first entry, so sorting by it puts
// queries that gather the same K/V rows next to each other.
__global__ void gather_key_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int64_t nq,
                                  int hkv, int max_sel, int64_t q_pos0, int sink, int64_t pairs, int64_t ld_tokens,
                                  uint32_t* __restrict__ keys, int32_t* __restrict__ vals) {
    const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= pairs) return;
    const int64_t i = q_pos0 + (p / hkv) % nq;
    const int n = cnt[p];
    const int ns = (int)min((int64_t)sink, i + 1);
    uint32_t key = 0xFFFFFFFFu;
    if (n > ns && n <= max_sel) {
        // KV heads apart (their rows are different memory) when (head, token) fits in 32 bits
        const int64_t t = idx[p * max_sel + ns];
        const int64_t hk = (int64_t)(p % hkv) * ld_tokens + t;
        key = (uint32_t)(hkv * ld_tokens < 0xFFFFFFFFll ? hk : t);
    }
    keys[p] = key;
    vals[p] = (int32_t)p;
}

template <int D, int G>
int launch_band_g(const BandArgs& ba, const GatherArgs& ga, int64_t batch, cudaStream_t s) {
    constexpr int NT = (G + 7) / 8;
    const size_t smem_gat = (size_t)kGatWarps * 2 * kGatStages * kGatSlice * D * 2 + kGatWarps * kGatStages * 4;
    cudaError_t e = cudaFuncSetAttribute(attn_gather_kernel<D, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_gat);
    if (e != cudaSuccess) return cuda_status(e);
    const int st = launch_band_tc(ba.Q, ba.K, ba.V, batch, ba.nq, ba.q_pos0, ba.hq, ba.hkv, D, ba.ld_tokens, ba.sink,
                                  ba.window, ba.part_o, ba.part_ml, ga.err, s);
    if (st != LSA_OK) return st;
    note_launch();
    attn_gather_kernel<D, NT><<<(unsigned)((ga.pairs + kGatWarps - 1) / kGatWarps), kGatWarps * 32, smem_gat, s>>>(ga);
    return cuda_status(cudaGetLastError());
}

template <int D>
int launch_band_d(int G, const BandArgs& ba, const GatherArgs& ga, int64_t batch, cudaStream_t s) {
    switch (G) {
        case 1: return launch_band_g<D, 1>(ba, ga, batch, s);
        case 2: return launch_band_g<D, 2>(ba, ga, batch, s);
        case 4: return launch_band_g<D, 4>(ba, ga, batch, s);
        case 8: return launch_band_g<D, 8>(ba, ga, batch, s);
        case 16: return launch_band_g<D, 16>(ba, ga, batch, s);
        default: return LSA_ERR_INVALID_ARG;
    }
}

}  // namespace

int launch_banded_attn(const void* Q, const void* K, const void* V, const int32_t* idx, const int32_t* cnt,
                       int64_t batch, int64_t nq, int64_t q_pos0, int hq, int hkv, int d, int max_sel,
                       int64_t ld_tokens, int sink, int window, void* O, float* lse, int32_t* err, cudaStream_t s) {
    if (nq <= 0 || batch <= 0) return LSA_OK;
    // the band runs on TMA + tcgen05 (TMA coordinates are int32); otherwise
    // the per-row kernels attend every row whole, with the same result
    if (!tma_available() || batch * nq >= INT32_MAX || batch * ld_tokens >= INT32_MAX)
        return launch_sparse_attn(Q, K, V, idx, cnt, batch, nq, hq, hkv, d, LSA_BF16, max_sel, ld_tokens, O, lse,
                                  err, s);
    const int G = hq / hkv;
    const int64_t rows = batch * nq * hq;
    Arena scratch;
    scratch.async = true;
    scratch.stream = s;
    float* part_o = scratch.alloc<float>(rows * d);
    float2* part_ml = scratch.alloc<float2>(rows);
    if (scratch.status != LSA_OK) return scratch.status;
    BandArgs ba{(const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, nq, q_pos0, ld_tokens,
                hq, hkv, sink, window, 1.4426950408889634f / sqrtf((float)d), part_o, part_ml};
    const int64_t pairs = batch * nq * hkv;
    GatherArgs ga{(const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, idx, cnt, nq, q_pos0,
                  ld_tokens, hq, hkv, max_sel, sink, window, ba.scale_log2, part_o, part_ml,
                  (__nv_bfloat16*)O, lse, err, nullptr, pairs};
    if (pairs >= kGatOrderMinPairs) {
        // gather order: row lists sorted by their first long-range token
        uint32_t* k0 = scratch.alloc<uint32_t>(pairs);
        uint32_t* k1 = scratch.alloc<uint32_t>(pairs);
        int32_t* v0 = scratch.alloc<int32_t>(pairs);
        int32_t* v1 = scratch.alloc<int32_t>(pairs);
        int32_t* rs = scratch.alloc<int32_t>(radix_scratch_elems(pairs));
        if (scratch.status != LSA_OK) return scratch.status;
        note_launch();
        gather_key_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, s>>>(idx, cnt, nq, hkv, max_sel, q_pos0, sink,
                                                                         pairs, ld_tokens, k0, v0);
        uint32_t* ko;
        int32_t* vo;
        radix_sort(k0, v0, k1, v1, pairs, 32, rs, s, &ko, &vo);
        ga.order = vo;
    }
    int st = LSA_ERR_INVALID_ARG;
    if (d == 128) st = launch_band_d<128>(G, ba, ga, batch, s);
    else if (d == 64) st = launch_band_d<64>(G, ba, ga, batch, s);
    scratch.release();
    return st;
}

}  // namespace lsa
