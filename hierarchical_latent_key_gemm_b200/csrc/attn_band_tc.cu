// Dense sink/window band of the selection on the 5th-generation tensor cores.
//
// Same job as the mma.sync band kernel: for 128 (query, head) rows of one KV
// head (128/G consecutive queries x their G heads) attend over the contiguous
// key band [0, S) and [i0-W+1, i1] with the per-row mask
// j <= i && (j < S || j >= i-W+1), and write the unnormalised partial
// (acc, running max, sum of weights) that the long-range gather kernel
// continues from (LSA explainer, "How does LSA work?" step 3: attention
// covers the chosen distant keys, the first S tokens and the last W).
//
// One CTA per 128 rows (one UMMA M), two CTAs per SM:
//   warp 4   TMA: the Q tile once, then K and V tiles of 32 keys through a
//            3-stage ring (128-byte swizzle; K and Q K-major, V read MN-major)
//   warp 5   TMEM owner and MMA issuer (one thread): S = Q K^T into one of two
//            32-column TMEM buffers, then O += P_hi V + P_lo V into a D-column
//            TMEM accumulator (P_hi and P_lo are the two halves of one
//            128-byte row per query-head row)
//   warps 0-3  softmax, one row per thread: S row from TMEM, mask, running
//            max, P = 2^(s - m) split into two bf16 terms written to shared
//            memory; O is rescaled in TMEM only when the running max grows by
//            more than 2^8 (the stale max keeps every weight below 256)
// Every mbarrier wait is bounded; a timeout latches kErrTimeout and the CTA
// winds down (issued copies and MMAs are drained, TMEM is released).
#include "tma_util.cuh"

namespace lsa {
namespace {

constexpr int kRowsT = 128;       // (query, head) rows per CTA = UMMA M
#ifndef LSA_BAND_TC_KEYS
#define LSA_BAND_TC_KEYS 32
#endif
#ifndef LSA_BAND_TC_STAGES
#define LSA_BAND_TC_STAGES 3
#endif
constexpr int kKeysT = LSA_BAND_TC_KEYS;     // keys per tile (32: two CTAs fit an SM)
constexpr int kStagesT = LSA_BAND_TC_STAGES; // K/V tiles in flight
constexpr int kPBufs = kKeysT / 32;          // 128-byte P rows: hi and lo halves (32 keys) or buffers (64)
constexpr int kThreadsT = 192;
constexpr float kLazyLog2 = 8.f;  // rescale O when the max grows by more than this

struct BandTcArgs {
    int64_t nq, q_pos0, ld_tokens;
    int hq, hkv, sink, window;
    float scale_log2;
    float* part_o;
    float2* part_ml;
    int32_t* err;
};

// K-major operand, 128-byte swizzle: 8-row x 128-byte atoms, 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t addr) {
    return ((uint64_t)(addr >> 4) & 0x3FFFull) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
           (2ull << 61);
}
// MN-major operand, 128-byte swizzle: every K row is a 128-byte line of 64
// MN elements, 8 K rows form a 1024-byte atom (SBO: the next 8 K rows), and
// the next 64 MN elements start lbo bytes further.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t addr, uint32_t lbo) {
    return ((uint64_t)(addr >> 4) & 0x3FFFull) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
// kind::f16 with bf16 A and B, fp32 D, M = 128; b_mn: B is MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kRowsT >> 4) << 24);
}
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}" ::"r"(tmem_d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(0u));
}
__device__ __forceinline__ void umma_commit_to(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(bar))
                 : "memory");
}
__device__ __forceinline__ void tmem_load32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,"
        "%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_store32(uint32_t taddr, const float* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// 2^x by the hardware approximation (flush-to-zero; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

template <int D>
constexpr size_t band_tc_smem() {
    return (size_t)(D / 64) * kRowsT * 128 + kStagesT * (size_t)(2 * (D / 64) * kKeysT * 128) +
           kPBufs * (size_t)kRowsT * 128 + 512 + 1024;
}

template <int D, int G>
__global__ void __launch_bounds__(kThreadsT, kKeysT == 32 ? 2 : 1)
    attn_band_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                        const __grid_constant__ CUtensorMap map_v, const BandTcArgs a) {
    constexpr int QT = kRowsT / G;                // queries per CTA
    constexpr int NB = D / 64;                    // 64-column boxes of d
    constexpr int Q_BYTES = kRowsT * 128;         // one Q box: 128 rows x 64 d
    constexpr int KV_BYTES = kKeysT * 128;        // one K or V box: kKeysT keys x 64 d
    constexpr int STAGE = 2 * NB * KV_BYTES;      // K boxes then V boxes of one tile
    constexpr int P_BYTES = kRowsT * 128;         // one buffer of 128-byte P rows
    constexpr int HC = kKeysT / 8;                // 16-byte chunks of a row's hi (and of its lo) part
    constexpr uint32_t kCols = 256;               // S: 2 x kKeysT columns; O: D columns at 128
    constexpr uint32_t kIdescS = idesc_bf16(kKeysT, false);
    constexpr uint32_t kIdescO = idesc_bf16(D, true);
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                           ~uintptr_t(1023));
    unsigned char* Qs = smem;
    unsigned char* KVs = Qs + NB * Q_BYTES;
    unsigned char* Ps = KVs + kStagesT * STAGE;   // row r: hi chunks then lo chunks (chunk c in buffer c / 8)
    uint64_t* bars = reinterpret_cast<uint64_t*>(Ps + kPBufs * P_BYTES);
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 1;                  // [kStagesT]
    uint64_t* kv_empty = kv_full + kStagesT;       // [kStagesT]
    uint64_t* s_full = kv_empty + kStagesT;        // [2]
    uint64_t* s_free = s_full + 2;                 // [2]
    uint64_t* p_full = s_free + 2;
    uint64_t* p_free = p_full + 1;
    uint64_t* drain = p_free + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.y;
    const int64_t b = u / a.hkv;
    const int h = u % a.hkv;
    const int64_t q0 = (int64_t)blockIdx.x * QT;
    const int64_t qlast = min(a.nq, q0 + QT) - 1;
    const int64_t i0 = a.q_pos0 + q0, i1 = a.q_pos0 + qlast;
    const int64_t s_end = min((int64_t)a.sink, i1 + 1);
    const int64_t w_beg = max((int64_t)a.sink, i0 - a.window + 1);
    const int64_t w_end = i1 + 1;
    const int nt_s = (int)((s_end + kKeysT - 1) / kKeysT);
    const int nt_w = w_end > w_beg ? (int)((w_end - w_beg + kKeysT - 1) / kKeysT) : 0;
    const int ntile = nt_s + nt_w;
    auto tile_start = [&](int t) -> int64_t { return t < nt_s ? (int64_t)t * kKeysT : w_beg + (int64_t)(t - nt_s) * kKeysT; };

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kStagesT; ++s) {
            mbar_init(kv_full + s, 1);
            mbar_init(kv_empty + s, 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(s_full + s, 1);
            mbar_init(s_free + s, 128);
        }
        mbar_init(p_full, 128);
        mbar_init(p_free, 1);
        mbar_init(drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                     "r"(kCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_o = tmem + 128;

    if (warp == 4) {
        if (lane == 0) {
            bool ok = true;
            int issued = 0;
            mbar_expect_tx(q_full, NB * Q_BYTES);
            for (int nb = 0; nb < NB; ++nb)
                tma_load_3d(Qs + nb * Q_BYTES, &map_q, q_full, nb * 64, h * G, (int)(b * a.nq + q0));
            for (int t = 0; t < ntile; ++t) {
                const int s = t % kStagesT;
                if (!mbar_wait(kv_empty + s, ((uint32_t)(t / kStagesT) & 1u) ^ 1u)) { ok = false; break; }
                mbar_expect_tx(kv_full + s, STAGE);
                const int z = (int)(b * a.ld_tokens + tile_start(t));
                unsigned char* st = KVs + s * STAGE;
                for (int nb = 0; nb < NB; ++nb) tma_load_3d(st + nb * KV_BYTES, &map_k, kv_full + s, nb * 64, h, z);
                for (int nb = 0; nb < NB; ++nb)
                    tma_load_3d(st + (NB + nb) * KV_BYTES, &map_v, kv_full + s, nb * 64, h, z);
                ++issued;
            }
            if (!ok) {
                latch(a.err, kErrTimeout);
                // let the copies already issued land before the CTA exits
                for (int k = issued - 1; k >= 0 && k >= issued - kStagesT; --k)
                    mbar_wait(kv_full + k % kStagesT, (uint32_t)(k / kStagesT) & 1u);
                mbar_wait(q_full, 0);
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            bool ok = mbar_wait(q_full, 0);
            tc_fence_after();
            for (int t = 0; ok && t <= ntile; ++t) {
                if (t < ntile) {
                    const int s = t % kStagesT, sb = t & 1;
                    if (!mbar_wait(kv_full + s, (uint32_t)(t / kStagesT) & 1u)) { ok = false; break; }
                    if (t >= 2 && !mbar_wait(s_free + sb, ((uint32_t)(t - 2) >> 1) & 1u)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t kb = su32(KVs + s * STAGE);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t da = desc_kmajor(su32(Qs) + (kk / 4) * Q_BYTES + (kk % 4) * 32);
                        const uint64_t db = desc_kmajor(kb + (kk / 4) * KV_BYTES + (kk % 4) * 32);
                        umma_bf16(tmem + sb * kKeysT, da, db, kIdescS, kk > 0 ? 1u : 0u);
                    }
                    umma_commit_to(s_full + sb);
                }
                if (t >= 1) {
                    const int tp = t - 1, sp = tp % kStagesT;
                    if (!mbar_wait(p_full, (uint32_t)tp & 1u)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t vb = su32(KVs + sp * STAGE + NB * KV_BYTES);
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
#pragma unroll
                        for (int kk = 0; kk < kKeysT / 16; ++kk) {
                            // chunk 2 kk of the hi part, or of the lo part (chunks HC ..), of every row
                            const int ch = part * HC + 2 * kk;
                            const uint64_t da = desc_kmajor(su32(Ps) + (ch / 8) * P_BYTES + (ch % 8) * 16);
                            const uint64_t db = desc_mnmajor(vb + kk * 16 * 128, KV_BYTES);
                            umma_bf16(tmem_o, da, db, kIdescO, (tp > 0 || part > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    umma_commit_to(p_free);
                    umma_commit_to(kv_empty + sp);
                }
            }
            if (!ok) latch(a.err, kErrTimeout);
            umma_commit_to(drain);
            mbar_wait(drain, 0);
        }
    } else {
        // softmax: thread r owns row r = TMEM lane r
        const int r = threadIdx.x;
        const int64_t q = q0 + r / G;
        const bool row_ok = q <= qlast;
        const int64_t i = a.q_pos0 + q;
        const uint32_t lrow = (uint32_t)(32 * warp) << 16;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int t = 0; t < ntile; ++t) {
            const int s = t & 1;
            if (!mbar_wait(s_full + s, ((uint32_t)t >> 1) & 1u)) { ok = false; break; }
            tc_fence_after();
            float x[kKeysT];
#pragma unroll
            for (int c = 0; c < kKeysT; c += 32) tmem_load32(tmem + lrow + s * kKeysT + c, x + c);
            tc_fence_before();
            mbar_arrive(s_free + s);
            // valid keys of this row in the tile: offsets c in [cmin, cmax] (positions fit in int32)
            const int64_t jb = tile_start(t);
            const int64_t je = min(jb + kKeysT, t < nt_s ? s_end : w_end);
            const bool sink_tile = t < nt_s;
            int cmin = 0, cmax = -1;
            if (row_ok) {
                cmax = (int)(min(je - 1, i) - jb);
                if (!sink_tile) cmin = (int)max((int64_t)0, i - a.window + 1 - jb);
            }
            const bool full = cmin == 0 && cmax == kKeysT - 1;
            // raw scores: the scale is positive, so it is applied inside the exponent
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < kKeysT; ++c) {
                if (!full) x[c] = (c >= cmin && c <= cmax) ? x[c] : -INFINITY;
                mx = fmaxf(mx, x[c]);
            }
            mx *= a.scale_log2;
            // new reference max (lazy: kept unless the max grows by more than 2^8)
            const float m_new = fmaxf(m_ref, mx);
            float alpha = 1.f;
            if (m_ref == -INFINITY) {
                m_ref = m_new;                       // O row is still zero
            } else if (m_new > m_ref + kLazyLog2) {
                alpha = exp2f(m_ref - m_new);
                m_ref = m_new;
            }
            // P = 2^(s scale - m_ref) as hi + lo bf16 pairs (computed while the
            // previous P V runs); masked keys are -inf and give 0, so does a row
            // with no valid key yet (its reference is taken as 0)
            const float nm = m_ref == -INFINITY ? 0.f : -m_ref;
            float ls = 0.f;
            uint32_t hw[kKeysT / 2], lw[kKeysT / 2];
#pragma unroll
            for (int c = 0; c < kKeysT; c += 2) {
                const float p0 = ex2_approx(__fmaf_rn(x[c], a.scale_log2, nm));
                const float p1 = ex2_approx(__fmaf_rn(x[c + 1], a.scale_log2, nm));
                ls += p0 + p1;
                const __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
                const float2 hf = __bfloat1622float2(hb);
                const __nv_bfloat162 lb = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
                hw[c / 2] = *reinterpret_cast<const uint32_t*>(&hb);
                lw[c / 2] = *reinterpret_cast<const uint32_t*>(&lb);
            }
            l = l * alpha + ls;
            // the previous P V has finished: O may be rescaled and P rewritten
            if (t >= 1 && !mbar_wait(p_free, (uint32_t)(t - 1) & 1u)) { ok = false; break; }
            tc_fence_after();
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    float o[32];
                    tmem_load32(tmem_o + lrow + c, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= alpha;
                    tmem_store32(tmem_o + lrow + c, o);
                }
            }
#pragma unroll
            for (int ch = 0; ch < 2 * HC; ++ch) {
                const uint32_t* w = ch < HC ? hw + 4 * ch : lw + 4 * (ch - HC);
                unsigned char* dst = Ps + (ch / 8) * P_BYTES + r * 128 + (((ch % 8) ^ (r & 7)) << 4);
                *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            mbar_arrive(p_full);
        }
        if (ok && ntile > 0 && !mbar_wait(p_free, (uint32_t)(ntile - 1) & 1u)) ok = false;
        if (!ok) {
            latch(a.err, kErrTimeout);
        } else {
            tc_fence_after();
            const int64_t grow = (b * a.nq + q) * a.hq + (int64_t)h * G + r % G;
#pragma unroll 1
            for (int c = 0; c < D; c += 32) {
                float o[32];
                if (ntile > 0) {
                    tmem_load32(tmem_o + lrow + c, o);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = 0.f;
                }
                if (row_ok) {
                    float4* dst = reinterpret_cast<float4*>(a.part_o + grow * D + c);
#pragma unroll
                    for (int e = 0; e < 8; ++e) dst[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
                }
            }
            if (row_ok) a.part_ml[grow] = make_float2(m_ref, l);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols));
}

template <int D, int G>
int launch_tc_g(const void* Q, const void* K, const void* V, int64_t batch, const BandTcArgs& ba, cudaStream_t s) {
    constexpr int QT = kRowsT / G;
    CUtensorMap mq, mk, mv;
    const int64_t dq[3] = {D, ba.hq, batch * ba.nq};
    const int64_t sq[2] = {(int64_t)D * 2, (int64_t)ba.hq * D * 2};
    const int bq[3] = {64, G, QT};
    const int64_t dk[3] = {D, ba.hkv, batch * ba.ld_tokens};
    const int64_t sk[2] = {(int64_t)D * 2, (int64_t)ba.hkv * D * 2};
    const int bk[3] = {64, 1, kKeysT};
    if (!make_tensor_map_3d(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, dq, sq, bq) ||
        !make_tensor_map_3d(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, dk, sk, bk) ||
        !make_tensor_map_3d(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, V, dk, sk, bk))
        return LSA_ERR_CUDA;
    const size_t smem = band_tc_smem<D>();
    cudaError_t e = cudaFuncSetAttribute(attn_band_tc_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return cuda_status(e);
    note_launch();
    attn_band_tc_kernel<D, G><<<dim3((unsigned)((ba.nq + QT - 1) / QT), (unsigned)(batch * ba.hkv)), kThreadsT,
                                smem, s>>>(mq, mk, mv, ba);
    return cuda_status(cudaGetLastError());
}

template <int D>
int launch_tc_d(int G, const void* Q, const void* K, const void* V, int64_t batch, const BandTcArgs& ba,
                cudaStream_t s) {
    switch (G) {
        case 1: return launch_tc_g<D, 1>(Q, K, V, batch, ba, s);
        case 2: return launch_tc_g<D, 2>(Q, K, V, batch, ba, s);
        case 4: return launch_tc_g<D, 4>(Q, K, V, batch, ba, s);
        case 8: return launch_tc_g<D, 8>(Q, K, V, batch, ba, s);
        case 16: return launch_tc_g<D, 16>(Q, K, V, batch, ba, s);
        default: return LSA_ERR_INVALID_ARG;
    }
}

}  // namespace

int launch_band_tc(const void* Q, const void* K, const void* V, int64_t batch, int64_t nq, int64_t q_pos0, int hq,
                   int hkv, int d, int64_t ld_tokens, int sink, int window, float* part_o, float2* part_ml,
                   int32_t* err, cudaStream_t s) {
    if (!tma_available()) return LSA_ERR_CUDA;
    BandTcArgs ba{nq, q_pos0, ld_tokens, hq, hkv, sink, window, 1.4426950408889634f / sqrtf((float)d),
                  part_o, part_ml, err};
    const int G = hq / hkv;
    if (d == 128) return launch_tc_d<128>(G, Q, K, V, batch, ba, s);
    if (d == 64) return launch_tc_d<64>(G, Q, K, V, batch, ba, s);
    return LSA_ERR_INVALID_ARG;
}

}  // namespace lsa
