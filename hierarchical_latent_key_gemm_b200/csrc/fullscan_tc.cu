// The full-scan indexer (the previous indexer: every candidate block is
// scored; tree-search wiki note, flowchart, red path) as a tensor-core GEMM
// that filters, followed by an exact top-K over the survivors.
//
// For a tile of 128 queries of one KV head (rows) and every candidate block
// (columns, 256 per tile), tcgen05 forms approximate scores q.k from the
// fp16 roundings of both sides (one power of two scaling both, exact; K = r
// padded to 64): |approximate - exact| stays below eps = 2^-9 |q| max|k|
// (fp16 keeps 11 significant bits: about 2^-10 from the two roundings, the
// fp32 accumulations far below).  Only whether a block can be in the top K
// is decided here, so no split is needed.  Two sweeps over the blocks:
//   pass 0  each row's histogram of approximate scores over 128 equal bins of
//           [-R, R], R = |q| max|k| (Cauchy-Schwarz bound); from it the lower
//           edge L of the bin that holds the ceil(K/P)-th largest, and the
//           threshold T = L - 2 eps (eps bounds |approximate - exact|)
//   pass 1  every eligible block whose approximate score is >= T is
//           appended to the row's candidate list (two lists, one per
//           column half, no atomics)
// Why T is safe: at least ceil(K/P) blocks have an approximate score >= L,
// so their exact scores are >= L - eps and the exact ceil(K/P)-th largest
// score s* >= L - eps; any block with an exact score >= s* then has an
// approximate score >= s* - eps >= L - 2 eps = T.  So the lists hold every
// block of the exact top ceil(K/P), ties at s* included, and the per-query
// kernel of select.cu ranks the lists with its exact arithmetic: the result
// is bit-identical to scoring every block there.  A list that would overflow
// sends its query back to the per-query full scan.
#include <cuda_fp16.h>

#include <algorithm>
#include <new>

#include "tc_common.cuh"

namespace lsa {
namespace {

constexpr int kFM = kTcM;           // queries per CTA
constexpr int kFN = kTcN;           // blocks per tile
constexpr int kFKC = 64;            // fp16 per K chunk (one 128-byte swizzle row)
constexpr int kFStages = 4;         // key tiles in flight (one K chunk each)
constexpr int kFThreads = 320;      // producer, MMA issuer, 8 epilogue warps
constexpr int kBins = 128;
constexpr int kBinLd = kBins + 1;   // padded histogram row
constexpr int kHalfCap = 2048;      // candidates per (query, column half)
constexpr float kEpsRel = 1.f / 512.f;     // eps = 2^-9 R: twice the roundings' and accumulations' bound
constexpr float kEpsAbs = 1.f / 128.f;     // + 2^-7 (scaled units): the subnormal range's share, doubled

__host__ __device__ constexpr int fs_k(int r) { return (r + kFKC - 1) / kFKC * kFKC; }

struct FsArgs {
    int64_t nq, nq_pad;       // queries of the chunk; rows per unit of the split queries
    int64_t nb, nb_pad;       // indexed blocks per unit; rows per unit of the split keys
    int64_t b_lo;             // first candidate block (sink rule)
    int hkv, pool, window, kb;
    const int64_t* q_pos;     // [batch][nq] positions of the chunk's queries, or null
    int64_t q_pos0;           // position of the chunk's first query
    int64_t q_stride;         // q_pos row stride (queries per sequence in the call)
    const float* qnorm;       // [units][nq_pad] |q'| (scaled)
    const float* kmax;        // [units] max |k'| (scaled)
    float* thr;               // [units][nq_pad] threshold (scaled units)
    int32_t* cand;            // [units][nq_pad][2][kHalfCap] block ids
    int32_t* ccount;          // [units][nq_pad][2]
    int32_t* err;
    // split of each tile's block range over gridDim.z CTAs (small calls):
    // pass 0 adds its counts into ghist [units][nq_pad][kBins] and the
    // thresholds come from fs_thr_kernel; pass 1 appends through atomics on
    // ccount (zeroed before)
    int nsplit;
    int32_t* ghist;
};

__device__ __forceinline__ int64_t fs_bhi(const FsArgs& a, int u, int64_t qi) {
    const int64_t b = u / a.hkv;
    const int64_t pos = a.q_pos ? a.q_pos[b * a.q_stride + qi] : a.q_pos0 + qi;
    const int64_t bound = pos - a.window - a.pool + 1;
    const int64_t bh = bound >= 0 ? bound / a.pool : -1;
    return bh < a.nb - 1 ? bh : a.nb - 1;
}

// Largest |value| of the latent queries and latent keys, as float bits.
__global__ void fs_absmax_kernel(const float* __restrict__ q, int64_t nqv, const float* __restrict__ Kl,
                                 int64_t units, int64_t nb, int64_t nb_cap, int r, uint32_t* __restrict__ out) {
    uint32_t m = 0;
    const int64_t tk = units * nb * r;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < nqv + tk;
         e += (int64_t)gridDim.x * blockDim.x) {
        float v;
        if (e < nqv) {
            v = q[e];
        } else {
            const int64_t f = e - nqv, c = f % r, row = f / r;
            v = Kl[((row / nb) * nb_cap + row % nb) * r + c];
        }
        m = max(m, __float_as_uint(fabsf(v)));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(out, m);
}

// Scaled values below 2^10 (the products then stay far inside fp32).
__device__ __forceinline__ int fs_scale_exp(const uint32_t* absmax) {
    const float m = __uint_as_float(*absmax);
    if (!(m > 0.f) || isinf(m)) return 0;
    return max(-60, min(60, ilogbf(m) - 9));
}

// One warp per row: the scaled row rounded to fp16 (zero-padded to K), and
// the row's scaled norm (fp64 sum, rounded up).
__global__ void fs_split_kernel(const float* __restrict__ src, int64_t units, int64_t n, int64_t n_pad, int r,
                                int64_t row_stride, int64_t unit_stride_b, int64_t unit_stride_h, int hkv,
                                const uint32_t* __restrict__ absmax, __half* __restrict__ dst,
                                float* __restrict__ norm) {
    const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= units * n_pad) return;
    const int64_t u = row / n_pad, i = row % n_pad;
    const int kp = fs_k(r);
    const int sc = -fs_scale_exp(absmax);
    const float* s = src + (u / hkv) * unit_stride_b + (u % hkv) * unit_stride_h + i * row_stride;
    __half* o = dst + row * kp;
    double nn = 0.0;
    for (int c = lane; c < kp; c += 32) {
        const float x = (i < n && c < r) ? ldexpf(s[c], sc) : 0.f;
        nn = fma((double)x, (double)x, nn);
        o[c] = __float2half_rn(x);
    }
#pragma unroll
    for (int of = 16; of >= 1; of >>= 1) nn += __shfl_xor_sync(0xffffffffu, nn, of);
    if (lane == 0) norm[row] = (float)sqrt(nn) * (1.f + 1e-6f);   // (rounded up: a bound)
}

__global__ void fs_kmax_kernel(const float* __restrict__ knorm, int64_t n, int64_t n_pad, float* __restrict__ kmax) {
    const int u = blockIdx.x;
    float m = 0.f;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, knorm[u * n_pad + i]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float w[32];
    if ((threadIdx.x & 31) == 0) w[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int k = 1; k < (int)(blockDim.x >> 5); ++k) m = fmaxf(m, w[k]);
        kmax[u] = fmaxf(m, w[0]);
    }
}

// Thresholds of a split pass 0: the same rule as in the kernel, on the summed
// histogram of every row.
__global__ void fs_thr_kernel(const int32_t* __restrict__ ghist, const float* __restrict__ qnorm,
                              const float* __restrict__ kmax, int64_t nq, int64_t nq_pad, int64_t units, int kb,
                              float* __restrict__ thr) {
    const int64_t gr = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gr >= units * nq_pad) return;
    const int64_t u = gr / nq_pad, qi = gr % nq_pad;
    if (qi >= nq) return;
    const float Rr = qnorm[gr] * kmax[u];
    const int32_t* h = ghist + gr * kBins;
    float t = -INFINITY;
    int cum = 0;
    for (int bin = kBins - 1; bin >= 0; --bin) {
        cum += h[bin];
        if (cum >= kb) {
            const float L = -Rr + (float)bin * (2.f * Rr / (float)kBins);
            t = L - 2.f * (kEpsRel * Rr + kEpsAbs);
            break;
        }
    }
    thr[gr] = t;
}

template <int R, int PASS>
__global__ void __launch_bounds__(kFThreads, 1)
    fs_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                 const FsArgs a) {
    constexpr int KS = fs_k(R) / kFKC;
    constexpr int A_CHUNK = kFM * 128;
    constexpr int B_CHUNK = kFN * 128;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                           ~uintptr_t(1023));
    unsigned char* As = smem;
    unsigned char* Bs = As + KS * A_CHUNK;
    int* hist = reinterpret_cast<int*>(Bs + kFStages * B_CHUNK);            // [kFM][kBinLd] (pass 0)
    uint64_t* bars = reinterpret_cast<uint64_t*>(hist + (PASS == 0 ? kFM * kBinLd : 0));
    uint64_t* a_full = bars;
    uint64_t* b_full = bars + 1;
    uint64_t* b_empty = b_full + kFStages;
    uint64_t* acc_full = b_empty + kFStages;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
    int* sh_tiles = reinterpret_cast<int*>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.y;
    const int64_t q0 = (int64_t)blockIdx.x * kFM;

    // the tile's block range: [b_lo, max row bound]
    if (threadIdx.x == 0) *sh_tiles = 0;
    if (PASS == 0)
        for (int e = threadIdx.x; e < kFM * kBinLd; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    if (threadIdx.x < kFM && q0 + threadIdx.x < a.nq) {
        const int64_t bh = fs_bhi(a, u, q0 + threadIdx.x);
        const int64_t nt = bh >= a.b_lo ? (bh - a.b_lo) / kFN + 1 : 0;
        atomicMax(sh_tiles, (int)nt);
    }
    if (threadIdx.x == 0) {
        mbar_init(a_full, 1);
        for (int s = 0; s < kFStages; ++s) {
            mbar_init(b_full + s, 1);
            mbar_init(b_empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full + b, 1);
            mbar_init(acc_empty + b, 256);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(su32(tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    const uint32_t tmem = *tmem_slot;
    // this CTA's share of the tile's block range: tiles [t_beg, t_beg + ntile)
    const int ntile_all = *sh_tiles;
    const int per = (ntile_all + a.nsplit - 1) / a.nsplit;
    const int t_beg = min(ntile_all, (int)blockIdx.z * per);
    const int ntile = min(ntile_all, t_beg + per) - t_beg;

    bool ok = true;
    if (warp == 0) {
        if (lane == 0 && ntile > 0) {
            mbar_expect_tx(a_full, KS * A_CHUNK);
            for (int c = 0; c < KS; ++c)
                tma_load_2d(As + c * A_CHUNK, &map_q, a_full, c * kFKC, (int)(u * a.nq_pad + q0));
            int issued = 0;
            for (int t = 0; t < ntile && ok; ++t) {
                for (int c = 0; c < KS && ok; ++c) {
                    const int it = t * KS + c, s = it % kFStages;
                    const uint32_t ph = (uint32_t)(it / kFStages) & 1u;
                    if (!mbar_wait(b_empty + s, ph ^ 1u)) { ok = false; break; }
                    mbar_expect_tx(b_full + s, B_CHUNK);
                    tma_load_2d(Bs + s * B_CHUNK, &map_k, b_full + s, c * kFKC,
                                (int)(u * a.nb_pad + a.b_lo + (int64_t)(t_beg + t) * kFN));
                    ++issued;
                }
            }
            if (!ok) {
                latch(a.err, kErrTimeout);
                for (int it = 0; it < issued && it < kFStages; ++it) {
                    const int last = issued - 1 - it;
                    mbar_wait(b_full + last % kFStages, (uint32_t)(last / kFStages) & 1u);
                }
                mbar_wait(a_full, 0);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && ntile > 0) {
            if (!mbar_wait(a_full, 0)) ok = false;
            for (int t = 0; t < ntile && ok; ++t) {
                const int buf = t & 1;
                if (!mbar_wait(acc_empty + buf, ((uint32_t)(t >> 1) & 1u) ^ 1u)) { ok = false; break; }
                asm volatile("tcgen05.fence::after_thread_sync;");
                const uint32_t d = tmem + buf * kFN;
                for (int c = 0; c < KS; ++c) {
                    const int it = t * KS + c, s = it % kFStages;
                    if (!mbar_wait(b_full + s, (uint32_t)(it / kFStages) & 1u)) { ok = false; break; }
                    asm volatile("tcgen05.fence::after_thread_sync;");
#pragma unroll
                    for (int kk = 0; kk < kFKC / 16; ++kk) {
                        const uint64_t da = umma_desc(As + c * A_CHUNK + kk * 32);
                        const uint64_t db = umma_desc(Bs + s * B_CHUNK + kk * 32);
                        umma_f16(d, da, db, (c | kk) ? 1u : 0u);
                    }
                    umma_commit(b_empty + s);
                }
                if (!ok) break;
                umma_commit(acc_full + buf);
            }
            if (!ok) latch(a.err, kErrTimeout);
        }
    } else {
        // epilogue: row = TMEM lane; warps 2-5 columns [0, 128), 6-9 [128, 256)
        const int qd = warp & 3;
        const int half = (warp - 2) >> 2;
        const int row = 32 * qd + lane;
        const int64_t qi = q0 + row;
        const bool live = qi < a.nq;
        const int64_t bh = live ? fs_bhi(a, u, qi) : -1;
        const int64_t gr = (int64_t)u * a.nq_pad + qi;
        const float Rr = live ? a.qnorm[gr] * a.kmax[u] : 0.f;
        const float inv = Rr > 0.f ? (float)kBins / (2.f * Rr) : 0.f;
        const float T = (PASS == 1 && live) ? a.thr[gr] : INFINITY;
        int* hr = hist + row * kBinLd;
        int32_t* lst = a.cand + ((gr * 2) + half) * kHalfCap;
        int n = 0;
        for (int t = 0; t < ntile; ++t) {
            const int buf = t & 1;
            if (!mbar_wait(acc_full + buf, (uint32_t)(t >> 1) & 1u)) { ok = false; latch(a.err, kErrTimeout); break; }
            asm volatile("tcgen05.fence::after_thread_sync;");
#pragma unroll
            for (int cb = 0; cb < kFN / 64; ++cb) {
                float v[32];
                const int col = half * (kFN / 2) + cb * 32;
                tmem_ld32(tmem + ((uint32_t)(32 * qd) << 16) + buf * kFN + col, v);
                const int64_t b0 = a.b_lo + (int64_t)(t_beg + t) * kFN + col;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (b0 + i <= bh) {
                        if (PASS == 0) {
                            const int bin = min(kBins - 1, max(0, (int)((v[i] + Rr) * inv)));
                            atomicAdd(hr + bin, 1);
                        } else if (v[i] >= T) {
                            if (a.nsplit == 1) {
                                if (n < kHalfCap) lst[n] = (int32_t)(b0 + i);
                                ++n;
                            } else {
                                const int pp = atomicAdd(a.ccount + gr * 2 + half, 1);
                                if (pp < kHalfCap) lst[pp] = (int32_t)(b0 + i);
                            }
                        }
                    }
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;");
            mbar_arrive(acc_empty + buf);
        }
        if (PASS == 0 && a.nsplit > 1) {
            asm volatile("bar.sync 1, 256;" ::: "memory");   // both halves' counts are in
            if (half == 0 && live)
                for (int bin = 0; bin < kBins; ++bin)
                    if (hr[bin]) atomicAdd(a.ghist + gr * kBins + bin, hr[bin]);
        } else if (PASS == 0) {
            asm volatile("bar.sync 1, 256;" ::: "memory");   // both halves' counts are in
            if (half == 0 && live) {
                float thr = -INFINITY;
                int cum = 0;
                for (int bin = kBins - 1; bin >= 0; --bin) {
                    cum += hr[bin];
                    if (cum >= a.kb) {
                        const float L = -Rr + (float)bin * (2.f * Rr / (float)kBins);
                        // (plus an absolute term for values that fp16 keeps
                        // only as subnormals: at most 2^-8 in scaled units)
                        thr = L - 2.f * (kEpsRel * Rr + kEpsAbs);
                        break;
                    }
                }
                a.thr[gr] = thr;
            }
        } else if (live && a.nsplit == 1) {
            a.ccount[gr * 2 + half] = n;
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}

template <int R, int PASS>
size_t fs_smem_bytes() {
    return (size_t)(fs_k(R) / kFKC) * kFM * 128 + (size_t)kFStages * kFN * 128 +
           (PASS == 0 ? (size_t)kFM * kBinLd * 4 : 0) + 256 + 1024;
}

template <int R>
int fs_run_passes(const CUtensorMap& mq, const CUtensorMap& mk, const FsArgs& a, int64_t units, cudaStream_t s) {
    dim3 grid((unsigned)(a.nq_pad / kFM), (unsigned)units, (unsigned)a.nsplit);
    const size_t s0 = fs_smem_bytes<R, 0>(), s1 = fs_smem_bytes<R, 1>();
    cudaError_t e = cudaFuncSetAttribute(fs_tc_kernel<R, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s0);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fs_tc_kernel<R, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
    if (e != cudaSuccess) return cuda_status(e);
    const int64_t rows = units * a.nq_pad;
    if (a.nsplit > 1) {
        e = cudaMemsetAsync(a.ghist, 0, (size_t)rows * kBins * sizeof(int32_t), s);
        if (e != cudaSuccess) return cuda_status(e);
    }
    note_launch();
    fs_tc_kernel<R, 0><<<grid, kFThreads, s0, s>>>(mq, mk, a);
    if (a.nsplit > 1) {
        note_launch();
        fs_thr_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(a.ghist, a.qnorm, a.kmax, a.nq, a.nq_pad, units,
                                                                      a.kb, a.thr);
        e = cudaMemsetAsync(a.ccount, 0, (size_t)rows * 2 * sizeof(int32_t), s);
        if (e != cudaSuccess) return cuda_status(e);
    }
    note_launch();
    fs_tc_kernel<R, 1><<<grid, kFThreads, s1, s>>>(mq, mk, a);
    return cuda_status(cudaGetLastError());
}

// first candidate block (the sink rule)
int64_t a_b_lo(const lsa_build_params& p) { return (p.sink + p.pool - 1) / p.pool; }

}  // namespace

bool fullscan_tc_applies(const lsa_index* ix, const lsa_select_params* sp) {
    const int r = ix->p.r;
    const int kb = (sp->topk + ix->p.pool - 1) / ix->p.pool;
    return (r == 16 || r == 32 || r == 64) && kb >= 1 && tma_available() && ix->nb > 0;
}

int launch_fullscan_tc(const lsa_index* ix, const lsa_select_params* sp, const float* qbar, int64_t nq,
                       const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int max_sel,
                       cudaStream_t s, Arena& A) {
    const lsa_build_params& p = ix->p;
    const int r = p.r, hkv = p.hkv;
    const int64_t U = ix->units, nb = ix->nb;
    const int kp = fs_k(r);
    const int kb = (sp->topk + p.pool - 1) / p.pool;
    const int64_t nb_pad = (nb + kFN - 1) / kFN * kFN + kFN;
    // queries per chunk: candidate lists of about 2 GiB
    int64_t cq = std::max<int64_t>(kFM, ((int64_t)2 << 30) / ((int64_t)2 * kHalfCap * 4 * U) / kFM * kFM);
    const int64_t nq_chunk_max = std::min<int64_t>(cq, (nq + kFM - 1) / kFM * kFM);
    uint32_t* absmax = A.alloc<uint32_t>(1);
    __half* Kk = A.alloc<__half>(U * nb_pad * kp);
    float* knorm = A.alloc<float>(U * nb_pad);
    float* kmax = A.alloc<float>(U);
    __half* Aq = A.alloc<__half>(U * nq_chunk_max * kp);
    float* qnorm = A.alloc<float>(U * nq_chunk_max);
    float* thr = A.alloc<float>(U * nq_chunk_max);
    int32_t* cand = A.alloc<int32_t>(U * nq_chunk_max * 2 * kHalfCap);
    int32_t* ccount = A.alloc<int32_t>(U * nq_chunk_max * 2);
    // small calls split each tile's block range so that about two CTAs run per SM
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t tiles_q = nq_chunk_max / kFM * U;
    const int64_t tiles_k = (nb - a_b_lo(p) + kFN - 1) / kFN;
    int64_t nsplit = (2 * (int64_t)sms + tiles_q - 1) / tiles_q;
    nsplit = std::max<int64_t>(1, std::min<int64_t>(nsplit, tiles_k / 8));
    int32_t* ghist = nsplit > 1 ? A.alloc<int32_t>(U * nq_chunk_max * kBins) : nullptr;
    if (A.status != LSA_OK) return A.status;
    cudaError_t e = cudaMemsetAsync(absmax, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return cuda_status(e);
    note_launch();
    fs_absmax_kernel<<<592, 256, 0, s>>>(qbar, p.batch * nq * hkv * (int64_t)r, ix->Kl, U, nb, ix->nb_cap, r, absmax);
    // keys: unit u = (sequence, head) rows of Kl [units][nb_cap][r]
    note_launch();
    fs_split_kernel<<<(unsigned)((U * nb_pad * 32 + 255) / 256), 256, 0, s>>>(
        ix->Kl, U, nb, nb_pad, r, r, (int64_t)hkv * ix->nb_cap * r, ix->nb_cap * r, hkv, absmax, Kk, knorm);
    note_launch();
    fs_kmax_kernel<<<(unsigned)U, 256, 0, s>>>(knorm, nb, nb_pad, kmax);
    CUtensorMap mk;
    if (!make_tensor_map_2d(&mk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Kk, U * nb_pad, kp, kp * 2, kFKC, kFN))
        return LSA_ERR_CUDA;
    FsArgs a{};
    a.nb = nb;
    a.nb_pad = nb_pad;
    a.b_lo = a_b_lo(p);
    a.hkv = hkv;
    a.pool = p.pool;
    a.window = sp->window;
    a.kb = kb;
    a.q_stride = nq;
    a.qnorm = qnorm;
    a.kmax = kmax;
    a.thr = thr;
    a.cand = cand;
    a.ccount = ccount;
    a.err = ix->err;
    a.nsplit = (int)nsplit;
    a.ghist = ghist;
    for (int64_t q0 = 0; q0 < nq; q0 += nq_chunk_max) {
        const int64_t nqc = std::min(nq_chunk_max, nq - q0);
        const int64_t nqc_pad = (nqc + kFM - 1) / kFM * kFM;
        // the chunk's latent queries: q̄ [batch][nq][hkv][r], unit u = (b, h)
        note_launch();
        fs_split_kernel<<<(unsigned)((U * nqc_pad * 32 + 255) / 256), 256, 0, s>>>(
            qbar + q0 * hkv * (int64_t)r, U, nqc, nqc_pad, r, (int64_t)hkv * r, nq * hkv * (int64_t)r, r, hkv,
            absmax, Aq, qnorm);
        CUtensorMap mq;
        if (!make_tensor_map_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Aq, U * nqc_pad, kp, kp * 2, kFKC, kFM))
            return LSA_ERR_CUDA;
        a.nq = nqc;
        a.nq_pad = nqc_pad;
        a.q_pos = q_pos ? q_pos + q0 : nullptr;
        a.q_pos0 = q_pos0 + q0;
        int st;
        switch (r) {
            case 16: st = fs_run_passes<16>(mq, mk, a, U, s); break;
            case 32: st = fs_run_passes<32>(mq, mk, a, U, s); break;
            default: st = fs_run_passes<64>(mq, mk, a, U, s); break;
        }
        if (st != LSA_OK) return st;
        // exact ranking of the lists (select.cu), per query of the chunk
        ListIn li{cand, ccount, nqc_pad, kHalfCap};
        st = launch_select_lists(ix, sp, qbar + q0 * hkv * (int64_t)r, nq, nqc, q_pos ? q_pos + q0 : nullptr,
                                 q_pos0 + q0, idx + q0 * hkv * (int64_t)max_sel, cnt + q0 * hkv, max_sel, li, s);
        if (st != LSA_OK) return st;
    }
    return cuda_status(cudaGetLastError());
}

}  // namespace lsa
