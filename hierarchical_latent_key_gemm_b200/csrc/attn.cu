// Exact softmax attention over the selected tokens.  LSA changes only which
// keys attention reads; the attention itself is ordinary exact softmax over
// that subset (LSA explainer, "How does LSA work?" step 3; tree-search wiki
// note, flowchart, the sparse-attention node).
//
// One CTA per (query, KV head): the G query heads of the group share the
// selected row list, so every gathered K/V row is read once for all G heads.
//
// bf16 path: the G heads (zero-padded to 16) are the M side of
// mma.sync.m16n8k16 tiles; S = Q K^T over 16-key slices, online softmax in
// fp32 registers, O += P V with P reused from the S accumulators (P split
// into two bf16 terms so the weights keep about 16 significant bits).  K/V rows
// are gathered with 16-byte cp.async into an XOR-swizzled 3-stage ring of
// 64-key tiles; each of the 4 warps owns 16 keys of every tile and the warps'
// partial (max, sum, O) are merged at the end.
// fp32 path: CUDA-core dot products, one warp per key, same merge.
#include <algorithm>

#include "lsa_internal.cuh"
#include "warp_mma.cuh"

namespace lsa {
namespace {

constexpr int kAttThreads = 128;
constexpr int kTileKeys = 64;
constexpr int kStages = 3;

template <int D>
__global__ __launch_bounds__(kAttThreads) void attn_bf16_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int64_t nq, int hq, int hkv, int max_sel,
    int64_t ld_tokens, __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int32_t* err, float scale_log2,
    int nsplit, float* __restrict__ part) {
    constexpr int CH = D / 8;                       // 16-byte chunks per row
    constexpr int TILE_BYTES = kTileKeys * D * 2;   // one K (or V) tile
    extern __shared__ __align__(128) unsigned char smem[];
    unsigned char* Ks = smem;                                   // [kStages][64][D]
    unsigned char* Vs = smem + kStages * TILE_BYTES;            // [kStages][64][D]
    unsigned char* Qs = smem + 2 * kStages * TILE_BYTES;        // [16][D]
    int* toks = reinterpret_cast<int*>(Qs + 16 * D * 2);        // [kStages][64]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = hq / hkv;
    const int64_t qi = blockIdx.x;
    const int u = blockIdx.y;
    const int64_t b = u / hkv;
    const int h = u % hkv;
    const int64_t row = (b * nq + qi) * hkv + h;
    int n = cnt[row];
    if (n < 0 || n > max_sel) {
        if (tid == 0) latch(err, kErrDevice);
        n = n < 0 ? 0 : max_sel;
    }
    const int32_t* ir = idx + row * max_sel;

    // Q tile (rows >= G are zero)
    for (int e = tid; e < 16 * CH; e += kAttThreads) {
        const int r = e / CH, c = e % CH;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < G) v = *reinterpret_cast<const uint4*>(Q + ((b * nq + qi) * hq + (int64_t)h * G + r) * D + c * 8);
        *reinterpret_cast<uint4*>(Qs + swz<D>(r, c)) = v;
    }

    // split-K: CTA z of nsplit takes a contiguous run of the row list's tiles
    const int ntile_all = (n + kTileKeys - 1) / kTileKeys;
    const int per_split = (ntile_all + nsplit - 1) / nsplit;
    const int tile0 = blockIdx.z * per_split;
    const int ntile = max(0, min(ntile_all, tile0 + per_split) - tile0);
    // Each thread gathers the same 16-byte column c of RPT rows of every tile;
    // its token ids are read one tile ahead into registers, so the gathers
    // never wait on an index load.
    constexpr int RPT = kTileKeys * CH / kAttThreads;
    constexpr int ROW_STEP = kAttThreads / CH;
    const int c_col = tid % CH, r_base = tid / CH;
    auto fetch_tokens = [&](int t, int* tk) {
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const int j = (tile0 + t) * kTileKeys + r_base + ROW_STEP * k;
            tk[k] = (t < ntile && j < n) ? __ldg(ir + j) : -1;
        }
    };
    const __nv_bfloat16* kcol = K + (b * ld_tokens * hkv + h) * D + c_col * 8;
    const __nv_bfloat16* vcol = V + (b * ld_tokens * hkv + h) * D + c_col * 8;
    auto load_tile = [&](int t, const int* tk) {
        const int st = t % kStages;
        const uint32_t kb = smem_u32(Ks + st * TILE_BYTES), vb = smem_u32(Vs + st * TILE_BYTES);
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const int r = r_base + ROW_STEP * k;
            int tok = tk[k];
            if (tok >= ld_tokens || tok < -1) { latch(err, kErrDevice); tok = -1; }
            const int64_t off = tok >= 0 ? (int64_t)tok * hkv * D : 0;
            const int bytes = tok >= 0 ? 16 : 0;
            cp_async16(kb + swz<D>(r, c_col), kcol + off, bytes);
            cp_async16(vb + swz<D>(r, c_col), vcol + off, bytes);
            if (c_col == 0) toks[st * kTileKeys + r] = tok;
        }
    };

    int tk_next[RPT];
#pragma unroll
    for (int t = 0; t < kStages - 1; ++t) {
        fetch_tokens(t, tk_next);
        if (t < ntile) load_tile(t, tk_next);
        cp_async_commit();
    }
    fetch_tokens(kStages - 1, tk_next);
    __syncthreads();

    // Q fragments for every 16-wide k step
    uint32_t qa[D / 16][4];
    {
        const uint32_t qb = smem_u32(Qs);
        const int r = (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int kt = 0; kt < D / 16; ++kt) {
            const int c = 2 * kt + (lane >> 4);
            ldsm_x4(qb + swz<D>(r, c), qa[kt][0], qa[kt][1], qa[kt][2], qa[kt][3]);
        }
    }

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int t = 0; t < ntile; ++t) {
        cp_async_wait<kStages - 2>();
        __syncthreads();
        if (t + kStages - 1 < ntile) load_tile(t + kStages - 1, tk_next);
        cp_async_commit();
        fetch_tokens(t + kStages, tk_next);
        const int st = t % kStages;
        const uint32_t kb = smem_u32(Ks + st * TILE_BYTES), vb = smem_u32(Vs + st * TILE_BYTES);
        const int key0 = warp * 16;  // this warp's 16 keys within the tile
        // S = Q K^T for 16 keys (two n8 tiles)
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const int kr = key0 + (lane & 7) + 8 * (lane >> 4);
#pragma unroll
            for (int kt = 0; kt < D / 16; ++kt) {
                const int c = 2 * kt + ((lane >> 3) & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kb + swz<D>(kr, c), b0, b1, b2, b3);
                mma_bf16(s[0], qa[kt], b0, b1);
                mma_bf16(s[1], qa[kt], b2, b3);
            }
        }
        // mask and scale
        const int* tk = toks + st * kTileKeys + key0;
        float x[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int kk = 8 * j + 2 * (lane & 3) + (e & 1);
                x[j][e] = tk[kk] >= 0 ? s[j][e] * scale_log2 : -INFINITY;
            }
        }
        float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
        float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = (mn0 == -INFINITY) ? 1.f : exp2f(m0 - mn0);
        const float al1 = (mn1 == -INFINITY) ? 1.f : exp2f(m1 - mn1);
        float p[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            p[j][0] = (mn0 == -INFINITY) ? 0.f : exp2f(x[j][0] - mn0);
            p[j][1] = (mn0 == -INFINITY) ? 0.f : exp2f(x[j][1] - mn0);
            p[j][2] = (mn1 == -INFINITY) ? 0.f : exp2f(x[j][2] - mn1);
            p[j][3] = (mn1 == -INFINITY) ? 0.f : exp2f(x[j][3] - mn1);
        }
        l0 = l0 * al0 + (p[0][0] + p[0][1] + p[1][0] + p[1][1]);
        l1 = l1 * al1 + (p[0][2] + p[0][3] + p[1][2] + p[1][3]);
        m0 = mn0;
        m1 = mn1;
        // rescale O only when some running maximum moved
        if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
            for (int i = 0; i < D / 8; ++i) {
                o[i][0] *= al0; o[i][1] *= al0;
                o[i][2] *= al1; o[i][3] *= al1;
            }
        }
        // P = hi + lo, both bf16: the weights keep ~16 significant bits
        uint32_t pa[4], pl[4];
        split_pack(p[0][0], p[0][1], pa[0], pl[0]);
        split_pack(p[0][2], p[0][3], pa[1], pl[1]);
        split_pack(p[1][0], p[1][1], pa[2], pl[2]);
        split_pack(p[1][2], p[1][3], pa[3], pl[3]);
        // O += P V
        {
            const int vr = key0 + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
            for (int nt = 0; nt < D / 8; nt += 2) {
                const int c = nt + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vb + swz<D>(vr, c), b0, b1, b2, b3);
                mma_bf16(o[nt], pa, b0, b1);
                mma_bf16(o[nt + 1], pa, b2, b3);
                mma_bf16(o[nt], pl, b0, b1);
                mma_bf16(o[nt + 1], pl, b2, b3);
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // merge the 4 warps: each writes (m, l, O) for its 16 rows
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    float* Om = reinterpret_cast<float*>(smem);          // [4][16][D]
    float* Mm = Om + 4 * 16 * D;                         // [4][16]
    float* Lm = Mm + 4 * 16;                             // [4][16]
    const int r0 = lane >> 2, r1 = r0 + 8;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
        const int c = nt * 8 + 2 * (lane & 3);
        Om[(warp * 16 + r0) * D + c] = o[nt][0];
        Om[(warp * 16 + r0) * D + c + 1] = o[nt][1];
        Om[(warp * 16 + r1) * D + c] = o[nt][2];
        Om[(warp * 16 + r1) * D + c + 1] = o[nt][3];
    }
    if ((lane & 3) == 0) {
        Mm[warp * 16 + r0] = m0; Mm[warp * 16 + r1] = m1;
        Lm[warp * 16 + r0] = l0; Lm[warp * 16 + r1] = l1;
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += kAttThreads) {
        const int r = e / D, c = e % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, Mm[w * 16 + r]);
        float Ls = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float f = exp2f(Mm[w * 16 + r] - M);
                Ls += f * Lm[w * 16 + r];
                acc += f * Om[(w * 16 + r) * D + c];
            }
        }
        if (part) {
            // partial of this split: unnormalised sum, running max (log2 units), sum of weights
            float* pp = part + ((row * nsplit + blockIdx.z) * G + r) * (D + 2);
            pp[c] = acc;
            if (c == 0) { pp[D] = M; pp[D + 1] = Ls; }
            continue;
        }
        const float outv = Ls > 0.f ? acc / Ls : 0.f;
        O[((b * nq + qi) * hq + (int64_t)h * G + r) * D + c] = __float2bfloat16_rn(outv);
        if (c == 0 && lse) lse[(b * nq + qi) * hq + (int64_t)h * G + r] = Ls > 0.f ? (M + log2f(Ls)) * 0.69314718055994531f : -INFINITY;
    }
}

// Merge the nsplit partials of every (query, KV head) row list by their
// maxima: O = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s.  One CTA per
// (row list, query head), one thread per output column.
template <int D>
__global__ __launch_bounds__(D) void attn_combine_kernel(const float* __restrict__ part, int nsplit, int G, int hq,
                                                         int hkv, __nv_bfloat16* __restrict__ O,
                                                         float* __restrict__ lse) {
    __shared__ float wsp[32];
    __shared__ float Msh, Lsh;
    const int64_t row = blockIdx.x / G;  // (b * nq + qi) * hkv + h
    const int r = blockIdx.x % G;
    const int h = (int)(row % hkv);
    const int64_t bq = row / hkv;        // b * nq + qi
    const int64_t stride = (int64_t)G * (D + 2);
    const float* p0 = part + (row * nsplit * G + r) * (D + 2);
    if (threadIdx.x < 32) {
        const int sp = threadIdx.x;
        const float m = sp < nsplit ? p0[sp * stride + D] : -INFINITY;
        float M = m;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float w = (M == -INFINITY || sp >= nsplit) ? 0.f : exp2f(m - M);
        float L = sp < nsplit ? w * p0[sp * stride + D + 1] : 0.f;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        wsp[sp] = w;
        if (sp == 0) { Msh = M; Lsh = L; }
    }
    __syncthreads();
    const int c = threadIdx.x;
    float acc = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) acc += wsp[sp] * p0[sp * stride + c];
    const float Ls = Lsh;
    O[(bq * hq + (int64_t)h * G + r) * D + c] = __float2bfloat16_rn(Ls > 0.f ? acc / Ls : 0.f);
    if (c == 0 && lse) lse[bq * hq + (int64_t)h * G + r] = Ls > 0.f ? (Msh + log2f(Ls)) * 0.69314718055994531f : -INFINITY;
}

template <int D, int GMAX>
__global__ __launch_bounds__(kAttThreads) void attn_f32_kernel(
    const float* __restrict__ Q, const float* __restrict__ K, const float* __restrict__ V,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt, int64_t nq, int hq, int hkv, int max_sel,
    int64_t ld_tokens, float* __restrict__ O, float* __restrict__ lse, int32_t* err, float scale_log2) {
    constexpr int PL = D / 32;  // dims per lane: lane + 32*t
    __shared__ float Om[4][GMAX][D];
    __shared__ float Mm[4][GMAX], Lm[4][GMAX];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = hq / hkv;
    const int64_t qi = blockIdx.x;
    const int u = blockIdx.y;
    const int64_t b = u / hkv;
    const int h = u % hkv;
    const int64_t row = (b * nq + qi) * hkv + h;
    int n = cnt[row];
    if (n < 0 || n > max_sel) {
        if (tid == 0) latch(err, kErrDevice);
        n = n < 0 ? 0 : max_sel;
    }
    const int32_t* ir = idx + row * max_sel;
    float qv[GMAX][PL], acc[GMAX][PL], m[GMAX], l[GMAX];
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int t = 0; t < PL; ++t) {
            acc[g][t] = 0.f;
            qv[g][t] = g < G ? Q[((b * nq + qi) * hq + (int64_t)h * G + g) * D + lane + 32 * t] : 0.f;
        }
    }
    for (int j = warp; j < n; j += 4) {
        int tok = ir[j];
        if (tok < 0 || tok >= ld_tokens) { if (lane == 0) latch(err, kErrDevice); continue; }
        const float* kr = K + ((b * ld_tokens + tok) * hkv + h) * D;
        const float* vr = V + ((b * ld_tokens + tok) * hkv + h) * D;
        float kv[PL], vv[PL];
#pragma unroll
        for (int t = 0; t < PL; ++t) { kv[t] = kr[lane + 32 * t]; vv[t] = vr[lane + 32 * t]; }
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
            if (g >= G) break;
            float s = 0.f;
#pragma unroll
            for (int t = 0; t < PL; ++t) s = fmaf(qv[g][t], kv[t], s);
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            const float x = s * scale_log2;
            const float mn = fmaxf(m[g], x);
            const float al = exp2f(m[g] - mn);
            const float pp = exp2f(x - mn);
            l[g] = l[g] * al + pp;
#pragma unroll
            for (int t = 0; t < PL; ++t) acc[g][t] = acc[g][t] * al + pp * vv[t];
            m[g] = mn;
        }
    }
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
#pragma unroll
        for (int t = 0; t < PL; ++t) Om[warp][g][lane + 32 * t] = acc[g][t];
        if (lane == 0) { Mm[warp][g] = m[g]; Lm[warp][g] = l[g]; }
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += kAttThreads) {
        const int g = e / D, c = e % D;
        float M = -INFINITY;
        for (int w = 0; w < 4; ++w) M = fmaxf(M, Mm[w][g]);
        float Ls = 0.f, a = 0.f;
        if (M != -INFINITY) {
            for (int w = 0; w < 4; ++w) {
                const float f = exp2f(Mm[w][g] - M);
                Ls += f * Lm[w][g];
                a += f * Om[w][g][c];
            }
        }
        O[((b * nq + qi) * hq + (int64_t)h * G + g) * D + c] = Ls > 0.f ? a / Ls : 0.f;
        if (c == 0 && lse) lse[(b * nq + qi) * hq + (int64_t)h * G + g] = Ls > 0.f ? (M + log2f(Ls)) * 0.69314718055994531f : -INFINITY;
    }
}

template <int D>
int launch_bf16(const void* Q, const void* K, const void* V, const int32_t* idx, const int32_t* cnt, int64_t batch,
                int64_t nq, int hq, int hkv, int max_sel, int64_t ld_tokens, void* O, float* lse, int32_t* err,
                cudaStream_t s) {
    const size_t pipe = (size_t)2 * kStages * kTileKeys * D * 2 + 16 * D * 2 + kStages * kTileKeys * 4;
    const size_t merge = (size_t)(4 * 16 * D + 8 * 16) * 4;
    const size_t smem = pipe > merge ? pipe : merge;
    cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_status(e);
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    // few row lists (decode): split each across CTAs, then merge
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t rows_n = batch * nq * hkv;
    int nsplit = 1;
    if (rows_n < 2 * (int64_t)sms) {
        const int64_t want = (4 * (int64_t)sms + rows_n - 1) / rows_n;
        const int64_t tiles = ((int64_t)max_sel + kTileKeys - 1) / kTileKeys;
        nsplit = (int)std::max<int64_t>(1, std::min<int64_t>({32, want, (tiles + 1) / 2}));
    }
    Arena scratch;
    scratch.async = true;
    scratch.stream = s;
    float* part = nullptr;
    if (nsplit > 1) {
        part = scratch.alloc<float>(rows_n * nsplit * (hq / hkv) * (D + 2));
        if (scratch.status != LSA_OK) return scratch.status;
    }
    dim3 grid((unsigned)nq, (unsigned)(batch * hkv), (unsigned)nsplit);
    note_launch();
    attn_bf16_kernel<D><<<grid, kAttThreads, smem, s>>>(
        (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, idx, cnt, nq, hq, hkv, max_sel,
        ld_tokens, (__nv_bfloat16*)O, lse, err, scale_log2, nsplit, part);
    if (nsplit > 1) {
        note_launch();
        attn_combine_kernel<D><<<(unsigned)(rows_n * (hq / hkv)), D, 0, s>>>(part, nsplit, hq / hkv, hq, hkv,
                                                                             (__nv_bfloat16*)O, lse);
    }
    const int st = cuda_status(cudaGetLastError());
    scratch.release();
    return st;
}

template <int D>
int launch_f32(const void* Q, const void* K, const void* V, const int32_t* idx, const int32_t* cnt, int64_t batch,
               int64_t nq, int hq, int hkv, int max_sel, int64_t ld_tokens, void* O, float* lse, int32_t* err,
               cudaStream_t s) {
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    dim3 grid((unsigned)nq, (unsigned)(batch * hkv));
    note_launch();
    attn_f32_kernel<D, 4><<<grid, kAttThreads, 0, s>>>((const float*)Q, (const float*)K, (const float*)V, idx, cnt,
                                                      nq, hq, hkv, max_sel, ld_tokens, (float*)O, lse, err,
                                                      scale_log2);
    return cuda_status(cudaGetLastError());
}

}  // namespace

int launch_sparse_attn(const void* Q, const void* K, const void* V, const int32_t* idx, const int32_t* cnt,
                       int64_t batch, int64_t nq, int hq, int hkv, int d, int dtype, int max_sel, int64_t ld_tokens,
                       void* O, float* lse, int32_t* err, cudaStream_t s) {
    if (nq <= 0 || batch <= 0) return LSA_OK;
    const int G = hq / hkv;
    if (dtype == LSA_BF16) {
        if (G > 16) return LSA_ERR_INVALID_ARG;
        if (d == 128) return launch_bf16<128>(Q, K, V, idx, cnt, batch, nq, hq, hkv, max_sel, ld_tokens, O, lse, err, s);
        if (d == 64) return launch_bf16<64>(Q, K, V, idx, cnt, batch, nq, hq, hkv, max_sel, ld_tokens, O, lse, err, s);
        return LSA_ERR_INVALID_ARG;
    }
    if (G > 4) return LSA_ERR_INVALID_ARG;
    if (d == 128) return launch_f32<128>(Q, K, V, idx, cnt, batch, nq, hq, hkv, max_sel, ld_tokens, O, lse, err, s);
    if (d == 64) return launch_f32<64>(Q, K, V, idx, cnt, batch, nq, hq, hkv, max_sel, ld_tokens, O, lse, err, s);
    return LSA_ERR_INVALID_ARG;
}

}  // namespace lsa
