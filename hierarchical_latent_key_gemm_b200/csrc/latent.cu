// Latent keys and latent queries.
//
// Keys: Kl[b] = W^T * mean(K[bP .. bP+P-1]) for every complete block of P
// keys: blocks of keys are averaged, then clustered in a learned low-rank
// space (LSA explainer, section "How does LSA work?", step 1).
// Queries: qbar = mean over a KV head's query heads of W^T q (the group shares
// one selection).
//
// Both are "mean of M rows, then a d x r map": an HBM stream (16 flop per key
// byte at P = 4), so CUDA cores suffice.  The arithmetic order (rows summed in
// order, one IEEE division by M, then one fused multiply-add chain over the d
// inputs in order) is fixed in latent_common.cuh and shared with the decode
// append, so both produce identical bits.
//
// stream_project_kernel: a CTA keeps W in shared memory and walks rounds of
// ITEMS items (grid-stride, so W is read once per CTA, not once per item
// tile).  Per round: the rows are read with 16-byte loads, consecutive threads
// on consecutive pieces of a row, all M rows of a piece in flight together,
// averaged into shared memory; then each thread forms a 4-item x 4-output
// tile of the product (per input k: one 16-byte W load and four mean values
// feed 16 FMAs), so shared memory does not bound the product.
#include "latent_common.cuh"

namespace lsa {
namespace {

// ------------------------------------------------------------ streaming form
constexpr int kPThreads = 256;

template <typename T>
struct Vec16;   // 16 bytes of T, widened to fp32
template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void widen(const uint4 v, float* f) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <>
struct Vec16<float> {
    static constexpr int N = 4;
    __device__ static void widen(const uint4 v, float* f) {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
};

template <int R>
constexpr int items_per_round() { return 4096 / R; }   // (ITEMS/4) x (R/4) = 256 tiles of 4 x 4

template <typename T, int D, int R, int M_MAX>
__global__ __launch_bounds__(kPThreads, 2) void stream_project_kernel(
    const T* __restrict__ src, const float* __restrict__ W, int M, int64_t n_items, int64_t row_stride,
    int64_t item_stride, int64_t unit_b_stride, int64_t unit_h_stride, int hpb, float* __restrict__ out,
    int64_t out_item_stride, int64_t out_b_stride, int64_t out_h_stride) {
    constexpr int ITEMS = items_per_round<R>();
    constexpr int VN = Vec16<T>::N;
    constexpr int CPR = D / VN;            // 16-byte pieces per row
    constexpr int LD = D + 4;              // padded mean row: 4 items apart land in other banks
    constexpr int OG = R / 4;              // output groups of 4
    extern __shared__ float4 smem4[];
    float* Ws = reinterpret_cast<float*>(smem4);   // [D][R]
    float* Ms = Ws + D * R;                         // [ITEMS][LD]
    const int unit = blockIdx.y;
    const int b = unit / hpb, h = unit % hpb;
    for (int e = threadIdx.x; e < D * R / 4; e += kPThreads)
        reinterpret_cast<float4*>(Ws)[e] = __ldg(reinterpret_cast<const float4*>(W) + e);
    const T* base = src + (int64_t)b * unit_b_stride + (int64_t)h * unit_h_stride;
    float* obase = out + (int64_t)b * out_b_stride + (int64_t)h * out_h_stride;
    const int og = threadIdx.x % OG, ig = threadIdx.x / OG;
    const int64_t rounds = (n_items + ITEMS - 1) / ITEMS;
    for (int64_t rd = blockIdx.x; rd < rounds; rd += gridDim.x) {
        const int64_t item0 = rd * ITEMS;
        // means of the round's items: piece c of item i by one thread, the M
        // rows of the piece loaded before any of them is summed
#pragma unroll 1
        for (int task = threadIdx.x; task < ITEMS * CPR; task += kPThreads) {
            const int it = task / CPR, c = task % CPR;
            const int64_t item = item0 + it;
            float s[VN];
#pragma unroll
            for (int j = 0; j < VN; ++j) s[j] = 0.f;
            if (item < n_items) {
                const T* p = base + item * item_stride + c * VN;
                uint4 raw[M_MAX];   // the M rows' 16-byte pieces, all in flight before the sum
#pragma unroll
                for (int m = 0; m < M_MAX; ++m)
                    if (m < M) raw[m] = __ldg(reinterpret_cast<const uint4*>(p + (int64_t)m * row_stride));
#pragma unroll
                for (int m = 0; m < M_MAX; ++m)
                    if (m < M) {
                        float v[VN];
                        Vec16<T>::widen(raw[m], v);
#pragma unroll
                        for (int j = 0; j < VN; ++j) s[j] = __fadd_rn(s[j], v[j]);
                    }
#pragma unroll
                for (int j = 0; j < VN; ++j) s[j] = __fdiv_rn(s[j], (float)M);
            }
            float* dst = Ms + it * LD + c * VN;
#pragma unroll
            for (int j = 0; j < VN; j += 4)
                *reinterpret_cast<float4*>(dst + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
        }
        __syncthreads();
        // 4 items x 4 outputs per thread, one fma chain per output over k in order
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int o = 0; o < 4; ++o) acc[i][o] = 0.f;
        const float* m0 = Ms + (ig * 4) * LD;
#pragma unroll 4
        for (int k = 0; k < D; ++k) {
            const float4 wv = *reinterpret_cast<const float4*>(Ws + k * R + og * 4);
            const float w4[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float mv = m0[i * LD + k];
#pragma unroll
                for (int o = 0; o < 4; ++o) acc[i][o] = __fmaf_rn(mv, w4[o], acc[i][o]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t item = item0 + ig * 4 + i;
            if (item < n_items) {
                float* op = obase + item * out_item_stride + og * 4;
#pragma unroll
                for (int o = 0; o < 4; ++o) op[o] = acc[i][o];
            }
        }
        __syncthreads();   // Ms is rewritten by the next round
    }
}

template <typename T, int D, int R>
int launch_stream(const T* src, const float* W, int M, int64_t n_items, int64_t row_stride, int64_t item_stride,
                  int64_t ub, int64_t uh, int64_t units, int hpb, float* out, int64_t ois, int64_t obs,
                  int64_t ohs, cudaStream_t s) {
    constexpr int ITEMS = items_per_round<R>();
    const size_t smem = (size_t)(D * R + ITEMS * (D + 4)) * sizeof(float);
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    auto kern = M <= 4 ? stream_project_kernel<T, D, R, 4>
                       : (M <= 8 ? stream_project_kernel<T, D, R, 8> : stream_project_kernel<T, D, R, 16>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_status(e);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kPThreads, smem);
    if (e != cudaSuccess) return cuda_status(e);
    const int64_t rounds = (n_items + ITEMS - 1) / ITEMS;
    int64_t gx = ((int64_t)sms * (per_sm > 0 ? per_sm : 1) + units - 1) / units;
    if (gx > rounds) gx = rounds;
    if (gx < 1) gx = 1;
    dim3 grid((unsigned)gx, (unsigned)units);
    note_launch();
    kern<<<grid, kPThreads, smem, s>>>(src, W, M, n_items, row_stride, item_stride, ub, uh, hpb, out, ois, obs,
                                       ohs);
    return cuda_status(cudaGetLastError());
}

template <typename T, int D>
int launch_stream_r(int r, const T* src, const float* W, int M, int64_t n_items, int64_t row_stride,
                    int64_t item_stride, int64_t ub, int64_t uh, int64_t units, int hpb, float* out, int64_t ois,
                    int64_t obs, int64_t ohs, cudaStream_t s) {
    switch (r) {
        case 16:
            return launch_stream<T, D, 16>(src, W, M, n_items, row_stride, item_stride, ub, uh, units, hpb, out, ois,
                                           obs, ohs, s);
        case 32:
            return launch_stream<T, D, 32>(src, W, M, n_items, row_stride, item_stride, ub, uh, units, hpb, out, ois,
                                           obs, ohs, s);
        case 64:
            return launch_stream<T, D, 64>(src, W, M, n_items, row_stride, item_stride, ub, uh, units, hpb, out, ois,
                                           obs, ohs, s);
        default:
            return launch_stream<T, D, (D >= 128 ? 128 : 64)>(src, W, M, n_items, row_stride, item_stride, ub, uh,
                                                              units, hpb, out, ois, obs, ohs, s);
    }
}

// ------------------------------------------------------------ general form
// (any d, r and M, any alignment; the same arithmetic)
constexpr int kItems = 32;      // items (blocks or queries) per CTA
constexpr int kThreads = 256;

template <typename T>
__global__ __launch_bounds__(kThreads) void mean_project_kernel(
    const T* __restrict__ src, const float* __restrict__ W, int d, int r, int M, int64_t n_items,
    int64_t row_stride, int64_t item_stride, int64_t unit_b_stride, int64_t unit_h_stride, int hpb,
    float* __restrict__ out, int64_t out_item_stride, int64_t out_b_stride, int64_t out_h_stride) {
    extern __shared__ float smem[];
    float* Ws = smem;               // [d][r]
    float* Ms = smem + d * r;       // [kItems][d]
    const int unit = blockIdx.y;
    const int b = unit / hpb, h = unit % hpb;
    const int64_t item0 = (int64_t)blockIdx.x * kItems;
    for (int e = threadIdx.x; e < d * r; e += kThreads) Ws[e] = W[e];
    const T* base = src + (int64_t)b * unit_b_stride + (int64_t)h * unit_h_stride;
    for (int e = threadIdx.x; e < kItems * d; e += kThreads) {
        const int it = e / d, k = e % d;
        const int64_t item = item0 + it;
        float m = 0.f;
        if (item < n_items) m = mean_of_rows(base + item * item_stride + k, row_stride, M);
        Ms[it * d + k] = m;
    }
    __syncthreads();
    float* obase = out + (int64_t)b * out_b_stride + (int64_t)h * out_h_stride;
    for (int e = threadIdx.x; e < kItems * r; e += kThreads) {
        const int it = e / r, o = e % r;
        const int64_t item = item0 + it;
        if (item < n_items) obase[item * out_item_stride + o] = latent_dot(Ms + it * d, Ws, d, r, o);
    }
}

template <typename T>
int launch_mean_project(const T* src, const float* W, int d, int r, int M, int64_t n_items,
                        int64_t row_stride, int64_t item_stride, int64_t ub, int64_t uh, int64_t units,
                        int hpb, float* out, int64_t ois, int64_t obs, int64_t ohs, cudaStream_t s) {
    if (n_items <= 0 || units <= 0) return LSA_OK;
    // streaming form: 16-byte aligned rows and W, d in {64, 128}, r in
    // {16, 32, 64, 128} (r <= d), M <= 16
    constexpr int VN = 16 / (int)sizeof(T);
    const bool aligned = ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(W)) & 15u) == 0 &&
                         row_stride % VN == 0 && item_stride % VN == 0 && ub % VN == 0 && uh % VN == 0;
    if (aligned && M >= 1 && M <= 16 && (r == 16 || r == 32 || r == 64 || r == 128) && r <= d) {
        if (d == 128)
            return launch_stream_r<T, 128>(r, src, W, M, n_items, row_stride, item_stride, ub, uh, units, hpb, out,
                                           ois, obs, ohs, s);
        if (d == 64)
            return launch_stream_r<T, 64>(r, src, W, M, n_items, row_stride, item_stride, ub, uh, units, hpb, out,
                                          ois, obs, ohs, s);
    }
    size_t smem = (size_t)(d * r + kItems * d) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(mean_project_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return cuda_status(e);
    dim3 grid((unsigned)((n_items + kItems - 1) / kItems), (unsigned)units);
    note_launch();
    mean_project_kernel<T><<<grid, kThreads, smem, s>>>(src, W, d, r, M, n_items, row_stride, item_stride,
                                                        ub, uh, hpb, out, ois, obs, ohs);
    return cuda_status(cudaGetLastError());
}

}  // namespace

int launch_project_pool(const void* K, const float* W, int64_t batch, int64_t n_blocks, int64_t ld_tokens,
                        int hkv, int d, int r, int pool, int dtype, float* Kl, int64_t kl_unit_stride,
                        cudaStream_t s) {
    const int64_t row_stride = (int64_t)hkv * d;
    const int64_t item_stride = (int64_t)pool * hkv * d;
    const int64_t ub = ld_tokens * hkv * d, uh = d;
    const int64_t obs = (int64_t)hkv * kl_unit_stride * r, ohs = kl_unit_stride * r;
    if (dtype == LSA_F32)
        return launch_mean_project((const float*)K, W, d, r, pool, n_blocks, row_stride, item_stride, ub, uh,
                                   batch * hkv, hkv, Kl, r, obs, ohs, s);
    return launch_mean_project((const __nv_bfloat16*)K, W, d, r, pool, n_blocks, row_stride, item_stride, ub,
                               uh, batch * hkv, hkv, Kl, r, obs, ohs, s);
}

int launch_query_latent(const void* Q, const float* W, int64_t batch, int64_t nq, int hq, int hkv, int d,
                        int r, int dtype, float* qbar, cudaStream_t s) {
    const int G = hq / hkv;
    const int64_t row_stride = d, item_stride = (int64_t)hq * d;
    const int64_t ub = nq * hq * d, uh = (int64_t)G * d;
    const int64_t ois = (int64_t)hkv * r, obs = nq * hkv * r, ohs = r;
    if (dtype == LSA_F32)
        return launch_mean_project((const float*)Q, W, d, r, G, nq, row_stride, item_stride, ub, uh,
                                   batch * hkv, hkv, qbar, ois, obs, ohs, s);
    return launch_mean_project((const __nv_bfloat16*)Q, W, d, r, G, nq, row_stride, item_stride, ub, uh,
                               batch * hkv, hkv, qbar, ois, obs, ohs, s);
}

}  // namespace lsa
