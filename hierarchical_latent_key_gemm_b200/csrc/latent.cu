// Latent keys and latent queries.
//
// Keys: Kl[b] = W^T * mean(K[bP .. bP+P-1]) for every complete block of P
// keys: blocks of keys are averaged, then clustered in a learned low-rank
// space (LSA explainer, section "How does LSA work?", step 1).
// Queries: qbar = mean over a KV head's query heads of W^T q (the group shares
// one selection).
//
// Both are "mean of M rows, then a d x r map": an HBM stream at P = 4 (16
// flop per key byte), so CUDA cores suffice; W sits in shared memory.  The
// arithmetic order (rows summed in order, one IEEE division by M, then one
// fused multiply-add chain over the d inputs) is fixed in latent_common.cuh
// and shared with the decode append, so both produce identical bits.
#include "latent_common.cuh"

namespace lsa {
namespace {

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
