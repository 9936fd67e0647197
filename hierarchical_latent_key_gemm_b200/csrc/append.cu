// Decode append ("each new token attends back over the whole history", LSA
// explainer, "Prefill, decode and training"; decode is the response phase of
// "Prompt processing is not response generation").
//
// Every block that the new tokens complete is pooled and mapped exactly as in
// the build (same arithmetic order, so identical bits), placed in its nearest
// leaf by squared distance over all leaves (frozen centroids, ties to the
// lower id) at the end of that leaf's ascending member run, and the minpos of
// the leaf and its ancestors is lowered.  One CTA per unit walks its new
// blocks in order.  A full leaf latches kErrCapacity and leaves the block
// unindexed.
#include "latent_common.cuh"

namespace lsa {
namespace {

constexpr int kAppThreads = 256;

struct AppArgs {
    const float* W;
    float* Kl;
    float* Klp;
    int32_t* blk;
    int32_t* leaf_start;
    int32_t* leaf_cnt;
    int32_t* leaf_cap;
    int32_t* leaf_of_block;
    const float* cent_leaf;
    int64_t* minpos[LSA_MAX_LEVELS];
    int64_t* ord_mp[LSA_MAX_LEVELS];
    const int32_t* ord_pos[LSA_MAX_LEVELS];
    const int32_t* parent[LSA_MAX_LEVELS];
    int n_l[LSA_MAX_LEVELS];
    int levels, L, d, r, pool, sink, hkv, grid_log2;
    int64_t nb_cap, ld_tokens, first_block, n_new;
    int32_t* err;
};

template <typename T>
__global__ __launch_bounds__(kAppThreads) void append_kernel(const T* __restrict__ K, const AppArgs a) {
    extern __shared__ float sm[];
    float* Ws = sm;                     // [d][r]
    float* mean = Ws + a.d * a.r;       // [d]
    float* x = mean + a.d;              // [r]
    __shared__ float bd[kAppThreads];
    __shared__ int bj[kAppThreads];
    __shared__ int slot_sh;
    const int u = blockIdx.x;
    const int64_t bseq = u / a.hkv;
    const int h = u % a.hkv;
    for (int e = threadIdx.x; e < a.d * a.r; e += kAppThreads) Ws[e] = a.W[e];
    const float* cl = a.cent_leaf + (int64_t)u * a.L * a.r;
    const float scale = a.grid_log2 > 0 ? (float)(1 << a.grid_log2) : 1.f;
    for (int64_t t = 0; t < a.n_new; ++t) {
        const int64_t b = a.first_block + t;
        __syncthreads();
        for (int k = threadIdx.x; k < a.d; k += kAppThreads) {
            const T* p = K + ((bseq * a.ld_tokens + b * a.pool) * a.hkv + h) * a.d + k;
            mean[k] = mean_of_rows(p, (int64_t)a.hkv * a.d, a.pool);
        }
        __syncthreads();
        for (int o = threadIdx.x; o < a.r; o += kAppThreads) {
            const float v = latent_dot(mean, Ws, a.d, a.r, o);
            x[o] = v;
            a.Kl[((int64_t)u * a.nb_cap + b) * a.r + o] = v;
        }
        __syncthreads();
        float best = INFINITY;
        int bestj = 0x7fffffff;
        for (int j = threadIdx.x; j < a.L; j += kAppThreads) {
            const float* c = cl + (int64_t)j * a.r;
            float dist;
            if (a.grid_log2 > 0) {
                long long s = 0;
                for (int e = 0; e < a.r; ++e) {
                    const long long dd = (long long)(x[e] * scale) - (long long)(c[e] * scale);
                    s += dd * dd;
                }
                dist = (float)s;  // exact ordering preserved below via integer compare
                // keep exactness: compare in integers by encoding into the float only when small
                if (s >= (1LL << 24)) latch(a.err, kErrInexact);
            } else {
                float s = 0.f;
                for (int e = 0; e < a.r; ++e) {
                    const float dd = __fsub_rn(x[e], c[e]);
                    s = __fmaf_rn(dd, dd, s);
                }
                dist = s;
            }
            if (dist < best) { best = dist; bestj = j; }
        }
        bd[threadIdx.x] = best;
        bj[threadIdx.x] = bestj;
        __syncthreads();
        for (int w = kAppThreads / 2; w >= 1; w >>= 1) {
            if (threadIdx.x < w) {
                const float od = bd[threadIdx.x + w];
                const int oj = bj[threadIdx.x + w];
                if (od < bd[threadIdx.x] || (od == bd[threadIdx.x] && oj < bj[threadIdx.x])) {
                    bd[threadIdx.x] = od;
                    bj[threadIdx.x] = oj;
                }
            }
            __syncthreads();
        }
        if (threadIdx.x == 0) {
            const int leaf = bj[0];
            const int64_t c = (int64_t)u * a.L + leaf;
            const int cnt = a.leaf_cnt[c];
            int slot = -1;
            if (cnt < a.leaf_cap[c]) {
                slot = a.leaf_start[c] + cnt;
                a.blk[slot] = (int32_t)b;
                a.leaf_cnt[c] = cnt + 1;
                a.leaf_of_block[(int64_t)u * a.nb_cap + b] = leaf;
                const int64_t start = b * a.pool;
                if (start >= a.sink) {
                    int node = leaf;
                    for (int l = a.levels - 1; l >= 0; --l) {
                        int64_t* mp = a.minpos[l] + (int64_t)u * a.n_l[l] + node;
                        if (start < *mp) *mp = start;
                        int64_t* omp = a.ord_mp[l] + (int64_t)u * a.n_l[l] + a.ord_pos[l][(int64_t)u * a.n_l[l] + node];
                        if (start < *omp) *omp = start;
                        if (l > 0) node = a.parent[l][(int64_t)u * a.n_l[l] + node];
                    }
                }
            } else {
                latch(a.err, kErrCapacity);
                a.leaf_of_block[(int64_t)u * a.nb_cap + b] = -1;
            }
            slot_sh = slot;
        }
        __syncthreads();
        const int slot = slot_sh;
        if (slot >= 0)
            for (int o = threadIdx.x; o < a.r; o += kAppThreads) a.Klp[(int64_t)slot * a.r + o] = x[o];
    }
}

}  // namespace

int launch_append(lsa_index* ix, const void* K, int64_t first_block, int64_t n_new_blocks, cudaStream_t s) {
    if (n_new_blocks <= 0) return LSA_OK;
    const lsa_build_params& p = ix->p;
    AppArgs a{};
    a.W = ix->W;
    a.Kl = ix->Kl;
    a.Klp = ix->Klp;
    a.blk = ix->blk;
    a.leaf_start = ix->leaf_start;
    a.leaf_cnt = ix->leaf_cnt;
    a.leaf_cap = ix->leaf_cap;
    a.leaf_of_block = ix->leaf_of_block;
    a.cent_leaf = ix->cent[p.levels - 1];
    for (int l = 0; l < p.levels; ++l) {
        a.minpos[l] = ix->minpos[l];
        a.ord_mp[l] = ix->ord_mp[l];
        a.ord_pos[l] = ix->ord_pos[l];
        a.parent[l] = ix->parent[l];
        a.n_l[l] = p.level_sizes[l];
    }
    a.levels = p.levels;
    a.L = ix->L;
    a.d = p.d;
    a.r = p.r;
    a.pool = p.pool;
    a.sink = p.sink;
    a.hkv = p.hkv;
    a.grid_log2 = p.grid_log2;
    a.nb_cap = ix->nb_cap;
    a.ld_tokens = p.ld_tokens;
    a.first_block = first_block;
    a.n_new = n_new_blocks;
    a.err = ix->err;
    const size_t smem = (size_t)(p.d * p.r + p.d + p.r) * sizeof(float);
    cudaError_t e;
    if (p.dtype == LSA_F32) {
        e = cudaFuncSetAttribute(append_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_status(e);
        note_launch();
        append_kernel<float><<<(unsigned)ix->units, kAppThreads, smem, s>>>((const float*)K, a);
    } else {
        e = cudaFuncSetAttribute(append_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return cuda_status(e);
        note_launch();
        append_kernel<__nv_bfloat16><<<(unsigned)ix->units, kAppThreads, smem, s>>>((const __nv_bfloat16*)K, a);
    }
    return cuda_status(cudaGetLastError());
}

}  // namespace lsa
