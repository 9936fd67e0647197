// Decode append.  In decode every generated token's query looks at the whole
// history, so the index must keep up with the tokens that decode adds (LSA
// explainer, section "Prefill, decode and training"; the decode phase is the
// subject of the 72.4x report's section "Prompt processing is not response
// generation").
//
// Every block that the new tokens complete is pooled and mapped exactly as in
// the build (same arithmetic order, so identical bits), placed in its nearest
// leaf by squared distance over all leaves (frozen centroids, ties to the
// lower id) at the end of that leaf's ascending member run, and the minpos of
// the leaf and its ancestors is lowered.  A full leaf latches kErrCapacity;
// the block keeps its leaf label but stays out of the buckets (and out of
// minpos) until the leaves are laid out again (relayout_leaves).
//
// Three launches: latents of the new blocks; the nearest-leaf scan spread over
// many CTAs (each takes a chunk of 128 leaves, eight lanes per leaf row, and
// folds its best (distance, leaf) into one 64-bit key per block with
// atomicMin, so ties go to the lower leaf); the ordered insertion, one CTA per
// unit.
#include "latent_common.cuh"

namespace lsa {
namespace {

constexpr int kAppThreads = 256;
constexpr int kLeavesPerCta = 128;
constexpr int kLanesPerLeaf = 8;

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
    unsigned long long* best;   // [units][n_new] packed (distance, leaf)
    int32_t* err;
};

// Latent of every new block: blockIdx.x = new block, blockIdx.y = unit.
template <typename T>
__global__ __launch_bounds__(kAppThreads) void append_latent_kernel(const T* __restrict__ K, const AppArgs a) {
    extern __shared__ float sm[];
    float* Ws = sm;                     // [d][r]
    float* mean = Ws + a.d * a.r;       // [d]
    const int u = blockIdx.y;
    const int64_t b = a.first_block + blockIdx.x;
    const int64_t bseq = u / a.hkv;
    const int h = u % a.hkv;
    for (int e = threadIdx.x; e < a.d * a.r; e += kAppThreads) Ws[e] = a.W[e];
    for (int k = threadIdx.x; k < a.d; k += kAppThreads) {
        const T* p = K + ((bseq * a.ld_tokens + b * a.pool) * a.hkv + h) * a.d + k;
        mean[k] = mean_of_rows(p, (int64_t)a.hkv * a.d, a.pool);
    }
    __syncthreads();
    for (int o = threadIdx.x; o < a.r; o += kAppThreads)
        a.Kl[((int64_t)u * a.nb_cap + b) * a.r + o] = latent_dot(mean, Ws, a.d, a.r, o);
}

// Nearest leaf, one chunk of leaves per CTA: blockIdx.x = chunk, blockIdx.y =
// unit.  Groups of kLanesPerLeaf lanes take one leaf row each (a lane sums
// every kLanesPerLeaf-th dimension, then the group adds by shuffles), so a
// warp has 32 / kLanesPerLeaf rows in flight; each warp folds its best
// (distance, leaf) key by shuffles and issues one atomicMin per new block.
__global__ __launch_bounds__(kAppThreads) void append_nearest_kernel(const AppArgs a) {
    extern __shared__ float xs[];       // [n_new][r] latents of the new blocks
    constexpr int kGroups = kAppThreads / kLanesPerLeaf;   // leaf rows in flight per CTA
    const int u = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane % kLanesPerLeaf;
    const int grp = warp * (32 / kLanesPerLeaf) + lane / kLanesPerLeaf;
    for (int e = threadIdx.x; e < a.n_new * a.r; e += kAppThreads)
        xs[e] = a.Kl[((int64_t)u * a.nb_cap + a.first_block + e / a.r) * a.r + e % a.r];
    __syncthreads();
    const float* cl = a.cent_leaf + (int64_t)u * a.L * a.r;
    const float scale = a.grid_log2 > 0 ? (float)(1 << a.grid_log2) : 1.f;
    const int j0 = blockIdx.x * kLeavesPerCta;
    const int j1 = min(a.L, j0 + kLeavesPerCta);
    for (int64_t nb = 0; nb < a.n_new; ++nb) {
        const float* x = xs + nb * a.r;
        unsigned long long best = ~0ull;
        // the trip count is the same for every lane (shuffles below); a group
        // past the chunk's end reads the chunk's first row and drops the result
        for (int jb = j0; jb < j1; jb += kGroups) {
            const int j = jb + grp;
            const bool valid = j < j1;
            const float* c = cl + (int64_t)(valid ? j : j0) * a.r;
            unsigned long long key = ~0ull;
            if (a.grid_log2 > 0) {
                long long s = 0;
                for (int e = sub; e < a.r; e += kLanesPerLeaf) {
                    const long long dd = (long long)(x[e] * scale) - (long long)(c[e] * scale);
                    s += dd * dd;
                }
#pragma unroll
                for (int o = kLanesPerLeaf / 2; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                if (valid) {
                    if (s >= (1ll << 43)) latch(a.err, kErrInexact);
                    key = ((unsigned long long)s << 20) | (unsigned)j;
                }
            } else {
                float s = 0.f;
                for (int e = sub; e < a.r; e += kLanesPerLeaf) {
                    const float dd = __fsub_rn(x[e], c[e]);
                    s = __fmaf_rn(dd, dd, s);
                }
#pragma unroll
                for (int o = kLanesPerLeaf / 2; o >= 1; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
                // distances are >= 0, so their bit patterns order like the values
                if (valid) key = ((unsigned long long)__float_as_uint(s) << 32) | (unsigned)j;
            }
            best = key < best ? key : best;
        }
#pragma unroll
        for (int o = 16; o >= kLanesPerLeaf; o >>= 1) {
            const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
            best = other < best ? other : best;
        }
        if (lane == 0 && best != ~0ull) atomicMin(a.best + (int64_t)u * a.n_new + nb, best);
    }
}

// Ordered insertion of the new blocks of one unit.
__global__ __launch_bounds__(kAppThreads) void append_insert_kernel(const AppArgs a) {
    __shared__ int slot_sh;
    const int u = blockIdx.x;
    for (int64_t t = 0; t < a.n_new; ++t) {
        const int64_t b = a.first_block + t;
        if (threadIdx.x == 0) {
            const unsigned long long key = a.best[(int64_t)u * a.n_new + t];
            const int leaf = a.grid_log2 > 0 ? (int)(key & 0xFFFFFull) : (int)(key & 0xFFFFFFFFull);
            int slot = -1;
            if (key == ~0ull || leaf < 0 || leaf >= a.L) {
                latch(a.err, kErrDevice);
                a.leaf_of_block[(int64_t)u * a.nb_cap + b] = -1;
            } else {
                const int64_t c = (int64_t)u * a.L + leaf;
                const int cnt = a.leaf_cnt[c];
                if (cnt < a.leaf_cap[c]) {
                    slot = a.leaf_start[c] + cnt;
                    a.blk[slot] = (int32_t)b;
                    a.leaf_cnt[c] = cnt + 1;
                    a.leaf_of_block[(int64_t)u * a.nb_cap + b] = leaf;
                    const int64_t start = b * a.pool;
                    if (start >= a.sink) {
                        int node = leaf;
                        for (int l = a.levels - 1; l >= 0; --l) {
                            const int64_t base = (int64_t)u * a.n_l[l];
                            int64_t* mp = a.minpos[l] + base + node;
                            if (start < *mp) *mp = start;
                            int64_t* omp = a.ord_mp[l] + base + a.ord_pos[l][base + node];
                            if (start < *omp) *omp = start;
                            if (l > 0) node = a.parent[l][base + node];
                        }
                    }
                } else {
                    // no free slot: the block keeps its label and waits for a relayout
                    latch(a.err, kErrCapacity);
                    a.leaf_of_block[(int64_t)u * a.nb_cap + b] = leaf;
                }
            }
            slot_sh = slot;
        }
        __syncthreads();
        const int slot = slot_sh;
        if (slot >= 0)
            for (int o = threadIdx.x; o < a.r; o += kAppThreads)
                a.Klp[(int64_t)slot * a.r + o] = a.Kl[((int64_t)u * a.nb_cap + b) * a.r + o];
        __syncthreads();
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
    const size_t smem_lat = (size_t)(p.d * p.r + p.d) * sizeof(float);
    const size_t smem_near = (size_t)n_new_blocks * p.r * sizeof(float);
    if (smem_near > 200 * 1024) return LSA_ERR_INVALID_ARG;
    Arena scratch;
    scratch.async = true;
    scratch.stream = s;
    a.best = scratch.alloc<unsigned long long>(ix->units * n_new_blocks);
    if (scratch.status != LSA_OK) return scratch.status;
    cudaMemsetAsync(a.best, 0xff, ix->units * n_new_blocks * sizeof(unsigned long long), s);
    cudaError_t e;
    dim3 glat((unsigned)n_new_blocks, (unsigned)ix->units);
    if (p.dtype == LSA_F32) {
        e = cudaFuncSetAttribute(append_latent_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem_lat);
        if (e != cudaSuccess) return cuda_status(e);
        note_launch();
        append_latent_kernel<float><<<glat, kAppThreads, smem_lat, s>>>((const float*)K, a);
    } else {
        e = cudaFuncSetAttribute(append_latent_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem_lat);
        if (e != cudaSuccess) return cuda_status(e);
        note_launch();
        append_latent_kernel<__nv_bfloat16><<<glat, kAppThreads, smem_lat, s>>>((const __nv_bfloat16*)K, a);
    }
    e = cudaFuncSetAttribute(append_nearest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_near);
    if (e != cudaSuccess) return cuda_status(e);
    dim3 gnear((unsigned)((ix->L + kLeavesPerCta - 1) / kLeavesPerCta), (unsigned)ix->units);
    note_launch();
    append_nearest_kernel<<<gnear, kAppThreads, smem_near, s>>>(a);
    note_launch();
    append_insert_kernel<<<(unsigned)ix->units, kAppThreads, 0, s>>>(a);
    const int st = cuda_status(cudaGetLastError());
    scratch.release();
    return st;
}

}  // namespace lsa
