// C ABI of the LSA hot path: argument checks, index lifecycle, build
// orchestration and error reporting.  Kernels live in the other files.
#include <atomic>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_set>

#include "lsa_internal.cuh"

namespace lsa {

namespace {
std::atomic<int32_t> g_fail_after{0};
std::mutex g_err_mu;
int32_t* g_err_words[128] = {nullptr};
}  // namespace

namespace {
std::atomic<int64_t> g_launches{0};
}  // namespace

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

bool debug_alloc_should_fail() {
    int32_t v = g_fail_after.load();
    while (v > 0) {
        if (g_fail_after.compare_exchange_weak(v, v - 1)) return v == 1;
    }
    return false;
}

bool Arena::alloc_raw(void** p, int64_t nbytes) {
    if (debug_alloc_should_fail()) return false;
    cudaError_t e = async ? cudaMallocAsync(p, (size_t)nbytes, stream) : cudaMalloc(p, (size_t)nbytes);
    if (e != cudaSuccess) {
        cudaGetLastError();  // clear the sticky-free error state of a failed allocation
        return false;
    }
    return true;
}

void Arena::release() {
    for (void* p : ptrs) {
        if (async) cudaFreeAsync(p, stream);
        else cudaFree(p);
    }
    ptrs.clear();
    bytes = 0;
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return LSA_OK;
    if (e == cudaErrorMemoryAllocation) return LSA_ERR_OOM;
    return LSA_ERR_CUDA;
}

int err_bits_to_status(int32_t bits) {
    if (bits & kErrDevice) return LSA_ERR_DEVICE;
    if (bits & kErrInexact) return LSA_ERR_INEXACT;
    if (bits & kErrCapacity) return LSA_ERR_CAPACITY;
    if (bits & kErrTimeout) return LSA_ERR_TIMEOUT;
    return LSA_OK;
}

int32_t* global_err_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
    std::lock_guard<std::mutex> lk(g_err_mu);
    if (!g_err_words[dev]) {
        int32_t* p = nullptr;
        if (cudaMalloc(&p, sizeof(int32_t)) != cudaSuccess) return nullptr;
        cudaMemset(p, 0, sizeof(int32_t));
        cudaDeviceSynchronize();
        g_err_words[dev] = p;
    }
    return g_err_words[dev];
}

}  // namespace lsa

using namespace lsa;

namespace {

// Live indexes; a pointer outside this set is never dereferenced.
std::mutex g_live_mu;
std::unordered_set<const lsa_index*> g_live;

bool is_device_ptr(const void* p) {
    if (!p) return false;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

bool valid_r(int r) { return r == 16 || r == 32 || r == 64 || r == 128; }
bool valid_d(int d) { return d == 64 || d == 128; }

int check_build_params(const lsa_build_params* p) {
    if (!p) return LSA_ERR_INVALID_ARG;
    if (p->batch < 1 || p->n_tokens < 1 || p->ld_tokens < p->n_tokens) return LSA_ERR_INVALID_ARG;
    if (p->hkv < 1 || !valid_d(p->d) || !valid_r(p->r)) return LSA_ERR_INVALID_ARG;
    if (p->pool < 1 || p->pool > 16) return LSA_ERR_INVALID_ARG;
    if (p->dtype != LSA_F32 && p->dtype != LSA_BF16) return LSA_ERR_INVALID_ARG;
    if (p->levels < 1 || p->levels > LSA_MAX_LEVELS) return LSA_ERR_INVALID_ARG;
    for (int l = 0; l < p->levels; ++l) {
        if (p->level_sizes[l] < 1) return LSA_ERR_INVALID_ARG;
        if (l > 0 && p->level_sizes[l] < p->level_sizes[l - 1]) return LSA_ERR_INVALID_ARG;
    }
    if (p->lloyd_iters < 1 || p->grid_log2 < 0 || p->grid_log2 > 8) return LSA_ERR_INVALID_ARG;
    if (p->sink < 0 || p->append_capacity < 0) return LSA_ERR_INVALID_ARG;
    if (p->n_tokens / p->pool < 1) return LSA_ERR_INVALID_ARG;
    if (p->n_tokens + p->append_capacity > p->ld_tokens) return LSA_ERR_INVALID_ARG;
    const int64_t units = p->batch * p->hkv;
    const int64_t nb_cap = p->ld_tokens / p->pool + 1;
    if (units > 65535 || units * nb_cap > INT32_MAX / 2 || units * (int64_t)p->level_sizes[p->levels - 1] > INT32_MAX / 4)
        return LSA_ERR_INVALID_ARG;
    return LSA_OK;
}

// The library allocates from the device's default stream-ordered pool.  Freed
// blocks stay cached in the pool (up to 16 GiB) so that rebuilding an index of
// the same shape does not go back to the driver.  This is a setting of this
// process's pool, not of the GPU.
void keep_pool_memory() {
    static std::mutex mu;
    static bool done[128] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return;
    std::lock_guard<std::mutex> lk(mu);
    if (done[dev]) return;
    cudaMemPool_t pool;
    if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
        uint64_t thr = uint64_t(16) << 30;
        cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr);
    }
    cudaGetLastError();
    done[dev] = true;
}

// Allocates every persistent array of an index (no kernel launched).
int alloc_index(const lsa_build_params* p, const float* W, cudaStream_t s, lsa_index** out) {
    keep_pool_memory();
    lsa_index* ix = new (std::nothrow) lsa_index();
    if (!ix) return LSA_ERR_OOM;
    std::memset(ix, 0, sizeof(*ix));
    ix->mem = new (std::nothrow) Arena();
    if (!ix->mem) { delete ix; return LSA_ERR_OOM; }
    ix->mem->async = true;
    ix->mem->stream = s;
    ix->p = *p;
    cudaGetDevice(&ix->device);
    ix->units = p->batch * p->hkv;
    ix->nb = p->n_tokens / p->pool;
    ix->n_tokens = p->n_tokens;
    ix->nb_cap = (p->n_tokens + p->append_capacity) / p->pool + 1;
    ix->L = p->level_sizes[p->levels - 1];
    const int64_t U = ix->units, r = p->r;
    const int64_t append_blocks = p->append_capacity > 0 ? (p->append_capacity + p->pool - 1) / p->pool + 1 : 0;
    const int64_t slots_per_unit = ix->nb + (append_blocks > 0 ? 3 * (int64_t)ix->L + 2 * append_blocks : 0) + 16;
    ix->slots = U * slots_per_unit;
    Arena& A = *ix->mem;
    ix->W = A.alloc<float>((int64_t)p->d * r);
    ix->Kl = A.alloc<float>(U * ix->nb_cap * r);
    ix->Klp = A.alloc<float>(ix->slots * r);
    ix->blk = A.alloc<int32_t>(ix->slots);
    ix->leaf_start = A.alloc<int32_t>(U * ix->L + 1);
    ix->leaf_cnt = A.alloc<int32_t>(U * ix->L);
    ix->leaf_cap = A.alloc<int32_t>(U * ix->L);
    ix->leaf_of_block = A.alloc<int32_t>(U * ix->nb_cap);
    for (int l = 0; l < p->levels; ++l) {
        const int64_t nl = p->level_sizes[l];
        ix->cent[l] = A.alloc<float>(U * nl * r);
        ix->minpos[l] = A.alloc<int64_t>(U * nl);
        ix->parent[l] = A.alloc<int32_t>(U * nl);
        ix->objective[l] = A.alloc<double>((int64_t)p->lloyd_iters * U);
        ix->ord_id[l] = A.alloc<int32_t>(U * nl);
        ix->ord_pos[l] = A.alloc<int32_t>(U * nl);
        ix->ord_cent[l] = A.alloc<float>(U * nl * r);
        ix->ord_mp[l] = A.alloc<int64_t>(U * nl);
        if (l + 1 < p->levels) {
            ix->child_off[l] = A.alloc<int32_t>(U * nl + 1);
            ix->child_ids[l] = A.alloc<int32_t>(U * (int64_t)p->level_sizes[l + 1]);
            ix->ord_coff[l] = A.alloc<int32_t>(U * nl + 1);
        }
    }
    ix->err = A.alloc<int32_t>(1);
    if (A.status != LSA_OK) {
        int st = A.status;
        A.release();
        delete ix->mem;
        delete ix;
        return st;
    }
    cudaMemsetAsync(ix->err, 0, sizeof(int32_t), s);
    cudaMemsetAsync(ix->leaf_of_block, 0xff, U * ix->nb_cap * sizeof(int32_t), s);
    cudaMemsetAsync(ix->blk, 0xff, ix->slots * sizeof(int32_t), s);
    cudaMemsetAsync(ix->Kl, 0, U * ix->nb_cap * r * sizeof(float), s);
    cudaMemsetAsync(ix->parent[0], 0xff, U * (int64_t)p->level_sizes[0] * sizeof(int32_t), s);
    for (int l = 0; l < p->levels; ++l)
        cudaMemsetAsync(ix->objective[l], 0, (int64_t)p->lloyd_iters * U * sizeof(double), s);
    cudaMemcpyAsync(ix->W, W, (size_t)p->d * r * sizeof(float), cudaMemcpyDefault, s);
    ix->magic = kIndexMagic;
    {
        std::lock_guard<std::mutex> lk(g_live_mu);
        g_live.insert(ix);
    }
    *out = ix;
    return cuda_status(cudaGetLastError());
}

void destroy_index(lsa_index* ix) {
    if (!ix) return;
    {
        std::lock_guard<std::mutex> lk(g_live_mu);
        g_live.erase(ix);
    }
    ix->magic = kFreedMagic;
    if (ix->mem) {
        // the caller's streams may still use the index: wait for them, then
        // return the memory to the pool on the legacy stream
        cudaDeviceSynchronize();
        ix->mem->stream = nullptr;
        ix->mem->release();
        delete ix->mem;
    }
    delete ix;
}

bool live(const lsa_index* ix) {
    if (!ix) return false;
    std::lock_guard<std::mutex> lk(g_live_mu);
    return g_live.count(ix) && ix->magic == kIndexMagic;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int build_common(const lsa_build_params* p, const void* K, const float* W, void* stream, lsa_index** out,
                 const int32_t* given_leaf, const int32_t* const* given_parents, const float* const* given_cent) {
    if (!out) return LSA_ERR_INVALID_ARG;
    *out = nullptr;
    int st = check_build_params(p);
    if (st != LSA_OK) return st;
    if (!is_device_ptr(K) || !is_device_ptr(W)) return LSA_ERR_INVALID_ARG;
    const bool given = given_leaf != nullptr;
    if (given) {
        if (!is_device_ptr(given_leaf) || !given_cent) return LSA_ERR_INVALID_ARG;
        for (int l = 0; l < p->levels; ++l)
            if (!is_device_ptr(given_cent[l])) return LSA_ERR_INVALID_ARG;
        for (int l = 1; l < p->levels; ++l)
            if (!given_parents || !is_device_ptr(given_parents[l])) return LSA_ERR_INVALID_ARG;
    }
    cudaStream_t s = as_stream(stream);
    lsa_index* ix = nullptr;
    st = alloc_index(p, W, s, &ix);
    if (st != LSA_OK) return st;
    const int64_t U = ix->units, nb = ix->nb;
    const int L = ix->L, r = p->r, levels = p->levels;
    Arena scratch;
    scratch.async = true;
    scratch.stream = s;
    st = launch_project_pool(K, ix->W, p->batch, nb, p->ld_tokens, p->hkv, p->d, r, p->pool, p->dtype, ix->Kl,
                             ix->nb_cap, s);
    int32_t* leaf_perm = scratch.alloc<int32_t>(U * nb);
    int32_t* leaf_off = scratch.alloc<int32_t>(U * (int64_t)L + 1);
    int32_t* up_perm[LSA_MAX_LEVELS] = {nullptr};
    int32_t* up_off[LSA_MAX_LEVELS] = {nullptr};
    for (int l = 0; l + 1 < levels; ++l) {
        up_perm[l] = scratch.alloc<int32_t>(U * (int64_t)p->level_sizes[l + 1]);
        up_off[l] = scratch.alloc<int32_t>(U * (int64_t)p->level_sizes[l] + 1);
    }
    if (st == LSA_OK) st = scratch.status;
    if (st == LSA_OK && !given) {
        KmeansOut ko{ix->leaf_of_block, ix->cent[levels - 1], leaf_perm, leaf_off, ix->objective[levels - 1]};
        st = run_kmeans(ix->Kl, ix->nb_cap, U, nb, r, L, p->lloyd_iters, p->grid_log2, ko, ix->nb_cap, ix->err, s,
                        scratch);
        for (int l = levels - 2; l >= 0 && st == LSA_OK; --l) {
            const int n_child = p->level_sizes[l + 1];
            KmeansOut ku{ix->parent[l + 1], ix->cent[l], up_perm[l], up_off[l], ix->objective[l]};
            st = run_kmeans(ix->cent[l + 1], n_child, U, n_child, r, p->level_sizes[l], p->lloyd_iters, p->grid_log2,
                            ku, n_child, ix->err, s, scratch);
        }
    } else if (st == LSA_OK) {
        for (int64_t u = 0; u < U && st == LSA_OK; ++u)
            st = cuda_status(cudaMemcpyAsync(ix->leaf_of_block + u * ix->nb_cap, given_leaf + u * nb,
                                             nb * sizeof(int32_t), cudaMemcpyDefault, s));
        for (int l = 0; l < levels && st == LSA_OK; ++l) {
            const int64_t nl = p->level_sizes[l];
            st = cuda_status(cudaMemcpyAsync(ix->cent[l], given_cent[l], U * nl * r * sizeof(float), cudaMemcpyDefault, s));
            if (st == LSA_OK && l > 0)
                st = cuda_status(cudaMemcpyAsync(ix->parent[l], given_parents[l], U * nl * sizeof(int32_t),
                                                 cudaMemcpyDefault, s));
        }
        if (st == LSA_OK) {
            GroupWork gw = alloc_group_work(U, nb, L, scratch);
            st = scratch.status;
            if (st == LSA_OK)
                st = group_by_label(ix->leaf_of_block, ix->nb_cap, U, nb, L, leaf_perm, leaf_off, ix->err, s, gw);
        }
        for (int l = levels - 2; l >= 0 && st == LSA_OK; --l) {
            const int n_child = p->level_sizes[l + 1];
            GroupWork gw = alloc_group_work(U, n_child, p->level_sizes[l], scratch);
            st = scratch.status;
            if (st == LSA_OK)
                st = group_by_label(ix->parent[l + 1], n_child, U, n_child, p->level_sizes[l], up_perm[l], up_off[l],
                                    ix->err, s, gw);
        }
    }
    if (st == LSA_OK) st = finish_tree(ix, leaf_perm, leaf_off, up_perm, up_off, s, scratch);
    scratch.release();
    if (st == LSA_OK) st = cuda_status(cudaGetLastError());
    if (st != LSA_OK) {
        destroy_index(ix);
        return st;
    }
    *out = ix;
    return LSA_OK;
}

int check_select(const lsa_index* ix, const lsa_select_params* sp, const void* Q, int64_t nq, const int64_t* q_pos,
                 int64_t q_pos0, const int32_t* idx, const int32_t* cnt, int32_t max_sel) {
    if (!live(ix) || !sp) return LSA_ERR_INVALID_ARG;
    const lsa_build_params& p = ix->p;
    if (sp->hq < p.hkv || sp->hq % p.hkv) return LSA_ERR_INVALID_ARG;
    if (sp->beam < 1 || sp->beam > 1024 || sp->topk < 0 || sp->window < 1 || sp->sink != p.sink)
        return LSA_ERR_INVALID_ARG;
    const int64_t kb = (sp->topk + p.pool - 1) / p.pool;
    if (kb > 4096) return LSA_ERR_INVALID_ARG;
    if ((int64_t)max_sel < kb * p.pool + p.sink + sp->window) return LSA_ERR_INVALID_ARG;
    if (nq < 0 || (nq > 0 && (!is_device_ptr(Q) || !is_device_ptr(idx) || !is_device_ptr(cnt))))
        return LSA_ERR_INVALID_ARG;
    if (q_pos && !is_device_ptr(q_pos)) return LSA_ERR_INVALID_ARG;
    if (!q_pos && (q_pos0 < 0 || q_pos0 + nq > INT32_MAX)) return LSA_ERR_INVALID_ARG;
    if (nq > INT32_MAX) return LSA_ERR_INVALID_ARG;
    return LSA_OK;
}

// Full scans of this many (query, KV head) pairs or more take the
// tensor-core filter (its CTAs split the block range when the query tiles
// alone would not fill the GPU); fewer pairs are scanned by the per-query
// kernel directly.
constexpr int64_t kFullscanTcMinPairs = 64;

int do_select(const lsa_index* ix, const lsa_select_params* sp, const void* Q, int64_t nq, const int64_t* q_pos,
              int64_t q_pos0, int32_t* idx, int32_t* cnt, int32_t max_sel, void* stream, bool fullscan,
              unsigned long long* work = nullptr) {
    int st = check_select(ix, sp, Q, nq, q_pos, q_pos0, idx, cnt, max_sel);
    if (st != LSA_OK || nq == 0) return st;
    cudaStream_t s = as_stream(stream);
    const lsa_build_params& p = ix->p;
    keep_pool_memory();
    Arena scratch;
    scratch.async = true;
    scratch.stream = s;
    float* qbar = scratch.alloc<float>(p.batch * nq * p.hkv * p.r);
    if (scratch.status != LSA_OK) return scratch.status;
    st = launch_query_latent(Q, ix->W, p.batch, nq, sp->hq, p.hkv, p.d, p.r, p.dtype, qbar, s);
    if (st == LSA_OK && fullscan && nq * ix->units >= kFullscanTcMinPairs && fullscan_tc_applies(ix, sp))
        st = launch_fullscan_tc(ix, sp, qbar, nq, q_pos, q_pos0, idx, cnt, max_sel, s, scratch);
    else if (st == LSA_OK && fullscan)
        st = launch_select(ix, sp, qbar, nq, q_pos, q_pos0, idx, cnt, max_sel, true, s, work);
    else if (st == LSA_OK)
        st = launch_select_tree(ix, sp, qbar, nq, q_pos, q_pos0, idx, cnt, max_sel, s, work, nullptr, scratch);
    scratch.release();
    return st;
}

// bf16 attention reads Q, K, V rows and writes O in 16-byte pieces
bool attn_aligned(int dtype, const void* Q, const void* K, const void* V, const void* O) {
    if (dtype != LSA_BF16) return true;
    return ((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V) |
             reinterpret_cast<uintptr_t>(O)) & 15u) == 0;
}

}  // namespace

extern "C" {

int lsa_build_index(const lsa_build_params* params, const void* K, const float* W, void* stream, lsa_index** out) {
    return build_common(params, K, W, stream, out, nullptr, nullptr, nullptr);
}

int lsa_build_index_from_tree(const lsa_build_params* params, const void* K, const float* W,
                              const int32_t* leaf_of_block, const int32_t* const* parents,
                              const float* const* centroids, void* stream, lsa_index** out) {
    if (!leaf_of_block) return LSA_ERR_INVALID_ARG;
    return build_common(params, K, W, stream, out, leaf_of_block, parents, centroids);
}

int lsa_select(const lsa_index* index, const lsa_select_params* params, const void* Q, int64_t nq,
               const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int32_t max_sel, void* stream) {
    return do_select(index, params, Q, nq, q_pos, q_pos0, idx, cnt, max_sel, stream, false);
}

int lsa_select_work(const lsa_index* index, const lsa_select_params* params, const void* Q, int64_t nq,
                    const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int32_t max_sel,
                    unsigned long long* scored, void* stream) {
    if (!scored || !is_device_ptr(scored)) return LSA_ERR_INVALID_ARG;
    return do_select(index, params, Q, nq, q_pos, q_pos0, idx, cnt, max_sel, stream, false, scored);
}

int lsa_fullscan_select(const lsa_index* index, const lsa_select_params* params, const void* Q, int64_t nq,
                        const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt, int32_t max_sel,
                        void* stream) {
    return do_select(index, params, Q, nq, q_pos, q_pos0, idx, cnt, max_sel, stream, true);
}

int lsa_select_blocks(const lsa_index* index, const lsa_select_params* params, const void* Q, int64_t nq,
                      const int64_t* q_pos, int64_t q_pos0, int64_t token_offset, float* scores, int32_t* blocks,
                      int32_t* count, int32_t kb_cap, void* stream) {
    if (!live(index) || !params) return LSA_ERR_INVALID_ARG;
    const lsa_build_params& p = index->p;
    const lsa_select_params& sp = *params;
    if (sp.hq < p.hkv || sp.hq % p.hkv || sp.beam < 1 || sp.beam > 1024 || sp.topk < 0 || sp.window < 1 ||
        sp.sink != p.sink)
        return LSA_ERR_INVALID_ARG;
    const int64_t kb = (sp.topk + p.pool - 1) / p.pool;
    if (kb > 4096 || kb_cap < kb || kb_cap < 1) return LSA_ERR_INVALID_ARG;
    if (token_offset < 0 || token_offset % p.pool || token_offset / p.pool + index->nb_cap > INT32_MAX)
        return LSA_ERR_INVALID_ARG;
    if (nq < 0 || nq > INT32_MAX) return LSA_ERR_INVALID_ARG;
    if (!q_pos && (q_pos0 < 0 || q_pos0 + nq > INT32_MAX)) return LSA_ERR_INVALID_ARG;
    if (nq == 0) return LSA_OK;
    if (!is_device_ptr(Q) || !is_device_ptr(scores) || !is_device_ptr(blocks) || !is_device_ptr(count))
        return LSA_ERR_INVALID_ARG;
    if (q_pos && !is_device_ptr(q_pos)) return LSA_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    keep_pool_memory();
    Arena scratch;
    scratch.async = true;
    scratch.stream = s;
    float* qbar = scratch.alloc<float>(p.batch * nq * p.hkv * p.r);
    if (scratch.status != LSA_OK) return scratch.status;
    ScoredOut so{token_offset, (int32_t)(token_offset / p.pool), kb_cap, scores, blocks, count};
    int st = launch_query_latent(Q, index->W, p.batch, nq, sp.hq, p.hkv, p.d, p.r, p.dtype, qbar, s);
    if (st == LSA_OK)
        st = launch_select_tree(index, params, qbar, nq, q_pos, q_pos0, nullptr, nullptr, 0, s, nullptr, &so, scratch);
    scratch.release();
    return st;
}

int lsa_merge_selection(int32_t parts, const float* scores, const int32_t* blocks, const int32_t* count,
                        int32_t kb_cap, int64_t batch, int64_t nq, int32_t hkv, const int64_t* q_pos, int64_t q_pos0,
                        int32_t pool, int32_t topk, int32_t sink, int32_t window, int32_t* idx, int32_t* cnt,
                        int32_t max_sel, void* stream) {
    if (parts < 1 || parts > 64 || kb_cap < 1 || (int64_t)parts * kb_cap > 16384) return LSA_ERR_INVALID_ARG;
    if (batch < 1 || nq < 0 || hkv < 1 || pool < 1 || pool > 16 || topk < 0 || sink < 0 || window < 1)
        return LSA_ERR_INVALID_ARG;
    const int64_t kb = ((int64_t)topk + pool - 1) / pool;
    if (kb > (int64_t)parts * kb_cap || (int64_t)max_sel < kb * pool + sink + window) return LSA_ERR_INVALID_ARG;
    if (batch * nq * hkv > INT32_MAX) return LSA_ERR_INVALID_ARG;
    if (!q_pos && (q_pos0 < 0 || q_pos0 + nq > INT32_MAX)) return LSA_ERR_INVALID_ARG;
    if (nq == 0) return LSA_OK;
    if (!is_device_ptr(scores) || !is_device_ptr(blocks) || !is_device_ptr(count) || !is_device_ptr(idx) ||
        !is_device_ptr(cnt))
        return LSA_ERR_INVALID_ARG;
    if (q_pos && !is_device_ptr(q_pos)) return LSA_ERR_INVALID_ARG;
    return launch_merge_selection(parts, scores, blocks, count, kb_cap, batch, nq, hkv, q_pos, q_pos0, pool, (int)kb,
                                  sink, window, idx, cnt, max_sel, as_stream(stream));
}

int lsa_localize_rows(const int32_t* idx, const int32_t* cnt, int64_t rows, int32_t max_sel, int64_t lo, int64_t hi,
                      int32_t* idx_out, int32_t* cnt_out, void* stream) {
    if (rows < 0 || max_sel < 1 || lo < 0 || hi < lo || rows > ((int64_t)1 << 36)) return LSA_ERR_INVALID_ARG;
    if (rows == 0) return LSA_OK;
    if (!is_device_ptr(idx) || !is_device_ptr(cnt) || !is_device_ptr(idx_out) || !is_device_ptr(cnt_out))
        return LSA_ERR_INVALID_ARG;
    // idx_out is idx, or does not overlap it
    const int64_t bytes = rows * max_sel * (int64_t)sizeof(int32_t);
    const char* a = reinterpret_cast<const char*>(idx);
    const char* b = reinterpret_cast<const char*>(idx_out);
    if (a != b && a < b + bytes && b < a + bytes) return LSA_ERR_INVALID_ARG;
    return launch_localize_rows(idx, cnt, rows, max_sel, lo, hi, idx_out, cnt_out, as_stream(stream));
}

int lsa_merge_attn(int32_t parts, const void* O_parts, const float* lse_parts, int64_t rows, int32_t hq, int32_t d,
                   int32_t dtype, void* O, float* lse, void* stream) {
    if (parts < 1 || rows < 0 || hq < 1 || d < 1 || d > 1024 || (dtype != LSA_F32 && dtype != LSA_BF16))
        return LSA_ERR_INVALID_ARG;
    if (rows * hq > ((int64_t)1 << 36)) return LSA_ERR_INVALID_ARG;
    if (rows == 0) return LSA_OK;
    if (!is_device_ptr(O_parts) || !is_device_ptr(lse_parts) || !is_device_ptr(O)) return LSA_ERR_INVALID_ARG;
    if (lse && !is_device_ptr(lse)) return LSA_ERR_INVALID_ARG;
    return launch_merge_attn(parts, O_parts, lse_parts, rows, hq, d, dtype, O, lse, as_stream(stream));
}

int lsa_sparse_attn(const void* Q, const void* K, const void* V, const int32_t* idx, const int32_t* cnt,
                    int64_t batch, int64_t nq, int32_t hq, int32_t hkv, int32_t d, int32_t dtype, int32_t max_sel,
                    int64_t ld_tokens, void* O, float* lse, void* stream) {
    if (batch < 1 || nq < 0 || hkv < 1 || hq < hkv || hq % hkv || !valid_d(d) || max_sel < 1 || ld_tokens < 1)
        return LSA_ERR_INVALID_ARG;
    if (dtype != LSA_F32 && dtype != LSA_BF16) return LSA_ERR_INVALID_ARG;
    if (batch * hkv > 65535 || nq > INT32_MAX) return LSA_ERR_INVALID_ARG;
    if (nq == 0) return LSA_OK;
    if (!is_device_ptr(Q) || !is_device_ptr(K) || !is_device_ptr(V) || !is_device_ptr(idx) || !is_device_ptr(cnt) ||
        !is_device_ptr(O))
        return LSA_ERR_INVALID_ARG;
    if (lse && !is_device_ptr(lse)) return LSA_ERR_INVALID_ARG;
    if (!attn_aligned(dtype, Q, K, V, O)) return LSA_ERR_INVALID_ARG;
    return launch_sparse_attn(Q, K, V, idx, cnt, batch, nq, hq, hkv, d, dtype, max_sel, ld_tokens, O, lse,
                              global_err_word(), as_stream(stream));
}

int lsa_sparse_attn_banded(const void* Q, const void* K, const void* V, const int32_t* idx, const int32_t* cnt,
                           int64_t batch, int64_t nq, int64_t q_pos0, int32_t hq, int32_t hkv, int32_t d,
                           int32_t dtype, int32_t max_sel, int64_t ld_tokens, int32_t sink, int32_t window, void* O,
                           float* lse, void* stream) {
    if (batch < 1 || nq < 0 || hkv < 1 || hq < hkv || hq % hkv || !valid_d(d) || max_sel < 1 || ld_tokens < 1)
        return LSA_ERR_INVALID_ARG;
    if (dtype != LSA_F32 && dtype != LSA_BF16) return LSA_ERR_INVALID_ARG;
    if (batch * hkv > 65535 || nq > INT32_MAX) return LSA_ERR_INVALID_ARG;
    if (q_pos0 < 0 || q_pos0 + nq > ld_tokens || sink < 0 || window < 1) return LSA_ERR_INVALID_ARG;
    if (nq == 0) return LSA_OK;
    if (!is_device_ptr(Q) || !is_device_ptr(K) || !is_device_ptr(V) || !is_device_ptr(idx) || !is_device_ptr(cnt) ||
        !is_device_ptr(O))
        return LSA_ERR_INVALID_ARG;
    if (lse && !is_device_ptr(lse)) return LSA_ERR_INVALID_ARG;
    if (!attn_aligned(dtype, Q, K, V, O)) return LSA_ERR_INVALID_ARG;
    const int G = hq / hkv;
    if (dtype == LSA_BF16 && (G == 1 || G == 2 || G == 4 || G == 8 || G == 16))
        return launch_banded_attn(Q, K, V, idx, cnt, batch, nq, q_pos0, hq, hkv, d, max_sel, ld_tokens, sink, window,
                                  O, lse, global_err_word(), as_stream(stream));
    return launch_sparse_attn(Q, K, V, idx, cnt, batch, nq, hq, hkv, d, dtype, max_sel, ld_tokens, O, lse,
                              global_err_word(), as_stream(stream));
}

int lsa_append(lsa_index* index, const void* K, int64_t n_new, void* stream) {
    if (!live(index) || n_new < 0) return LSA_ERR_INVALID_ARG;
    const lsa_build_params& p = index->p;
    if (index->n_tokens + n_new > p.n_tokens + p.append_capacity) return LSA_ERR_INVALID_ARG;
    if (n_new == 0) return LSA_OK;
    if (!is_device_ptr(K)) return LSA_ERR_INVALID_ARG;
    const int64_t new_tokens = index->n_tokens + n_new;
    const int64_t first = index->nb;
    const int64_t nb_new = new_tokens / p.pool;
    int st = launch_append(index, K, first, nb_new - first, as_stream(stream));
    if (st != LSA_OK) return st;
    index->n_tokens = new_tokens;
    index->nb = nb_new;
    return LSA_OK;
}

int lsa_relayout(lsa_index* index, void* stream) {
    if (!live(index)) return LSA_ERR_INVALID_ARG;
    Arena scratch;
    scratch.async = true;
    scratch.stream = as_stream(stream);
    int st = relayout_leaves(index, as_stream(stream), scratch);
    scratch.release();
    return st != LSA_OK ? st : cuda_status(cudaGetLastError());
}

int lsa_refresh_centroids(lsa_index* index, void* stream) {
    if (!live(index)) return LSA_ERR_INVALID_ARG;
    Arena scratch;
    scratch.async = true;
    scratch.stream = as_stream(stream);
    int st = refresh_centroids(index, as_stream(stream), scratch);
    scratch.release();
    return st != LSA_OK ? st : cuda_status(cudaGetLastError());
}

int lsa_project_pool(const void* K, const float* W, int64_t batch, int64_t n_tokens, int64_t ld_tokens, int32_t hkv,
                     int32_t d, int32_t r, int32_t pool, int32_t dtype, float* Kl, void* stream) {
    if (batch < 1 || n_tokens < 0 || ld_tokens < n_tokens || hkv < 1 || !valid_d(d) || !valid_r(r) || pool < 1 ||
        (dtype != LSA_F32 && dtype != LSA_BF16) || batch * hkv > 65535)
        return LSA_ERR_INVALID_ARG;
    const int64_t nb = n_tokens / pool;
    if (nb == 0) return LSA_OK;
    if (!is_device_ptr(K) || !is_device_ptr(W) || !is_device_ptr(Kl)) return LSA_ERR_INVALID_ARG;
    return launch_project_pool(K, W, batch, nb, ld_tokens, hkv, d, r, pool, dtype, Kl, nb, as_stream(stream));
}

int lsa_query_latent(const void* Q, const float* W, int64_t batch, int64_t nq, int32_t hq, int32_t hkv, int32_t d,
                     int32_t r, int32_t dtype, float* qbar, void* stream) {
    if (batch < 1 || nq < 0 || hkv < 1 || hq < hkv || hq % hkv || !valid_d(d) || !valid_r(r) ||
        (dtype != LSA_F32 && dtype != LSA_BF16) || batch * hkv > 65535)
        return LSA_ERR_INVALID_ARG;
    if (nq == 0) return LSA_OK;
    if (!is_device_ptr(Q) || !is_device_ptr(W) || !is_device_ptr(qbar)) return LSA_ERR_INVALID_ARG;
    return launch_query_latent(Q, W, batch, nq, hq, hkv, d, r, dtype, qbar, as_stream(stream));
}

int lsa_pca_map(const void* K, int64_t batch, int64_t n_tokens, int64_t ld_tokens, int32_t hkv, int32_t d,
                int32_t pool, int32_t dtype, int32_t r, float* W, double* eigvals, void* stream) {
    if (batch < 1 || n_tokens < 0 || ld_tokens < n_tokens || hkv < 1 || (d != 64 && d != 128) || pool < 1 ||
        (dtype != LSA_F32 && dtype != LSA_BF16) || r < 1 || r > d || batch * hkv > 65535)
        return LSA_ERR_INVALID_ARG;
    if (n_tokens / pool < 1 || batch * hkv * (n_tokens / pool) > ((int64_t)1 << 40)) return LSA_ERR_INVALID_ARG;
    if (!is_device_ptr(K) || !is_device_ptr(W)) return LSA_ERR_INVALID_ARG;
    if (eigvals && !is_device_ptr(eigvals)) return LSA_ERR_INVALID_ARG;
    return launch_pca_map(K, batch, n_tokens, ld_tokens, hkv, d, pool, dtype, r, W, eigvals, as_stream(stream));
}

int lsa_kmeans(const float* X, int64_t units, int64_t n, int32_t r, int32_t k, int32_t iters, int32_t grid_log2,
               int32_t* labels, float* C, const float* C_init, double* objective, void* stream) {
    if (units < 1 || units > 65535 || n < 1 || !valid_r(r) || k < 1 || iters < 1 || grid_log2 < 0 || grid_log2 > 8)
        return LSA_ERR_INVALID_ARG;
    if (units * n > INT32_MAX / 2 || units * (int64_t)k > INT32_MAX / 4) return LSA_ERR_INVALID_ARG;
    if (!is_device_ptr(X) || !is_device_ptr(labels) || !is_device_ptr(C)) return LSA_ERR_INVALID_ARG;
    if (objective && !is_device_ptr(objective)) return LSA_ERR_INVALID_ARG;
    if (C_init) {
        const int64_t bytes = units * (int64_t)k * r * (int64_t)sizeof(float);
        const char* a = reinterpret_cast<const char*>(C_init);
        const char* b = reinterpret_cast<const char*>(C);
        if (!is_device_ptr(C_init) || (a < b + bytes && b < a + bytes)) return LSA_ERR_INVALID_ARG;
    }
    cudaStream_t s = as_stream(stream);
    Arena scratch;
    scratch.async = true;
    scratch.stream = s;
    KmeansOut ko{labels, C, nullptr, nullptr, objective};
    int st = run_kmeans(X, n, units, n, r, k, iters, grid_log2, ko, n, global_err_word(), s, scratch, C_init);
    scratch.release();
    return st;
}

int lsa_index_info(const lsa_index* ix, lsa_index_info_t* out) {
    if (!live(ix) || !out) return LSA_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof(*out));
    out->units = ix->units;
    out->n_tokens = ix->n_tokens;
    out->n_blocks = ix->nb;
    out->block_capacity = ix->nb_cap;
    out->device_bytes = ix->mem->bytes;
    out->levels = ix->p.levels;
    for (int l = 0; l < ix->p.levels; ++l) out->level_sizes[l] = ix->p.level_sizes[l];
    out->r = ix->p.r;
    out->pool = ix->p.pool;
    out->sink = ix->p.sink;
    out->grid_log2 = ix->p.grid_log2;
    return LSA_OK;
}

int lsa_index_get(const lsa_index* ix, int32_t what, int32_t level, void* dst, int64_t dst_bytes, void* stream) {
    if (!live(ix) || !dst) return LSA_ERR_INVALID_ARG;
    const lsa_build_params& p = ix->p;
    const int64_t U = ix->units;
    cudaStream_t s = as_stream(stream);
    const bool lvl_ok = level >= 0 && level < p.levels;
    int64_t bytes = 0;
    cudaError_t e = cudaSuccess;
    switch (what) {
        case LSA_GET_CENTROIDS:
            if (!lvl_ok) return LSA_ERR_INVALID_ARG;
            bytes = U * p.level_sizes[level] * p.r * (int64_t)sizeof(float);
            if (dst_bytes < bytes) return LSA_ERR_INVALID_ARG;
            e = cudaMemcpyAsync(dst, ix->cent[level], bytes, cudaMemcpyDefault, s);
            break;
        case LSA_GET_PARENT:
            if (!lvl_ok || level == 0) return LSA_ERR_INVALID_ARG;
            bytes = U * p.level_sizes[level] * (int64_t)sizeof(int32_t);
            if (dst_bytes < bytes) return LSA_ERR_INVALID_ARG;
            e = cudaMemcpyAsync(dst, ix->parent[level], bytes, cudaMemcpyDefault, s);
            break;
        case LSA_GET_MINPOS:
            if (!lvl_ok) return LSA_ERR_INVALID_ARG;
            bytes = U * p.level_sizes[level] * (int64_t)sizeof(int64_t);
            if (dst_bytes < bytes) return LSA_ERR_INVALID_ARG;
            e = cudaMemcpyAsync(dst, ix->minpos[level], bytes, cudaMemcpyDefault, s);
            break;
        case LSA_GET_OBJECTIVE:
            if (!lvl_ok) return LSA_ERR_INVALID_ARG;
            bytes = (int64_t)p.lloyd_iters * U * (int64_t)sizeof(double);
            if (dst_bytes < bytes) return LSA_ERR_INVALID_ARG;
            e = cudaMemcpyAsync(dst, ix->objective[level], bytes, cudaMemcpyDefault, s);
            break;
        case LSA_GET_LEAF_OF_BLOCK:
        case LSA_GET_LATENT: {
            const int64_t w = what == LSA_GET_LATENT ? p.r * (int64_t)sizeof(float) : (int64_t)sizeof(int32_t);
            bytes = U * ix->nb * w;
            if (dst_bytes < bytes) return LSA_ERR_INVALID_ARG;
            const char* src = what == LSA_GET_LATENT ? (const char*)ix->Kl : (const char*)ix->leaf_of_block;
            e = cudaMemcpy2DAsync(dst, ix->nb * w, src, ix->nb_cap * w, ix->nb * w, U, cudaMemcpyDefault, s);
            break;
        }
        case LSA_GET_LEAF_COUNT:
            bytes = U * ix->L * (int64_t)sizeof(int32_t);
            if (dst_bytes < bytes) return LSA_ERR_INVALID_ARG;
            e = cudaMemcpyAsync(dst, ix->leaf_cnt, bytes, cudaMemcpyDefault, s);
            break;
        default:
            return LSA_ERR_INVALID_ARG;
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return cuda_status(e);
}

int lsa_check(lsa_index* ix, void* stream) {
    cudaStream_t s = as_stream(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e);
    int32_t* w = nullptr;
    if (ix) {
        if (!live(ix)) return LSA_ERR_INVALID_ARG;
        w = ix->err;
    } else {
        w = global_err_word();
    }
    if (!w) return LSA_ERR_CUDA;
    int32_t bits = 0;
    e = cudaMemcpy(&bits, w, sizeof(int32_t), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
    if (bits) {
        cudaMemset(w, 0, sizeof(int32_t));
        cudaDeviceSynchronize();
    }
    return err_bits_to_status(bits);
}

void lsa_free_index(lsa_index* ix) {
    if (!live(ix)) return;
    destroy_index(ix);
}

const char* lsa_strerror(int status) {
    switch (status) {
        case LSA_OK: return "ok";
        case LSA_ERR_INVALID_ARG: return "invalid argument";
        case LSA_ERR_CUDA: return "CUDA runtime error";
        case LSA_ERR_OOM: return "device allocation failed";
        case LSA_ERR_INEXACT: return "integer-grid value outside the exact range";
        case LSA_ERR_TIMEOUT: return "bounded device wait gave up";
        case LSA_ERR_DEVICE: return "kernel met an out-of-range index";
        case LSA_ERR_CAPACITY: return "leaf has no free slot for an appended block";
        default: return "unknown status";
    }
}

void lsa_debug_fail_alloc_after(int32_t n) { g_fail_after.store(n > 0 ? n : 0); }

int64_t lsa_launch_count(void) { return g_launches.load(); }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free selection.  The scratch of lsa_select (the latent queries)
// lives in a fixed device array here, for callers that cannot allocate while
// they serve.  In host code g_noalloc_qbar only stands in for the device
// variable: kernels receive the address cudaGetSymbolAddress returns for the
// current device.
namespace {

static __device__ __align__(256) float g_noalloc_qbar[LSA_SELECT_NOALLOC_MAX_FLOATS];

std::mutex g_noalloc_mu;
float* g_noalloc_ptr[128] = {nullptr};

// Device address of g_noalloc_qbar on the current device, looked up once per
// device with that device current.
int noalloc_scratch(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= 128) return LSA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_qbar);
        if (e != cudaSuccess) return cuda_status(e);
        g_noalloc_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_noalloc_ptr[dev];
    return LSA_OK;
}

}  // namespace

extern "C" int lsa_select_noalloc(const lsa_index* index, const lsa_select_params* params, const void* Q,
                                  int64_t nq, const int64_t* q_pos, int64_t q_pos0, int32_t* idx, int32_t* cnt,
                                  int32_t max_sel, void* stream) {
    int st = check_select(index, params, Q, nq, q_pos, q_pos0, idx, cnt, max_sel);
    if (st != LSA_OK || nq == 0) return st;
    const lsa_build_params& p = index->p;
    if (p.batch * nq * p.hkv * (int64_t)p.r > LSA_SELECT_NOALLOC_MAX_FLOATS) return LSA_ERR_INVALID_ARG;
    float* qbar = nullptr;
    st = noalloc_scratch(&qbar);
    if (st != LSA_OK) return st;
    cudaStream_t s = as_stream(stream);
    st = launch_query_latent(Q, index->W, p.batch, nq, params->hq, p.hkv, p.d, p.r, p.dtype, qbar, s);
    if (st == LSA_OK) st = launch_select(index, params, qbar, nq, q_pos, q_pos0, idx, cnt, max_sel, false, s);
    return st;
}
