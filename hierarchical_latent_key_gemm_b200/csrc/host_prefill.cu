// One prefill layer from host memory in one C-ABI call (lsa_prefill_run): the
// layer of the LSA explainer's "How does LSA work?" steps 1-3 (build the
// bucket hierarchy, select per query, attend exactly over the selection),
// with the host-device copies on their own streams so that they overlap the
// kernels.  Host code only: the arithmetic is in the build, select and
// attention calls it enqueues.
//
// Streams of a context: s_in copies K and W up, then V, then the queries in
// chunks; s_comp builds the index once K and W are up and, chunk by chunk,
// selects and attends as soon as a chunk's queries have arrived; s_out copies
// each chunk's output down while the next chunk computes.  Every copy is one
// cudaMemcpyAsync.
#include <cuda_runtime.h>

#include <algorithm>
#include <new>
#include <vector>

#include "lsa_internal.cuh"

struct lsa_prefill {
    lsa_build_params bp;
    lsa_select_params sp;
    int device = 0;
    int64_t nq = 0;
    int32_t max_sel = 0;
    size_t es = 0;                    // bytes per element of Q, K, V, O
    std::vector<int64_t> bounds;      // chunk c holds queries [bounds[c], bounds[c+1])
    void* dQ = nullptr;
    void* dK = nullptr;
    void* dV = nullptr;
    void* dO = nullptr;
    float* dW = nullptr;
    float* dlse = nullptr;
    int32_t* idx = nullptr;
    int32_t* cnt = nullptr;
    cudaStream_t st[3] = {nullptr, nullptr, nullptr};   // in, comp, out
    cudaEvent_t start = nullptr, ev_kw = nullptr, ev_v = nullptr;
    cudaEvent_t done[3] = {nullptr, nullptr, nullptr};  // end of the last run, per stream
    std::vector<cudaEvent_t> q_ev, o_ev;
};

namespace {

void destroy(lsa_prefill* pf) {
    for (cudaStream_t s : pf->st)
        if (s) cudaStreamSynchronize(s);
    for (void* p : {pf->dQ, pf->dK, pf->dV, pf->dO, (void*)pf->dW, (void*)pf->dlse, (void*)pf->idx, (void*)pf->cnt})
        if (p) cudaFree(p);
    for (cudaEvent_t e : {pf->start, pf->ev_kw, pf->ev_v, pf->done[0], pf->done[1], pf->done[2]})
        if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : pf->q_ev)
        if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : pf->o_ev)
        if (e) cudaEventDestroy(e);
    for (cudaStream_t s : pf->st)
        if (s) cudaStreamDestroy(s);
    delete pf;
}

// `stream` waits for everything the context's streams have been given
int join(lsa_prefill* pf, cudaStream_t stream) {
    for (int i = 0; i < 3; ++i) {
        cudaError_t e = cudaEventRecord(pf->done[i], pf->st[i]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, pf->done[i], 0);
        if (e != cudaSuccess) return lsa::cuda_status(e);
    }
    return LSA_OK;
}

int alloc(void** p, size_t bytes) {
    cudaError_t e = cudaMalloc(p, bytes > 0 ? bytes : 16);
    if (e == cudaErrorMemoryAllocation) {
        cudaGetLastError();
        *p = nullptr;
        return LSA_ERR_OOM;
    }
    return e == cudaSuccess ? LSA_OK : lsa::cuda_status(e);
}

}  // namespace

extern "C" int lsa_prefill_create(const lsa_build_params* bp, const lsa_select_params* sp, int64_t nq,
                                  int32_t chunks, lsa_prefill** out) {
    if (!out) return LSA_ERR_INVALID_ARG;
    *out = nullptr;
    if (!bp || !sp || bp->batch != 1 || nq < 1 || nq > bp->n_tokens || bp->ld_tokens < bp->n_tokens ||
        chunks < 1 || bp->hkv < 1 || bp->d < 1 || bp->r < 1 || bp->pool < 1 || sp->hq < 1 ||
        sp->hq % bp->hkv != 0 || sp->topk < 0 || sp->sink < 0 || sp->window < 1 ||
        (bp->dtype != LSA_F32 && bp->dtype != LSA_BF16))
        return LSA_ERR_INVALID_ARG;
    const int64_t max_sel = (sp->topk + bp->pool - 1) / bp->pool * bp->pool + sp->sink + sp->window;
    if (max_sel > INT32_MAX) return LSA_ERR_INVALID_ARG;
    lsa_prefill* pf = new (std::nothrow) lsa_prefill();
    if (!pf) return LSA_ERR_OOM;
    pf->bp = *bp;
    pf->sp = *sp;
    pf->nq = nq;
    pf->max_sel = (int32_t)max_sel;
    pf->es = bp->dtype == LSA_BF16 ? 2 : 4;
    const int64_t nc = chunks < nq ? chunks : nq;
    for (int64_t c = 0; c <= nc; ++c) pf->bounds.push_back(nq * c / nc);
    int64_t cmax = 0;
    for (int64_t c = 0; c < nc; ++c) cmax = std::max(cmax, pf->bounds[c + 1] - pf->bounds[c]);
    int st = lsa::cuda_status(cudaGetDevice(&pf->device));
    const size_t kv = (size_t)bp->ld_tokens * bp->hkv * bp->d * pf->es;
    const size_t qo = (size_t)nq * sp->hq * bp->d * pf->es;
    if (st == LSA_OK) st = alloc(&pf->dK, kv);
    if (st == LSA_OK) st = alloc(&pf->dV, kv);
    if (st == LSA_OK) st = alloc(&pf->dQ, qo);
    if (st == LSA_OK) st = alloc(&pf->dO, qo);
    if (st == LSA_OK) st = alloc((void**)&pf->dW, (size_t)bp->d * bp->r * sizeof(float));
    if (st == LSA_OK) st = alloc((void**)&pf->dlse, (size_t)nq * sp->hq * sizeof(float));
    if (st == LSA_OK) st = alloc((void**)&pf->idx, (size_t)cmax * bp->hkv * max_sel * sizeof(int32_t));
    if (st == LSA_OK) st = alloc((void**)&pf->cnt, (size_t)cmax * bp->hkv * sizeof(int32_t));
    for (int i = 0; i < 3 && st == LSA_OK; ++i)
        st = lsa::cuda_status(cudaStreamCreateWithFlags(&pf->st[i], cudaStreamNonBlocking));
    for (cudaEvent_t* e : {&pf->start, &pf->ev_kw, &pf->ev_v, &pf->done[0], &pf->done[1], &pf->done[2]})
        if (st == LSA_OK) st = lsa::cuda_status(cudaEventCreateWithFlags(e, cudaEventDisableTiming));
    pf->q_ev.assign(nc, nullptr);
    pf->o_ev.assign(nc, nullptr);
    for (int64_t c = 0; c < nc && st == LSA_OK; ++c) {
        st = lsa::cuda_status(cudaEventCreateWithFlags(&pf->q_ev[c], cudaEventDisableTiming));
        if (st == LSA_OK) st = lsa::cuda_status(cudaEventCreateWithFlags(&pf->o_ev[c], cudaEventDisableTiming));
    }
    if (st != LSA_OK) {
        destroy(pf);
        return st;
    }
    *out = pf;
    return LSA_OK;
}

extern "C" int lsa_prefill_run(lsa_prefill* pf, const void* hQ, const void* hK, const void* hV, const float* hW,
                               void* hO, float* hlse, void* stream, lsa_index** index_out) {
    if (index_out) *index_out = nullptr;
    if (!pf || !hQ || !hK || !hV || !hW || !hO || !index_out) return LSA_ERR_INVALID_ARG;
    int dev = -1;
    int st = lsa::cuda_status(cudaGetDevice(&dev));
    if (st != LSA_OK) return st;
    if (dev != pf->device) return LSA_ERR_INVALID_ARG;
    const cudaStream_t s = (cudaStream_t)stream;
    cudaStream_t s_in = pf->st[0], s_comp = pf->st[1], s_out = pf->st[2];
    const lsa_build_params& bp = pf->bp;
    const lsa_select_params& sp = pf->sp;
    const size_t kv = (size_t)bp.ld_tokens * bp.hkv * bp.d * pf->es;
    const size_t qrow = (size_t)sp.hq * bp.d * pf->es;   // bytes of one query position (all heads)
    cudaError_t e = cudaEventRecord(pf->start, s);
    // every stream waits for the caller's stream and for the previous run on
    // this context (its buffers are reused), whatever stream that was issued on
    for (int i = 0; i < 3 && e == cudaSuccess; ++i) {
        e = cudaStreamWaitEvent(pf->st[i], pf->start, 0);
        for (int j = 0; j < 3 && e == cudaSuccess; ++j) e = cudaStreamWaitEvent(pf->st[i], pf->done[j], 0);
    }
    // up: K and W first (the build needs them), V during the build, then the queries chunk by chunk
    if (e == cudaSuccess) e = cudaMemcpyAsync(pf->dK, hK, kv, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(pf->dW, hW, (size_t)bp.d * bp.r * sizeof(float), cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaEventRecord(pf->ev_kw, s_in);
    if (e == cudaSuccess) e = cudaMemcpyAsync(pf->dV, hV, kv, cudaMemcpyHostToDevice, s_in);
    if (e == cudaSuccess) e = cudaEventRecord(pf->ev_v, s_in);
    const size_t nc = pf->q_ev.size();
    for (size_t c = 0; c < nc && e == cudaSuccess; ++c) {
        const int64_t a = pf->bounds[c], n = pf->bounds[c + 1] - a;
        e = cudaMemcpyAsync((char*)pf->dQ + a * qrow, (const char*)hQ + a * qrow, n * qrow, cudaMemcpyHostToDevice,
                            s_in);
        if (e == cudaSuccess) e = cudaEventRecord(pf->q_ev[c], s_in);
    }
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_comp, pf->ev_kw, 0);
    if (e != cudaSuccess) {
        join(pf, s);
        return lsa::cuda_status(e);
    }
    lsa_index* ix = nullptr;
    st = lsa_build_index(&bp, pf->dK, pf->dW, s_comp, &ix);
    if (st == LSA_OK) st = lsa::cuda_status(cudaStreamWaitEvent(s_comp, pf->ev_v, 0));
    for (size_t c = 0; c < nc && st == LSA_OK; ++c) {
        const int64_t a = pf->bounds[c], n = pf->bounds[c + 1] - a;
        const void* q = (const char*)pf->dQ + a * qrow;
        void* o = (char*)pf->dO + a * qrow;
        float* lse = pf->dlse + a * sp.hq;
        st = lsa::cuda_status(cudaStreamWaitEvent(s_comp, pf->q_ev[c], 0));
        if (st == LSA_OK)
            st = lsa_select(ix, &sp, q, n, nullptr, a, pf->idx, pf->cnt, pf->max_sel, s_comp);
        if (st == LSA_OK)
            st = lsa_sparse_attn_banded(q, pf->dK, pf->dV, pf->idx, pf->cnt, 1, n, a, sp.hq, bp.hkv, bp.d, bp.dtype,
                                        pf->max_sel, bp.ld_tokens, sp.sink, sp.window, o, lse, s_comp);
        // down: this chunk's output while the next one computes
        if (st == LSA_OK) st = lsa::cuda_status(cudaEventRecord(pf->o_ev[c], s_comp));
        if (st == LSA_OK) st = lsa::cuda_status(cudaStreamWaitEvent(s_out, pf->o_ev[c], 0));
        if (st == LSA_OK)
            st = lsa::cuda_status(cudaMemcpyAsync((char*)hO + a * qrow, o, n * qrow, cudaMemcpyDeviceToHost, s_out));
        if (st == LSA_OK && hlse)
            st = lsa::cuda_status(cudaMemcpyAsync(hlse + a * sp.hq, lse, (size_t)n * sp.hq * sizeof(float),
                                                  cudaMemcpyDeviceToHost, s_out));
    }
    const int sj = join(pf, s);
    if (st == LSA_OK) st = sj;
    if (st != LSA_OK) {
        if (ix) {
            cudaStreamSynchronize(s_comp);
            lsa_free_index(ix);
        }
        return st;
    }
    *index_out = ix;
    return LSA_OK;
}

extern "C" void lsa_prefill_free(lsa_prefill* pf) {
    if (pf) destroy(pf);
}
