// Context parallelism: one sequence's context split over shards (ranks).
//
// The 10M-token runs on the pages split one sequence over several GPUs (LSA
// explainer, "What do 22.7x and 72.4x actually compare?" and "Can I run
// LSA?"); the pages give no algorithm, so this follows the plainest reading:
// every shard holds a contiguous token range with its own index, selects its
// local top blocks with their scores (select.cu, scored mode), the picks of all
// shards are merged into the global top blocks (select.cu, merge), and
// attention over the merged selection is computed per shard on the shard's own
// rows and combined by the log-sum-exp rule.  This file holds the two
// elementwise steps of that attention:
//   localize_kernel   rows of a selection inside [lo, hi), shifted by -lo
//   merge_attn_kernel O = sum_s exp(lse_s - m) O_s / sum_s exp(lse_s - m),
//                     lse = m + log(sum_s exp(lse_s - m)), m = max_s lse_s
#include "lsa_internal.cuh"

namespace lsa {
namespace {

// One warp per row: the entries of [lo, hi), in order, compacted by ballots.
// (idx_out may be idx itself: no __restrict__ on either)
__global__ void localize_kernel(const int32_t* idx, const int32_t* cnt, int64_t rows, int max_sel, int64_t lo,
                                int64_t hi, int32_t* idx_out, int32_t* cnt_out) {
    const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    int n = cnt[row];
    n = n < 0 ? 0 : (n > max_sel ? max_sel : n);
    const int32_t* in = idx + row * max_sel;
    int32_t* out = idx_out + row * max_sel;
    uint32_t lt;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt));
    int w = 0;
    for (int base = 0; base < n; base += 32) {
        const int e = base + lane;
        const int v = e < n ? in[e] : -1;
        const bool keep = e < n && v >= lo && v < hi;
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        // (every lane has read its entry before any lane writes: out may be in)
        __syncwarp();
        if (keep) out[w + __popc(bal & lt)] = (int32_t)(v - lo);
        w += __popc(bal);
    }
    for (int e = w + lane; e < max_sel; e += 32) out[e] = -1;
    if (lane == 0) cnt_out[row] = w;
}

__device__ __forceinline__ float ldf(const float* p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stf(float* p, float v) { *p = v; }
__device__ __forceinline__ void stf(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// One warp per (query, head): parts summed in order s = 0, 1, ...
template <typename T>
__global__ void merge_attn_kernel(int parts, const T* __restrict__ Op, const float* __restrict__ lsep,
                                  int64_t rh, int d, T* __restrict__ O, float* __restrict__ lse) {
    const int64_t g = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (g >= rh) return;
    float m = -INFINITY;
    for (int s = 0; s < parts; ++s) m = fmaxf(m, lsep[(int64_t)s * rh + g]);
    T* o = O + g * d;
    if (m == -INFINITY) {
        for (int k = lane; k < d; k += 32) stf(o + k, 0.f);
        if (lse && lane == 0) lse[g] = -INFINITY;
        return;
    }
    float den = 0.f;
    for (int s = 0; s < parts; ++s) den += expf(lsep[(int64_t)s * rh + g] - m);
    const float inv = 1.f / den;
    for (int k = lane; k < d; k += 32) {
        float acc = 0.f;
        for (int s = 0; s < parts; ++s) {
            const float wgt = expf(lsep[(int64_t)s * rh + g] - m);
            acc = fmaf(wgt, ldf(Op + ((int64_t)s * rh + g) * d + k), acc);
        }
        stf(o + k, acc * inv);
    }
    if (lse && lane == 0) lse[g] = m + logf(den);
}

}  // namespace

int launch_localize_rows(const int32_t* idx, const int32_t* cnt, int64_t rows, int max_sel, int64_t lo, int64_t hi,
                         int32_t* idx_out, int32_t* cnt_out, cudaStream_t s) {
    if (rows <= 0) return LSA_OK;
    const int threads = 256;
    const int64_t blocks = (rows * 32 + threads - 1) / threads;
    note_launch();
    localize_kernel<<<(unsigned)blocks, threads, 0, s>>>(idx, cnt, rows, max_sel, lo, hi, idx_out, cnt_out);
    return cuda_status(cudaGetLastError());
}

int launch_merge_attn(int parts, const void* O_parts, const float* lse_parts, int64_t rows, int hq, int d, int dtype,
                      void* O, float* lse, cudaStream_t s) {
    const int64_t rh = rows * hq;
    if (rh <= 0) return LSA_OK;
    const int threads = 256;
    const int64_t blocks = (rh * 32 + threads - 1) / threads;
    note_launch();
    if (dtype == LSA_F32)
        merge_attn_kernel<float><<<(unsigned)blocks, threads, 0, s>>>(parts, (const float*)O_parts, lse_parts, rh,
                                                                      d, (float*)O, lse);
    else
        merge_attn_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, s>>>(
            parts, (const __nv_bfloat16*)O_parts, lse_parts, rh, d, (__nv_bfloat16*)O, lse);
    return cuda_status(cudaGetLastError());
}

}  // namespace lsa
