// Arithmetic shared by every place that forms a latent vector, so that the
// build, the query path and the decode append round identically.
#pragma once

#include "lsa_internal.cuh"

namespace lsa {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Mean of M values spaced `stride` elements apart: summed in order, then one
// IEEE division.
template <typename T>
__device__ __forceinline__ float mean_of_rows(const T* p, int64_t stride, int M) {
    float s = 0.f;
    for (int m = 0; m < M; ++m) s = __fadd_rn(s, to_f32(p[(int64_t)m * stride]));
    return __fdiv_rn(s, (float)M);
}

// Output o of mean (length d) times W [d][r]: one fma chain over inputs in order.
__device__ __forceinline__ float latent_dot(const float* mean, const float* W, int d, int r, int o) {
    float acc = 0.f;
    for (int k = 0; k < d; ++k) acc = __fmaf_rn(mean[k], W[k * r + o], acc);
    return acc;
}

}  // namespace lsa
