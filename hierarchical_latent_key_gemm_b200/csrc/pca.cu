// Training-free latent map: W = the r leading principal directions of the
// pooled keys (LSA explainer, "How does LSA work?": one of the D-LSA options
// needs no training and takes its map from a PCA).
//
// Pooled keys of every (sequence, KV head) form one sample; their covariance
// (centred, divided by the count) is accumulated in fp64 and diagonalised by a
// parallel cyclic Jacobi method; the eigenvectors of the r largest
// eigenvalues, in descending order, are the columns of W, each signed so that
// its entry of largest magnitude (lowest index among equal magnitudes) is
// positive.
//
//   pca_gram_kernel   each CTA pools a run of blocks (fp64 mean of the block's
//                     keys) and accumulates sum(x) and x x^T over
//                     them in fp64 registers (one T x T tile of the D x D Gram
//                     per thread), then adds them to the global sums atomically
//   pca_jacobi_kernel one CTA: C = G / n - mu mu^T in shared memory (fp64),
//                     sweeps of n - 1 rounds of n / 2 disjoint rotations
//                     (round-robin pairing) until the off-diagonal mass is
//                     below 1e-30 of the total (or 40 sweeps); V^T accumulates the
//                     rotations in global memory; then the top-r selection and
//                     the sign convention
#include "latent_common.cuh"

namespace lsa {
namespace {

constexpr int kGramThreads = 256;   // 16 x 16 tiles
constexpr int kGramRows = 8;        // pooled rows staged per pass
constexpr int kJacThreads = 1024;

template <typename T, int D>
__global__ __launch_bounds__(kGramThreads) void pca_gram_kernel(const T* __restrict__ K, int64_t units, int64_t nb,
                                                               int64_t ld_tokens, int hkv, int pool,
                                                               double* __restrict__ G, double* __restrict__ S) {
    constexpr int TS = D / 16;   // tile side per thread
    __shared__ double xs[kGramRows][D];
    const int tid = threadIdx.x;
    const int ti = tid / 16, tj = tid % 16;
    double acc[TS][TS];
#pragma unroll
    for (int i = 0; i < TS; ++i)
#pragma unroll
        for (int j = 0; j < TS; ++j) acc[i][j] = 0.0;
    double sum = 0.0;   // thread t < D: sum of column t
    const int64_t total = units * nb;
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    const int64_t r0 = (int64_t)blockIdx.x * per, r1 = min(total, r0 + per);
    for (int64_t base = r0; base < r1; base += kGramRows) {
        const int nrow = (int)min((int64_t)kGramRows, r1 - base);
        for (int e = tid; e < kGramRows * D; e += kGramThreads) {
            const int rr = e / D, k = e % D;
            double v = 0.0;
            if (rr < nrow) {
                const int64_t row = base + rr;
                const int64_t u = row / nb, b = row % nb;
                const int64_t bseq = u / hkv;
                const int h = (int)(u % hkv);
                const T* p = K + ((bseq * ld_tokens + b * pool) * hkv + h) * D + k;
                for (int t = 0; t < pool; ++t) v += (double)to_f32(p[(int64_t)t * hkv * D]);
                v /= (double)pool;
            }
            xs[rr][k] = v;
        }
        __syncthreads();
        for (int rr = 0; rr < nrow; ++rr) {
            double xi[TS], xj[TS];
#pragma unroll
            for (int i = 0; i < TS; ++i) {
                xi[i] = xs[rr][ti * TS + i];
                xj[i] = xs[rr][tj * TS + i];
            }
#pragma unroll
            for (int i = 0; i < TS; ++i)
#pragma unroll
                for (int j = 0; j < TS; ++j) acc[i][j] = fma(xi[i], xj[j], acc[i][j]);
            if (tid < D) sum += xs[rr][tid];
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < TS; ++i)
#pragma unroll
        for (int j = 0; j < TS; ++j) atomicAdd(G + (int64_t)(ti * TS + i) * D + tj * TS + j, acc[i][j]);
    if (tid < D) atomicAdd(S + tid, sum);
}

template <int D>
__global__ __launch_bounds__(kJacThreads, 1) void pca_jacobi_kernel(const double* __restrict__ G,
                                                                    const double* __restrict__ S, double count, int r,
                                                                    double* __restrict__ VT, float* __restrict__ W,
                                                                    double* __restrict__ evals_out) {
    extern __shared__ double A[];                       // [D][D]
    __shared__ double cs_c[D / 2], cs_s[D / 2];
    __shared__ int pp[D / 2], qq[D / 2];
    __shared__ double red[kJacThreads / 32];
    __shared__ int order[D];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < D * D; e += kJacThreads) {
        const int i = e / D, j = e % D;
        const double mi = S[i] / count, mj = S[j] / count;
        A[e] = G[e] / count - mi * mj;
        VT[e] = i == j ? 1.0 : 0.0;
    }
    __syncthreads();
    auto offdiag = [&]() -> double2 {   // (off-diagonal mass, total mass)
        double o = 0.0, t = 0.0;
        for (int e = tid; e < D * D; e += kJacThreads) {
            const double v = A[e] * A[e];
            t += v;
            if (e / D != e % D) o += v;
        }
#pragma unroll
        for (int k = 16; k >= 1; k >>= 1) {
            o += __shfl_xor_sync(0xffffffffu, o, k);
            t += __shfl_xor_sync(0xffffffffu, t, k);
        }
        __syncthreads();
        if (lane == 0) red[warp] = o;
        __syncthreads();
        double oo = 0.0;
        for (int w = 0; w < kJacThreads / 32; ++w) oo += red[w];
        __syncthreads();
        if (lane == 0) red[warp] = t;
        __syncthreads();
        double tt = 0.0;
        for (int w = 0; w < kJacThreads / 32; ++w) tt += red[w];
        __syncthreads();
        return make_double2(oo, tt);
    };
    for (int sweep = 0; sweep < 40; ++sweep) {
        const double2 m = offdiag();
        if (m.x <= 1e-30 * m.y) break;
        for (int round = 0; round < D - 1; ++round) {
            if (tid < D / 2) {
                // round-robin pairing: D - 1 fixed against the round, the rest in a circle
                int p, q;
                if (tid == 0) {
                    p = round;
                    q = D - 1;
                } else {
                    p = (round + tid) % (D - 1);
                    q = (round - tid + (D - 1)) % (D - 1);
                }
                if (p > q) { const int t = p; p = q; q = t; }
                const double apq = A[p * D + q];
                double c = 1.0, s = 0.0;
                if (apq != 0.0) {
                    const double theta = (A[q * D + q] - A[p * D + p]) / (2.0 * apq);
                    const double t = (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
                    c = 1.0 / sqrt(t * t + 1.0);
                    s = t * c;
                }
                pp[tid] = p;
                qq[tid] = q;
                cs_c[tid] = c;
                cs_s[tid] = s;
            }
            __syncthreads();
            // rows p, q of every pair: A <- J^T A, and V^T <- J^T V^T (V <- V J);
            // consecutive threads walk a row: coalesced
            for (int e = tid; e < (D / 2) * D; e += kJacThreads) {
                const int k = e / D, j = e % D;
                const int p = pp[k], q = qq[k];
                const double c = cs_c[k], s = cs_s[k];
                const double ap = A[p * D + j], aq = A[q * D + j];
                A[p * D + j] = c * ap - s * aq;
                A[q * D + j] = s * ap + c * aq;
                const double vp = VT[p * D + j], vq = VT[q * D + j];
                VT[p * D + j] = c * vp - s * vq;
                VT[q * D + j] = s * vp + c * vq;
            }
            __syncthreads();
            // columns p, q: A <- A J, walked row by row (consecutive threads take
            // different pairs of one row, not one column: no bank-wide conflicts)
            for (int e = tid; e < (D / 2) * D; e += kJacThreads) {
                const int k = e % (D / 2), i = e / (D / 2);
                const int p = pp[k], q = qq[k];
                const double c = cs_c[k], s = cs_s[k];
                const double ap = A[i * D + p], aq = A[i * D + q];
                A[i * D + p] = c * ap - s * aq;
                A[i * D + q] = s * ap + c * aq;
            }
            __syncthreads();
        }
    }
    // rank of eigenvalue i: by (value desc, index asc)
    if (tid < D) {
        const double x = A[tid * D + tid];
        int rank = 0;
        for (int j = 0; j < D; ++j) {
            const double y = A[j * D + j];
            rank += y > x || (y == x && j < tid);
        }
        order[rank] = tid;
    }
    __syncthreads();
    // column c of W = eigenvector order[c], signed so its largest-magnitude entry is positive
    if (tid < r) {
        const int src = order[tid];
        int jm = 0;
        double best = -1.0;
        for (int j = 0; j < D; ++j) {
            const double a = fabs(VT[src * D + j]);
            if (a > best) { best = a; jm = j; }
        }
        const double sg = VT[src * D + jm] < 0.0 ? -1.0 : 1.0;
        for (int j = 0; j < D; ++j) W[(int64_t)j * r + tid] = (float)(sg * VT[src * D + j]);
        if (evals_out) evals_out[tid] = A[src * D + src];
    }
}

template <int D>
int launch_pca_d(const void* K, int64_t batch, int64_t n_tokens, int64_t ld_tokens, int hkv, int pool, int dtype,
                 int r, float* W, double* evals, cudaStream_t s) {
    const int64_t units = batch * hkv;
    const int64_t nb = n_tokens / pool;
    Arena scratch;
    scratch.async = true;
    scratch.stream = s;
    double* G = scratch.alloc<double>((int64_t)D * D + D);
    double* Vm = scratch.alloc<double>((int64_t)D * D);
    if (scratch.status != LSA_OK) return scratch.status;
    double* Sv = G + D * D;
    cudaMemsetAsync(G, 0, ((size_t)D * D + D) * sizeof(double), s);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t rows = units * nb;
    const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(4 * (int64_t)sms, (rows + 63) / 64));
    note_launch();
    if (dtype == LSA_BF16)
        pca_gram_kernel<__nv_bfloat16, D><<<grid, kGramThreads, 0, s>>>((const __nv_bfloat16*)K, units, nb, ld_tokens,
                                                                         hkv, pool, G, Sv);
    else
        pca_gram_kernel<float, D><<<grid, kGramThreads, 0, s>>>((const float*)K, units, nb, ld_tokens, hkv, pool, G, Sv);
    const size_t smem = (size_t)D * D * sizeof(double);
    cudaError_t e = cudaFuncSetAttribute(pca_jacobi_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_status(e);
    note_launch();
    pca_jacobi_kernel<D><<<1, kJacThreads, smem, s>>>(G, Sv, (double)rows, r, Vm, W, evals);
    const int st = cuda_status(cudaGetLastError());
    scratch.release();
    return st;
}

}  // namespace

int launch_pca_map(const void* K, int64_t batch, int64_t n_tokens, int64_t ld_tokens, int hkv, int d, int pool,
                   int dtype, int r, float* W, double* evals, cudaStream_t s) {
    if (d == 128) return launch_pca_d<128>(K, batch, n_tokens, ld_tokens, hkv, pool, dtype, r, W, evals, s);
    if (d == 64) return launch_pca_d<64>(K, batch, n_tokens, ld_tokens, hkv, pool, dtype, r, W, evals, s);
    return LSA_ERR_INVALID_ARG;
}

}  // namespace lsa
