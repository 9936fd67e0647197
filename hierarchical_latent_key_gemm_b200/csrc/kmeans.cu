// Lloyd k-means for the bucket hierarchy: the keys are grouped into clusters
// before any query is scored (10M-token attention post), and the buckets form
// a hierarchy (LSA explainer, "How does LSA work?" step 1).
//
// Rules: centroid j starts at point floor(j*n/k); assign = argmin squared
// distance with ties to the lower centroid id; update = mean of the members,
// an empty cluster keeps its centroid; optional integer grid (means rounded
// half-to-even onto multiples of 2^-g, exact integer arithmetic).
//
// Assign (float): distance = ||c||^2 - 2 x.c (||x||^2 is common to a row);
// for r = 32 or 64 on the tensor cores (kmeans_tc.cu), otherwise a
// register-tiled fp32 product on CUDA cores with the running argmin kept in
// registers.  Assign (grid): exact int64 sum of squared grid differences.
// Update: members are grouped by a stable sort, so each cluster sums its
// points in ascending order (float64 accumulation): deterministic bits.
#include <algorithm>

#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kAsgThreads = 256;
constexpr int kTileP = 128;   // points per CTA
constexpr int kTileC = 128;   // centroids per inner tile

__global__ void transpose_kernel(const float* __restrict__ src, int64_t rows, int64_t ld_src_unit, int cols,
                                 float* __restrict__ dst, int64_t ld_dst) {
    // src: [units][ld_src_unit][cols] (rows used); dst: [units][cols][ld_dst]
    __shared__ float t[32][33];
    const int u = blockIdx.z;
    const int64_t r0 = (int64_t)blockIdx.x * 32;
    const int c0 = blockIdx.y * 32;
    const float* s = src + (int64_t)u * ld_src_unit * cols;
    float* dd = dst + (int64_t)u * cols * ld_dst;
    for (int y = threadIdx.y; y < 32; y += blockDim.y) {
        int64_t rr = r0 + y;
        int cc = c0 + threadIdx.x;
        t[y][threadIdx.x] = (rr < rows && cc < cols) ? s[rr * cols + cc] : 0.f;
    }
    __syncthreads();
    for (int y = threadIdx.y; y < 32; y += blockDim.y) {
        int cc = c0 + y;
        int64_t rr = r0 + threadIdx.x;
        if (cc < cols && rr < ld_dst) dd[(int64_t)cc * ld_dst + rr] = t[threadIdx.x][y];
    }
}

void launch_transpose(const float* src, int64_t units, int64_t rows, int64_t ld_src_unit, int cols, float* dst,
                      int64_t ld_dst, cudaStream_t s) {
    dim3 grid((unsigned)((ld_dst + 31) / 32), (unsigned)((cols + 31) / 32), (unsigned)units);
    note_launch();
    transpose_kernel<<<grid, dim3(32, 8), 0, s>>>(src, rows, ld_src_unit, cols, dst, ld_dst);
}

__global__ void init_kernel(const float* __restrict__ X, int64_t ldx, int64_t units, int64_t n, int k, int r,
                            float* __restrict__ C) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = units * k * r;
    if (e >= total) return;
    const int64_t u = e / ((int64_t)k * r);
    const int64_t j = (e / r) % k;
    const int c = (int)(e % r);
    const int64_t src = (j * n) / k;
    C[e] = X[(u * ldx + src) * r + c];
}

__global__ void cnorm_kernel(const float* __restrict__ C, int64_t count, int r, float* __restrict__ cc) {
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= count) return;
    float s = 0.f;
    for (int c = 0; c < r; ++c) {
        float v = C[j * r + c];
        s = __fmaf_rn(v, v, s);
    }
    cc[j] = s;
}

// XT: [units][R][ldxt]; CT: [units][R][ldct]; cc: [units*k]
template <int R>
__global__ __launch_bounds__(kAsgThreads) void assign_f32_kernel(
    const float* __restrict__ XT, int64_t ldxt, int64_t n, const float* __restrict__ CT, int64_t ldct,
    const float* __restrict__ cc, int k, int32_t* __restrict__ labels, int64_t ldl) {
    extern __shared__ float4 smem4[];
    float* Xs = reinterpret_cast<float*>(smem4);   // [R][kTileP]
    float* Cs = Xs + R * kTileP;                    // [R][kTileC]
    float* ccs = Cs + R * kTileC;                   // [kTileC]
    const int u = blockIdx.y;
    const int64_t p0 = (int64_t)blockIdx.x * kTileP;
    const int tid = threadIdx.x;
    const int ty = tid >> 4, tx = tid & 15;
    const float* xt = XT + (int64_t)u * R * ldxt;
    const float* ct = CT + (int64_t)u * R * ldct;
    // points tile, float4 along points (ldxt is a multiple of 4, padded with zeros)
    for (int e = tid; e < R * (kTileP / 4); e += kAsgThreads) {
        const int row = e / (kTileP / 4), q4 = e % (kTileP / 4);
        const int64_t p = p0 + q4 * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p < ldxt) v = *reinterpret_cast<const float4*>(xt + (int64_t)row * ldxt + p);
        reinterpret_cast<float4*>(Xs + row * kTileP)[q4] = v;
    }
    float best[8];
    int bestj[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { best[i] = INFINITY; bestj[i] = 0; }
    for (int c0 = 0; c0 < k; c0 += kTileC) {
        __syncthreads();
        for (int e = tid; e < R * (kTileC / 4); e += kAsgThreads) {
            const int row = e / (kTileC / 4), q4 = e % (kTileC / 4);
            const int64_t j = c0 + q4 * 4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j < ldct) v = *reinterpret_cast<const float4*>(ct + (int64_t)row * ldct + j);
            reinterpret_cast<float4*>(Cs + row * kTileC)[q4] = v;
        }
        for (int e = tid; e < kTileC; e += kAsgThreads) {
            const int64_t j = c0 + e;
            ccs[e] = (j < k) ? cc[(int64_t)u * k + j] : 0.f;
        }
        __syncthreads();
        float acc[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 4
        for (int e = 0; e < R; ++e) {
            const float4 a0 = reinterpret_cast<const float4*>(Xs + e * kTileP)[ty];
            const float4 a1 = reinterpret_cast<const float4*>(Xs + e * kTileP + 64)[ty];
            const float4 b0 = reinterpret_cast<const float4*>(Cs + e * kTileC)[tx];
            const float4 b1 = reinterpret_cast<const float4*>(Cs + e * kTileC + 64)[tx];
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
        }
        // centroid order within the thread: tx*4+t then 64+tx*4+t, both ascending
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int jl = (j < 4) ? (tx * 4 + j) : (64 + tx * 4 + (j - 4));
            const int jj = c0 + jl;
            if (jj < k) {
                const float cj = ccs[jl];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float dist = __fmaf_rn(-2.f, acc[i][j], cj);
                    if (dist < best[i]) { best[i] = dist; bestj[i] = jj; }
                }
            }
        }
    }
    // combine the 16 column threads of each point row (lexicographic (dist, id))
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float bd = best[i];
        int bj = bestj[i];
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) {
            float od = __shfl_xor_sync(0xffffffffu, bd, o);
            int oj = __shfl_xor_sync(0xffffffffu, bj, o);
            if (od < bd || (od == bd && oj < bj)) { bd = od; bj = oj; }
        }
        if (tx == 0) {
            const int pl = (i < 4) ? (ty * 4 + i) : (64 + ty * 4 + (i - 4));
            const int64_t p = p0 + pl;
            if (p < n) labels[(int64_t)u * ldl + p] = bj;
        }
    }
}

// Exact assign on the 2^-g grid: sum over dims of (x*2^g - c*2^g)^2 in int64.
__global__ void assign_grid_kernel(const float* __restrict__ X, int64_t ldx, int64_t n, int r,
                                   const float* __restrict__ C, int k, int grid_log2,
                                   int32_t* __restrict__ labels, int64_t ldl, int32_t* err) {
    extern __shared__ int32_t cs[];   // [chunk][r]
    const int u = blockIdx.y;
    const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const float scale = (float)(1 << grid_log2);
    const int chunk = 256;
    int32_t x[128];
    bool ok = true;
    if (p < n) {
        for (int c = 0; c < r; ++c) {
            float v = X[((int64_t)u * ldx + p) * r + c] * scale;
            if (!(fabsf(v) < 8388608.f) || v != rintf(v)) ok = false;
            x[c] = (int32_t)v;
        }
    }
    if (!ok) latch(err, kErrInexact);
    int64_t bestd = INT64_MAX;
    int bestj = 0;
    for (int c0 = 0; c0 < k; c0 += chunk) {
        __syncthreads();
        for (int e = threadIdx.x; e < chunk * r; e += blockDim.x) {
            const int j = c0 + e / r;
            int32_t q = 0;
            if (j < k) {
                float v = C[((int64_t)u * k + j) * r + (e % r)] * scale;
                if (!(fabsf(v) < 8388608.f) || v != rintf(v)) latch(err, kErrInexact);
                q = (int32_t)v;
            }
            cs[e] = q;
        }
        __syncthreads();
        if (p < n) {
            const int lim = min(chunk, k - c0);
            for (int j = 0; j < lim; ++j) {
                int64_t s = 0;
                for (int c = 0; c < r; ++c) {
                    int64_t dlt = (int64_t)x[c] - cs[j * r + c];
                    s += dlt * dlt;
                }
                if (s < bestd) { bestd = s; bestj = c0 + j; }
            }
        }
    }
    if (p < n) labels[(int64_t)u * ldl + p] = bestj;
}

__global__ void keys_kernel(const int32_t* __restrict__ labels, int64_t ldl, int64_t units, int64_t n, int k,
                            uint32_t* __restrict__ keys, int32_t* __restrict__ vals, int32_t* __restrict__ counts,
                            int32_t* err) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= units * n) return;
    const int64_t u = e / n, i = e % n;
    int32_t lab = labels[u * ldl + i];
    if (lab < 0 || lab >= k) { latch(err, kErrDevice); lab = 0; }
    const uint32_t key = (uint32_t)(u * k + lab);
    keys[e] = key;
    vals[e] = (int32_t)e;
    atomicAdd(&counts[key], 1);
}

// One warp per cluster: members in ascending point order, float64 sums.
__global__ void update_kernel(const float* __restrict__ X, int64_t ldx, int64_t n, int r, int k,
                              const int32_t* __restrict__ perm, const int32_t* __restrict__ off,
                              const float* __restrict__ Cold, float* __restrict__ Cnew, int grid_log2,
                              double* __restrict__ cobj, int64_t nclusters, int32_t* err) {
    const int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (c >= nclusters) return;
    const int64_t u = c / k;
    const int32_t s = off[c], e = off[c + 1];
    const int cnt = e - s;
    double sum[4] = {0, 0, 0, 0};
    long long isum[4] = {0, 0, 0, 0};
    double obj = 0.0;
    long long iobj = 0;
    float cold[4];
    const float scale = (float)(1 << (grid_log2 > 0 ? grid_log2 : 0));
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int dim = lane + 32 * t;
        cold[t] = dim < r ? Cold[c * r + dim] : 0.f;
    }
    for (int m = s; m < e; ++m) {
        const int64_t pid = perm[m];
        const int64_t row = u * ldx + (pid - u * n);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int dim = lane + 32 * t;
            if (dim < r) {
                const float x = X[row * r + dim];
                if (grid_log2 > 0) {
                    const long long xi = (long long)(x * scale);
                    const long long ci = (long long)(cold[t] * scale);
                    isum[t] += xi;
                    iobj += (xi - ci) * (xi - ci);
                } else {
                    sum[t] += (double)x;
                    const double dd = (double)x - (double)cold[t];
                    obj += dd * dd;
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int dim = lane + 32 * t;
        if (dim >= r) continue;
        float out = cold[t];
        if (cnt > 0) {
            if (grid_log2 > 0) {
                // round-half-even(isum / cnt) with floor division
                long long q = isum[t] / cnt, rem = isum[t] % cnt;
                if (rem < 0) { rem += cnt; q -= 1; }
                const long long tw = 2 * rem;
                if (tw > cnt || (tw == cnt && (q & 1))) q += 1;
                if (q >= 8388608LL || q <= -8388608LL) latch(err, kErrInexact);
                out = (float)q / scale;
            } else {
                out = (float)(sum[t] / (double)cnt);
            }
        }
        Cnew[c * r + dim] = out;
    }
    if (grid_log2 > 0) {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) iobj += __shfl_xor_sync(0xffffffffu, iobj, o);
        if (lane == 0) cobj[c] = (double)iobj / ((double)scale * (double)scale);
    } else {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) obj += __shfl_xor_sync(0xffffffffu, obj, o);
        if (lane == 0) cobj[c] = obj;
    }
}

__global__ void obj_reduce_kernel(const double* __restrict__ cobj, int k, double* __restrict__ out) {
    __shared__ double sh[256];
    const int u = blockIdx.x;
    double s = 0.0;
    for (int j = threadIdx.x; j < k; j += 256) s += cobj[(int64_t)u * k + j];
    sh[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w >= 1; w >>= 1) {
        if (threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) out[u] = sh[0];
}

template <int R>
int launch_assign_f32(const float* XT, int64_t ldxt, int64_t n, const float* CT, int64_t ldct, const float* cc,
                      int k, int64_t units, int32_t* labels, int64_t ldl, cudaStream_t s) {
    const size_t smem = (size_t)(R * kTileP + R * kTileC + kTileC) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(assign_f32_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return cuda_status(e);
    dim3 grid((unsigned)((n + kTileP - 1) / kTileP), (unsigned)units);
    note_launch();
    assign_f32_kernel<R><<<grid, kAsgThreads, smem, s>>>(XT, ldxt, n, CT, ldct, cc, k, labels, ldl);
    return cuda_status(cudaGetLastError());
}

int bits_for(int64_t count) {
    int b = 1;
    while ((int64_t(1) << b) < count) ++b;
    return b;
}

}  // namespace

GroupWork alloc_group_work(int64_t units, int64_t n, int k, Arena& A) {
    GroupWork w;
    w.total = units * n;
    w.nc = units * (int64_t)k;
    w.k0 = A.alloc<uint32_t>(w.total);
    w.v0 = A.alloc<int32_t>(w.total);
    w.k1 = A.alloc<uint32_t>(w.total);
    w.v1 = A.alloc<int32_t>(w.total);
    w.counts = A.alloc<int32_t>(w.nc);
    w.scratch = A.alloc<int32_t>(std::max(radix_scratch_elems(w.total), scan_scratch_elems(w.nc)) + 1);
    return w;
}

// Group points of every unit by label with a stable sort; perm holds global
// point ids (u*n + i) in (u, label, i) order; off[u*k + j] is where cluster
// (u, j) starts, off[units*k] = units*n.
int group_by_label(const int32_t* labels, int64_t ldl, int64_t units, int64_t n, int k, int32_t* perm,
                   int32_t* off, int32_t* err, cudaStream_t s, const GroupWork& w) {
    const int64_t total = units * n;
    const int64_t nc = units * (int64_t)k;
    if (total != w.total || nc != w.nc) return LSA_ERR_INVALID_ARG;
    cudaMemsetAsync(w.counts, 0, nc * sizeof(int32_t), s);
    if (total > 0) {
        note_launch();
        keys_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(labels, ldl, units, n, k, w.k0, w.v0,
                                                                    w.counts, err);
    }
    scan_exclusive(w.counts, off, nc, w.scratch, s);
    uint32_t* ks;
    int32_t* vs;
    radix_sort(w.k0, w.v0, w.k1, w.v1, total, bits_for(nc), w.scratch, s, &ks, &vs);
    if (total > 0) cudaMemcpyAsync(perm, vs, total * sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    return cuda_status(cudaGetLastError());
}

// Decode maintenance (lsa_refresh_centroids): every centroid becomes the
// mean of its current members, memberships fixed, bottom-up (leaves from the
// latent keys of their blocks, each upper level from the refreshed level
// below), by the update of the Lloyd rounds (fp64 sums in ascending member
// order, empty keeps, grid rounding); then the tree-order copies.
int refresh_centroids(lsa_index* ix, cudaStream_t s, Arena& A) {
    const lsa_build_params& p = ix->p;
    const int levels = p.levels, r = p.r;
    const int64_t U = ix->units;
    for (int l = levels - 1; l >= 0; --l) {
        const int k = p.level_sizes[l];
        const bool leaf = l == levels - 1;
        const int64_t n = leaf ? ix->nb : p.level_sizes[l + 1];
        const float* X = leaf ? ix->Kl : ix->cent[l + 1];
        const int64_t ldx = leaf ? ix->nb_cap : n;
        const int32_t* labels = leaf ? ix->leaf_of_block : ix->parent[l + 1];
        const int64_t nc = U * (int64_t)k;
        int32_t* perm = A.alloc<int32_t>(U * n);
        int32_t* off = A.alloc<int32_t>(nc + 1);
        float* Cn = A.alloc<float>(nc * r);
        double* cobj = A.alloc<double>(nc);
        GroupWork gw = alloc_group_work(U, n, k, A);
        if (A.status != LSA_OK) return A.status;
        int st = group_by_label(labels, ldx, U, n, k, perm, off, ix->err, s, gw);
        if (st != LSA_OK) return st;
        note_launch();
        update_kernel<<<(unsigned)((nc * 32 + 255) / 256), 256, 0, s>>>(X, ldx, n, r, k, perm, off, ix->cent[l], Cn,
                                                                       p.grid_log2, cobj, nc, ix->err);
        cudaMemcpyAsync(ix->cent[l], Cn, nc * r * sizeof(float), cudaMemcpyDeviceToDevice, s);
    }
    gather_tree_order(ix, s);
    return cuda_status(cudaGetLastError());
}

int run_kmeans(const float* X, int64_t ldx, int64_t units, int64_t n, int r, int k, int iters, int grid_log2,
               KmeansOut out, int64_t ldl, int32_t* err, cudaStream_t s, Arena& A, const float* C_init) {
    if (units <= 0 || n <= 0 || k <= 0) return LSA_OK;
    if (r != 16 && r != 32 && r != 64 && r != 128) return LSA_ERR_INVALID_ARG;
    const int64_t nc = units * (int64_t)k;
    const int64_t ldxt = (n + 3) / 4 * 4;
    const int64_t ldct = ((int64_t)k + 3) / 4 * 4;
    const bool tc = assign_tc_supported(r, grid_log2);
    const bool simt = grid_log2 == 0 && !tc;
    float* XT = simt ? A.alloc<float>(units * r * ldxt) : nullptr;
    float* CT = simt ? A.alloc<float>(units * r * ldct) : nullptr;
    float* cc = A.alloc<float>(nc);
    float* Cb = A.alloc<float>(nc * r);
    double* cobj = A.alloc<double>(nc);
    int32_t* perm = out.perm ? out.perm : A.alloc<int32_t>(units * n);
    int32_t* off = out.off ? out.off : A.alloc<int32_t>(nc + 1);
    GroupWork gw = alloc_group_work(units, n, k, A);
    if (A.status != LSA_OK) return A.status;
    const int64_t tot = nc * r;
    if (C_init) {
        const cudaError_t e = cudaMemcpyAsync(out.C, C_init, tot * sizeof(float), cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return cuda_status(e);
    } else {
        note_launch();
        init_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, s>>>(X, ldx, units, n, k, r, out.C);
    }
    if (simt) launch_transpose(X, units, n, ldx, r, XT, ldxt, s);
    void* tcw = nullptr;
    if (tc) {
        const int st = assign_tc_prepare_points(X, ldx, units, n, r, k, out.C, A, s, &tcw);
        if (st != LSA_OK) return st;
    }
    float* cur = out.C;
    float* nxt = Cb;
    int rc = LSA_OK;
    for (int it = 0; it < iters && rc == LSA_OK; ++it) {
        if (grid_log2 > 0) {
            const int threads = 128;
            dim3 grid((unsigned)((n + threads - 1) / threads), (unsigned)units);
            const size_t smem = 256 * r * sizeof(int32_t);
            cudaFuncSetAttribute(assign_grid_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            note_launch();
            assign_grid_kernel<<<grid, threads, smem, s>>>(X, ldx, n, r, cur, k, grid_log2, out.labels, ldl, err);
            rc = cuda_status(cudaGetLastError());
        } else if (tc) {
            note_launch();
            cnorm_kernel<<<(unsigned)((nc + 255) / 256), 256, 0, s>>>(cur, nc, r, cc);
            rc = assign_tc_run(tcw, cur, cc, units, n, r, k, out.labels, ldl, err, s);
        } else {
            launch_transpose(cur, units, k, k, r, CT, ldct, s);
            note_launch();
            cnorm_kernel<<<(unsigned)((nc + 255) / 256), 256, 0, s>>>(cur, nc, r, cc);
            switch (r) {
                case 16: rc = launch_assign_f32<16>(XT, ldxt, n, CT, ldct, cc, k, units, out.labels, ldl, s); break;
                case 32: rc = launch_assign_f32<32>(XT, ldxt, n, CT, ldct, cc, k, units, out.labels, ldl, s); break;
                case 64: rc = launch_assign_f32<64>(XT, ldxt, n, CT, ldct, cc, k, units, out.labels, ldl, s); break;
                default: rc = launch_assign_f32<128>(XT, ldxt, n, CT, ldct, cc, k, units, out.labels, ldl, s); break;
            }
        }
        if (rc != LSA_OK) break;
        rc = group_by_label(out.labels, ldl, units, n, k, perm, off, err, s, gw);
        if (rc != LSA_OK) break;
        const int64_t threads = nc * 32;
        note_launch();
        update_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(X, ldx, n, r, k, perm, off, cur, nxt,
                                                                       grid_log2, cobj, nc, err);
        if (out.objective) {
            note_launch();
            obj_reduce_kernel<<<(unsigned)units, 256, 0, s>>>(cobj, k, out.objective + (int64_t)it * units);
        }
        float* t = cur; cur = nxt; nxt = t;
        rc = cuda_status(cudaGetLastError());
    }
    if (tcw) assign_tc_release(tcw);
    if (rc == LSA_OK && cur != out.C)
        cudaMemcpyAsync(out.C, cur, tot * sizeof(float), cudaMemcpyDeviceToDevice, s);
    return rc != LSA_OK ? rc : cuda_status(cudaGetLastError());
}

}  // namespace lsa
