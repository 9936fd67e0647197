// k-means assign on the 5th-generation tensor cores (tcgen05).
//
// distance(x, c_j) = ||c_j||^2 - 2 x.c_j (||x||^2 is common to a row); the
// x.c products of a 128-point tile against 256-centroid tiles are one dense
// GEMM per tile.  Operands are fp32; each is scaled by one power of two
// (exact; chosen from the largest magnitude so that every value is below
// 2^10) and split into two fp16 parts (x = xh + xl, c = ch + cl).  The GEMM
// runs over K = 3r + 2 (zero-padded to a multiple of 64) with
// A = [xh | xh | xl | 2^12 | 2^12], B = [ch | cl | ch | -nh | -nl], nh + nl =
// |c|^2 / 2^13 split the same way, so the accumulator holds
// x.c - |c|^2 / 2 (scaled) and the nearest centroid is the largest entry: the
// norms ride in the product and the epilogue is one compare per entry.  fp16
// keeps 11 significant bits like tf32, so the dropped xl.cl term and the
// roundings leave an error near 2^-21 of |x||c| (fp32-like assignments), at
// the f16 MMA rate, twice the tf32 one.
//
// One CTA per 128 points, persistent over all centroid tiles of its unit:
//   warp 0    TMA producer: the point tile once (all K-chunks resident), then
//             centroid K-chunks through a 3-stage ring (128B swizzle)
//   warp 1    TMEM owner and MMA issuer (one thread): tcgen05.mma kind::f16
//             (fp16 A and B), M=128, N=256, K=16 per instruction, into one of
//             two TMEM accumulators (2 x 256 columns)
//   warps 2-9 epilogue: tcgen05.ld of the accumulator rows, two warps per
//             TMEM lane quarter (each on half of the columns), running
//             (value, id) maximum per point, ties to the lower id, the two
//             halves merged at the end
// Every mbarrier wait is bounded; a timeout latches kErrTimeout and the CTA
// winds down (TMEM is always released).
#include <cuda_fp16.h>

#include <mutex>
#include <new>

#include "tc_common.cuh"

namespace lsa {
namespace {

constexpr int kTM = kTcM;         // points per CTA (UMMA M)
constexpr int kTN = kTcN;         // centroids per tile (UMMA N)
constexpr int kKC = 64;           // fp16 per K-chunk: one 128-byte swizzle row
constexpr int kStagesB = 3;
constexpr int kThreadsTC = 320;   // producer, MMA issuer, 8 epilogue warps
// K extent of the split operands: 3r + 2 rounded up to whole 64-element chunks.
__host__ __device__ constexpr int split_k(int r) { return (3 * r + 2 + kKC - 1) / kKC * kKC; }

// Largest |value| of the points and the starting centroids, as float bits
// (non-negative floats order like their bit patterns).
__global__ void absmax_kernel(const float* __restrict__ X, int64_t ldx, int64_t n, int r, int64_t units,
                              const float* __restrict__ C, int64_t nc, uint32_t* __restrict__ out) {
    uint32_t m = 0;
    const int64_t tot = units * n * r;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < tot + nc;
         e += (int64_t)gridDim.x * blockDim.x) {
        float v;
        if (e < tot) {
            const int64_t c = e % r, row = e / r;
            v = X[((row / n) * ldx + row % n) * r + c];
        } else {
            v = C[e - tot];
        }
        m = max(m, __float_as_uint(fabsf(v)));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(out, m);
}

// The power of two 2^-e that brings the largest magnitude into [2^9, 2^10):
// scaled coordinates fit fp16, and |scaled c|^2 / 2^13 <= r 2^7 does too.
__device__ __forceinline__ int scale_exp(const uint32_t* absmax) {
    const float m = __uint_as_float(*absmax);
    if (!(m > 0.f) || isinf(m)) return 0;
    return max(-60, min(60, ilogbf(m) - 9));
}

// Xs[u*n_pad + p] = [xh | xh | xl | 2^12 | 2^12 | 0], x scaled by 2^-e, zero
// rows past n.
__global__ void split_points_kernel(const float* __restrict__ X, int64_t ldx, int64_t n, int64_t n_pad, int r,
                                    int64_t units, const uint32_t* __restrict__ absmax, __half* __restrict__ Xs) {
    const int kp = split_k(r);
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= units * n_pad * kp) return;
    const int c = (int)(e % kp);
    const int64_t row = e / kp;
    const int64_t u = row / n_pad, p = row % n_pad;
    const int sc = -scale_exp(absmax);
    const int src = c < r ? c : (c < 2 * r ? c - r : (c < 3 * r ? c - 2 * r : -1));
    float x = 0.f;
    if (p < n && src >= 0) x = ldexpf(X[(u * ldx + p) * r + src], sc);
    const __half xh = __float2half_rn(x);
    const __half xl = __float2half_rn(x - __half2float(xh));
    __half out = __float2half_rn(0.f);
    if (c < 2 * r) out = xh;
    else if (c < 3 * r) out = xl;
    else if (c < 3 * r + 2 && p < n) out = __float2half_rn(4096.f);
    Xs[row * kp + c] = out;
}

// Cs[u*k_pad + j] = [ch | cl | ch | -nh | -nl | 0], c scaled by 2^-e,
// nh + nl = |scaled c|^2 / 2^13 (summed in fp64, split in two fp16 parts);
// zero rows past k.  One thread per row.
__global__ void split_centroids_kernel(const float* __restrict__ C, int k, int k_pad, int r, int64_t units,
                                       const uint32_t* __restrict__ absmax, __half* __restrict__ Cs) {
    const int kp = split_k(r);
    const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= units * k_pad) return;
    const int64_t u = row / k_pad, j = row % k_pad;
    const int sc = -scale_exp(absmax);
    __half* o = Cs + row * kp;
    double nrm = 0.0;   // (in fp64: the norm then carries only the split's error)
    for (int c = 0; c < r; ++c) {
        float x = 0.f;
        if (j < k) x = ldexpf(C[(u * k + j) * r + c], sc);
        nrm = fma((double)x, (double)x, nrm);
        const __half xh = __float2half_rn(x);
        const __half xl = __float2half_rn(x - __half2float(xh));
        o[c] = xh;
        o[r + c] = xl;
        o[2 * r + c] = xh;
    }
    const double hn = ldexp(nrm, -13);
    const __half nh = __double2half(hn);
    const __half nl = __double2half(hn - (double)__half2float(nh));
    o[3 * r] = __hneg(nh);
    o[3 * r + 1] = __hneg(nl);
    for (int c = 3 * r + 2; c < kp; ++c) o[c] = __float2half_rn(0.f);
}

template <int R>
__global__ void __launch_bounds__(kThreadsTC, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_c,
                     int64_t n, int64_t n_pad, int k, int k_pad, const float* __restrict__ cc,
                     const uint32_t* __restrict__ absmax, int32_t* __restrict__ labels, int64_t ldl, int32_t* err) {
    constexpr int KS = split_k(R) / kKC;             // K-chunks
    constexpr int KSTEPS = (3 * R + 2 + 15) / 16;    // 16-wide MMA steps that hold data (the rest are zero)
    constexpr int A_CHUNK = kTM * 128;               // bytes per A chunk
    constexpr int B_CHUNK = kTN * 128;               // bytes per B stage
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                           ~uintptr_t(1023));
    unsigned char* As = smem;                                    // KS x 16 KB
    unsigned char* Bs = smem + KS * A_CHUNK;                     // kStagesB x 32 KB
    uint64_t* bars = reinterpret_cast<uint64_t*>(Bs + kStagesB * B_CHUNK);
    uint64_t* a_full = bars;                                     // 1
    uint64_t* b_full = bars + 1;                                 // kStagesB
    uint64_t* b_empty = b_full + kStagesB;                       // kStagesB
    uint64_t* acc_full = b_empty + kStagesB;                     // 2
    uint64_t* acc_empty = acc_full + 2;                          // 2
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.y;
    const int64_t p0 = (int64_t)blockIdx.x * kTM;
    const int ntile = (k + kTN - 1) / kTN;

    if (threadIdx.x == 0) {
        mbar_init(a_full, 1);
        for (int s = 0; s < kStagesB; ++s) {
            mbar_init(b_full + s, 1);
            mbar_init(b_empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full + b, 1);
            mbar_init(acc_empty + b, 256);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(su32(tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    const uint32_t tmem = *tmem_slot;

    bool ok = true;
    if (warp == 0) {
        if (lane == 0) {
            mbar_expect_tx(a_full, KS * A_CHUNK);
            for (int c = 0; c < KS; ++c)
                tma_load_2d(As + c * A_CHUNK, &map_x, a_full, c * kKC, (int)(u * n_pad + p0));
            int issued = 0;
            for (int t = 0; t < ntile && ok; ++t) {
                for (int c = 0; c < KS && ok; ++c) {
                    const int it = t * KS + c, s = it % kStagesB;
                    const uint32_t ph = (uint32_t)(it / kStagesB) & 1u;
                    if (!mbar_wait(b_empty + s, ph ^ 1u)) { ok = false; break; }
                    mbar_expect_tx(b_full + s, B_CHUNK);
                    tma_load_2d(Bs + s * B_CHUNK, &map_c, b_full + s, c * kKC, u * k_pad + t * kTN);
                    ++issued;
                }
            }
            if (!ok) {
                latch(err, kErrTimeout);
                // let the copies already issued land before the CTA exits
                for (int it = 0; it < issued && it < kStagesB; ++it) {
                    const int last = issued - 1 - it;
                    mbar_wait(b_full + last % kStagesB, (uint32_t)(last / kStagesB) & 1u);
                }
                mbar_wait(a_full, 0);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            if (!mbar_wait(a_full, 0)) ok = false;
            for (int t = 0; t < ntile && ok; ++t) {
                const int buf = t & 1;
                if (!mbar_wait(acc_empty + buf, ((uint32_t)(t >> 1) & 1u) ^ 1u)) { ok = false; break; }
                asm volatile("tcgen05.fence::after_thread_sync;");
                const uint32_t d = tmem + buf * kTN;
                for (int c = 0; c < KS; ++c) {
                    const int it = t * KS + c, s = it % kStagesB;
                    if (!mbar_wait(b_full + s, (uint32_t)(it / kStagesB) & 1u)) { ok = false; break; }
                    asm volatile("tcgen05.fence::after_thread_sync;");
#pragma unroll
                    for (int kk = 0; kk < kKC / 16; ++kk) {
                        // the zero padding after column 3r + 2 adds nothing: its steps are skipped
                        if (c * (kKC / 16) + kk >= KSTEPS) break;
                        const uint64_t da = umma_desc(As + c * A_CHUNK + kk * 32);
                        const uint64_t db = umma_desc(Bs + s * B_CHUNK + kk * 32);
                        umma_f16(d, da, db, (c | kk) ? 1u : 0u);
                    }
                    umma_commit(b_empty + s);
                }
                if (!ok) break;
                umma_commit(acc_full + buf);
            }
            if (!ok) latch(err, kErrTimeout);
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31, one point per
        // thread; warps 2-5 take columns [0, 128) of every tile, warps 6-9
        // columns [128, 256)
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const int row = 32 * q + lane;
        const int64_t p = p0 + row;
        float best = -INFINITY;
        int bestj = INT32_MAX;
        for (int t = 0; t < ntile; ++t) {
            const int buf = t & 1;
            if (!mbar_wait(acc_full + buf, (uint32_t)(t >> 1) & 1u)) { ok = false; latch(err, kErrTimeout); break; }
            asm volatile("tcgen05.fence::after_thread_sync;");
#pragma unroll
            for (int cb = 0; cb < kTN / 64; ++cb) {
                float v[32];
                const int col = half * (kTN / 2) + cb * 32;
                tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + buf * kTN + col, v);
                const int j0 = t * kTN + col;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (v[i] > best && j0 + i < k) { best = v[i]; bestj = j0 + i; }
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;");
            mbar_arrive(acc_empty + buf);
        }
        // the two halves of each point: the larger value, ties to the lower id
        float* mv = reinterpret_cast<float*>(tmem_slot + 4);    // [128] values of the second half
        int* mj = reinterpret_cast<int*>(mv + kTM);            // [128] their ids
        if (half == 1) {
            mv[row] = best;
            mj[row] = bestj;
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");   // the 8 epilogue warps only
        if (half == 0) {
            const float ob = mv[row];
            const int oj = mj[row];
            if (ob > best || (ob == best && oj < bestj)) { best = ob; bestj = oj; }
            if (bestj == INT32_MAX) bestj = 0;
            if (ok && p < n) labels[(int64_t)u * ldl + p] = bestj;
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
}

template <int R>
size_t tc_smem_bytes() {
    // operand tiles + barriers and TMEM slot (256 B) + the halves' merge (1 KB) + alignment
    return (size_t)(split_k(R) / kKC) * kTM * 128 + (size_t)kStagesB * kTN * 128 + 256 + 1024 + 1024;
}

}  // namespace

bool assign_tc_supported(int r, int grid_log2) { return (r == 32 || r == 64) && grid_log2 == 0 && tma_available(); }

// Scratch for the tensor-core assign of (units, n, k, r): split points and
// split centroids.
struct AssignTcWork {
    __half* Xs = nullptr;
    __half* Cs = nullptr;
    uint32_t* absmax = nullptr;
    int64_t n_pad = 0;
    int k_pad = 0;
};

int assign_tc_prepare_points(const float* X, int64_t ldx, int64_t units, int64_t n, int r, int k, const float* C0,
                             Arena& A, cudaStream_t s, void** work_out) {
    AssignTcWork* w = new (std::nothrow) AssignTcWork();
    if (!w) return LSA_ERR_OOM;
    w->n_pad = (n + kTM - 1) / kTM * kTM;
    w->k_pad = (k + kTN - 1) / kTN * kTN;
    const int kp = split_k(r);
    w->Xs = A.alloc<__half>(units * w->n_pad * kp);
    w->Cs = A.alloc<__half>(units * (int64_t)w->k_pad * kp);
    w->absmax = A.alloc<uint32_t>(1);
    if (A.status != LSA_OK) { delete w; return A.status; }
    // one scale for the run: the points, and the centroids it starts from
    // (later centroids are means of points, never larger)
    cudaError_t e = cudaMemsetAsync(w->absmax, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) { delete w; return cuda_status(e); }
    note_launch();
    absmax_kernel<<<592, 256, 0, s>>>(X, ldx, n, r, units, C0, units * (int64_t)k * r, w->absmax);
    const int64_t tot = units * w->n_pad * kp;
    note_launch();
    split_points_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, s>>>(X, ldx, n, w->n_pad, r, units, w->absmax,
                                                                      w->Xs);
    *work_out = w;
    return cuda_status(cudaGetLastError());
}

void assign_tc_release(void* work) { delete static_cast<AssignTcWork*>(work); }

int assign_tc_run(void* work, const float* C, const float* cc, int64_t units, int64_t n, int r, int k,
                  int32_t* labels, int64_t ldl, int32_t* err, cudaStream_t s) {
    AssignTcWork* w = static_cast<AssignTcWork*>(work);
    const int kp = split_k(r);
    const int64_t tot = units * (int64_t)w->k_pad;
    note_launch();
    split_centroids_kernel<<<(unsigned)((tot + 127) / 128), 128, 0, s>>>(C, k, w->k_pad, r, units, w->absmax,
                                                                         w->Cs);
    CUtensorMap mx, mc;
    if (!make_tensor_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, w->Xs, units * w->n_pad, kp, kp * 2, kKC, kTM) ||
        !make_tensor_map_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, w->Cs, units * w->k_pad, kp, kp * 2, kKC, kTN))
        return LSA_ERR_CUDA;
    dim3 grid((unsigned)(w->n_pad / kTM), (unsigned)units);
    cudaError_t e;
    if (r == 64) {
        const size_t smem = tc_smem_bytes<64>();
        e = cudaFuncSetAttribute(assign_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_status(e);
        note_launch();
        assign_tc_kernel<64><<<grid, kThreadsTC, smem, s>>>(mx, mc, n, w->n_pad, k, w->k_pad, cc, w->absmax, labels,
                                                             ldl, err);
    } else {
        const size_t smem = tc_smem_bytes<32>();
        e = cudaFuncSetAttribute(assign_tc_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_status(e);
        note_launch();
        assign_tc_kernel<32><<<grid, kThreadsTC, smem, s>>>(mx, mc, n, w->n_pad, k, w->k_pad, cc, w->absmax, labels,
                                                             ldl, err);
    }
    return cuda_status(cudaGetLastError());
}

}  // namespace lsa
