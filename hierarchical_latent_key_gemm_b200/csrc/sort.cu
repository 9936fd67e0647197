// Device-wide exclusive scan and stable LSD radix sort.
//
// The bucket layout and the k-means update both need, for every cluster, its
// members in ascending point order (so sums run in one fixed order and the
// result is deterministic).  A stable sort of (cluster id, point id) pairs by
// cluster id gives exactly that.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

constexpr int kScanThreads = 1024;
constexpr int kScanItems = 4;
constexpr int kScanChunk = kScanThreads * kScanItems;

__device__ __forceinline__ int32_t warp_incl_scan(int32_t v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int32_t t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// Exclusive scan of one chunk of (n_items) values; item i < n reads in[i],
// items in [n, n_items) read 0.  Writes out[i] for i < n_items and, when sums
// is not null, the chunk total to sums[blockIdx.x].
__global__ void scan_chunk_kernel(const int32_t* __restrict__ in, int32_t* __restrict__ out,
                                  int64_t n, int64_t n_items, int32_t* __restrict__ sums) {
    __shared__ int32_t warp_tot[kScanThreads / 32];
    const int64_t base = (int64_t)blockIdx.x * kScanChunk + (int64_t)threadIdx.x * kScanItems;
    int32_t v[kScanItems];
    int32_t local = 0;
#pragma unroll
    for (int t = 0; t < kScanItems; ++t) {
        int64_t i = base + t;
        v[t] = (i < n) ? in[i] : 0;
        local += v[t];
    }
    int32_t incl = warp_incl_scan(local);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t w = (lane < kScanThreads / 32) ? warp_tot[lane] : 0;
        int32_t wi = warp_incl_scan(w);
        if (lane < kScanThreads / 32) warp_tot[lane] = wi - w;
    }
    __syncthreads();
    int32_t run = warp_tot[warp] + incl - local;
#pragma unroll
    for (int t = 0; t < kScanItems; ++t) {
        int64_t i = base + t;
        if (i < n_items) out[i] = run;
        run += v[t];
    }
    if (sums && threadIdx.x == kScanThreads - 1) sums[blockIdx.x] = run;
}

__global__ void scan_add_kernel(int32_t* __restrict__ out, int64_t n_items, const int32_t* __restrict__ offs) {
    const int64_t i = (int64_t)blockIdx.x * kScanChunk + threadIdx.x;
    const int32_t add = offs[blockIdx.x];
#pragma unroll
    for (int t = 0; t < kScanItems; ++t) {
        int64_t j = i + (int64_t)t * kScanThreads;
        if (j < n_items) out[j] += add;
    }
}

// ------------------------------------------------------------------ radix
constexpr int kRsThreads = 256;
constexpr int kRsItems = 16;
constexpr int kRsTile = kRsThreads * kRsItems;
constexpr int kRsWarps = kRsThreads / 32;

__global__ void radix_hist_kernel(const uint32_t* __restrict__ keys, int64_t n, int shift,
                                  int32_t* __restrict__ hist, int64_t ntiles) {
    __shared__ int32_t h[256];
    h[threadIdx.x] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kRsTile;
#pragma unroll 4
    for (int it = 0; it < kRsItems; ++it) {
        int64_t i = base + (int64_t)it * kRsThreads + threadIdx.x;
        if (i < n) atomicAdd(&h[(keys[i] >> shift) & 255u], 1);
    }
    __syncthreads();
    hist[(int64_t)threadIdx.x * ntiles + blockIdx.x] = h[threadIdx.x];
}

// Items of a tile are taken in rounds: round t holds items base + t*256 + tid,
// so (round, warp, lane) order is index order and the rank below is stable.
__global__ void radix_scatter_kernel(const uint32_t* __restrict__ kin, const int32_t* __restrict__ vin,
                                     uint32_t* __restrict__ kout, int32_t* __restrict__ vout, int64_t n,
                                     int shift, const int32_t* __restrict__ offs, int64_t ntiles) {
    __shared__ int32_t wcnt[kRsWarps][256];
    __shared__ int32_t wbase[kRsWarps][256];
    __shared__ int32_t tile_off[256];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    tile_off[tid] = offs[(int64_t)tid * ntiles + blockIdx.x];
    for (int w = 0; w < kRsWarps; ++w) wcnt[w][tid] = 0;
    int32_t run = 0;  // items of digit `tid` placed so far in this tile
    uint32_t lt_mask;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt_mask));
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kRsTile;
    for (int it = 0; it < kRsItems; ++it) {
        const int64_t i = base + (int64_t)it * kRsThreads + tid;
        const bool valid = i < n;
        uint32_t key = valid ? kin[i] : 0u;
        int32_t val = valid ? vin[i] : 0;
        uint32_t dg = valid ? ((key >> shift) & 255u) : (256u + lane);
        uint32_t peers = __match_any_sync(0xffffffffu, dg);
        int rank = __popc(peers & lt_mask);
        if (valid && rank == 0) wcnt[warp][dg] = __popc(peers);
        __syncthreads();
        {
            int32_t r = run;
#pragma unroll
            for (int w = 0; w < kRsWarps; ++w) {
                int32_t c = wcnt[w][tid];
                wbase[w][tid] = r;
                r += c;
                wcnt[w][tid] = 0;
            }
            run = r;
        }
        __syncthreads();
        if (valid) {
            int32_t pos = tile_off[dg] + wbase[warp][dg] + rank;
            kout[pos] = key;
            vout[pos] = val;
        }
    }
}

}  // namespace

int64_t scan_scratch_elems(int64_t n) {
    int64_t items = n + 1;
    if (items <= kScanChunk) return 0;
    int64_t nb = (items + kScanChunk - 1) / kScanChunk;
    return 2 * nb + 1 + scan_scratch_elems(nb);
}

// out has n+1 entries; out[n] = total.
void scan_exclusive(const int32_t* in, int32_t* out, int64_t n, int32_t* scratch, cudaStream_t s) {
    const int64_t items = n + 1;
    if (items <= kScanChunk) {
        note_launch();
        scan_chunk_kernel<<<1, kScanThreads, 0, s>>>(in, out, n, items, nullptr);
        return;
    }
    const int64_t nb = (items + kScanChunk - 1) / kScanChunk;
    int32_t* sums = scratch;
    int32_t* sums_scan = scratch + nb;
    note_launch();
    scan_chunk_kernel<<<(unsigned)nb, kScanThreads, 0, s>>>(in, out, n, items, sums);
    scan_exclusive(sums, sums_scan, nb, scratch + 2 * nb + 1, s);
    note_launch();
    scan_add_kernel<<<(unsigned)nb, kScanThreads, 0, s>>>(out, items, sums_scan);
}

int64_t radix_scratch_elems(int64_t n) {
    int64_t ntiles = (n + kRsTile - 1) / kRsTile;
    if (ntiles < 1) ntiles = 1;
    int64_t h = 256 * ntiles;
    return h + (h + 1) + scan_scratch_elems(h);
}

void radix_sort(uint32_t* k0, int32_t* v0, uint32_t* k1, int32_t* v1, int64_t n, int bits,
                int32_t* scratch, cudaStream_t s, uint32_t** kout, int32_t** vout) {
    uint32_t* kin = k0;
    int32_t* vin = v0;
    uint32_t* kalt = k1;
    int32_t* valt = v1;
    if (n > 0) {
        int64_t ntiles = (n + kRsTile - 1) / kRsTile;
        int64_t h = 256 * ntiles;
        int32_t* hist = scratch;
        int32_t* offs = scratch + h;
        int32_t* sc = scratch + 2 * h + 1;
        for (int shift = 0; shift < bits; shift += 8) {
            note_launch();
            radix_hist_kernel<<<(unsigned)ntiles, kRsThreads, 0, s>>>(kin, n, shift, hist, ntiles);
            scan_exclusive(hist, offs, h, sc, s);
            note_launch();
            radix_scatter_kernel<<<(unsigned)ntiles, kRsThreads, 0, s>>>(kin, vin, kalt, valt, n, shift,
                                                                        offs, ntiles);
            uint32_t* tk = kin; kin = kalt; kalt = tk;
            int32_t* tv = vin; vin = valt; valt = tv;
        }
    }
    *kout = kin;
    *vout = vin;
}

}  // namespace lsa
