// Bucket layout of a built tree.
//
// Leaves store their blocks contiguously (a query reads whole buckets once
// it has descended into them, tree-search wiki note, TL;DR): slots [leaf_start, leaf_start +
// leaf_cnt) hold the member blocks in ascending block order, followed by
// free slots that decode appends fill.  The latent keys are copied into the
// same order (Klp), so scoring a bucket reads one contiguous run.  Child
// lists of every upper node are ascending child ids.  minpos of a node is the
// smallest start position of a member block at or after the sink (kNoPos if
// none); a node is eligible for the query at i iff minpos <= i - W - P + 1.
//
// relayout_leaves lays the leaves out again from the current block labels
// (decode maintenance, lsa_relayout): blocks that found their leaf full on
// append take their place, every leaf gets fresh free slots for the append
// capacity that is left, and minpos is recomputed; memberships and centroids
// do not change.
#include "lsa_internal.cuh"

namespace lsa {
namespace {

__global__ void leaf_cap_kernel(const int32_t* __restrict__ off, int64_t nc, int64_t append_blocks, int64_t denom,
                                int32_t* __restrict__ cap) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= nc) return;
    const int64_t cnt = off[c + 1] - off[c];
    int64_t slack = 0;
    if (append_blocks > 0) slack = 2 + (2 * append_blocks * (cnt + 1) + denom - 1) / denom;
    cap[c] = (int32_t)(cnt + slack);
}

__global__ void leaf_layout_kernel(const int32_t* __restrict__ perm, const int32_t* __restrict__ off, int64_t nb,
                                   int L, int64_t nc, const int32_t* __restrict__ leaf_start,
                                   int32_t* __restrict__ leaf_cnt, const float* __restrict__ Kl, int64_t nb_cap,
                                   int r, float* __restrict__ Klp, int32_t* __restrict__ blk, int pool, int sink,
                                   int64_t* __restrict__ minpos, int64_t slots, int32_t* err) {
    const int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (c >= nc) return;
    const int64_t u = c / L;
    const int32_t s = off[c], e = off[c + 1];
    const int32_t st = leaf_start[c];
    if ((int64_t)st + (e - s) > slots) {   // the slot arrays cannot hold this leaf
        if (lane == 0) {
            latch(err, kErrCapacity);
            leaf_cnt[c] = 0;
            minpos[c] = kNoPos;
        }
        return;
    }
    int64_t mp = kNoPos;
    for (int32_t m = s; m < e; ++m) {
        const int64_t i = perm[m] - u * nb;
        const int64_t slot = st + (m - s);
        if (lane == 0) blk[slot] = (int32_t)i;
        for (int dim = lane; dim < r; dim += 32) Klp[slot * r + dim] = Kl[(u * nb_cap + i) * r + dim];
        if (mp == kNoPos && i * pool >= sink) mp = i * pool;
    }
    if (lane == 0) {
        leaf_cnt[c] = e - s;
        minpos[c] = mp;
    }
}

__global__ void child_ids_kernel(const int32_t* __restrict__ perm, int64_t total, int64_t n_child,
                                 int32_t* __restrict__ child_ids) {
    const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= total) return;
    const int64_t g = perm[p];
    child_ids[p] = (int32_t)(g % n_child);
}

__global__ void minpos_up_kernel(const int32_t* __restrict__ child_off, const int32_t* __restrict__ child_ids,
                                 int64_t nc, int n_l, int n_child, const int64_t* __restrict__ mp_child,
                                 int64_t* __restrict__ mp) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= nc) return;
    const int64_t u = c / n_l;
    int64_t best = kNoPos;
    for (int32_t q = child_off[c]; q < child_off[c + 1]; ++q) {
        const int64_t v = mp_child[u * n_child + child_ids[q]];
        if (v < best) best = v;
    }
    mp[c] = best;
}

// Tree order: level 0 keeps its ids; the children of the node at position q
// of level l take the positions [coff[q], coff[q+1]) of level l+1, in
// ascending child id.
__global__ void order_identity_kernel(int32_t* __restrict__ ord_id, int64_t total, int n_l) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e < total) ord_id[e] = (int32_t)(e % n_l);
}

__global__ void order_counts_kernel(const int32_t* __restrict__ ord_id, const int32_t* __restrict__ child_off,
                                    int64_t total, int n_l, int32_t* __restrict__ cnt) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= total) return;
    const int64_t u = e / n_l;
    const int64_t node = u * n_l + ord_id[e];
    cnt[e] = child_off[node + 1] - child_off[node];
}

__global__ void order_children_kernel(const int32_t* __restrict__ ord_id, const int32_t* __restrict__ child_off,
                                      const int32_t* __restrict__ child_ids, const int32_t* __restrict__ coff,
                                      int64_t total, int n_l, int n_child, int32_t* __restrict__ ord_id_child) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= total) return;
    const int64_t u = e / n_l;
    const int64_t node = u * n_l + ord_id[e];
    const int32_t s = child_off[node], n = child_off[node + 1] - s;
    for (int32_t k = 0; k < n; ++k) ord_id_child[coff[e] + k] = child_ids[s + k];
}

__global__ void order_gather_kernel(const int32_t* __restrict__ ord_id, int64_t total, int n_l, int r,
                                    const float* __restrict__ cent, const int64_t* __restrict__ mp,
                                    float* __restrict__ ocent, int64_t* __restrict__ omp, int32_t* __restrict__ opos) {
    const int64_t e = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (e >= total) return;
    const int64_t u = e / n_l;
    const int64_t node = u * n_l + ord_id[e];
    for (int c = lane; c < r; c += 32) ocent[e * r + c] = cent[node * r + c];
    if (lane == 0) {
        omp[e] = mp[node];
        opos[node] = (int32_t)(e - u * n_l);
    }
}

__global__ void clear_bits_kernel(int32_t* err, int32_t bits) { atomicAnd(err, ~bits); }

// Slots for every leaf (its members + free slots for `append_blocks` more
// blocks, shared in proportion to the leaf's size), then the members of every
// leaf in ascending block order with their latent keys, and leaf minpos.
int lay_out_leaves(lsa_index* ix, const int32_t* leaf_perm, const int32_t* leaf_off, int64_t append_blocks,
                   cudaStream_t s, Arena& A) {
    const lsa_build_params& p = ix->p;
    const int L = ix->L;
    const int64_t nc = ix->units * L;
    int32_t* cap = A.alloc<int32_t>(nc);
    int32_t* sc = A.alloc<int32_t>(scan_scratch_elems(nc) + 1);
    if (A.status != LSA_OK) return A.status;
    note_launch();
    leaf_cap_kernel<<<(unsigned)((nc + 255) / 256), 256, 0, s>>>(leaf_off, nc, append_blocks, ix->nb + L, cap);
    cudaMemcpyAsync(ix->leaf_cap, cap, nc * sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    scan_exclusive(cap, ix->leaf_start, nc, sc, s);
    note_launch();
    leaf_layout_kernel<<<(unsigned)((nc * 32 + 255) / 256), 256, 0, s>>>(
        leaf_perm, leaf_off, ix->nb, L, nc, ix->leaf_start, ix->leaf_cnt, ix->Kl, ix->nb_cap, p.r, ix->Klp, ix->blk,
        p.pool, p.sink, ix->minpos[p.levels - 1], ix->slots, ix->err);
    return cuda_status(cudaGetLastError());
}

// minpos of every upper node from its children's, bottom-up.
void minpos_upper(lsa_index* ix, cudaStream_t s) {
    const lsa_build_params& p = ix->p;
    const int64_t U = ix->units;
    for (int l = p.levels - 2; l >= 0; --l) {
        const int n_l = p.level_sizes[l], n_child = p.level_sizes[l + 1];
        note_launch();
        minpos_up_kernel<<<(unsigned)((U * n_l + 255) / 256), 256, 0, s>>>(ix->child_off[l], ix->child_ids[l],
                                                                           U * n_l, n_l, n_child,
                                                                           ix->minpos[l + 1], ix->minpos[l]);
    }
}

}  // namespace

void gather_tree_order(lsa_index* ix, cudaStream_t s) {
    const lsa_build_params& p = ix->p;
    for (int l = 0; l < p.levels; ++l) {
        const int64_t tot = ix->units * p.level_sizes[l];
        note_launch();
        order_gather_kernel<<<(unsigned)((tot * 32 + 255) / 256), 256, 0, s>>>(
            ix->ord_id[l], tot, p.level_sizes[l], p.r, ix->cent[l], ix->minpos[l], ix->ord_cent[l], ix->ord_mp[l],
            ix->ord_pos[l]);
    }
}

int finish_tree(lsa_index* ix, const int32_t* leaf_perm, const int32_t* leaf_off, const int32_t* const* up_perm,
                const int32_t* const* up_off, cudaStream_t s, Arena& A) {
    const lsa_build_params& p = ix->p;
    const int levels = p.levels;
    const int L = ix->L;
    const int64_t U = ix->units;
    const int64_t append_blocks = p.append_capacity > 0 ? (p.append_capacity + p.pool - 1) / p.pool + 1 : 0;
    int st = lay_out_leaves(ix, leaf_perm, leaf_off, append_blocks, s, A);
    if (st != LSA_OK) return st;
    for (int l = levels - 2; l >= 0; --l) {
        const int n_l = p.level_sizes[l], n_child = p.level_sizes[l + 1];
        const int64_t tot = U * n_child;
        cudaMemcpyAsync(ix->child_off[l], up_off[l], (U * n_l + 1) * sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
        note_launch();
        child_ids_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, s>>>(up_perm[l], tot, n_child, ix->child_ids[l]);
    }
    minpos_upper(ix, s);
    // tree order of every level
    int32_t* ocnt = A.alloc<int32_t>(U * (int64_t)p.level_sizes[levels - 1]);
    int32_t* osc = A.alloc<int32_t>(scan_scratch_elems(U * (int64_t)p.level_sizes[levels - 1]) + 1);
    if (A.status != LSA_OK) return A.status;
    {
        const int64_t t0 = U * p.level_sizes[0];
        note_launch();
        order_identity_kernel<<<(unsigned)((t0 + 255) / 256), 256, 0, s>>>(ix->ord_id[0], t0, p.level_sizes[0]);
    }
    for (int l = 0; l + 1 < levels; ++l) {
        const int n_l = p.level_sizes[l], n_child = p.level_sizes[l + 1];
        const int64_t tot = U * n_l;
        note_launch();
        order_counts_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, s>>>(ix->ord_id[l], ix->child_off[l], tot, n_l,
                                                                          ocnt);
        scan_exclusive(ocnt, ix->ord_coff[l], tot, osc, s);
        note_launch();
        order_children_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, s>>>(
            ix->ord_id[l], ix->child_off[l], ix->child_ids[l], ix->ord_coff[l], tot, n_l, n_child, ix->ord_id[l + 1]);
    }
    gather_tree_order(ix, s);
    return cuda_status(cudaGetLastError());
}

int relayout_leaves(lsa_index* ix, cudaStream_t s, Arena& A) {
    const lsa_build_params& p = ix->p;
    const int L = ix->L;
    const int64_t U = ix->units, nb = ix->nb;
    const int64_t left = p.n_tokens + p.append_capacity - ix->n_tokens;
    const int64_t append_blocks = left > 0 ? (left + p.pool - 1) / p.pool + 1 : 0;
    // every leaf's slots: members + 2 + ceil(2 A (members + 1) / (nb + L)),
    // at most nb + 3 L + 2 A per unit in all
    const int64_t worst = nb + (append_blocks > 0 ? 3 * (int64_t)L + 2 * append_blocks : 0);
    if (U * worst > ix->slots) return LSA_ERR_CAPACITY;
    int32_t* perm = A.alloc<int32_t>(U * nb);
    int32_t* off = A.alloc<int32_t>(U * (int64_t)L + 1);
    GroupWork gw = alloc_group_work(U, nb, L, A);
    if (A.status != LSA_OK) return A.status;
    // the blocks that found their leaf full are placed below
    note_launch();
    clear_bits_kernel<<<1, 1, 0, s>>>(ix->err, kErrCapacity);
    int st = group_by_label(ix->leaf_of_block, ix->nb_cap, U, nb, L, perm, off, ix->err, s, gw);
    if (st == LSA_OK) st = lay_out_leaves(ix, perm, off, append_blocks, s, A);
    if (st != LSA_OK) return st;
    minpos_upper(ix, s);
    gather_tree_order(ix, s);
    return cuda_status(cudaGetLastError());
}

}  // namespace lsa
