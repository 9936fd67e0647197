"""Context parallelism: one long sequence split over the ranks of a process
group, one GPU per rank (orchestration only; every step is a library call).

The pages report 10M-token runs that split one sequence's context over
several GPUs (LSA explainer, "What do 22.7x and 72.4x actually compare?" and
"Can I run LSA?") without saying how.  Reading used here:

  - rank s holds the block-aligned token range [t0, t1) of K and V (the last
    rank also the tail and every token decode appends) and builds its own
    index over it, with the sink rule moved to its own positions
    (sink = max(0, S - t0));
  - select: every rank picks its local top ceil(K/P) blocks with their scores
    (lsa_select_blocks); one all-gather of the picks; every rank merges them
    into the same global top ceil(K/P) and writes the selection rows
    (lsa_merge_selection);
  - attend: every rank attends the rows of that selection it holds
    (lsa_localize_rows + lsa_sparse_attn with lse); one all-gather of the
    parts; every rank merges them by their log-sum-exps (lsa_merge_attn).

The exchange is `torch.distributed` (NCCL between GPUs, gloo on CPU).  The
phases are also exposed one by one (local_picks / merge_picks, local_attend /
merge_parts) so that a caller can run the shards of one sequence without a
process group, e.g. all on one device.
"""
from __future__ import annotations

import torch

from . import lsa


def shard_range(n_tokens: int, world: int, rank: int, pool: int):
    """Token range [t0, t1) of `rank`: the complete blocks are dealt in
    contiguous runs, the first (nb % world) ranks one block more; the last
    rank also takes the partial block at the end."""
    nb = n_tokens // pool
    base, extra = divmod(nb, world)
    b0 = rank * base + min(rank, extra)
    nbs = base + (1 if rank < extra else 0)
    t0 = b0 * pool
    t1 = (b0 + nbs) * pool if rank < world - 1 else n_tokens
    return t0, t1


def all_gather(t: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *t.shape]: every rank's tensor, stacked in rank order."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    t = t.contiguous()
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out.view(-1), t.view(-1), group=group)
        return out
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t, group=group)
    return torch.stack(parts)


class ContextShard:
    """One rank's part of a context-parallel sequence.

    n_tokens: tokens of the whole sequence at build time; pool, sink: the
    build's P and S (whole-sequence sink); gather: exchange function
    (default: all_gather over `group`)."""

    def __init__(self, rank: int, world: int, n_tokens: int, pool: int, sink: int, group=None, gather=None):
        self.rank, self.world = rank, world
        self.pool, self.sink = pool, sink
        self.t0, self.t1 = shard_range(n_tokens, world, rank, pool)
        self.local_sink = max(0, sink - self.t0)
        self.group = group
        self.gather = gather or (lambda t: all_gather(t, group))

    @property
    def last(self) -> bool:
        return self.rank == self.world - 1

    def build_params(self, batch, ld_tokens, hkv, d, r, dtype, level_sizes, lloyd_iters, grid_log2,
                     append_capacity=0):
        """The shard's build parameters: its own tokens, its sink."""
        return lsa.make_build_params(batch, self.t1 - self.t0, ld_tokens, hkv, d, r, self.pool, dtype, level_sizes,
                                     lloyd_iters, grid_log2, self.local_sink,
                                     append_capacity if self.last else 0)

    def local_params(self, sp):
        """Selection parameters with the sink in the shard's positions."""
        return lsa.make_select_params(sp.hq, sp.beam, sp.topk, self.local_sink, sp.window)

    # ------------------------------------------------------------ select
    def local_picks(self, index, sp, Q, q_pos=None, q_pos0=0, stream=None):
        """This shard's top blocks with scores (whole-sequence positions and
        block ids)."""
        return lsa.lsa_select_blocks(index, self.local_params(sp), Q, self.t0, q_pos=q_pos, q_pos0=q_pos0,
                                     stream=stream)

    def merge_picks(self, scores, blocks, count, sp, q_pos=None, q_pos0=0, max_sel=None, idx=None, cnt=None,
                    stream=None):
        """Selection rows from the picks of every shard ([world, ...] each)."""
        return lsa.lsa_merge_selection(scores, blocks, count, self.pool, sp.topk, self.sink, sp.window,
                                       q_pos=q_pos, q_pos0=q_pos0, max_sel=max_sel, idx=idx, cnt=cnt,
                                       stream=stream)

    def select(self, index, sp, Q, q_pos=None, q_pos0=0, max_sel=None, stream=None):
        """Selection rows of the whole sequence (the same on every rank)."""
        s, b, c = self.local_picks(index, sp, Q, q_pos=q_pos, q_pos0=q_pos0, stream=stream)
        return self.merge_picks(self.gather(s), self.gather(b), self.gather(c), sp, q_pos=q_pos, q_pos0=q_pos0,
                                max_sel=max_sel, stream=stream)

    # ------------------------------------------------------------ attend
    def local_attend(self, Q, K_local, V_local, idx, cnt, hkv, stream=None):
        """Attention over the selection's rows held here (O normalised over
        them, lse; no rows -> O = 0, lse = -inf)."""
        # the last shard also holds the tokens decode appended after t1
        t1 = self.t0 + K_local.shape[1] if self.last else self.t1
        li, lc = lsa.lsa_localize_rows(idx, cnt, self.t0, t1, stream=stream)
        return lsa.lsa_sparse_attn(Q, K_local, V_local, li, lc, hkv, stream=stream)

    @staticmethod
    def merge_parts(O_parts, lse_parts, stream=None):
        return lsa.lsa_merge_attn(O_parts, lse_parts, stream=stream)

    def attend(self, Q, K_local, V_local, idx, cnt, hkv, stream=None):
        """Attention over the whole selection (the same on every rank)."""
        o, l = self.local_attend(Q, K_local, V_local, idx, cnt, hkv, stream=stream)
        return self.merge_parts(self.gather(o), self.gather(l), stream=stream)

    # ------------------------------------------------------------ decode
    def append(self, index, K_local, n_new, stream=None):
        """Decode appends: only the last shard's range grows."""
        if self.last:
            lsa.lsa_append(index, K_local, n_new, stream=stream)
