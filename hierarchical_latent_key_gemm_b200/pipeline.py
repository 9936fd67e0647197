"""Orchestration of the library calls on streams and graphs (no arithmetic).

HostPrefill: a whole prefill layer from host memory, with the copies
overlapped.  Binding calls and torch copies on three CUDA streams: K and W go
up first, and the index is built while V and then the queries go up chunk by chunk;
each chunk of consecutive queries is selected and attended (banded attention)
as soon as its queries have arrived, and its output goes back to the host
while the next chunk computes.  Every step moves all of Q, K, V and W up and
all of O down; the overlap only hides the transfers behind the kernels.

DecodeStep: decode with select + attention replayed from one CUDA graph.
"""
from __future__ import annotations

import torch

from . import lsa


class HostPrefill:
    """Device buffers and streams for repeated host-to-host prefill layers of
    one shape (batch 1).  `run` enqueues one layer and makes the current
    stream wait for it; it returns the layer's index (free it when done)."""

    def __init__(self, bp, sp, hQ, hK, hV, hW, hO, sink: int, window: int, chunks: int = 8, device=None):
        if hQ.shape[0] != 1:
            raise ValueError("HostPrefill handles batch 1 (O chunks are contiguous ranges of queries)")
        for t in (hQ, hK, hV, hW, hO):
            if not t.is_pinned():
                raise ValueError("host tensors must be pinned")
        self.dev = device or torch.device("cuda", torch.cuda.current_device())
        self.bp, self.sp = bp, sp
        self.hQ, self.hK, self.hV, self.hW, self.hO = hQ, hK, hV, hW, hO
        self.sink, self.window = sink, window
        self.dQ = torch.empty(hQ.shape, dtype=hQ.dtype, device=self.dev)
        self.dK = torch.empty(hK.shape, dtype=hK.dtype, device=self.dev)
        self.dV = torch.empty(hV.shape, dtype=hV.dtype, device=self.dev)
        self.dW = torch.empty(hW.shape, dtype=hW.dtype, device=self.dev)
        self.dO = torch.empty(hO.shape, dtype=hO.dtype, device=self.dev)
        nq = hQ.shape[1]
        self.bounds = [(nq * c) // chunks for c in range(chunks + 1)]
        self.bounds = sorted(set(self.bounds))
        cmax = max(b - a for a, b in zip(self.bounds[:-1], self.bounds[1:]))
        kb = -(-sp.topk // bp.pool)
        self.max_sel = kb * bp.pool + bp.sink + sp.window
        self.idx = torch.empty((1, cmax, bp.hkv, self.max_sel), dtype=torch.int32, device=self.dev)
        self.cnt = torch.empty((1, cmax, bp.hkv), dtype=torch.int32, device=self.dev)
        self.lse = torch.empty((1, nq, hQ.shape[2]), dtype=torch.float32, device=self.dev)
        self.s_in = torch.cuda.Stream(self.dev)
        self.s_comp = torch.cuda.Stream(self.dev)
        self.s_out = torch.cuda.Stream(self.dev)

    @property
    def h2d_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.hQ, self.hK, self.hV, self.hW))

    @property
    def d2h_bytes(self) -> int:
        return self.hO.numel() * self.hO.element_size()

    def run(self):
        """Enqueue one layer after the work already on the current stream; the
        current stream waits for all of it (the output is on the host once the
        current stream reaches this point)."""
        cur = torch.cuda.current_stream(self.dev)
        start = torch.cuda.Event()
        start.record(cur)
        for s in (self.s_in, self.s_comp, self.s_out):
            s.wait_event(start)
        ev_kw, ev_v = torch.cuda.Event(), torch.cuda.Event()
        q_ev, o_ev = [], []
        with torch.cuda.stream(self.s_in):
            # K and W first (the build needs them); V goes up during the build
            self.dK.copy_(self.hK, non_blocking=True)
            self.dW.copy_(self.hW, non_blocking=True)
            ev_kw.record(self.s_in)
            self.dV.copy_(self.hV, non_blocking=True)
            ev_v.record(self.s_in)
            for a, b in zip(self.bounds[:-1], self.bounds[1:]):
                self.dQ[:, a:b].copy_(self.hQ[:, a:b], non_blocking=True)
                e = torch.cuda.Event()
                e.record(self.s_in)
                q_ev.append(e)
        self.s_comp.wait_event(ev_kw)
        ix = lsa.lsa_build_index(self.bp, self.dK, self.dW, stream=self.s_comp)
        self.s_comp.wait_event(ev_v)
        for c, (a, b) in enumerate(zip(self.bounds[:-1], self.bounds[1:])):
            self.s_comp.wait_event(q_ev[c])
            n = b - a
            q = self.dQ[:, a:b]
            idx, cnt = self.idx[:, :n], self.cnt[:, :n]
            lsa.lsa_select(ix, self.sp, q, idx=idx, cnt=cnt, max_sel=self.max_sel, q_pos0=a, stream=self.s_comp)
            lsa.lsa_sparse_attn_banded(q, self.dK, self.dV, idx, cnt, self.bp.hkv, self.sink, self.window,
                                       q_pos0=a, O=self.dO[:, a:b], lse=self.lse[:, a:b], stream=self.s_comp)
            e = torch.cuda.Event()
            e.record(self.s_comp)
            o_ev.append(e)
            self.s_out.wait_event(e)
            with torch.cuda.stream(self.s_out):
                self.hO[:, a:b].copy_(self.dO[:, a:b], non_blocking=True)
        # the index lives until the compute stream is done with it
        done_comp = torch.cuda.Event()
        done_comp.record(self.s_comp)
        for s in (self.s_in, self.s_comp, self.s_out):
            e = torch.cuda.Event()
            e.record(s)
            cur.wait_event(e)
        return ix


class DecodeStep:
    """Decode steps with little host work: the append runs as a plain call
    (whether it launches depends on the token completing a block), and select +
    attention for the new queries replay one CUDA graph captured at set-up.
    The graph reads the queries and their positions from fixed device buffers,
    and the index's device arrays carry every appended block, so one capture
    serves all later steps (tree selection reads no host-side block count)."""

    def __init__(self, index, sp, K, V, hq: int, max_sel: int, device=None):
        p = index.params
        self.dev = device or K.device
        self.index, self.sp, self.K, self.V = index, sp, K, V
        self.hkv, self.max_sel = p.hkv, max_sel
        B, d = p.batch, p.d
        self.q = torch.zeros((B, 1, hq, d), dtype=K.dtype, device=self.dev)
        self.pos = torch.full((B, 1), max(0, p.n_tokens - 1), dtype=torch.int64, device=self.dev)
        self.idx = torch.empty((B, 1, p.hkv, max_sel), dtype=torch.int32, device=self.dev)
        self.cnt = torch.empty((B, 1, p.hkv), dtype=torch.int32, device=self.dev)
        self.O = torch.empty((B, 1, hq, d), dtype=K.dtype, device=self.dev)
        self.lse = torch.empty((B, 1, hq), dtype=torch.float32, device=self.dev)
        side = torch.cuda.Stream(self.dev)
        side.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(side):
            self._select_attend()          # eager once: kernel attributes, scratch pool
        torch.cuda.current_stream(self.dev).wait_stream(side)
        torch.cuda.synchronize(self.dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=side):
            self._select_attend()

    def _select_attend(self):
        lsa.lsa_select(self.index, self.sp, self.q, q_pos=self.pos, idx=self.idx, cnt=self.cnt,
                       max_sel=self.max_sel)
        lsa.lsa_sparse_attn(self.q, self.K, self.V, self.idx, self.cnt, self.hkv, O=self.O, lse=self.lse)

    def step(self, q_new, pos: int):
        """Index the token at `pos` (already written into K), then select and
        attend for q_new [batch, 1, hq, d] at that position; returns (O, lse)
        buffers that the next step overwrites."""
        lsa.lsa_append(self.index, self.K, 1)
        self.q.copy_(q_new)
        self.pos.fill_(pos)
        self.graph.replay()
        return self.O, self.lse
