"""Seeded synthetic workloads for the LSA hot path.

This module only draws inputs (keys, queries, values, the latent map and the
planted needles).  It holds none of the method's arithmetic, so the CUDA path
and the CPU oracle can both consume what it produces.  Every tensor comes from
torch's own generator on the requested device, seeded per stream, so a given
(workload, seed, device) always yields the same bytes.

Workload shapes (one attention layer each):
  flat_4k_f32    causal prefill of 4096 tokens, 1 query / 1 KV head, d=128 fp32,
                 flat 64-bucket index, r=32, no pooling
  int_exact_16k  16384 tokens, GQA 4:1, d=64, integer-valued bf16 inputs, a
                 {-1,0,+1} map, 16x16 tree on the 1/16 grid (bit-exact indexing)
  gqa_128k       131072 tokens, 32 query / 4 KV heads, d=128 bf16, r=64, pool 4,
                 32x32 tree, 64 planted needles
  prefill_1m     1,048,576 tokens, 16 / 2 heads, 16x32x32 tree, drifting mixture
                 weights every 64K tokens, 256 needles
  decode_10m_x4  4 sequences of 10,000,000 cached tokens, 16 / 1 heads,
                 32x32x64 tree, then 256 decode steps, 1024 needles
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    n_tokens: int            # context length per sequence at build time
    batch: int               # sequences
    hq: int                  # query heads
    hkv: int                 # KV heads
    d: int                   # head dimension
    dtype: str               # "f32" or "bf16" (Q, K, V and O)
    r: int                   # latent rank
    pool: int                # keys per pooled block
    level_sizes: tuple       # nodes per tree level, top first, leaves last
    lloyd_iters: int
    grid_log2: int           # 0: float centroids; g > 0: centroids on multiples of 2**-g
    beam: int                # B
    topk: int                # K, in tokens
    sink: int                # S
    window: int              # W
    kind: str = "mixture"    # "mixture" (Gaussian mixture) or "int" (uniform integers)
    components: int = 0      # mixture components
    sigma: float = 0.3       # mixture noise
    needles: int = 0         # planted needle keys (total over sequences and KV heads)
    needle_gap: int = 100_000
    drift_every: int = 0     # tokens per segment of constant mixture weights (0: uniform)
    decode_steps: int = 0

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def n_blocks(self) -> int:
        return self.n_tokens // self.pool

    @property
    def topk_blocks(self) -> int:
        return -(-self.topk // self.pool)

    @property
    def max_sel(self) -> int:
        """Upper bound on selected tokens per (query, KV head)."""
        return self.topk_blocks * self.pool + self.sink + self.window

    def scaled(self, **kw) -> "Workload":
        """Same recipe at other sizes (used for parity cases the oracle finishes)."""
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "flat_4k_f32": Workload(
        "flat_4k_f32", 4096, 1, 1, 1, 128, "f32", 32, 1, (64,), 10, 0, 8, 256, 4, 128,
        kind="mixture", components=64, sigma=0.3),
    "int_exact_16k": Workload(
        "int_exact_16k", 16384, 1, 4, 1, 64, "bf16", 16, 1, (16, 256), 5, 4, 16, 512, 4, 256,
        kind="int"),
    "gqa_128k": Workload(
        "gqa_128k", 131072, 1, 32, 4, 128, "bf16", 64, 4, (32, 1024), 8, 0, 32, 2048, 64, 512,
        kind="mixture", components=4096, sigma=0.25, needles=64),
    "prefill_1m": Workload(
        "prefill_1m", 1 << 20, 1, 16, 2, 128, "bf16", 64, 4, (16, 512, 16384), 6, 0, 64, 2048, 64, 1024,
        kind="mixture", components=16384, sigma=0.25, needles=256, drift_every=1 << 16),
    "decode_10m_x4": Workload(
        "decode_10m_x4", 10_000_000, 4, 16, 1, 128, "bf16", 64, 4, (32, 1024, 65536), 6, 0, 64, 2048, 64, 2048,
        kind="mixture", components=65536, sigma=0.25, needles=1024, decode_steps=256),
}

# stream ids: each input draws from its own seeded generator
_S_CENTRES, _S_KCOMP, _S_KNOISE, _S_QCOMP, _S_QNOISE, _S_V, _S_W, _S_NEEDLE, _S_DRIFT = range(9)


def _gen(device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1009 + stream * 7919 + 17)
    return g


def torch_dtype(w: Workload):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def make_map(w: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    """The seeded latent map W [d, r] (fp32).  Integer workload: every row has
    4 nonzeros in {-1, +1} at seeded positions.  Otherwise: orthonormal columns
    (Gram-Schmidt of a seeded Gaussian matrix)."""
    g = _gen("cpu", seed, _S_W)
    if w.kind == "int":
        Wm = torch.zeros(w.d, w.r, dtype=torch.float32)
        nnz = min(4, w.r)
        for row in range(w.d):
            cols = torch.randperm(w.r, generator=g)[:nnz]
            signs = torch.randint(0, 2, (nnz,), generator=g).float() * 2 - 1
            Wm[row, cols] = signs
    else:
        # modified Gram-Schmidt in float64: the same bits on every host (a
        # threaded LAPACK QR need not be bitwise reproducible)
        A = torch.randn(w.d, w.r, generator=g, dtype=torch.float64).numpy()
        Qm = np.zeros_like(A)
        for j in range(w.r):
            v = A[:, j].copy()
            for i in range(j):
                v -= float(np.dot(Qm[:, i], v)) * Qm[:, i]
            Qm[:, j] = v / float(np.sqrt(np.dot(v, v)))
        Wm = torch.from_numpy(Qm).to(torch.float32)
    return Wm.contiguous().to(device)


def _segment_cdfs(w: Workload, n: int, seed: int) -> np.ndarray | None:
    """Cumulative mixture weights per drift segment (float64, CPU): logits
    take a Gaussian random walk (step 0.5) from one segment to the next.
    None = uniform weights."""
    if not w.drift_every:
        return None
    nseg = -(-n // w.drift_every)
    g = _gen("cpu", seed, _S_DRIFT)
    steps = torch.randn(nseg, w.components, generator=g, dtype=torch.float64) * 0.5
    logits = torch.cumsum(steps, dim=0)
    weights = torch.softmax(logits, dim=1).numpy()
    cdf = np.cumsum(weights, axis=1)
    cdf[:, -1] = 1.0
    return cdf


def _components(w: Workload, n: int, count_per_pos: int, seed: int, stream: int, device) -> torch.Tensor:
    """Mixture component per (position, slot): [n, count_per_pos] int64.
    Drifting weights are sampled by inverse CDF (uniform draws located in the
    segment's cumulative weights), which gives the same draws on any device."""
    g = _gen(device, seed, stream)
    cdfs = _segment_cdfs(w, n, seed)
    if cdfs is None:
        return torch.randint(0, w.components, (n, count_per_pos), generator=g, device=device)
    out = torch.empty(n, count_per_pos, dtype=torch.int64, device=device)
    for s in range(cdfs.shape[0]):
        lo, hi = s * w.drift_every, min(n, (s + 1) * w.drift_every)
        cdf = torch.from_numpy(cdfs[s]).to(device)
        u = torch.rand((hi - lo) * count_per_pos, generator=g, device=device, dtype=torch.float64)
        c = torch.searchsorted(cdf, u, right=True).clamp_(max=w.components - 1)
        out[lo:hi] = c.view(hi - lo, count_per_pos)
    return out


def make_inputs(w: Workload, seed: int = 0, device="cpu", chunk: int = 1 << 18) -> dict:
    """Draw one workload's inputs.

    Returns a dict with
      K, V  [batch, n_cap, hkv, d]  (n_cap = n_tokens + decode_steps; rows past
            n_tokens are the keys/values the decode steps append)
      Q     [batch, n_tokens, hq, d] for prefill workloads, or
            [batch, decode_steps, hq, d] for decode workloads (query of the
            token at position n_tokens + step)
      W     [d, r] fp32
      needles: list of (seq, kv_head, key_pos, query_pos)
    """
    dt = torch_dtype(w)
    B, N, Hq, Hkv, d = w.batch, w.n_tokens, w.hq, w.hkv, w.d
    G = w.group
    n_cap = N + w.decode_steps
    Wm = make_map(w, seed, device)
    if w.kind == "int":
        gk, gq, gv = _gen(device, seed, _S_KNOISE), _gen(device, seed, _S_QNOISE), _gen(device, seed, _S_V)
        K = torch.randint(-4, 5, (B, n_cap, Hkv, d), generator=gk, device=device).to(dt)
        V = torch.randint(-4, 5, (B, n_cap, Hkv, d), generator=gv, device=device).to(dt)
        nq = N if not w.decode_steps else w.decode_steps
        Q = torch.randint(-4, 5, (B, nq, Hq, d), generator=gq, device=device).to(dt)
        return {"K": K, "V": V, "Q": Q, "W": Wm, "needles": []}

    gc = _gen(device, seed, _S_CENTRES)
    mu = torch.randn(w.components, d, generator=gc, device=device)
    K = torch.empty(B, n_cap, Hkv, d, dtype=dt, device=device)
    V = torch.empty(B, n_cap, Hkv, d, dtype=dt, device=device)
    gkn, gv = _gen(device, seed, _S_KNOISE), _gen(device, seed, _S_V)
    for b in range(B):
        comp = _components(w, n_cap, Hkv, seed + 7 * b, _S_KCOMP, device)
        for lo in range(0, n_cap, chunk):
            hi = min(n_cap, lo + chunk)
            noise = torch.randn(hi - lo, Hkv, d, generator=gkn, device=device)
            K[b, lo:hi] = (mu[comp[lo:hi]] + w.sigma * noise).to(dt)
            V[b, lo:hi] = torch.randn(hi - lo, Hkv, d, generator=gv, device=device).to(dt)

    gqn = _gen(device, seed, _S_QNOISE)
    decode = w.decode_steps > 0
    nq = w.decode_steps if decode else N
    Q = torch.empty(B, nq, Hq, d, dtype=dt, device=device)
    for b in range(B):
        comp = _components(w, n_cap, Hkv, seed + 7 * b + 3, _S_QCOMP, device)
        if decode:
            comp = comp[N:N + nq]
        for lo in range(0, nq, chunk):
            hi = min(nq, lo + chunk)
            base = mu[comp[lo:hi]]                                   # [n, Hkv, d]
            base = base.repeat_interleave(G, dim=1)                  # [n, Hq, d]
            noise = torch.randn(hi - lo, Hq, d, generator=gqn, device=device)
            Q[b, lo:hi] = (base + w.sigma * noise).to(dt)

    needles = []
    if w.needles:
        gn = _gen("cpu", seed, _S_NEEDLE)
        kn = K[0, : min(N, 4096)].float().norm(dim=-1).flatten()
        qn = Q[0, : min(nq, 4096)].float().norm(dim=-1).flatten()
        k_scale = 2.0 * float(kn.median())
        q_scale = float(qn.median())
        gap = min(w.needle_gap, N // 2)
        per = -(-w.needles // (B * Hkv))
        used = set()
        for b in range(B):
            for h in range(Hkv):
                for _ in range(per):
                    if len(needles) >= w.needles:
                        break
                    u = torch.randn(d, generator=gn, dtype=torch.float64)
                    u = (u / u.norm()).to(torch.float32).to(device)
                    lo_k = w.sink + w.pool
                    while True:
                        p = int(torch.randint(lo_k, N - gap, (1,), generator=gn))
                        if decode:
                            qp = N + int(torch.randint(0, nq, (1,), generator=gn))
                        else:
                            qp = int(torch.randint(p + gap, N, (1,), generator=gn))
                        if (b, p) not in used and (b, qp) not in used:
                            used.add((b, p)); used.add((b, qp))
                            break
                    K[b, p, h] = (u * k_scale).to(dt)
                    qrow = qp - N if decode else qp
                    noise = torch.randn(G, d, generator=gn).to(device)
                    Q[b, qrow, h * G:(h + 1) * G] = (u[None, :] * q_scale + w.sigma * noise).to(dt)
                    needles.append((b, h, p, qp))
    return {"K": K, "V": V, "Q": Q, "W": Wm, "needles": needles}


def input_bytes(w: Workload) -> dict:
    """Bytes of each input tensor (for memory planning and e2e accounting)."""
    es = 4 if w.dtype == "f32" else 2
    n_cap = w.n_tokens + w.decode_steps
    nq = w.decode_steps if w.decode_steps else w.n_tokens
    return {"K": w.batch * n_cap * w.hkv * w.d * es, "V": w.batch * n_cap * w.hkv * w.d * es,
            "Q": w.batch * nq * w.hq * w.d * es, "W": w.d * w.r * 4}


def describe(w: Workload) -> str:
    return (f"{w.name}: N={w.n_tokens} x{w.batch}, Hq/Hkv={w.hq}/{w.hkv}, d={w.d} {w.dtype}, r={w.r}, "
            f"P={w.pool}, tree={'x'.join(str(s) for s in _fanouts(w.level_sizes))}, iters={w.lloyd_iters}, "
            f"B={w.beam}, K={w.topk}, S={w.sink}, W={w.window}")


def _fanouts(sizes):
    out, prev = [], 1
    for s in sizes:
        out.append(max(1, s // prev))
        prev = s
    return out


__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_map", "input_bytes", "describe", "torch_dtype"]
