"""Seeded synthetic inputs for the ETA decode step.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no bound, threshold, gate or attention).  Both the CUDA
path and the float64 oracle are fed from it, so the two always see the same
bytes.

Workload shapes follow the decode-benchmark description of "Elastic Threshold
Attention: Learned Contextual Sparsity for Long-Context Decoding" (arXiv
2609.20888, abstract: batch >= 64, contexts up to 512K tokens, bf16 caches),
with clustered keys so that block-level screening has structure to find:

* cluster centroids mu_c = g / ||g||, g ~ N(0, I_d)
* the token axis of every (batch row, KV head) is cut into segments; each
  segment takes a cluster uniformly at random and its keys are
  k = mu_c + sigma_k * N(0, I_d)        (sigma_k = 0.3 per coordinate)
* every query head picks a cluster c uniformly and q = mu_c + N(0, 0.5 I_d)
  (0.5 read as the per-coordinate variance)
* V ~ N(0, 1) per coordinate
* the threshold predictor weight is W = alpha * N(0, 1/d), alpha = 0.1,
  shape [Hq*d, Hq] (rows follow the concatenated query heads)
* optional "needles": a fresh key of a query head's cluster, scaled 3x,
  planted at a uniform position of that head's KV sequence.

All tensors are torch tensors on the requested device; K/V/q are bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Tuple, Union

import torch


@dataclass(frozen=True)
class Workload:
    """Shape and structure of one synthetic decode workload."""

    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    ctx: int                       # context length (tokens per row)
    blk: int                       # KV block size
    n_clusters: int
    seg: Union[int, Tuple[int, int]]   # fixed segment length or inclusive range
    needles: int = 0               # planted needle keys per batch row
    gate_T: float = 0.0            # 0 = hard gate
    bound: str = "exact"           # "exact" | "prob"
    z: float = 3.0
    density: float = 0.38          # target density
    density_kind: str = "head"     # "head" (per query head) | "union"
    tau_mode: str = "predictor"    # "predictor" | "const"
    sigma_k: float = 0.3
    q_var: float = 0.5
    alpha: float = 0.1
    q_scale: float = 1.0           # >1 gives the "sharp" variant
    seed: int = 1000

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def T_max(self) -> int:
        return ((self.ctx + self.blk - 1) // self.blk) * self.blk

    @property
    def NB(self) -> int:
        return self.T_max // self.blk

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


# The five decode workloads of the ETA decode benchmark (see module doc).
TINY = Workload("tiny-b1-h4x1-d64-ctx4k-blk64", B=1, Hq=4, Hkv=1, d=64, ctx=4096,
                blk=64, n_clusters=8, seg=256, gate_T=0.0, density=0.38,
                density_kind="head", seed=1001)
MID = Workload("mid-b8-h16x4-d128-ctx32k-blk64-needles", B=8, Hq=16, Hkv=4, d=128,
               ctx=32768, blk=64, n_clusters=64, seg=256, needles=16, gate_T=0.05,
               density=0.38, density_kind="head", seed=1002)
LONG128K = Workload("long-b64-h16x4-d128-ctx128k-blk64", B=64, Hq=16, Hkv=4, d=128,
                    ctx=131072, blk=64, n_clusters=256, seg=(384, 640), gate_T=0.0,
                    density=0.16, density_kind="union", seed=1003)
EXTREME512K = Workload("extreme-b64-h16x4-d128-ctx512k-blk128", B=64, Hq=16, Hkv=4,
                       d=128, ctx=524288, blk=128, n_clusters=256, seg=(384, 640),
                       gate_T=0.0, bound="prob", z=3.0, density=0.16,
                       density_kind="union", seed=1004)
CALIB256K = Workload("calibrated-b64-h16x4-d128-ctx256k-blk64", B=64, Hq=16, Hkv=4,
                     d=128, ctx=262144, blk=64, n_clusters=256, seg=(384, 640),
                     gate_T=0.0, density=0.38, density_kind="head", tau_mode="const",
                     seed=1005)

WORKLOADS = {w.name: w for w in (TINY, MID, LONG128K, EXTREME512K, CALIB256K)}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def centroids(n: int, d: int, gen: torch.Generator, device) -> torch.Tensor:
    g = torch.randn(n, d, generator=gen, device=device, dtype=torch.float32)
    return g / g.norm(dim=1, keepdim=True)


def _segment_clusters(T: int, seg, n_clusters: int, gen, device) -> torch.Tensor:
    """Cluster id of every token of one (row, KV head) sequence, int64 [T]."""
    if isinstance(seg, int):
        nseg = (T + seg - 1) // seg
        cid = torch.randint(0, n_clusters, (nseg,), generator=gen, device=device)
        return cid.repeat_interleave(seg)[:T]
    lo, hi = seg
    nseg = (T + lo - 1) // lo + 1
    seglen = torch.randint(lo, hi + 1, (nseg,), generator=gen, device=device)
    ends = torch.cumsum(seglen, 0)
    cid = torch.randint(0, n_clusters, (nseg,), generator=gen, device=device)
    pos = torch.arange(T, device=device)
    which = torch.searchsorted(ends, pos, right=True)
    return cid[which]


def generate(w: Workload, device="cpu", seed: Optional[int] = None,
             lengths: Optional[torch.Tensor] = None, with_values: bool = True):
    """Draw one workload.

    Returns a dict with
      K, V      bf16 [B, Hkv, T_max, d]   (rows beyond lengths[b] are zero)
      lengths   int32 [B]
      q         bf16 [B, Hq, d]
      W         fp32 [Hq*d, Hq]
      mu        fp32 [n_clusters, d]
      q_cluster int64 [B, Hq]
    Generation is row by row so that very large caches never need a second
    full-size temporary.
    """
    seed = w.seed if seed is None else seed
    gen = _gen(device, seed)
    B, Hq, Hkv, d, Tm = w.B, w.Hq, w.Hkv, w.d, w.T_max
    mu = centroids(w.n_clusters, d, gen, device)
    if lengths is None:
        lengths = torch.full((B,), w.ctx, dtype=torch.int32, device=device)
    else:
        lengths = lengths.to(device=device, dtype=torch.int32)

    q_cluster = torch.randint(0, w.n_clusters, (B, Hq), generator=gen, device=device)
    qn = torch.randn(B, Hq, d, generator=gen, device=device) * math.sqrt(w.q_var)
    q = ((mu[q_cluster] + qn) * w.q_scale).to(torch.bfloat16)

    W = (torch.randn(Hq * d, Hq, generator=gen, device=device)
         * (w.alpha / math.sqrt(d))).contiguous()

    K = torch.zeros(B, Hkv, Tm, d, dtype=torch.bfloat16, device=device)
    V = torch.zeros(B, Hkv, Tm, d, dtype=torch.bfloat16, device=device) if with_values else None
    for b in range(B):
        L = int(lengths[b])
        for h in range(Hkv):
            cid = _segment_clusters(L, w.seg, w.n_clusters, gen, device)
            noise = torch.randn(L, d, generator=gen, device=device)
            K[b, h, :L] = (mu[cid] + w.sigma_k * noise).to(torch.bfloat16)
            if with_values:
                V[b, h, :L] = torch.randn(L, d, generator=gen, device=device).to(torch.bfloat16)
        for i in range(w.needles):
            if L == 0:
                break
            g = int(torch.randint(0, Hkv, (1,), generator=gen, device=device))
            hq = g * w.G + (i % w.G)
            c = q_cluster[b, hq]
            key = mu[c] + w.sigma_k * torch.randn(d, generator=gen, device=device)
            t = int(torch.randint(0, L, (1,), generator=gen, device=device))
            K[b, g, t] = (3.0 * key).to(torch.bfloat16)
    return dict(K=K, V=V, lengths=lengths, q=q, W=W, mu=mu, q_cluster=q_cluster)


def calibration_queries(w: Workload, mu: torch.Tensor, n: int = 64,
                        seed: Optional[int] = None) -> torch.Tensor:
    """n seeded calibration queries, bf16 [n, Hq, d], drawn like the step's q."""
    seed = (w.seed + 500) if seed is None else seed
    device = mu.device
    gen = _gen(device, seed)
    cl = torch.randint(0, w.n_clusters, (n, w.Hq), generator=gen, device=device)
    qn = torch.randn(n, w.Hq, w.d, generator=gen, device=device) * math.sqrt(w.q_var)
    return ((mu[cl] + qn) * w.q_scale).to(torch.bfloat16)


def ragged_lengths(B: int, ctx: int, blk: int, gen_seed: int = 7) -> torch.Tensor:
    """Row lengths <= ctx that are mostly not multiples of blk (edge-case tests)."""
    g = _gen("cpu", gen_seed)
    L = torch.randint(max(1, ctx // 2), ctx + 1, (B,), generator=g)
    L[0] = ctx
    if B > 1:
        L[1] = max(1, ctx - blk // 2 - 1)
    return L.to(torch.int32)
