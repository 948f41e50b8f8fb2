"""Seeded synthetic workloads for the attention forward pass.

This module only describes workloads and draws random numbers.  It holds none
of the attention arithmetic, so both the CUDA path and the CPU oracle can take
their inputs from here without sharing any of the method's code.

Recipe (the pages name no dataset; every input is synthetic):
  * Q, K, V are drawn i.i.d. N(0, 1) as fp32 from one CPU ``torch.Generator``
    seeded per workload, in the order Q, then K, then V, and rounded to bf16
    (round-to-nearest-even) by ``Tensor.to(torch.bfloat16)``.
  * Layout is ``[B, N, H, d]`` with ``d`` contiguous.
  * The long-sequence workload additionally scales 1 % of the Q entries and,
    independently, 1 % of the K entries by 8 before rounding: for each tensor,
    ``round(0.01 * numel)`` positions are picked by ``randperm`` from the same
    generator (Q's positions first, then K's).
  * ``softmax_scale = 1 / sqrt(d)``.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int = 0
    outlier_frac: float = 0.0
    outlier_scale: float = 8.0
    description: str = field(default="", compare=False)
    # local (sliding-window) attention: key j visible to row i iff
    # g - window_left <= j <= g + window_right, g = i + Nk - Nq; -1 = open side
    window_left: int = -1
    window_right: int = -1

    @property
    def windowed(self) -> bool:
        return self.window_left >= 0 or self.window_right >= 0

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    # ---- bookkeeping used by the benchmark (counts, not attention math) ----
    def flops(self) -> float:
        """Algorithmic FLOPs: 4*B*Hq*Nq*Nk*d, halved when causal; with a window,
        4*B*Hq*d per visible (query, key) pair, counted exactly."""
        if not self.windowed:
            f = 4.0 * self.B * self.Hq * self.Nq * self.Nk * self.d
            return f / 2.0 if self.causal else f
        return 4.0 * self.B * self.Hq * self.d * float(self.visible_pairs())

    def visible_pairs(self) -> int:
        """Number of visible (query row, key) pairs of one head (a count of index ranges)."""
        g = np.arange(self.Nq, dtype=np.int64) + (self.Nk - self.Nq)
        hi = np.full(self.Nq, self.Nk - 1, dtype=np.int64)
        lo = np.zeros(self.Nq, dtype=np.int64)
        if self.causal:
            hi = np.minimum(hi, g)
        if self.window_right >= 0:
            hi = np.minimum(hi, g + self.window_right)
        if self.window_left >= 0:
            lo = np.maximum(lo, g - self.window_left)
        return int(np.maximum(hi - lo + 1, 0).sum())

    def compulsory_bytes(self) -> int:
        """Read Q, K, V once (bf16), write O once (bf16) and LSE (fp32)."""
        q = self.B * self.Nq * self.Hq * self.d * 2
        kv = 2 * self.B * self.Nk * self.Hkv * self.d * 2
        o = self.B * self.Nq * self.Hq * self.d * 2
        lse = self.B * self.Hq * self.Nq * 4
        return q + kv + o + lse


# The five workloads the forward pass is specified and measured on.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 2, 256, 256, 64, False, seed=0,
                     description="tiny non-causal, B=1 H=2 N=256 d=64"),
    "noncausal_2k": Workload("noncausal_2k", 4, 16, 16, 2048, 2048, 128, False,
                             description="non-causal, B=4 H=16 N=2048 d=128"),
    "causal_8k": Workload("causal_8k", 2, 16, 16, 8192, 8192, 128, True,
                          description="causal, B=2 H=16 N=8192 d=128"),
    "long_32k": Workload("long_32k", 1, 2, 2, 32768, 32768, 128, True,
                         outlier_frac=0.01, outlier_scale=8.0,
                         description="long single-sequence causal, B=1 H=2 N=32768 d=128, "
                                     "1% of Q/K entries x8"),
    "gqa_4k": Workload("gqa_4k", 4, 32, 8, 4096, 4096, 128, True,
                       description="GQA causal, B=4 Hq=32 Hkv=8 N=4096 d=128"),
}

# Further workloads for the variants built on the same path (not among the
# five above): local attention with a causal window of 1024 keys per row, and
# a short query block against a long key sequence (16 units of 256 K/V tiles:
# one block per unit leaves most SMs idle; the split-KV schedule does not).
EXTRA_WORKLOADS = {
    "shortq_32k": Workload("shortq_32k", 1, 16, 16, 256, 32768, 128, False,
                           description="short query vs long keys, B=1 H=16 Nq=256 Nk=32768 d=128"),
    "local_8k": Workload("local_8k", 2, 16, 16, 8192, 8192, 128, True, window_left=1023,
                         description="causal sliding window of 1024 keys, B=2 H=16 N=8192 d=128"),
}


def make_qkv(w: Workload, seed: int | None = None):
    """Draw (q, k, v) as CPU bf16 tensors ``[B, N, H, d]`` following the recipe above."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    q = torch.randn((w.B, w.Nq, w.Hq, w.d), generator=g, dtype=torch.float32)
    k = torch.randn((w.B, w.Nk, w.Hkv, w.d), generator=g, dtype=torch.float32)
    v = torch.randn((w.B, w.Nk, w.Hkv, w.d), generator=g, dtype=torch.float32)
    if w.outlier_frac > 0.0:
        for t in (q, k):
            n = t.numel()
            cnt = int(round(w.outlier_frac * n))
            idx = torch.randperm(n, generator=g)[:cnt]
            flat = t.view(-1)
            flat[idx] = flat[idx] * w.outlier_scale
    return (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16))


def shard_seed(w: Workload, rank: int) -> int:
    """Seed of rank `rank`'s share of a multi-GPU job (rank 0's equals the
    single-GPU inputs)."""
    return w.seed + rank


def global_workload(w: Workload, world: int) -> Workload:
    """The whole job of `world` ranks that each hold workload `w`: the KV-head
    groups of one problem are split across the ranks, rank r holding query
    heads [r*Hq, (r+1)*Hq) and KV heads [r*Hkv, (r+1)*Hkv) (whole groups, so
    no rank needs another's K or V)."""
    return w.with_(name=f"{w.name}_x{world}", Hq=w.Hq * world, Hkv=w.Hkv * world)


def make_global_qkv(w: Workload, world: int):
    """Inputs of the whole job in the single-GPU layout ``[B, N, H, d]``: rank
    r's head slice is ``make_qkv(w, seed=shard_seed(w, r))``."""
    parts = [make_qkv(w, seed=shard_seed(w, r)) for r in range(world)]
    return tuple(torch.cat([p[i] for p in parts], dim=2) for i in range(3))


def sample_rows(w: Workload, n_sample: int = 1024, seed: int | None = None) -> np.ndarray:
    """Seeded sample of query rows used when every row is too many for the oracle.

    Always includes the tile edges 0, 127, 128, 255 and the last row; the rest
    are drawn uniformly without replacement.  Returned sorted, int32.
    """
    if n_sample >= w.Nq:
        return np.arange(w.Nq, dtype=np.int32)
    g = torch.Generator(device="cpu")
    g.manual_seed(1 + (seed if seed is not None else 0))
    must = sorted({r for r in (0, 127, 128, 255, w.Nq - 1) if 0 <= r < w.Nq})
    perm = torch.randperm(w.Nq, generator=g).numpy()
    rest = [int(r) for r in perm if int(r) not in must][: max(0, n_sample - len(must))]
    return np.array(sorted(must + rest), dtype=np.int32)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 array of its bit patterns (no rounding, no copy of values)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
