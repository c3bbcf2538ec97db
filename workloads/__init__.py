"""Seeded synthetic inputs for the activation-sparse gated FFN.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
bench. It holds random-number generation and the workload shapes only: none of
the FFN's arithmetic (gate, activation, selection, projections) lives here.

Every tensor comes from its own torch CPU generator, seeded from
``(seed, tensor name)``, so a tensor does not change when another one is added
or resized.  Values are drawn in fp32 from N(0, 1), scaled, and rounded to the
storage dtype (round-to-nearest-even for bf16).

The shapes stand in for the pages' models (trained LLaMA-like FFNs evaluated
on C4 / MMLU / ARC / PIQA / TruthfulQA in "Mixture-of-Channels", section
"Cosa cambia nei numeri"), which are not available here: Gaussian weights with
variance 1/d make the dense gate pre-activation z ~ N(0, 1) per channel, so a
threshold tau = Phi^-1(s) gives sparsity s.
"""
from __future__ import annotations

import math
import statistics
import zlib
from dataclasses import dataclass, field
from typing import Dict, Optional

import torch

DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}


def _seed_for(seed: int, name: str) -> int:
    return (int(seed) * 0x9E3779B1 + zlib.crc32(name.encode())) & 0x7FFF_FFFF_FFFF


def normal(shape, std: float, dtype: str, seed: int, name: str) -> torch.Tensor:
    """N(0, std^2) samples of ``shape`` rounded to ``dtype`` ("bf16" or "f32")."""
    g = torch.Generator().manual_seed(_seed_for(seed, name))
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(DTYPES[dtype]).contiguous()


def tau_for_sparsity(s: float) -> float:
    """Threshold that leaves a fraction ``s`` of N(0,1) gate values inactive.

    The population quantile Phi^-1(s), rounded to fp32 so that the host, the
    oracle and the kernels all compare against the same number.
    """
    if s <= 0.0:
        return float("-inf")
    if s >= 1.0:
        return float("inf")
    q = statistics.NormalDist().inv_cdf(s)
    return float(torch.tensor(q, dtype=torch.float32).item())


def ffn_weights(d: int, d_ff: int, dtype: str = "bf16", seed: int = 0,
                gate: str = "dense", r: int = 0, tag: str = "") -> Dict[str, torch.Tensor]:
    """Weights of one gated FFN in the API layout (row-major, CPU).

    ``w_gate``: d x d_ff (gate == "dense"), ``A``: d x r and ``B``: r x d_ff
    (gate == "lopa"), ``w_up``: d x d_ff, ``w_down``: d_ff x d.
    Dense weights are N(0, 1/d).  LoPA factors each have variance
    1/sqrt(d*r), so that z = (x A) B has unit variance for x ~ N(0, 1).
    """
    out: Dict[str, torch.Tensor] = {}
    std = 1.0 / math.sqrt(d)
    if gate in ("dense", "both"):
        out["w_gate"] = normal((d, d_ff), std, dtype, seed, tag + "w_gate")
    if gate in ("lopa", "both"):
        if r <= 0:
            raise ValueError("a LoPA gate needs a rank r > 0")
        sab = (d * r) ** -0.25
        out["A"] = normal((d, r), sab, dtype, seed, tag + f"A{r}")
        out["B"] = normal((r, d_ff), sab, dtype, seed, tag + f"B{r}")
    out["w_up"] = normal((d, d_ff), std, dtype, seed, tag + "w_up")
    out["w_down"] = normal((d_ff, d), std, dtype, seed, tag + "w_down")
    return out


def tokens(n: int, d: int, dtype: str = "bf16", seed: int = 0, tag: str = "") -> torch.Tensor:
    """``n`` independent tokens x ~ N(0, 1)^d, shape n x d."""
    return normal((n, d), 1.0, dtype, seed, tag + f"x{n}")


def hot_channels(d_ff: int, frac: float, seed: int = 0) -> torch.Tensor:
    """A seeded random set of round(frac * d_ff) channels, ascending (int64)."""
    m = int(round(frac * d_ff))
    if m <= 0:
        return torch.zeros(0, dtype=torch.int64)
    g = torch.Generator().manual_seed(_seed_for(seed, "hot"))
    return torch.sort(torch.randperm(d_ff, generator=g)[:m]).values


def outlier_feature(d: int, seed: int = 0) -> int:
    """The input feature that carries the heavy hitters' common large value."""
    g = torch.Generator().manual_seed(_seed_for(seed, "outlier"))
    return int(torch.randint(d, (1,), generator=g).item())


@dataclass
class Workload:
    """One of the pages' workload shapes, as a synthetic stand-in."""
    name: str
    d: int
    d_ff: int
    n: int
    dtype: str
    gate: str                 # "dense" or "lopa"
    select: str               # "threshold", "topk" or "topp"
    r: int = 0
    sparsity: Optional[float] = None
    tau: Optional[float] = None
    k: int = 0
    p: float = 0.0            # top-p budget
    seed: int = 0
    extra: dict = field(default_factory=dict)
    hot_frac: float = 0.0     # heavy hitters: fraction of channels active for every token
    outlier: float = 0.0      # ... driven by this value in one feature of every token

    def __post_init__(self):
        if self.select == "threshold" and self.tau is None:
            self.tau = tau_for_sparsity(self.sparsity)

    def weights(self, gate: Optional[str] = None) -> Dict[str, torch.Tensor]:
        w = ffn_weights(self.d, self.d_ff, self.dtype, self.seed, gate or self.gate, self.r)
        if self.hot_frac > 0.0:
            # the outlier feature's gate weight of a hot channel sets its mean
            # pre-activation to tau + 3 (active with probability Phi(3))
            if "w_gate" not in w:
                raise ValueError("heavy hitters are defined for a dense gate")
            w["w_gate"][outlier_feature(self.d, self.seed), self.hot()] = (self.tau + 3.0) / self.outlier
        return w

    def x(self, n: Optional[int] = None, tag: str = "") -> torch.Tensor:
        x = tokens(self.n if n is None else n, self.d, self.dtype, self.seed, tag)
        if self.outlier:
            x[:, outlier_feature(self.d, self.seed)] = self.outlier
        return x

    def hot(self) -> torch.Tensor:
        """The heavy-hitter channels (ascending), empty without them."""
        return hot_channels(self.d_ff, self.hot_frac, self.seed)

    def describe(self) -> str:
        sel = (f"tau={self.tau:.5f}" if self.select == "threshold" else
               f"top-p p={self.p:g}" if self.select == "topp" else f"top-k k={self.k}")
        sp = f" sparsity={self.sparsity:g}" if self.sparsity is not None else ""
        rr = f" r={self.r}" if self.gate == "lopa" else ""
        hh = (f" heavy-hitters={len(self.hot())} outlier={self.outlier:g}" if self.hot_frac > 0.0 else "")
        return (f"{self.name}: d={self.d} d_ff={self.d_ff} n={self.n} {self.dtype} "
                f"{self.gate}-gate{rr} {sel}{sp}{hh}")


def tiny() -> Workload:
    """d=256, d_ff=1024, 4 tokens, fp32, ReLU(z - 1.2816) (about 90 % zeros)."""
    return Workload("tiny-relu", 256, 1024, 4, "f32", "dense", "threshold", tau=1.2816)


def llama7b_decode(sparsity: float = 0.9) -> Workload:
    """Llama-7B-shaped FFN decode: d=4096, d_ff=11008, one token, dense gate."""
    return Workload("llama7b-ffn-decode", 4096, 11008, 1, "bf16", "dense", "threshold",
                    sparsity=sparsity)


def lopa7b(sparsity: float = 0.9, n: int = 1) -> Workload:
    """LoPA gate A (4096 x 256) B (256 x 11008) on the Llama-7B FFN shapes."""
    return Workload("lopa7b-ffn-decode", 4096, 11008, n, "bf16", "lopa", "threshold",
                    r=256, sparsity=sparsity)


def moc_topk(n: int = 16) -> Workload:
    """Mixture-of-Channels top-K: d=2048, d_ff=5632, 16 tokens, K = d_ff / 8."""
    return Workload("moc-topk", 2048, 5632, n, "bf16", "dense", "topk", k=5632 // 8)


def heavy7b(n: int = 1, hot_frac: float = 0.02) -> Workload:
    """Llama-7B-shaped decode whose activations have heavy hitters: every
    token carries the value 16 in one input feature, and a fraction hot_frac
    of the channels respond to it strongly enough to be active for every
    token (the heavy-hitter abstract in the "FFN modules" paper listing: a
    few neurons have a large output for any input); the rest stay about 90 %
    sparse."""
    return Workload("heavy7b-ffn-decode", 4096, 11008, n, "bf16", "dense", "threshold",
                    sparsity=0.9, hot_frac=hot_frac, outlier=16.0)


def llama70b(n: int = 1, gate: str = "dense", sparsity: float = 0.9) -> Workload:
    """70B-shaped FFN: d=8192, d_ff=28672, dense gate or LoPA r=512."""
    return Workload("llama70b-ffn", 8192, 28672, n, "bf16", gate, "threshold",
                    r=512 if gate == "lopa" else 0, sparsity=sparsity)


LOPA_SPARSITIES = (0.8, 0.9, 0.95, 0.99)
SWEEP_70B_BATCHES = (1, 4, 16, 64)
SWEEP_70B_SPARSITIES = (0.5, 0.7, 0.8, 0.9, 0.95, 0.99)
