"""Seeded synthetic packed-document workloads.

This module holds NO arithmetic of the attention method: it only draws document
lengths and random tensors.  It is the one module that both the CUDA path's
callers (tests, bench) and the CPU oracle's callers use, so that both sides see
the same bf16 bits.

Recipe (all CPU, deterministic for a given seed):
  * document lengths and outlier indices: ``numpy.random.default_rng(seed)``;
  * tensors: ``torch.Generator().manual_seed(seed)``, one ``torch.randn`` call
    per tensor in the order Q, K, V, dO, in fp32, outliers applied in fp32,
    then rounded to bf16.

The FLAMIA page measures on unnamed "causal packed-document workloads" and
gives no shapes, so the shapes below are synthetic stand-ins of the kind the
page describes (packed variable-length documents, long context, GQA).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, Dict, List, Optional

import numpy as np
import torch


def lengths_uniform(rng: np.random.Generator, T: int, lo: int, hi: int,
                    first: Optional[List[int]] = None) -> List[int]:
    """Draw L ~ U{lo..hi} (inclusive) until the lengths cover T; the last
    document is truncated so that the lengths sum to exactly T (it may be short,
    even one token).  ``first`` lengths are placed before the drawn ones."""
    out = list(first or [])
    total = sum(out)
    while total < T:
        L = int(rng.integers(lo, hi + 1))
        L = min(L, T - total)
        out.append(L)
        total += L
    return out


def lengths_lognormal(rng: np.random.Generator, T: int, median: float, sigma: float,
                      lo: int, hi: int) -> List[int]:
    """L = clip(round(exp(N(ln median, sigma))), lo, hi), fill then truncate."""
    out: List[int] = []
    total = 0
    mu = math.log(median)
    while total < T:
        L = int(np.clip(np.rint(np.exp(rng.normal(mu, sigma))), lo, hi))
        L = min(L, T - total)
        out.append(L)
        total += L
    return out


def cu_from_lengths(lengths: List[int]) -> np.ndarray:
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu


@dataclasses.dataclass
class Workload:
    """One synthetic packed-document attention problem."""
    name: str
    T: int
    Hq: int
    Hkv: int
    d: int
    seed: int
    cu: np.ndarray                     # int32 [n_docs + 1]
    scale: float
    outliers: str = "none"             # "none" | "channels_x20" | "tokens_1pct_x8"

    @property
    def n_docs(self) -> int:
        return len(self.cu) - 1

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.cu.astype(np.int64))

    @property
    def max_seqlen(self) -> int:
        return int(self.lengths.max()) if self.n_docs else 0

    def pairs(self) -> int:
        """Unmasked (query, key) pairs per query head: sum_k L_k (L_k + 1) / 2."""
        L = self.lengths
        return int(np.sum(L * (L + 1) // 2))

    def flops(self) -> float:
        """Algorithmic causal fwd+bwd FLOPs: 4 d pairs Hq (QK^T, PV) forward plus
        10 d pairs Hq (S recompute, dP, dV, dK, dQ) backward."""
        return 14.0 * self.d * self.Hq * self.pairs()

    def describe(self) -> Dict:
        return {"workload": self.name, "T": self.T, "Hq": self.Hq, "Hkv": self.Hkv, "d": self.d,
                "n_docs": self.n_docs, "max_seqlen": self.max_seqlen, "seed": self.seed,
                "outliers": self.outliers}

    def tensors(self, with_dout: bool = True):
        """CPU bf16 tensors (q, k, v, dout) drawn from the seed (dout None if
        not requested)."""
        g = torch.Generator().manual_seed(self.seed)
        rng = np.random.default_rng(self.seed + 1_000_003)
        shapes = [(self.T, self.Hq, self.d), (self.T, self.Hkv, self.d), (self.T, self.Hkv, self.d)]
        out = []
        for shp in shapes:
            x = torch.randn(shp, generator=g, dtype=torch.float32)
            if self.outliers == "channels_x20":
                # per head, 4 random channels scaled x20 (Q, K, V independently)
                for h in range(shp[1]):
                    ch = rng.choice(self.d, size=4, replace=False)
                    x[:, h, torch.from_numpy(ch)] *= 20.0
            elif self.outliers == "tokens_1pct_x8":
                # 1% of tokens, all heads and channels, scaled x8
                n = max(1, self.T // 100)
                tok = rng.choice(self.T, size=n, replace=False)
                x[torch.from_numpy(tok)] *= 8.0
            out.append(x.to(torch.bfloat16))
        if with_dout:
            out.append(torch.randn((self.T, self.Hq, self.d), generator=g,
                                   dtype=torch.float32).to(torch.bfloat16))
        else:
            out.append(None)
        return tuple(out)


def single_doc(seed: int = 0) -> Workload:
    """One 256-token document, Hq=Hkv=2, d=64, scale 1/8 (bf16 path only)."""
    return Workload("single-doc-256-h2-d64", 256, 2, 2, 64, seed,
                    cu_from_lengths([256]), 1.0 / math.sqrt(64))


def packed_8k(seed: int = 0) -> Workload:
    """8192 packed tokens, lengths U{128..2048}, Hq=Hkv=16, d=128."""
    rng = np.random.default_rng(seed)
    return Workload("packed-8k-uniform128-2048-h16-d128", 8192, 16, 16, 128, seed,
                    cu_from_lengths(lengths_uniform(rng, 8192, 128, 2048)), 1.0 / math.sqrt(128))


def packed_16k_outliers(seed: int = 0) -> Workload:
    """16384 packed tokens, lengths U{128..2048}, Hq=Hkv=16, d=128, 4 outlier
    channels x20 per head in Q, K, V (the MXFP8 workload)."""
    rng = np.random.default_rng(seed)
    return Workload("packed-16k-uniform128-2048-h16-d128-outlierch", 16384, 16, 16, 128, seed,
                    cu_from_lengths(lengths_uniform(rng, 16384, 128, 2048)), 1.0 / math.sqrt(128),
                    outliers="channels_x20")


def packed_32k_lognormal(seed: int = 0) -> Workload:
    """32768 packed tokens, log-normal lengths (median 2048, sigma 1, clipped to
    [64, 16384]), Hq=Hkv=32, d=128, 1% of tokens x8."""
    rng = np.random.default_rng(seed)
    return Workload("packed-32k-lognormal2048-h32-d128", 32768, 32, 32, 128, seed,
                    cu_from_lengths(lengths_lognormal(rng, 32768, 2048.0, 1.0, 64, 16384)),
                    1.0 / math.sqrt(128), outliers="tokens_1pct_x8")


def gqa_128k(seed: int = 0) -> Workload:
    """131072 tokens: one 65536-token document first, then U{512..8192}
    documents filling the rest; Hq=32 sharing Hkv=8 (G=4), d=128."""
    rng = np.random.default_rng(seed)
    return Workload("gqa-128k-doc64k-uniform512-8192-hq32-hkv8-d128", 131072, 32, 8, 128, seed,
                    cu_from_lengths(lengths_uniform(rng, 131072, 512, 8192, first=[65536])),
                    1.0 / math.sqrt(128))


CONFIGS: Dict[int, Callable[[int], Workload]] = {
    1: single_doc,
    2: packed_8k,
    3: packed_16k_outliers,
    4: packed_32k_lognormal,
    5: gqa_128k,
}


def config(n: int, seed: int = 0) -> Workload:
    return CONFIGS[n](seed)


def custom(lengths: List[int], Hq: int, Hkv: int, d: int, seed: int = 0,
           scale: Optional[float] = None, name: str = "custom") -> Workload:
    """A workload with explicit document lengths (tests: ragged tails, empty and
    one-token documents)."""
    cu = cu_from_lengths(lengths)
    return Workload(name, int(cu[-1]), Hq, Hkv, d, seed, cu,
                    scale if scale is not None else 1.0 / math.sqrt(d))
