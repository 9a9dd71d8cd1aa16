"""Seeded synthetic inputs for the MACAQ linear (shared by tests, smoke and bench).

This module draws random numbers and lays out input tensors.  It holds none of
the method's arithmetic: no scaling, no rotation, no quantisation.  The
channel factor D is produced here because the pages treat calibration as an
offline step outside the kernel; the recipe below replaces calibration with a
closed form computed from the generated tensors.

Recipe (numpy ``default_rng``; one ``SeedSequence(seed).spawn`` stream per
tensor):

* x: fp32 N(0, 1) of shape [M, K]; ``max(1, round(0.01 K))`` outlier channels
  chosen by a seeded permutation are multiplied by 20; then rounded to bf16
  (round-to-nearest-even) and kept as uint16 bit patterns.
* W: fp32 N(0, 0.02) (0.02 = standard deviation) of shape [E, N, K].
* D[k] = clamp(sqrt(max_m |x[m,k]| / max_n |W[n,k]|), 1e-2, 1e2), in binary64,
  then rounded to fp32; 0/0 or NaN gives 1.  Grouped: per expert over that
  expert's rows; an expert with no rows gets D = 1.
* group counts: E=4 uses multinomial(T, uniform); E=128 uses p_e proportional
  to rank_e^-1.1 with ranks a seeded permutation, and p = 0 for a seeded 1/16
  of the experts so that some groups are empty.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round-to-nearest-even via torch."""
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _streams(seed: int, n: int):
    return [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(n)]


def make_x(M: int, K: int, rng: np.random.Generator, outlier_frac: float = 0.01,
           outlier_mult: float = 20.0) -> np.ndarray:
    x = rng.standard_normal((M, K), dtype=np.float32)
    n_out = max(1, int(round(outlier_frac * K)))
    idx = rng.permutation(K)[:n_out]
    x[:, idx] *= outlier_mult
    return to_bf16_bits(x)


def make_w(E: int, N: int, K: int, rng: np.random.Generator, std: float = 0.02) -> np.ndarray:
    return rng.normal(0.0, std, size=(E, N, K)).astype(np.float32)


def make_d(x_bits: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Closed-form channel factor for one expert: x bits [m, K], W [N, K]."""
    K = W.shape[1]
    if x_bits.shape[0] == 0:
        return np.ones(K, np.float32)
    xa = np.abs(bf16_bits_to_f32(x_bits).astype(np.float64)).max(axis=0)
    wa = np.abs(W.astype(np.float64)).max(axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        d = np.sqrt(xa / wa)
    d = np.where(np.isfinite(d), d, np.where(xa > 0, 1e2, 1.0))
    d = np.where((xa == 0) & (wa == 0), 1.0, d)
    return np.clip(d, 1e-2, 1e2).astype(np.float32)


@dataclass
class Problem:
    """One linear problem.  Dense problems have E == 1 and group_list None."""
    x: np.ndarray            # uint16 bf16 bits [M, K]
    W: np.ndarray            # fp32 [E, N, K]
    D: np.ndarray            # fp32 [E, K]
    M: int
    N: int
    K: int
    E: int = 1
    group_list: np.ndarray | None = None   # int64 [E]
    group_list_type: int = 0               # 0 cumulative sum, 1 counts
    name: str = ""

    @property
    def counts(self) -> np.ndarray:
        if self.group_list is None:
            return np.array([self.M], np.int64)
        if self.group_list_type == 1:
            return self.group_list.copy()
        return np.diff(np.concatenate([[0], self.group_list])).astype(np.int64)

    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K

    def algorithmic_bytes(self) -> float:
        """x read once, codes + E8M0 scales of non-empty experts, D, y written once."""
        live = int((self.counts > 0).sum())
        w = live * (self.N * self.K // 2 + self.N * self.K // 32)
        return float(self.M * self.K * 2 + w + live * self.K * 4 + self.M * self.N * 2)


def dense(M: int, K: int, N: int, seed: int = 0, name: str = "") -> Problem:
    sx, sw = _streams(seed, 2)
    x = make_x(M, K, sx)
    W = make_w(1, N, K, sw)
    D = make_d(x, W[0])[None, :]
    return Problem(x=x, W=W, D=D, M=M, N=N, K=K, name=name or f"dense M={M} K={K} N={N}")


def zipf_counts(T: int, E: int, rng: np.random.Generator, s: float = 1.1,
                empty_frac: float = 1 / 16) -> np.ndarray:
    ranks = rng.permutation(E) + 1
    p = ranks.astype(np.float64) ** (-s)
    n_empty = int(round(empty_frac * E))
    if n_empty:
        p[rng.permutation(E)[:n_empty]] = 0.0
    p /= p.sum()
    return rng.multinomial(T, p).astype(np.int64)


def grouped(T: int, E: int, K: int, N: int, seed: int = 0, dist: str = "uniform",
            group_list_type: int = 1, name: str = "") -> Problem:
    sc, sx, sw = _streams(seed, 3)
    if dist == "uniform":
        counts = sc.multinomial(T, [1.0 / E] * E).astype(np.int64)
    elif dist == "zipf":
        counts = zipf_counts(T, E, sc)
    else:
        raise ValueError(dist)
    x = make_x(T, K, sx)
    W = make_w(E, N, K, sw)
    off = np.concatenate([[0], np.cumsum(counts)])
    D = np.stack([make_d(x[off[e]:off[e + 1]], W[e]) for e in range(E)])
    gl = counts.copy() if group_list_type == 1 else np.cumsum(counts).astype(np.int64)
    return Problem(x=x, W=W, D=D, M=T, N=N, K=K, E=E, group_list=gl,
                   group_list_type=group_list_type,
                   name=name or f"grouped E={E} T={T} K={K} N={N}")


# The five workloads: (K, N) pairs are Qwen3-0.6B-shaped projections.
QWEN_PAIRS = [(1024, 2048), (1024, 1024), (2048, 1024), (1024, 3072), (3072, 1024)]


def config(idx: int, seed: int = 0) -> list[Problem]:
    """Problems of workload idx: 0 dense M=16 K=N=1024; 1 dense M=128 x five
    (K,N); 2 dense M=4096 x five (K,N); 3 grouped E=4 over 4096 tokens
    (counts); 4 grouped E=128 over 8192 tokens, Zipf(1.1) (cumsum)."""
    if idx == 0:
        return [dense(16, 1024, 1024, seed, "c0 dense M=16 K=1024 N=1024")]
    if idx == 1:
        return [dense(128, k, n, seed, f"c1 dense M=128 K={k} N={n}") for k, n in QWEN_PAIRS]
    if idx == 2:
        return [dense(4096, k, n, seed, f"c2 dense M=4096 K={k} N={n}") for k, n in QWEN_PAIRS]
    if idx == 3:
        return [grouped(4096, 4, k, n, seed, "uniform", 1, f"c3 grouped E=4 K={k} N={n}")
                for k, n in [(1024, 3072), (3072, 1024)]]
    if idx == 4:
        return [grouped(8192, 128, k, n, seed, "zipf", 0, f"c4 grouped E=128 K={k} N={n}")
                for k, n in [(2048, 768), (768, 2048)]]
    raise ValueError(idx)
