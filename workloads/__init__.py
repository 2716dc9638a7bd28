"""Seeded synthetic inputs for the LLM.int8() mixed-precision matmul.

This module is shared by the CPU oracle's tests, the GPU parity tests and the
benchmark.  It only draws random numbers and builds fp16 arrays; it holds none
of the method's arithmetic (no outlier detection, no quantization, no matmul).

Recipe (the pages measure on trained OPT/BLOOM models and text datasets, which
are not available; these synthetic inputs stand in for them with the statistics
the pages give):

* activations X [M, K]: i.i.d. N(0, 1) drawn in fp32 by numpy's PCG64
  ``default_rng(seed)``, then a fixed set of feature columns is multiplied by 20
  (outliers "up to 20x larger", Compress your LLMs; ~0.1 % of the feature
  dimensions, 6 of 4096 at the 6.7B scale, 8-bit Matrix Multiplication for Large
  Language Models, Summary & Methodology Analysis), then rounded to fp16 (RNE).
  The planted column set is drawn first from the same generator, without
  replacement, and sorted; Tiny uses the fixed columns {3, 200}.
* weights W [K, N]: i.i.d. N(0, sigma^2) drawn in fp32 from ``default_rng(seed +
  100)``, rounded to fp16.  Large W is drawn in row chunks; a numpy Generator
  produces the same stream whether a draw is split or not (checked by a test).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = ["Workload", "WORKLOADS", "get", "make_x", "make_w", "make_inputs", "planted_columns"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic problem Y[M,N] = X[M,K] . W[K,N] with threshold ``tau``."""

    name: str
    M: int
    K: int
    N: int
    seed: int
    n_planted: int = 0
    planted: Optional[Tuple[int, ...]] = None  # explicit columns (overrides n_planted)
    w_sigma: float = 0.02
    tau: float = 6.0
    note: str = ""

    @property
    def ops(self) -> int:
        """2*M*N*K: the effective-operation count the throughput metric uses."""
        return 2 * self.M * self.N * self.K

    def with_tau(self, tau: float, suffix: str) -> "Workload":
        return dataclasses.replace(self, tau=tau, name=self.name + suffix)


def _n_frac(K: int, frac: float) -> int:
    return max(1, int(round(frac * K))) if frac > 0 else 0


def _build_registry():
    w = {}

    def add(wl: Workload):
        w[wl.name] = wl

    add(Workload("tiny", 16, 256, 256, seed=0, planted=(3, 200), w_sigma=0.02,
                 note="X [16,256] with 2 fixed columns x20; W [256,256] N(0,0.02^2)"))
    add(Workload("ffn_6p7b_prefill", 2048, 4096, 16384, seed=2, n_planted=6, w_sigma=0.02,
                 note="6.7B-style FFN up-projection prefill, 6 of 4096 columns x20"))
    for m in (1, 8, 32):
        add(Workload(f"decode_m{m}", m, 4096, 4096, seed=3, n_planted=6, w_sigma=0.02,
                     note=f"decode-shaped X [{m},4096], W [4096,4096], 6 planted columns"))
    add(Workload("hidden_175b", 4096, 12288, 49152, seed=4, n_planted=25, w_sigma=0.015,
                 note="175B-style hidden projection, 25 of 12288 columns x20"))
    for n, tag in ((0, "0"), (8, "0p1"), (82, "1")):
        add(Workload(f"sweep8k_o{tag}", 8192, 8192, 8192, seed=5, n_planted=n, w_sigma=0.02,
                     note=f"[8192,8192]^2 with {n} planted columns"))
    for (m, n, k) in ((1000, 1000, 1000), (2047, 4095, 4100), (129, 257, 520), (1, 1001, 1000), (3, 33, 24)):
        add(Workload(f"ragged_{m}x{n}x{k}", m, k, n, seed=6, n_planted=_n_frac(k, 0.0015), w_sigma=0.02,
                     note="ragged shape, ~0.15% of columns x20"))
    return w


WORKLOADS = _build_registry()


def get(name: str) -> Workload:
    return WORKLOADS[name]


def planted_columns(wl: Workload) -> np.ndarray:
    """The sorted feature columns of X that are scaled by 20."""
    if wl.planted is not None:
        return np.asarray(sorted(wl.planted), dtype=np.int64)
    if wl.n_planted == 0:
        return np.zeros(0, dtype=np.int64)
    rng = np.random.default_rng(wl.seed)
    return np.sort(rng.choice(wl.K, size=wl.n_planted, replace=False)).astype(np.int64)


def make_x(wl: Workload, M: Optional[int] = None) -> np.ndarray:
    """fp16 activations [M, K] (M defaults to the workload's)."""
    M = wl.M if M is None else M
    rng = np.random.default_rng(wl.seed)
    if wl.planted is None and wl.n_planted > 0:
        rng.choice(wl.K, size=wl.n_planted, replace=False)  # same draw as planted_columns()
    x = rng.standard_normal((M, wl.K), dtype=np.float32)
    cols = planted_columns(wl)
    if cols.size:
        x[:, cols] *= np.float32(20.0)
    return x.astype(np.float16)


def make_w(wl: Workload, chunk_rows: int = 1024) -> np.ndarray:
    """fp16 weights [K, N] ~ N(0, w_sigma^2), drawn in row chunks."""
    rng = np.random.default_rng(wl.seed + 100)
    out = np.empty((wl.K, wl.N), dtype=np.float16)
    sigma = np.float32(wl.w_sigma)
    for r0 in range(0, wl.K, chunk_rows):
        r1 = min(wl.K, r0 + chunk_rows)
        blk = rng.standard_normal((r1 - r0, wl.N), dtype=np.float32)
        blk *= sigma
        out[r0:r1] = blk.astype(np.float16)
    return out


def make_inputs(wl: Workload) -> Tuple[np.ndarray, np.ndarray]:
    return make_x(wl), make_w(wl)


def random_small(rng: np.random.Generator, M: int, K: int, N: int, n_planted: int,
                 w_sigma: float = 0.02) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Small random problem for brute-force comparisons: (X16, W16, planted cols)."""
    cols = np.sort(rng.choice(K, size=min(n_planted, K), replace=False)) if n_planted else np.zeros(0, np.int64)
    x = rng.standard_normal((M, K), dtype=np.float32)
    if cols.size:
        x[:, cols] *= np.float32(20.0)
    w = rng.standard_normal((K, N), dtype=np.float32) * np.float32(w_sigma)
    return x.astype(np.float16), w.astype(np.float16), cols


def sample_rows(M: int, n: int = 64, seed: int = 12345) -> np.ndarray:
    """Rows checked at full size: n seeded random rows plus the first and last."""
    rng = np.random.default_rng(seed)
    pick = rng.choice(M, size=min(n, M), replace=False)
    return np.unique(np.concatenate([pick, [0, M - 1]])).astype(np.int64)
