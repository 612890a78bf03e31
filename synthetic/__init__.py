"""Seeded synthetic inputs for the Avey-B ranker + neural-processor path.

This module is shared by the fp64 oracle (``oracle/``) and the CUDA library
(``attention_free_long_b200``).  It only draws random numbers and shapes them;
it contains none of the method's arithmetic (no normalisation, similarity,
selection, compression or layer math).

Workloads (shapes from the Avey-B summary pages; the pages' downstream
benchmarks are not available, so seeded Gaussian mixtures stand in for them):

========== ==== ====== ===== ====== ====== ========== ==== =========== =====
name        B    N      S     n      d      m (h/t)    k    layers      dtype
========== ==== ====== ===== ====== ====== ========== ==== =========== =====
tiny_f32    1    256    16    16     64     128 64/64  3    D           f32
base_bf16   8    4096   64    64     768    1536       7    S,D         bf16
mid_bf16    2    16384  64    256    768    1536       7    S,D,S,D     bf16
long_bf16   1    98304  64    1536   768    1536       7    S,D,S,D     bf16
large_bf16  4    32768  128   256    1024   2048       15   (S,D)x6     bf16
========== ==== ====== ===== ====== ====== ========== ==== =========== =====

Draw recipe (numpy ``Generator(PCG64(seed))``; embeddings seed 0, weights
seed 1; the order of draws below is fixed):

1. ``K`` mixture centres, each ``N(0, I_d)`` (float64 draws).
2. Per sequence: one centre index per split, uniform over ``0..K-1``.
3. Per sequence: token noise ``sigma * N(0, I_d)`` (float32 draws); token
   ``x = centre[split] + noise``.
4. mid_bf16 only: per sequence, ``ceil(0.05 n)`` destination splits without
   replacement, then as many distinct source splits from the remaining ones;
   each destination split becomes an exact copy of its source.
5. Weights ``N(0, 1/fan_in)``: P (fan_in ``(k+1)S``) first, then per layer U
   and its bias (fan_in d), V for static layers (fan_in S), O (fan_in m).
6. bf16 workloads round every value to the nearest bf16 (ties to even); both
   sides then read identical values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np

STATIC = 0
DYNAMIC = 1
COUPLED = 2  # original Avey: V * cosine, causal mask (not in the named workloads)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    S: int
    d: int
    m: int
    m_h: int
    k: int
    pattern: tuple  # layer kinds, STATIC / DYNAMIC
    dtype: str  # "f32" or "bf16"
    centers: int
    sigma: float
    dup_frac: float = 0.0
    eps: float = 1e-8
    prenorm: bool = False

    @property
    def n(self) -> int:
        return -(-self.N // self.S)

    @property
    def m_t(self) -> int:
        return self.m - self.m_h

    @property
    def T(self) -> int:
        """Padded token count B * n * S."""
        return self.B * self.n * self.S

    @property
    def layers(self) -> int:
        return len(self.pattern)


def _alt(L: int) -> tuple:
    return tuple(STATIC if i % 2 == 0 else DYNAMIC for i in range(L))


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 256, 16, 64, 128, 64, 3, (DYNAMIC,), "f32", 4, 0.3),
    "base_bf16": Workload("base_bf16", 8, 4096, 64, 768, 1536, 768, 7, _alt(2), "bf16", 32, 0.5),
    "mid_bf16": Workload("mid_bf16", 2, 16384, 64, 768, 1536, 768, 7, _alt(4), "bf16", 32, 0.5,
                         dup_frac=0.05),
    "long_bf16": Workload("long_bf16", 1, 98304, 64, 768, 1536, 768, 7, _alt(4), "bf16", 64, 0.5),
    "large_bf16": Workload("large_bf16", 4, 32768, 128, 1024, 2048, 1024, 15, _alt(12), "bf16", 64,
                           0.5, prenorm=True),
}


def custom(name="custom", B=1, N=256, S=16, d=64, m=128, m_h=None, k=3, pattern=(DYNAMIC,),
           dtype="bf16", centers=4, sigma=0.3, dup_frac=0.0, eps=1e-8, prenorm=False) -> Workload:
    """A workload with arbitrary shapes (parity sweeps, edge cases)."""
    return Workload(name, B, N, S, d, m, m // 2 if m_h is None else m_h, k, tuple(pattern), dtype,
                    centers, sigma, dup_frac, eps, prenorm)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), kept as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


@dataclasses.dataclass
class Embeddings:
    X: np.ndarray  # [B, N, d] float32 (bf16-representable for bf16 workloads)
    split_center: np.ndarray  # [B, n] int64
    dup_pairs: List[List[tuple]]  # per sequence: (dst, src) split pairs


def gen_embeddings(w: Workload, seed: int = 0) -> Embeddings:
    rng = np.random.Generator(np.random.PCG64(seed))
    centers = rng.standard_normal((w.centers, w.d))  # float64
    X = np.empty((w.B, w.N, w.d), dtype=np.float32)
    split_center = np.empty((w.B, w.n), dtype=np.int64)
    dup_pairs: List[List[tuple]] = []
    for b in range(w.B):
        split_center[b] = rng.integers(0, w.centers, size=w.n)
        noise = rng.standard_normal((w.N, w.d), dtype=np.float32)
        tok_center = np.repeat(split_center[b], w.S)[: w.N]
        X[b] = (centers[tok_center] + w.sigma * noise).astype(np.float32)
        pairs = []
        if w.dup_frac > 0:
            n_dup = math.ceil(w.dup_frac * w.n)
            dst = rng.choice(w.n, size=n_dup, replace=False)
            rest = np.setdiff1d(np.arange(w.n), dst)
            src = rng.choice(rest, size=n_dup, replace=False)
            for t, s in zip(dst.tolist(), src.tolist()):
                lo_s, hi_s = s * w.S, min((s + 1) * w.S, w.N)
                lo_t, hi_t = t * w.S, min((t + 1) * w.S, w.N)
                if hi_s - lo_s == hi_t - lo_t:  # full splits only
                    X[b, lo_t:hi_t] = X[b, lo_s:hi_s]
                    pairs.append((t, s))
        dup_pairs.append(pairs)
    if w.dtype == "bf16":
        X = round_bf16(X)
    return Embeddings(X, split_center, dup_pairs)


@dataclasses.dataclass
class LayerWeights:
    kind: int  # STATIC, DYNAMIC or COUPLED
    U: np.ndarray  # [d, m]   enricher weight (Z = X U + b)
    bU: np.ndarray  # [m]
    V: Optional[np.ndarray]  # [S, S] for static and coupled layers, None for dynamic
    O: np.ndarray  # [m, d]   fuser weight


@dataclasses.dataclass
class Weights:
    P: np.ndarray  # [S, (k+1) S] compressor
    layers: List[LayerWeights]


def gen_weights(w: Workload, seed: int = 1, block: int = 0) -> Weights:
    """Seeded weights in a fixed draw order (P, then per layer U, bU, V, O).

    ``block`` is the contextualizer's token block (V is block x block); the
    default is the split size S.  The uncompressed processor mixes blocks of
    (k+1)S tokens and takes block=(k+1)S: its V are drawn from a second stream
    (seed, 1000 + layer), while the main stream makes the same draws as for
    block=S, so P, U, bU and O are identical.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    blk = block if block else w.S

    def draw(shape, fan_in):
        a = (rng.standard_normal(shape, dtype=np.float32) * np.float32(1.0 / math.sqrt(fan_in)))
        return round_bf16(a) if w.dtype == "bf16" else a.astype(np.float32)

    P = draw((w.S, (w.k + 1) * w.S), (w.k + 1) * w.S)
    layers = []
    for li, kind in enumerate(w.pattern):
        U = draw((w.d, w.m), w.d)
        bU = draw((w.m,), w.d)
        V = draw((w.S, w.S), w.S) if kind in (STATIC, COUPLED) else None
        if V is not None and blk != w.S:
            r2 = np.random.Generator(np.random.PCG64([seed, 1000 + li]))
            a = r2.standard_normal((blk, blk), dtype=np.float32) * np.float32(1.0 / math.sqrt(blk))
            V = round_bf16(a) if w.dtype == "bf16" else a.astype(np.float32)
        O = draw((w.m, w.d), w.m)
        layers.append(LayerWeights(kind, U, bU, V, O))
    return Weights(P, layers)


def sample_targets(w: Workload, per_seq: int, seed: int = 2, must=None) -> np.ndarray:
    """Seeded (batch, target split) pairs for split-sampled checks.

    ``must`` optionally lists (b, t) pairs that are always included (e.g. the
    planted duplicate splits).  Returns an int32 array [n_sel, 2] sorted by
    (b, t) without repeats.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    sel = set()
    for b in range(w.B):
        cnt = min(per_seq, w.n)
        for t in rng.choice(w.n, size=cnt, replace=False).tolist():
            sel.add((b, t))
    if must:
        sel.update((int(b), int(t)) for b, t in must)
    return np.array(sorted(sel), dtype=np.int32).reshape(-1, 2)
