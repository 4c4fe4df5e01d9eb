"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds no entmax arithmetic.  It draws Q, K, V, dO on the host with
numpy's counter-based Philox generator and rounds them to the storage dtype, so
the CUDA path and the float64 oracle see the same quantised values (every bf16
value is exact in float32 and float64).

Workloads (shapes and value distributions as the AdaSplash pages' synthetic
stand-ins; the pages measure only on trained models and public datasets):

* ``tiny``  -- B1 H2 N256 d64 fp32, non-causal, alpha 1.5, iid N(0,1).
* ``iid``   -- B4 H16 N4096 d128 bf16, causal, alpha 1.5, iid N(0,1); the
  temperature beta (1, 2, 4, 8) multiplies Q, which scales s = QK^T/sqrt(d) by
  beta exactly because beta is a power of two.
* ``alpha`` -- B2 H16 N8192 d64 bf16, causal, beta 4, alpha in {1.25, 1.5, 2}.
* ``long``  -- B1 H16 N32768 d128 bf16, causal, alpha 1.5, beta 4, clustered:
  64 centres c ~ N(0, I); key j = c[(j // 512) % 64] + 0.1 N(0, I) (each
  cluster a contiguous span of 512 keys); each 128-row query tile draws 1-4
  distinct centres and every row of the tile is their mean + 0.1 N(0, I).
* ``lm``    -- B8 H12 N2048 d64 bf16, causal, alpha 1.5; Q, K, V are heads of
  X W with X ~ N(0,1) [B, N, 768] and W Xavier-uniform [768, 2304].
* ``clustered4k`` (supplementary) -- the ``long`` generator at the iid shape
  (B4 H16 N4096 d128, beta 4); the cluster span (keys per centre, default 512)
  sets the block sparsity, for a sweep between the dense iid case and ~95 %.
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str          # "f32" or "bf16"
    causal: bool
    alpha: float
    beta: float
    kind: str           # "iid", "clustered", "lm"
    span: int = 512     # clustered: contiguous keys per cluster

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def shape(self):
        return (self.B, self.H, self.N, self.d)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 256, 64, "f32", False, 1.5, 1.0, "iid"),
    "iid": Workload("iid", 4, 16, 4096, 128, "bf16", True, 1.5, 1.0, "iid"),
    "alpha": Workload("alpha", 2, 16, 8192, 64, "bf16", True, 1.5, 4.0, "iid"),
    "long": Workload("long", 1, 16, 32768, 128, "bf16", True, 1.5, 4.0, "clustered"),
    "lm": Workload("lm", 8, 12, 2048, 64, "bf16", True, 1.5, 1.0, "lm"),
    # supplementary (not one of the five configurations): the long workload's clustered
    # generator at the iid shape, for a block-sparsity sweep over the cluster span
    "clustered4k": Workload("clustered4k", 4, 16, 4096, 128, "bf16", True, 1.5, 4.0, "clustered"),
}


def rng(seed: int) -> np.random.Generator:
    """Counter-based generator (Philox 4x64) keyed by ``seed``."""
    return np.random.Generator(np.random.Philox(key=seed))


def row_scores(rows: int, n: int, seed: int = 0, scale: float = 1.0) -> np.ndarray:
    """[rows, n] float32 scores ~ N(0, scale^2) (Philox stream (seed, 7)) for the
    row-wise entmax op: the distribution of s = q.k/sqrt(d) on the iid workload."""
    return (scale * _normal(rng(seed * 16 + 7), (rows, n))).astype(np.float32)


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """float32 array whose values are ``a`` rounded to bfloat16 (nearest, ties even)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(a)
    out = (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32).copy()
    out[nan] = np.nan
    return out


def _quantise(a: np.ndarray, dtype: str) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    return round_to_bf16(a) if dtype == "bf16" else a


def _normal(g: np.random.Generator, shape) -> np.ndarray:
    return g.standard_normal(size=shape, dtype=np.float32)


def make_inputs(w: Workload, seed: int = 0):
    """(q, k, v, do) as float32 [B,H,N,d] arrays holding values of ``w.dtype``.

    ``q`` already carries the temperature beta.  Each tensor has its own
    Philox stream (seed, tensor index), so one tensor can be regenerated alone.
    """
    B, H, N, d = w.shape
    if w.kind == "iid":
        q = _normal(rng(seed * 16 + 0), (B, H, N, d))
        k = _normal(rng(seed * 16 + 1), (B, H, N, d))
        v = _normal(rng(seed * 16 + 2), (B, H, N, d))
    elif w.kind == "clustered":
        g = rng(seed * 16 + 0)
        centres = _normal(g, (B, H, 64, d))
        span = np.arange(N) // w.span % 64
        k = centres[:, :, span, :] + 0.1 * _normal(rng(seed * 16 + 1), (B, H, N, d))
        T = -(-N // 128)
        q = np.empty((B, H, T * 128, d), np.float32)
        gq = rng(seed * 16 + 3)
        for b in range(B):
            for h in range(H):
                for t in range(T):
                    n = int(gq.integers(1, 5))
                    pick = gq.choice(64, size=n, replace=False)
                    q[b, h, t * 128:(t + 1) * 128] = centres[b, h, pick].mean(axis=0)
        q = q[:, :, :N] + 0.1 * _normal(rng(seed * 16 + 4), (B, H, N, d))
        v = _normal(rng(seed * 16 + 2), (B, H, N, d))
    elif w.kind == "lm":
        hidden, nh = 768, w.H
        assert nh * d == hidden
        x = _normal(rng(seed * 16 + 0), (B, N, hidden))
        lim = np.float32(np.sqrt(6.0 / (hidden + 3 * hidden)))
        wqkv = rng(seed * 16 + 1).uniform(-lim, lim, size=(hidden, 3 * hidden)).astype(np.float32)
        qkv = (x.reshape(B * N, hidden) @ wqkv).reshape(B, N, 3, nh, d)
        q, k, v = (np.ascontiguousarray(qkv[:, :, i].transpose(0, 2, 1, 3)) for i in range(3))
    else:
        raise ValueError(f"unknown workload kind {w.kind!r}")
    do = _normal(rng(seed * 16 + 5), (B, H, N, d))
    q = _quantise(q, w.dtype)
    if w.beta != 1.0:
        q = _quantise(q * np.float32(w.beta), w.dtype)
    return q, _quantise(k, w.dtype), _quantise(v, w.dtype), _quantise(do, w.dtype)


def small_case(B=1, H=2, N=384, d=64, dtype="bf16", causal=True, alpha=1.5, beta=1.0,
               kind="iid", seed=0):
    """A custom-size workload and its inputs (for tests that need odd shapes)."""
    w = Workload(f"custom-{kind}", B, H, N, d, dtype, causal, alpha, beta, kind)
    return w, make_inputs(w, seed)
