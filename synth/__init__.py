"""Seeded synthetic inputs for the LSCD SpMM workloads.

This module only draws numbers: pruned fp16 weight matrices A (M x K,
row-major), skinny fp16 activation matrices B (stored as ``[N, K]``, i.e. the
K x N operand in column-major order) and the workload tables.  It holds none
of the method's arithmetic (no encoding, no product), so both the CPU oracle
and the GPU path can be fed from it without sharing any computation.

Workload shapes follow Flash-LLM's skinny decoder MatMuls (Flash-LLM paper
review, section 3, table of the four decoder-layer MatMuls: QKV, output
projection, MLP1, MLP2 with the token batch as N) and its kernel benchmark
set-up (section 6, "experimental setup": OPT shapes, 70/80/90 % random
unstructured sparsity, batch 8-64).  The moderate-sparsity
LLaMA layer and the stress sweep widen that set.

Recipe (every draw is reproducible from its key):

* generator: ``numpy.random.Generator(PCG64(SeedSequence(key)))`` with
  ``key = [config, layer, sparsity_pct, structure, role, N]``;
* weights: ``0.02 * standard_normal(float32)`` rounded to fp16 (RNE);
* activations: ``standard_normal(float32)`` rounded to fp16;
* masks are applied after the fp16 cast; structures:
  - ``uniform``: element zeroed iff ``u < s`` for a row-major float32 draw u;
  - ``row_magnitude``: each row drops ``(s_pct*K + 50) // 100`` entries of
    smallest fp16 magnitude, ties broken by dropping the higher column first;
  - ``power_law``: row density d_r drawn from p(d) ~ d^-alpha on [0.02, 0.60]
    with alpha set by bisection so that E[d] = 1 - s; each row keeps
    ``round(d_r*K)`` columns chosen uniformly without replacement;
  - ``column_clustered``: 25 % of the 64-wide column blocks are hot, with
    density d_h = min(0.95, 3d); the rest get d_c = (d - 0.25 d_h) / 0.75;
    Bernoulli per element.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

STRUCTURES = {"uniform": 0, "row_magnitude": 1, "power_law": 2, "column_clustered": 3}
ROLE_WEIGHT, ROLE_MASK, ROLE_B = 0, 1, 2
_ROW_CHUNK = 1024


def rng_for(*key: int) -> np.random.Generator:
    """Generator for one draw, keyed by small non-negative integers."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def weights_fp16(M: int, K: int, key) -> np.ndarray:
    """Dense N(0, 0.02) weights in fp16, row-major M x K."""
    g = rng_for(*key, ROLE_WEIGHT)
    out = np.empty((M, K), dtype=np.float16)
    for r0 in range(0, M, _ROW_CHUNK):
        r1 = min(M, r0 + _ROW_CHUNK)
        x = g.standard_normal((r1 - r0, K), dtype=np.float32)
        x *= np.float32(0.02)
        out[r0:r1] = x.astype(np.float16)
    return out


def activations_fp16(N: int, K: int, key) -> np.ndarray:
    """Activations B as an [N, K] fp16 array (K contiguous per token)."""
    g = rng_for(*key, ROLE_B, N)
    return g.standard_normal((N, K), dtype=np.float32).astype(np.float16)


def _mask_uniform(W: np.ndarray, s: float, g: np.random.Generator) -> None:
    M, K = W.shape
    for r0 in range(0, M, _ROW_CHUNK):
        r1 = min(M, r0 + _ROW_CHUNK)
        u = g.random((r1 - r0, K), dtype=np.float32)
        W[r0:r1][u < np.float32(s)] = 0


def row_magnitude_drop_count(K: int, s_pct: int) -> int:
    return (s_pct * K + 50) // 100


def _mask_row_magnitude(W: np.ndarray, s_pct: int) -> None:
    M, K = W.shape
    nz = row_magnitude_drop_count(K, s_pct)
    if nz <= 0:
        return
    if nz >= K:
        W[:] = 0
        return
    cols = np.arange(K, dtype=np.uint32)
    tiebreak = np.uint32(0xFFFF) - cols  # equal magnitude: higher column drops first
    bits = W.view(np.uint16)
    for r0 in range(0, M, _ROW_CHUNK):
        r1 = min(M, r0 + _ROW_CHUNK)
        mag = (bits[r0:r1] & np.uint16(0x7FFF)).astype(np.uint32)
        keys = (mag << np.uint32(16)) | tiebreak
        drop = np.argpartition(keys, nz - 1, axis=1)[:, :nz]
        np.put_along_axis(W[r0:r1], drop, np.float16(0), axis=1)


def _power_law_moments(alpha: float, a: float, b: float):
    """(mean, normaliser) of p(d) ~ d^-alpha on [a, b], stable near alpha = 1, 2."""
    L = math.log(b / a)

    def integral(p: float) -> float:  # int_a^b d^p dd
        x = (p + 1.0) * L
        f = math.expm1(x) / x if abs(x) > 1e-12 else 1.0
        return a ** (p + 1.0) * L * f

    z = integral(-alpha)
    return integral(1.0 - alpha) / z, z


def power_law_alpha(mean: float, a: float = 0.02, b: float = 0.60) -> float:
    """Exponent alpha with E[d] = mean for p(d) ~ d^-alpha on [a, b] (bisection)."""
    if not (a < mean < b):
        raise ValueError(f"mean density {mean} outside ({a}, {b})")
    lo, hi = -200.0, 200.0  # mean decreases as alpha grows
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        m, _ = _power_law_moments(mid, a, b)
        if m > mean:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def power_law_sample(u: np.ndarray, alpha: float, a: float = 0.02, b: float = 0.60) -> np.ndarray:
    """Inverse CDF of p(d) ~ d^-alpha on [a, b] applied to uniforms u."""
    L = math.log(b / a)
    q = 1.0 - alpha
    x = q * L
    if abs(x) < 1e-12:
        return a * np.exp(u * L)
    return a * np.exp(np.log1p(u * math.expm1(x)) / q)


def _mask_power_law(W: np.ndarray, s: float, g: np.random.Generator) -> np.ndarray:
    M, K = W.shape
    alpha = power_law_alpha(1.0 - s)
    d = power_law_sample(g.random(M), alpha)
    keep = np.rint(d * K).astype(np.int64)
    keep = np.clip(keep, 0, K)
    for r in range(M):
        row_keep = np.zeros(K, dtype=bool)
        row_keep[g.choice(K, size=int(keep[r]), replace=False)] = True
        W[r, ~row_keep] = 0
    return d


def column_cluster_densities(s: float):
    d = 1.0 - s
    d_h = min(0.95, 3.0 * d)
    d_c = (d - 0.25 * d_h) / 0.75
    return d_h, d_c


def _mask_column_clustered(W: np.ndarray, s: float, g: np.random.Generator) -> np.ndarray:
    M, K = W.shape
    nblk = (K + 63) // 64
    hot = g.choice(nblk, size=int(round(0.25 * nblk)), replace=False)
    d_h, d_c = column_cluster_densities(s)
    dens = np.full(K, d_c, dtype=np.float32)
    for blk in hot:
        dens[blk * 64:min(K, blk * 64 + 64)] = d_h
    for r0 in range(0, M, _ROW_CHUNK):
        r1 = min(M, r0 + _ROW_CHUNK)
        u = g.random((r1 - r0, K), dtype=np.float32)
        W[r0:r1][u >= dens[None, :]] = 0
    return np.sort(hot)


def sparse_weight(M: int, K: int, s_pct: int, structure: str, key) -> np.ndarray:
    """Pruned fp16 weight matrix (row-major M x K) for a workload key.

    ``key`` is ``(config, layer)``; sparsity and structure are appended so every
    (matrix, sparsity, structure) cell has its own stream.
    """
    sid = STRUCTURES[structure]
    full = (*key, s_pct, sid)
    W = weights_fp16(M, K, full)
    s = s_pct / 100.0
    g = rng_for(*full, ROLE_MASK)
    if structure == "uniform":
        _mask_uniform(W, s, g)
    elif structure == "row_magnitude":
        _mask_row_magnitude(W, s_pct)
    elif structure == "power_law":
        _mask_power_law(W, s, g)
    elif structure == "column_clustered":
        _mask_column_clustered(W, s, g)
    else:
        raise ValueError(structure)
    return W


# ---------------------------------------------------------------------------
# Workload tables
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class MatMul:
    name: str
    M: int
    K: int


@dataclass(frozen=True)
class Workload:
    cfg: int
    name: str
    matmuls: tuple
    sparsities: tuple
    structures: tuple
    Ns: tuple
    note: str = field(default="")


def _layer(h: int, ffn: int):
    return (MatMul("qkv", 3 * h, h), MatMul("out_proj", h, h),
            MatMul("mlp1", ffn, h), MatMul("mlp2", h, ffn))


WORKLOADS = {
    1: Workload(1, "single_1024", (MatMul("spmm", 1024, 1024),), (80,), ("uniform",), (8,),
                "1024 x 1024, 80 % uniform, N = 8, 64 x 64 tiles"),
    2: Workload(2, "opt66b_layer", _layer(9216, 4 * 9216), (80,), ("uniform",), (8, 16, 32, 64),
                "OPT-66B decoder layer (H = 9216), 80 % uniform"),
    3: Workload(3, "opt175b_layer", _layer(12288, 4 * 12288), (70, 80, 90), ("row_magnitude",),
                (8, 16, 32), "OPT-175B decoder layer (H = 12288), per-row magnitude pruning"),
    4: Workload(4, "llama7b_layer",
                (MatMul("qkv", 12288, 4096), MatMul("out_proj", 4096, 4096),
                 MatMul("gate", 11008, 4096), MatMul("up", 11008, 4096),
                 MatMul("down", 4096, 11008)),
                (50,), ("row_magnitude",), (8, 16, 32, 64, 128),
                "LLaMA-7B layer (hidden 4096, FFN 11008), 50 % per-row magnitude"),
    5: Workload(5, "stress_12288", (MatMul("square", 12288, 12288),), (50, 60, 70, 80, 90, 95),
                ("uniform", "power_law", "column_clustered"), (8, 16, 32, 64, 128),
                "12288^2 sweep of sparsity x N x mask structure"),
}


def layer_key(cfg: int, layer_index: int):
    return (cfg, layer_index)
