"""Seeded synthetic inputs for the block-sparse linear layer.

This module only draws inputs: activations X, dense weights W (with values
everywhere; the block mask decides which survive), block masks and upstream
gradients dY.  It contains none of the layer's arithmetic, so both the CPU
oracle (``oracle/``) and the CUDA path (``sparse_gemm_b200``) may use it.

Seed scheme: ``numpy.random.default_rng(seed * 10 + s)`` with sub-stream
``s`` = 0 for X, 1 for the mask, 2 for W, 3 for dY.  Every draw is fp32 and is
rounded to bf16 by round-to-nearest-even (torch's fp32->bf16 conversion).

Workload shapes follow the layer sizes of the pages' subject, the Hugging
Face "pytorch_block_sparse" BlockSparseLinear (a drop-in for nn.Linear with a
``density`` knob): a BERT-base FFN input projection (768 -> 3072), and two
LLM MLP projections (4096 -> 14336, 4096 -> 11008).  No datasets and no
trained weights are involved; the values are random.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

__all__ = [
    "Workload", "WORKLOADS", "bf16_bits", "bits_to_f32", "mask_uniform",
    "zipf_row_counts", "mask_zipf_rows", "make_inputs", "round_half_even",
    "semi24_weight", "Semi24Workload", "SEMI24_WORKLOADS", "make_semi24_inputs",
    "BSR24_WORKLOADS", "make_bsr24_inputs",
]


def round_half_even(x: float) -> int:
    """Nearest integer, ties to even (Python's built-in ``round``)."""
    return int(round(x))


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round-to-nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_f32(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the exactly equal fp32 values."""
    return (h.astype(np.uint32) << 16).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    draw = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        draw = draw * np.float32(std)
    return bf16_bits(draw)


def mask_uniform(R: int, C: int, nnz: int, rng: np.random.Generator) -> np.ndarray:
    """Exactly ``nnz`` of the R*C blocks, uniformly without replacement.

    The chosen blocks are the first ``nnz`` entries of one seeded permutation
    of the block ids, so masks drawn from the same seed at decreasing
    densities are nested.
    """
    if not 0 <= nnz <= R * C:
        raise ValueError("nnz out of range")
    perm = rng.permutation(R * C)
    m = np.zeros(R * C, dtype=np.uint8)
    m[perm[:nnz]] = 1
    return m.reshape(R, C)


def zipf_row_counts(R: int, C: int, total: int, s: float,
                    rng: np.random.Generator) -> np.ndarray:
    """Per-block-row block counts skewed by a Zipf(s) law over the rows.

    Each row gets a rank 1..R from a seeded permutation and a weight
    rank**-s; the targets total*w/sum(w) are capped at C by water-filling
    (rows over the cap are clamped and their excess is spread over the
    uncapped rows in proportion to their targets, repeated until none is
    over), then made integral by flooring and handing the remaining units to
    the largest fractional parts (ties: lower row id).  The counts sum to
    ``total`` exactly.
    """
    if not 0 <= total <= R * C:
        raise ValueError("total out of range")
    rank = rng.permutation(R).astype(np.float64) + 1.0
    w = rank ** (-s)
    t = total * w / w.sum()
    capped = np.zeros(R, dtype=bool)
    while True:
        over = (t > C) & ~capped
        if not over.any():
            break
        excess = float((t[over] - C).sum())
        t[over] = C
        capped |= over
        free = ~capped
        t[free] += excess * t[free] / t[free].sum()
    base = np.floor(t).astype(np.int64)
    rem = total - int(base.sum())
    frac = t - base
    order = sorted(range(R), key=lambda r: (-frac[r], r))
    for r in order[:rem]:
        base[r] += 1
    return base


def mask_zipf_rows(R: int, C: int, total: int, s: float,
                   rng: np.random.Generator) -> np.ndarray:
    """Block mask whose row counts follow :func:`zipf_row_counts`; the
    columns inside each row are uniform without replacement."""
    counts = zipf_row_counts(R, C, total, s, rng)
    m = np.zeros((R, C), dtype=np.uint8)
    for r in range(R):
        cols = rng.choice(C, size=int(counts[r]), replace=False)
        m[r, cols] = 1
    return m


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    N: int
    K: int
    b: int
    density: float          # requested density (the packed one is nnz/(R*C))
    seed: int
    mask_kind: str = "uniform"   # "uniform" | "zipf"
    zipf_s: float = 1.1
    with_dy: bool = False
    description: str = ""

    @property
    def R(self) -> int:
        return self.N // self.b

    @property
    def C(self) -> int:
        return self.K // self.b

    @property
    def nnz(self) -> int:
        return round_half_even(self.density * self.R * self.C)

    def flops(self) -> int:
        """Algorithmic flops of one contraction: 2*M*N*K*(nnz/(R*C))."""
        return 2 * self.M * self.b * self.b * self.nnz


WORKLOADS: dict[str, Workload] = {w.name: w for w in [
    Workload("tiny_fwd", 64, 256, 256, 32, 0.25, 1,
             description="X[64,256], W[256,256], 32x32 blocks, 16 of 64 kept"),
    Workload("enc_fwd", 4096, 3072, 768, 32, 0.25, 2,
             description="BERT-base FFN-in forward, 75% block-sparse"),
    Workload("enc_train_d1.0", 4096, 3072, 768, 32, 1.0, 3, with_dy=True,
             description="encoder training step (fwd, dX, dW), density 1.0"),
    Workload("enc_train_d0.5", 4096, 3072, 768, 32, 0.5, 3, with_dy=True,
             description="encoder training step, density 0.5"),
    Workload("enc_train_d0.25", 4096, 3072, 768, 32, 0.25, 3, with_dy=True,
             description="encoder training step, density 0.25"),
    Workload("enc_train_d0.1", 4096, 3072, 768, 32, 0.1, 3, with_dy=True,
             description="encoder training step, density 0.1"),
    Workload("large_fwd", 8192, 14336, 4096, 64, 0.1, 4, mask_kind="zipf",
             description="LLM-MLP forward, 90% block-sparse, Zipf(1.1) rows"),
    Workload("decode_fwd", 16, 11008, 4096, 32, 0.25, 5,
             description="decode forward, 16 tokens, 75% block-sparse"),
]}


def make_mask(w: Workload) -> np.ndarray:
    rng = np.random.default_rng(w.seed * 10 + 1)
    if w.mask_kind == "uniform":
        return mask_uniform(w.R, w.C, w.nnz, rng)
    if w.mask_kind == "zipf":
        return mask_zipf_rows(w.R, w.C, w.nnz, w.zipf_s, rng)
    raise ValueError(w.mask_kind)


def make_inputs(w: Workload, *, M: int | None = None, with_dy: bool | None = None):
    """Seeded inputs of a workload as bf16 bit arrays (uint16) + uint8 mask.

    Returns a dict with X [M,K], W [N,K] (dense, values everywhere), mask
    [R,C] and, for training workloads, dY [M,N].  ``M`` may override the
    token count (rows are drawn from the same stream, so a smaller M gives a
    prefix of the full X only when the draw order allows it; callers should
    not rely on that).
    """
    M = w.M if M is None else M
    out = {}
    out["X"] = _normal_bf16(np.random.default_rng(w.seed * 10 + 0), (M, w.K), 1.0)
    out["mask"] = make_mask(w)
    out["W"] = _normal_bf16(np.random.default_rng(w.seed * 10 + 2), (w.N, w.K),
                            1.0 / math.sqrt(w.K))
    if w.with_dy if with_dy is None else with_dy:
        out["dY"] = _normal_bf16(np.random.default_rng(w.seed * 10 + 3), (M, w.N), 1.0)
    return out


def random_case(M: int, N: int, K: int, b: int, nnz: int, seed: int, *,
                integer_values: bool = False, empty_rows=(), empty_cols=()):
    """Small seeded case for parity and edge-case tests.

    With ``integer_values`` the entries are drawn from {-3..3}, exactly
    representable in bf16 and fp64, so sums are exact integers.
    ``empty_rows`` / ``empty_cols`` list block rows / columns whose mask is
    cleared after drawing.
    """
    R, C = N // b, K // b
    rng = np.random.default_rng(seed)
    mask = mask_uniform(R, C, nnz, rng)
    for r in empty_rows:
        mask[r, :] = 0
    for c in empty_cols:
        mask[:, c] = 0

    def draw(shape, std):
        if integer_values:
            return bf16_bits(rng.integers(-3, 4, size=shape).astype(np.float32))
        return _normal_bf16(rng, shape, std)

    return {
        "X": draw((M, K), 1.0),
        "W": draw((N, K), 1.0 / math.sqrt(K)),
        "dY": draw((M, N), 1.0),
        "mask": mask,
    }


# ---------------------------------------------------------------- 2:4 semi-structured weights

_PAIRS = ((0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3))


def semi24_weight(N: int, K: int, rng: np.random.Generator, *, std: float = 1.0,
                  fewer: float = 0.0, integer_values: bool = False) -> np.ndarray:
    """Dense bf16 weight [N, K] (bit patterns) with zeros in place, at most
    two nonzeros in every group of four consecutive elements of a row: the
    2:4 semi-structured pattern.  Each group's two unpruned positions are one
    of the six pairs, uniformly; the other two are +0.  With ``fewer`` > 0
    each unpruned value is replaced, with that probability, by +0 or -0 (half
    each), so groups with one or no nonzero and signed zeros appear.  Values
    are normal(0, std) rounded to bf16, or integers in {-3..3} without 0 with
    ``integer_values``."""
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    G = N * (K // 4)
    pick = rng.integers(0, 6, size=G)
    pairs = np.asarray(_PAIRS, dtype=np.int64)[pick]          # [G, 2]
    if integer_values:
        mag = rng.integers(1, 4, size=(G, 2)).astype(np.float32)
        val = bf16_bits(mag * np.where(rng.random((G, 2)) < 0.5, -1.0, 1.0).astype(np.float32))
    else:
        val = _normal_bf16(rng, (G, 2), std)
    if fewer > 0:
        drop = rng.random((G, 2)) < fewer
        signed = rng.random((G, 2)) < 0.5
        val = np.where(drop, np.where(signed, np.uint16(0x8000), np.uint16(0)), val).astype(np.uint16)
    out = np.zeros((G, 4), dtype=np.uint16)
    rows = np.arange(G)
    out[rows, pairs[:, 0]] = val[:, 0]
    out[rows, pairs[:, 1]] = val[:, 1]
    return out.reshape(N, K)


@dataclasses.dataclass(frozen=True)
class Semi24Workload:
    """A linear layer whose weight has the 2:4 semi-structured pattern."""
    name: str
    M: int
    N: int
    K: int
    seed: int
    description: str = ""

    def flops(self) -> int:
        """Algorithmic flops of the forward: 2*M*N*(K/2), the products with
        the unpruned half of the weight."""
        return self.M * self.N * self.K


SEMI24_WORKLOADS: dict[str, Semi24Workload] = {w.name: w for w in [
    Semi24Workload("semi24_fwd", 8192, 14336, 4096, 6,
                   description="LLM-MLP forward, X[8192,4096], W[14336,4096] 2:4 semi-structured"),
]}


def make_semi24_inputs(w: Semi24Workload, *, M: int | None = None):
    """Seeded X [M,K] and 2:4 weight W [N,K] (bf16 bits) of a 2:4 workload.
    Sub-streams as for the block-sparse workloads: 0 for X, 2 for W."""
    M = w.M if M is None else M
    return {
        "X": _normal_bf16(np.random.default_rng(w.seed * 10 + 0), (M, w.K), 1.0),
        "W": semi24_weight(w.N, w.K, np.random.default_rng(w.seed * 10 + 2),
                           std=1.0 / math.sqrt(w.K / 2)),
    }


# ---------------------------------------------------------------- block-sparse with 2:4 blocks

BSR24_WORKLOADS: dict[str, Workload] = {w.name: w for w in [
    Workload("bsr24_fwd", 8192, 14336, 4096, 64, 0.1, 7, mask_kind="zipf",
             description="LLM-MLP forward, 90% block-sparse (Zipf rows), 2:4 inside the kept blocks"),
]}


def make_bsr24_inputs(w: Workload, *, M: int | None = None):
    """Seeded X [M,K], block mask and a dense weight W [N,K] with the 2:4
    pattern along K everywhere (the mask then keeps whole blocks of it), as
    bf16 bits.  Sub-streams as :func:`make_inputs`: 0 X, 1 mask, 2 W."""
    M = w.M if M is None else M
    return {
        "X": _normal_bf16(np.random.default_rng(w.seed * 10 + 0), (M, w.K), 1.0),
        "mask": make_mask(w),
        "W": semi24_weight(w.N, w.K, np.random.default_rng(w.seed * 10 + 2), std=math.sqrt(2.0 / w.K)),
    }
