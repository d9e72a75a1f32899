"""Seeded synthetic inputs shared by the tests, the CPU oracle and bench.py.

This module only draws random numbers and lays them out; it contains none of
the GEMM's arithmetic (no quantisation, no scale rule, no packing).  Every
generator takes an explicit seed and uses numpy's PCG64 ``default_rng``.

Workload shapes follow the DeepSeek-V3 inference GEMMs that the DeepGEMM
release measured ("DeepSeek 开源第三弹 ... DeepGEMM" (app.myzaker.com),
section "性能"): dense projections with N,K in {(2112,7168), (24576,1536),
(32768,512), (7168,16384), (4096,7168), (7168,2048)}, MoE prefill through the
contiguous layout and MoE decode through the masked layout.
"""
from __future__ import annotations

import ml_dtypes
import numpy as np

DENSE_NK = [(2112, 7168), (24576, 1536), (32768, 512), (7168, 16384), (4096, 7168), (7168, 2048)]
DENSE_M = [64, 128, 4096]
GROUPED_NK = [(4096, 7168), (7168, 2048)]
MK_ALIGNMENT = 128


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def normal_f32(seed: int, shape) -> np.ndarray:
    """Independent N(0, 1) float32 samples."""
    return rng(seed).standard_normal(size=shape, dtype=np.float32)


def normal_bf16_bits(seed: int, shape) -> np.ndarray:
    """N(0, 1) samples stored as bfloat16 bit patterns (uint16)."""
    return normal_f32(seed, shape).astype(ml_dtypes.bfloat16).view(np.uint16)


def junk_bytes(seed: int, shape) -> np.ndarray:
    """Uniform random bytes; about 1 in 128 of them is an E4M3 NaN code."""
    return rng(seed).integers(0, 256, size=shape, dtype=np.uint8)


def contiguous_layout(seed: int, num_groups: int, lo: int, hi: int, align: int = MK_ALIGNMENT):
    """Rows per group ~ U[lo, hi] (inclusive integers); each group is padded to a
    multiple of ``align`` rows.  Returns (rows_per_group, m_indices) where
    m_indices[m] is the group of row m or -1 for a padding row."""
    r = rng(seed).integers(lo, hi, size=num_groups, endpoint=True)
    idx = []
    for g, n in enumerate(r):
        padded = (int(n) + align - 1) // align * align
        idx.append(np.full(int(n), g, np.int32))
        idx.append(np.full(padded - int(n), -1, np.int32))
    m_indices = np.concatenate(idx) if idx else np.zeros(0, np.int32)
    return r.astype(np.int64), m_indices


def k_grouped_sizes(seed: int, num_groups: int, lo: int, hi: int, align: int = MK_ALIGNMENT) -> np.ndarray:
    """K rows per group of a K-grouped (weight-gradient) call: U[lo, hi]
    (inclusive integers) rounded up to a multiple of ``align``."""
    r = rng(seed).integers(lo, hi, size=num_groups, endpoint=True)
    return ((r + align - 1) // align * align).astype(np.int32)


def masked_counts(seed: int, num_groups: int, expected_m: int, max_m: int) -> np.ndarray:
    """masked_m[g] = min(max_m, U{0 .. 2*expected_m})."""
    r = rng(seed).integers(0, 2 * expected_m, size=num_groups, endpoint=True)
    return np.minimum(r, max_m).astype(np.int32)


def sample_points(seed: int, rows: np.ndarray, N: int, count: int):
    """``count`` (m, n) output positions, m drawn from ``rows``, n from [0, N)."""
    g = rng(seed)
    pm = g.choice(rows, size=count, replace=True).astype(np.int64)
    pn = g.integers(0, N, size=count).astype(np.int64)
    return pm, pn
