"""CPU oracle for the fine-grained-scaled GEMM D = C + A * B^T.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm may import this package.  The
product (``moe_grouped_gemm_06_b200``) never imports it, and it never imports
the product: the two share no code.

The arithmetic lives in ``dg_oracle.c`` (plain C, double precision, table
decode of E4M3 / E2M1 / UE8M0); this module only builds that file with gcc and
marshals numpy arrays into it.

Sources (page title, section):
  * "DeepSeek 开源第三弹 ... DeepGEMM" (app.myzaker.com), section "DeepGEMM":
    FP8 GEMM with DeepSeek-V3 fine-grained scaling.
  * "DeepGEMM：统一高性能张量核心 GEMM 计算库编译与使用指南" (zhouruolin.cn),
    section 五 "使用方法": D = C + A @ B, NT layout, SM100 packed UE8M0 scale
    factors, M-grouped contiguous and masked layouts.
  * "DeepSeek 发布 DeepGEMM 重大更新" (linlog.top), section "FP4 精度支持":
    FP8 x FP4 GEMM, UE8M0 scales packed 4 per int32; its Mega MoE section and
    "DeepGEMM：FP8 GEMM 与 Mega-MoE" (charles2530.github.io): each expert runs
    linear1 -> SwiGLU -> linear2 (swiglu_interleaved below).

Every function is pinned by a ``-m "not gpu"`` test in ``tests/test_oracle.py``
against something other than itself (ml_dtypes code tables, numpy float64
matmul on independently decoded operands, closed forms, exact power-of-two
invariants, per-group slicing).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dg_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile dg_oracle.c into liboracle.so (gcc, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
    return _lib


def _p(arr):
    return arr.ctypes.data_as(ctypes.c_void_p) if arr is not None else None


def _c(arr, dtype):
    return np.ascontiguousarray(arr, dtype=dtype)


I64 = ctypes.c_int64


def tables():
    """(e4m3[256], e2m1[16], ue8m0[256]) float64 value tables, from bit fields."""
    lib = _load()
    e4, e2, ue = np.zeros(256), np.zeros(16), np.zeros(256)
    lib.or_tables(_p(e4), _p(e2), _p(ue))
    return e4, e2, ue


def num_threads() -> int:
    return int(_load().or_num_threads())


def encode_e4m3(v) -> np.ndarray:
    v = _c(v, np.float64).ravel()
    out = np.zeros(v.size, np.uint8)
    _load().or_encode_e4m3(_p(v), I64(v.size), _p(out))
    return out


def encode_e2m1(v) -> np.ndarray:
    v = _c(v, np.float64).ravel()
    out = np.zeros(v.size, np.uint8)
    _load().or_encode_e2m1(_p(v), I64(v.size), _p(out))
    return out


def scale_exponents(amax, qmax: float) -> np.ndarray:
    """i = min{i : qmax * 2^i >= amax}, clamped to [-127, 127] (0 for amax = 0)."""
    amax = _c(amax, np.float64).ravel()
    out = np.zeros(amax.size, np.int32)
    _load().or_scale_exponents_probe(_p(amax), I64(amax.size), ctypes.c_double(qmax), _p(out))
    return out


def quantize_fp8(x, gr: int, gc: int = 128):
    """E4M3 codes [rows, cols] and UE8M0 codes [ceil(rows/gr), cols/gc].

    gr = 1 is the activation recipe (one scale per 1x128 row-group), gr = 128
    the weight recipe (one scale per 128x128 block)."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    assert cols % gc == 0
    q = np.zeros((rows, cols), np.uint8)
    e = np.zeros(((rows + gr - 1) // gr, cols // gc), np.uint8)
    _load().or_quantize_fp8(_p(x), I64(rows), I64(cols), ctypes.c_int(gr), ctypes.c_int(gc),
                            _p(q), _p(e))
    return q, e


def quantize_fp4(x, gc: int = 32):
    """E2M1 codes packed two per byte [rows, cols/2] (low nibble = even column)
    and UE8M0 codes [rows, cols/gc]."""
    x = _c(x, np.float32)
    rows, cols = x.shape
    assert cols % gc == 0 and gc % 2 == 0
    q = np.zeros((rows, cols // 2), np.uint8)
    e = np.zeros((rows, cols // gc), np.uint8)
    _load().or_quantize_fp4(_p(x), I64(rows), I64(cols), ctypes.c_int(gc), _p(q), _p(e))
    return q, e


def pack_sf(e, rows: int, row_div: int = 1) -> np.ndarray:
    """Pack UE8M0 codes 4 per int32 into the library's scale layout.

    ``e`` is uint8 [ceil(rows/row_div), ng].  Returns int32 [Q, Cr, 128],
    Q = ceil(ng/4), Cr = ceil(rows/128); the word of (row r, group q) is at
    [q, r//128, (r%32)*4 + (r%128)//32] and its byte j holds column 4q+j."""
    e = _c(e, np.uint8)
    ng = e.shape[1]
    q, cr = (ng + 3) // 4, (rows + 127) // 128
    out = np.zeros((q, cr, 128), np.int32)
    _load().or_pack_sf(_p(e), I64(rows), I64(ng), ctypes.c_int(row_div), _p(out))
    return out


def _gemm_args(a, sfa, b, sfb, b_fp4, c):
    a = _c(a, np.uint8)
    sfa = _c(sfa, np.uint8)
    b = _c(b, np.uint8)
    sfb = _c(sfb, np.uint8)
    c = _c(c, np.uint16) if c is not None else None
    return a, sfa, b, sfb, int(bool(b_fp4)), c


def gemm(a, sfa, b, sfb, c=None, b_fp4=False) -> np.ndarray:
    """Dense NT reference, float64 [M, N].

    a: e4m3 [M, K]; sfa: UE8M0 [M, K/128].
    b: e4m3 [N, K] with sfb [ceil(N/128), K/128], or (b_fp4) packed e2m1
       [N, K/2] with sfb [N, K/32].
    c: bf16 bit patterns (uint16) [M, N] or None."""
    a, sfa, b, sfb, fp4, c = _gemm_args(a, sfa, b, sfb, b_fp4, c)
    M, K = a.shape
    N = b.shape[0]
    out = np.zeros((M, N), np.float64)
    _load().or_gemm(_p(a), _p(sfa), _p(b), _p(sfb), ctypes.c_int(fp4), _p(c),
                    I64(M), I64(N), I64(K), _p(out))
    return out


def gemm_points(a, sfa, b, sfb, pm, pn, c=None, b_fp4=False) -> np.ndarray:
    """The dense reference at the points (pm[t], pn[t]) only."""
    a, sfa, b, sfb, fp4, c = _gemm_args(a, sfa, b, sfb, b_fp4, c)
    M, K = a.shape
    N = b.shape[0]
    pm = _c(pm, np.int64)
    pn = _c(pn, np.int64)
    out = np.zeros(pm.size, np.float64)
    _load().or_gemm_points(_p(a), _p(sfa), _p(b), _p(sfb), ctypes.c_int(fp4), _p(c),
                           I64(M), I64(N), I64(K), _p(pm), _p(pn), I64(pm.size), _p(out))
    return out


def gemm_contiguous(a, sfa, b, sfb, m_indices, c=None, b_fp4=False, out=None) -> np.ndarray:
    """M-grouped contiguous reference.  b: [G, N, K] (or [G, N, K/2] for fp4),
    sfb: [G, ...].  Rows with m_indices < 0 keep the values of ``out``
    (NaN when ``out`` is not given)."""
    a, sfa, b, sfb, fp4, c = _gemm_args(a, sfa, b, sfb, b_fp4, c)
    M, K = a.shape
    G, N = b.shape[0], b.shape[1]
    mi = _c(m_indices, np.int32)
    res = np.full((M, N), np.nan) if out is None else _c(out, np.float64).copy()
    _load().or_gemm_contiguous(_p(a), _p(sfa), _p(b), _p(sfb), ctypes.c_int(fp4), _p(c),
                               _p(mi), I64(M), I64(N), I64(K), I64(G), _p(res))
    return res


def gemm_masked(a, sfa, b, sfb, masked_m, b_fp4=False, out=None) -> np.ndarray:
    """M-grouped masked reference.  a: [G, max_m, K], sfa: [G, max_m, K/128],
    b: [G, N, K], sfb: [G, ...].  Rows m >= masked_m[g] keep the values of
    ``out`` (NaN when ``out`` is not given)."""
    a, sfa, b, sfb, fp4, _ = _gemm_args(a, sfa, b, sfb, b_fp4, None)
    G, max_m, K = a.shape
    N = b.shape[1]
    mm = _c(masked_m, np.int32)
    res = np.full((G, max_m, N), np.nan) if out is None else _c(out, np.float64).copy()
    _load().or_gemm_masked(_p(a), _p(sfa), _p(b), _p(sfb), ctypes.c_int(fp4), _p(mm),
                           I64(G), I64(max_m), I64(N), I64(K), _p(res))
    return res


def gemm_layout(a, sfa, b, sfb, layout: str, c=None) -> np.ndarray:
    """Dense FP8 reference in one of the layouts "nt", "nn", "tn", "tt": the
    first letter is A ("n": [M, K], "t": stored [K, M]), the second B ("t":
    [N, K], "n": stored [K, N]).  sfa [M, K/128], sfb [ceil(N/128), K/128]
    whatever the storage.  Float64 [M, N]."""
    assert layout in ("nt", "nn", "tn", "tt")
    a_mn, b_mn = layout[0] == "t", layout[1] == "n"
    a, sfa, b, sfb, _, c = _gemm_args(a, sfa, b, sfb, False, c)
    K, M = a.shape if a_mn else a.shape[::-1]
    N = b.shape[1] if b_mn else b.shape[0]
    assert (b.shape[0] if b_mn else b.shape[1]) == K
    out = np.zeros((M, N), np.float64)
    _load().or_gemm_layout(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), ctypes.c_int(int(a_mn)), ctypes.c_int(int(b_mn)),
                           I64(M), I64(N), I64(K), _p(out))
    return out


def gemm_nn_contiguous(a, sfa, b, sfb, m_indices, c=None, out=None) -> np.ndarray:
    """M-grouped contiguous reference with B not transposed (NN).
    b: e4m3 [G, K, N]; sfb: UE8M0 [G, ceil(N/128), K/128] (block (n/128,
    k/128), the NT indexing).  Rows with m_indices < 0 keep ``out`` (NaN)."""
    a, sfa, b, sfb, _, c = _gemm_args(a, sfa, b, sfb, False, c)
    M, K = a.shape
    G, N = b.shape[0], b.shape[2]
    assert b.shape[1] == K
    mi = _c(m_indices, np.int32)
    res = np.full((M, N), np.nan) if out is None else _c(out, np.float64).copy()
    _load().or_gemm_nn_contiguous(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(mi),
                                  I64(M), I64(N), I64(K), I64(G), _p(res))
    return res


def gemm_k_grouped_tn(a, sfa, b, sfb, ks, c=None) -> np.ndarray:
    """K-grouped TN reference (weight gradient), float64 [G, M, N].
    a: e4m3 [Kt, M]; sfa: UE8M0 [M, Kt/128]; b: e4m3 [Kt, N]; sfb: UE8M0
    [N, Kt/128]; ks: K rows per group (multiples of 128, sum <= Kt);
    c: bf16 bits [G, M, N] or None.  D[g] = C[g] + A_g^T B_g."""
    a, sfa, b, sfb, _, c = _gemm_args(a, sfa, b, sfb, False, c)
    Kt, M = a.shape
    N = b.shape[1]
    ks = _c(ks, np.int32)
    G = ks.size
    assert b.shape[0] == Kt and int(ks.sum()) <= Kt and np.all(ks % 128 == 0) and np.all(ks >= 0)
    out = np.zeros((G, M, N), np.float64)
    _load().or_gemm_k_grouped_tn(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(ks),
                                 I64(G), I64(M), I64(N), I64(Kt), _p(out))
    return out


def gemm_k_grouped_tn_points(a, sfa, b, sfb, ks, pg, pi, pj, c=None) -> np.ndarray:
    """The K-grouped TN reference at the points (pg[t], pi[t], pj[t]) only."""
    a, sfa, b, sfb, _, c = _gemm_args(a, sfa, b, sfb, False, c)
    Kt, M = a.shape
    N = b.shape[1]
    ks = _c(ks, np.int32)
    assert b.shape[0] == Kt and int(ks.sum()) <= Kt and np.all(ks % 128 == 0) and np.all(ks >= 0)
    pg, pi, pj = _c(pg, np.int64), _c(pi, np.int64), _c(pj, np.int64)
    out = np.zeros(pg.size, np.float64)
    _load().or_gemm_k_grouped_tn_points(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(ks), I64(ks.size), I64(M),
                                        I64(N), I64(Kt), _p(pg), _p(pi), _p(pj), I64(pg.size), _p(out))
    return out


SWIGLU_BLOCK = 64


def silu(x) -> np.ndarray:
    """silu(x) = x / (1 + exp(-x)) = x * sigmoid(x), in float64."""
    x = np.asarray(x, np.float64)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def swiglu_interleaved(g, block: int = SWIGLU_BLOCK) -> np.ndarray:
    """SwiGLU of a linear1 output whose columns hold gate and up projections
    interleaved in blocks: columns [2jb, 2jb + b) are gate columns jb.., the
    next b the matching up columns.  out[..., jb + i] = silu(g[..., 2jb + i])
    * g[..., 2jb + b + i]; the last axis halves.  float64 in, float64 out
    (the library rounds this once to bf16)."""
    g = np.asarray(g, np.float64)
    n = g.shape[-1]
    if n % (2 * block):
        raise ValueError("columns must be a multiple of 2 * block")
    blocks = g.reshape(g.shape[:-1] + (n // (2 * block), 2, block))
    out = silu(blocks[..., 0, :]) * blocks[..., 1, :]
    return out.reshape(g.shape[:-1] + (n // 2,))



def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64: the upper half of an IEEE
    binary32 (sign, 8 exponent bits, 7 mantissa bits)."""
    bits = np.asarray(bits, np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def gemm_bf16(a_bits, b_bits, c_bits=None) -> np.ndarray:
    """Plain bf16 GEMM reference D = C + A * B^T in float64 (no scales):
    a_bits [M, K], b_bits [N, K], c_bits [M, N] or None, bf16 bit patterns."""
    d = bf16_to_f64(a_bits) @ bf16_to_f64(b_bits).T
    if c_bits is not None:
        d = d + bf16_to_f64(c_bits)
    return d
