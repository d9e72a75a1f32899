"""B200 (sm_100a) fine-grained-scaled FP8 / FP8xFP4 GEMM:  D = C + A @ B^T.

Thin Python binding over the C ABI in ``include/dg.h`` (``libdg.so``, built
in-tree by ``moe_grouped_gemm_06_b200/build.py``).  Each function here has
the name of the C entry point it calls and does argument marshalling only:
it reads shapes and device pointers off torch tensors and passes the current
CUDA stream.  Every step of the computation runs in the library's kernels;
there is no fallback of any kind, and importing this package raises if the
library has not been built.

torch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "DGError", "lib", "dg_fp8_gemm_nt", "dg_m_grouped_fp8_gemm_nt_contiguous",
    "dg_m_grouped_fp8_gemm_nt_masked", "dg_m_grouped_fp8_fp4_gemm_nt_masked",
    "dg_m_grouped_fp8_gemm_nt_masked_swiglu", "dg_m_grouped_fp8_fp4_gemm_nt_masked_swiglu", "dg_fp8_gemm_nt_noalloc", "dg_noalloc_scratch_bytes", "dg_fp8_gemm_nt_promoted", "dg_fp8_fp4_gemm_nt", "dg_bf16_gemm_nt", "dg_m_grouped_fp8_fp4_gemm_nt_contiguous",
    "dg_m_grouped_fp8_gemm_nn_contiguous", "dg_k_grouped_fp8_gemm_tn_contiguous", "dg_fp8_gemm_nn",
    "dg_fp8_gemm_tn", "dg_fp8_gemm_tt",
    "dg_quantize_fp8", "dg_quantize_fp4", "dg_pack_sf", "dg_packed_sf_words", "dg_get_num_sms",
    "dg_set_num_sms", "dg_set_pdl", "dg_get_pdl", "dg_set_tile_config", "dg_get_mk_alignment_for_contiguous_layout", "dg_get_last_error",
    "dg_debug_starved_wait", "dg_launch_count", "dg_query_dense_config", "dg_query_dense_cluster_split", "dg_debug_cluster_capacity", "dg_query_config", "dg_probe_mma_peak", "dg_num_tiles", "dg_debug_fastdiv", "dg_shutdown",
    "SYMBOLS",
]

# DG_LIBRARY may name another build of the same library (e.g. one compiled
# with -DDG_SELF_CHECK); by default the in-tree libdg.so is loaded.
LIB_PATH = os.environ.get("DG_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdg.so")

_VP, _I32P, _INT, _I64 = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64

# C signatures of every exported entry point (name -> (restype, argtypes)).
SYMBOLS = {
    "dg_fp8_gemm_nt": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _VP, _INT, _INT, _INT, _VP]),
    "dg_m_grouped_fp8_gemm_nt_contiguous": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _VP, _I32P, _INT, _INT, _INT,
                                                   _INT, _VP]),
    "dg_m_grouped_fp8_gemm_nt_masked": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _I32P, _INT, _INT, _INT, _INT, _INT, _VP]),
    "dg_m_grouped_fp8_fp4_gemm_nt_masked": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _I32P, _INT, _INT, _INT, _INT, _INT, _VP]),
    "dg_m_grouped_fp8_gemm_nt_masked_swiglu": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _I32P, _INT, _INT, _INT, _INT, _INT, _VP]),
    "dg_m_grouped_fp8_fp4_gemm_nt_masked_swiglu": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _I32P, _INT, _INT, _INT, _INT,
                                                          _INT, _VP]),
    "dg_fp8_gemm_nt_promoted": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _VP, _INT, _INT, _INT, _VP]),
    "dg_fp8_gemm_nt_noalloc": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _VP, _INT, _INT, _INT, _VP]),
    "dg_fp8_gemm_nn": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _VP, _INT, _INT, _INT, _VP]),
    "dg_fp8_gemm_tn": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _VP, _INT, _INT, _INT, _VP]),
    "dg_fp8_gemm_tt": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _VP, _INT, _INT, _INT, _VP]),
    "dg_noalloc_scratch_bytes": (ctypes.c_size_t, []),
    "dg_fp8_fp4_gemm_nt": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _VP, _INT, _INT, _INT, _VP]),
    "dg_bf16_gemm_nt": (_INT, [_VP, _VP, _VP, _VP, _INT, _INT, _INT, _VP]),
    "dg_m_grouped_fp8_fp4_gemm_nt_contiguous": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _VP, _I32P, _INT, _INT,
                                                       _INT, _INT, _VP]),
    "dg_m_grouped_fp8_gemm_nn_contiguous": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _VP, _I32P, _INT, _INT, _INT,
                                                   _INT, _VP]),
    "dg_k_grouped_fp8_gemm_tn_contiguous": (_INT, [_VP, _I32P, _VP, _I32P, _VP, _VP, _I32P, _INT, _INT, _INT,
                                                   _INT, _VP]),
    "dg_quantize_fp8": (_INT, [_VP, _INT, _INT, _INT, _VP, _VP, _VP]),
    "dg_quantize_fp4": (_INT, [_VP, _INT, _INT, _VP, _VP, _VP]),
    "dg_pack_sf": (_INT, [_VP, _INT, _INT, _INT, _VP, _VP]),
    "dg_packed_sf_words": (_I64, [_INT, _INT]),
    "dg_get_num_sms": (_INT, []),
    "dg_set_num_sms": (_INT, [_INT]),
    "dg_get_mk_alignment_for_contiguous_layout": (_INT, []),
    "dg_set_pdl": (_INT, [_INT]),
    "dg_set_tile_config": (_INT, [_INT, _INT]),
    "dg_get_pdl": (_INT, []),
    "dg_get_last_error": (_INT, [_VP]),
    "dg_debug_starved_wait": (_INT, [ctypes.c_uint, _VP]),
    "dg_status_string": (ctypes.c_char_p, [_INT]),
    "dg_launch_count": (ctypes.c_uint64, []),
    "dg_query_dense_config": (_INT, [_INT, _INT, _INT, _I64, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "dg_query_dense_cluster_split": (_INT, [_INT, _INT, _INT, _I64]),
    "dg_debug_cluster_capacity": (_INT, [_INT, _INT, _INT]),
    "dg_query_config": (_INT, [_INT, _INT, _INT, _INT, _INT, _INT, _INT, _INT, _VP, _VP, _VP]),
    "dg_probe_mma_peak": (_INT, [_INT, _INT, _INT, _VP]),
    "dg_num_tiles": (_I64, [_INT, _INT, _INT, _INT]),
    "dg_debug_fastdiv": (ctypes.c_uint32, [ctypes.c_uint32, ctypes.c_uint32]),
    "dg_shutdown": (None, []),
}

_lib = None


class DGError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} ({status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libdg.so (raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m moe_grouped_gemm_06_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SYMBOLS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().dg_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise DGError(status, where)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _bytes2(t):
    """2-D byte view [rows, cols] of a uint8 / float8 / packed tensor."""
    return t.shape[-2], t.shape[-1]


# ------------------------------------------------------------------ GEMMs

def dg_fp8_gemm_nt(a, sfa, b, sfb, c, d, stream=None) -> None:
    """D = C + A @ B^T.  a: e4m3 [m, k]; b: e4m3 [n, k]; sfa/sfb: packed sf
    words (int32); c: bf16 [m, n] or None; d: bf16 [m, n]."""
    m, k = a.shape
    n = b.shape[0]
    _check(lib().dg_fp8_gemm_nt(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(d), m, n, k, _stream(stream)),
           "dg_fp8_gemm_nt")


def dg_fp8_gemm_nt_promoted(a, sfa, b, sfb, c, d, stream=None) -> None:
    """As dg_fp8_gemm_nt, with the scales applied by per-K-block promotion
    (unscaled MMA per K-block, scaled and summed in FP32 by the epilogue)."""
    m, k = a.shape
    n = b.shape[0]
    _check(lib().dg_fp8_gemm_nt_promoted(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(d), m, n, k, _stream(stream)),
           "dg_fp8_gemm_nt_promoted")


def dg_fp8_gemm_nt_noalloc(a, sfa, b, sfb, c, d, stream=None) -> None:
    """As dg_fp8_gemm_nt, for callers that cannot allocate device memory at
    call time: split-K partials use the library's fixed 32 MiB device array
    (dg_noalloc_scratch_bytes()).  Calls that overlap on the GPU share that
    array and race; the first call on a device must precede stream capture."""
    m, k = a.shape
    n = b.shape[0]
    _check(lib().dg_fp8_gemm_nt_noalloc(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(d), m, n, k, _stream(stream)),
           "dg_fp8_gemm_nt_noalloc")


def dg_noalloc_scratch_bytes() -> int:
    return int(lib().dg_noalloc_scratch_bytes())


def _dense_layout_call(name, a_mn, b_mn, a, sfa, b, sfb, c, d, stream):
    k, m = a.shape if a_mn else (a.shape[1], a.shape[0])
    n = b.shape[1] if b_mn else b.shape[0]
    _check(getattr(lib(), name)(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(d), m, n, k, _stream(stream)), name)


def dg_fp8_gemm_nn(a, sfa, b, sfb, c, d, stream=None) -> None:
    """a: e4m3 [m, k]; b: e4m3 [k, n] (not transposed); sfa / sfb as for dg_fp8_gemm_nt."""
    _dense_layout_call("dg_fp8_gemm_nn", False, True, a, sfa, b, sfb, c, d, stream)


def dg_fp8_gemm_tn(a, sfa, b, sfb, c, d, stream=None) -> None:
    """a: e4m3 [k, m] (A stored transposed); b: e4m3 [k, n]."""
    _dense_layout_call("dg_fp8_gemm_tn", True, True, a, sfa, b, sfb, c, d, stream)


def dg_fp8_gemm_tt(a, sfa, b, sfb, c, d, stream=None) -> None:
    """a: e4m3 [k, m]; b: e4m3 [n, k] (as for dg_fp8_gemm_nt)."""
    _dense_layout_call("dg_fp8_gemm_tt", True, False, a, sfa, b, sfb, c, d, stream)


def dg_fp8_fp4_gemm_nt(a, sfa, b, sfb, c, d, stream=None) -> None:
    """As dg_fp8_gemm_nt with b: e2m1 packed [n, k/2] and per-1x32 sfb."""
    m, k = a.shape
    n = b.shape[0]
    _check(lib().dg_fp8_fp4_gemm_nt(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(d), m, n, k, _stream(stream)),
           "dg_fp8_fp4_gemm_nt")


def dg_bf16_gemm_nt(a, b, c, d, stream=None) -> None:
    """a: bf16 [m, k]; b: bf16 [n, k]; c: bf16 [m, n] or None; d: bf16 [m, n]."""
    m, k = a.shape
    n = b.shape[0]
    _check(lib().dg_bf16_gemm_nt(_p(a), _p(b), _p(c), _p(d), m, n, k, _stream(stream)), "dg_bf16_gemm_nt")


def dg_m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, c, d, m_indices, stream=None) -> None:
    """a: e4m3 [m_total, k]; b: e4m3 [groups, n, k]; m_indices: int32 [m_total]."""
    m_total, k = a.shape
    g, n = b.shape[0], b.shape[1]
    _check(lib().dg_m_grouped_fp8_gemm_nt_contiguous(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(d), _p(m_indices),
                                                     m_total, n, k, g, _stream(stream)),
           "dg_m_grouped_fp8_gemm_nt_contiguous")


def dg_m_grouped_fp8_fp4_gemm_nt_contiguous(a, sfa, b, sfb, c, d, m_indices, stream=None) -> None:
    """a: e4m3 [m_total, k]; b: e2m1 [groups, n, k/2]; m_indices: int32 [m_total]."""
    m_total, k = a.shape
    g, n = b.shape[0], b.shape[1]
    _check(lib().dg_m_grouped_fp8_fp4_gemm_nt_contiguous(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(d),
                                                         _p(m_indices), m_total, n, k, g, _stream(stream)),
           "dg_m_grouped_fp8_fp4_gemm_nt_contiguous")


def dg_m_grouped_fp8_gemm_nn_contiguous(a, sfa, b, sfb, c, d, m_indices, stream=None) -> None:
    """a: e4m3 [m_total, k]; b: e4m3 [groups, k, n] (not transposed);
    m_indices: int32 [m_total]."""
    m_total, k = a.shape
    g, n = b.shape[0], b.shape[2]
    _check(lib().dg_m_grouped_fp8_gemm_nn_contiguous(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(d), _p(m_indices),
                                                     m_total, n, k, g, _stream(stream)),
           "dg_m_grouped_fp8_gemm_nn_contiguous")


def dg_k_grouped_fp8_gemm_tn_contiguous(a, sfa, b, sfb, c, d, ks, stream=None) -> None:
    """a: e4m3 [k_total, m]; b: e4m3 [k_total, n]; ks: int32 [groups] on the
    device (K rows per group); c: bf16 [groups, m, n] or None; d: bf16
    [groups, m, n]."""
    k_total, m = a.shape
    n = b.shape[1]
    g = ks.shape[0]
    _check(lib().dg_k_grouped_fp8_gemm_tn_contiguous(_p(a), _p(sfa), _p(b), _p(sfb), _p(c), _p(d), _p(ks), g, m, n,
                                                     k_total, _stream(stream)),
           "dg_k_grouped_fp8_gemm_tn_contiguous")


def dg_m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, d, masked_m, expected_m: int = 0, stream=None) -> None:
    """a: e4m3 [groups, max_m, k]; b: e4m3 [groups, n, k]; d: bf16 [groups, max_m, n];
    masked_m: int32 [groups] on the device."""
    g, max_m, k = a.shape
    n = b.shape[1]
    _check(lib().dg_m_grouped_fp8_gemm_nt_masked(_p(a), _p(sfa), _p(b), _p(sfb), _p(d), _p(masked_m), g, max_m,
                                                 n, k, int(expected_m), _stream(stream)),
           "dg_m_grouped_fp8_gemm_nt_masked")


def _masked_call(name, a, sfa, b, sfb, d, masked_m, expected_m, stream):
    g, max_m, k = a.shape
    n = b.shape[1]
    _check(getattr(lib(), name)(_p(a), _p(sfa), _p(b), _p(sfb), _p(d), _p(masked_m), g, max_m, n, k,
                                int(expected_m), _stream(stream)), name)


def dg_m_grouped_fp8_fp4_gemm_nt_masked(a, sfa, b, sfb, d, masked_m, expected_m: int = 0, stream=None) -> None:
    """a: e4m3 [groups, max_m, k]; b: e2m1 [groups, n, k/2]; d: bf16 [groups, max_m, n]."""
    _masked_call("dg_m_grouped_fp8_fp4_gemm_nt_masked", a, sfa, b, sfb, d, masked_m, expected_m, stream)


def dg_m_grouped_fp8_gemm_nt_masked_swiglu(a, sfa, b, sfb, d, masked_m, expected_m: int = 0, stream=None) -> None:
    """b: e4m3 [groups, n, k], gate/up rows interleaved in blocks of 64; d: bf16 [groups, max_m, n/2]."""
    _masked_call("dg_m_grouped_fp8_gemm_nt_masked_swiglu", a, sfa, b, sfb, d, masked_m, expected_m, stream)


def dg_m_grouped_fp8_fp4_gemm_nt_masked_swiglu(a, sfa, b, sfb, d, masked_m, expected_m: int = 0,
                                               stream=None) -> None:
    """b: e2m1 [groups, n, k/2], gate/up rows interleaved in blocks of 64; d: bf16 [groups, max_m, n/2]."""
    _masked_call("dg_m_grouped_fp8_fp4_gemm_nt_masked_swiglu", a, sfa, b, sfb, d, masked_m, expected_m, stream)


# ------------------------------------------------------- input preparation

def dg_quantize_fp8(x, q, sf, block_rows: int, stream=None) -> None:
    """x: float32 [rows, cols] -> q: e4m3 [rows, cols], sf: ue8m0 [ceil(rows/block_rows), cols/128]."""
    rows, cols = x.shape
    _check(lib().dg_quantize_fp8(_p(x), rows, cols, int(block_rows), _p(q), _p(sf), _stream(stream)),
           "dg_quantize_fp8")


def dg_quantize_fp4(x, q, sf, stream=None) -> None:
    """x: float32 [rows, cols] -> q: e2m1 [rows, cols/2], sf: ue8m0 [rows, cols/32]."""
    rows, cols = x.shape
    _check(lib().dg_quantize_fp4(_p(x), rows, cols, _p(q), _p(sf), _stream(stream)), "dg_quantize_fp4")


def dg_pack_sf(sf, rows: int, packed, row_div: int = 1, stream=None) -> None:
    """sf: ue8m0 [ceil(rows/row_div), cols] -> packed int32 [dg_packed_sf_words(rows, cols)]."""
    cols = sf.shape[-1]
    _check(lib().dg_pack_sf(_p(sf), int(rows), int(cols), int(row_div), _p(packed), _stream(stream)),
           "dg_pack_sf")


def dg_packed_sf_words(rows: int, cols: int) -> int:
    return int(lib().dg_packed_sf_words(int(rows), int(cols)))


# ---------------------------------------------------------------- utilities

def dg_get_num_sms() -> int:
    return int(lib().dg_get_num_sms())


def dg_set_num_sms(n: int) -> None:
    _check(lib().dg_set_num_sms(int(n)), "dg_set_num_sms")


def dg_set_pdl(enable: bool) -> None:
    _check(lib().dg_set_pdl(int(bool(enable))), "dg_set_pdl")


def dg_set_tile_config(block_n: int = 0, schedule: int = 0) -> None:
    """block_n: 0 = heuristic; schedule: 0 heuristic, 1 whole tiles, 2 per-tile K-slices, 3 stream-K."""
    _check(lib().dg_set_tile_config(int(block_n), int(schedule)), "dg_set_tile_config")


def dg_get_pdl() -> bool:
    return bool(lib().dg_get_pdl())


def dg_get_mk_alignment_for_contiguous_layout() -> int:
    return int(lib().dg_get_mk_alignment_for_contiguous_layout())


def dg_get_last_error(stream=None) -> int:
    """Synchronises the stream; returns and clears the device-side error (0 = none)."""
    return int(lib().dg_get_last_error(_stream(stream)))


def dg_debug_starved_wait(limit_us: int, stream=None) -> None:
    _check(lib().dg_debug_starved_wait(int(limit_us), _stream(stream)), "dg_debug_starved_wait")


def dg_launch_count() -> int:
    return int(lib().dg_launch_count())


def dg_query_dense_config(m: int, n: int, k: int, workspace_cap: int = 0) -> dict:
    vals = [ctypes.c_int(0) for _ in range(6)] + [ctypes.c_int64(0)]
    _check(lib().dg_query_dense_config(m, n, k, int(workspace_cap), *[ctypes.byref(v) for v in vals]),
           "dg_query_dense_config")
    keys = ("block_n", "dp_tiles", "sk_tiles", "sk_split", "max_segments", "grid", "workspace_bytes")
    return dict(zip(keys, (v.value for v in vals)))


def dg_query_dense_cluster_split(m: int, n: int, k: int, workspace_cap: int = 0) -> int:
    """S > 0 when the dense plan splits every tile over a cluster of S CTAs."""
    return int(lib().dg_query_dense_cluster_split(m, n, k, int(workspace_cap)))


def dg_debug_cluster_capacity(block_n: int, cluster: int, fp4: bool = False) -> int:
    """Clusters of `cluster` CTAs of the split kernel the device holds at once."""
    return int(lib().dg_debug_cluster_capacity(block_n, int(fp4), cluster))


LAYOUTS = {"dense": 0, "contiguous": 1, "masked": 2}


def dg_query_config(layout: str, rows: int, n: int, k: int, groups: int = 1, fp4: bool = False,
                    expected_m: int = 0, swiglu: bool = False) -> dict:
    """Plan of an NT call (block_n, grid, units = output tiles) as the
    library would launch it; nothing is launched."""
    bn, grid, units = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int64(0)
    _check(lib().dg_query_config(LAYOUTS[layout], int(fp4), int(swiglu), rows, n, k, groups, expected_m,
                                 ctypes.byref(bn), ctypes.byref(grid), ctypes.byref(units)), "dg_query_config")
    return {"block_n": bn.value, "grid": grid.value, "units": units.value}


PROBE_KINDS = {"fp8_block_scaled": 0, "fp8_plain": 1, "bf16": 2}


def dg_probe_mma_peak(kind: str, block_n: int, kblocks: int, stream=None) -> float:
    """Enqueues the tensor-core throughput probe; returns the FLOPs that one
    launch performs (time it with CUDA events on the same stream)."""
    _check(lib().dg_probe_mma_peak(PROBE_KINDS[kind], block_n, kblocks, _stream(stream)), "dg_probe_mma_peak")
    k_per_mma = 16 if kind == "bf16" else 32
    return float(dg_get_num_sms_device()) * kblocks * 4 * 2 * 128 * block_n * k_per_mma


def dg_get_num_sms_device() -> int:
    """SMs of the current device (the probe's grid), ignoring dg_set_num_sms."""
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


def dg_num_tiles(m: int, n: int, block_m: int, block_n: int) -> int:
    return int(lib().dg_num_tiles(m, n, block_m, block_n))


def dg_debug_fastdiv(d: int, n: int) -> int:
    return int(lib().dg_debug_fastdiv(d, n))


def dg_shutdown() -> None:
    lib().dg_shutdown()
