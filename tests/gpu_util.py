"""Helpers shared by the GPU parity tests: seeded inputs (synth), quantised and
packed by the CPU oracle, uploaded with torch; comparison under the
tolerances of the method:

  per element  |D - ref| <= 2^-7 |ref| + 1e-3 rms(ref)
  globally     1 - 2<D, ref> / (|D|^2 + |ref|^2) <= 1e-3

(D is one bf16 rounding of the FP32 sum, so half of the per-element budget is
the bf16 half-ulp; the rest covers FP32 accumulation order.)
"""
from __future__ import annotations

import ml_dtypes
import numpy as np
import torch

import oracle
import synth

REL_TOL = 2.0 ** -7
ABS_TOL_RMS = 1e-3
GLOBAL_TOL = 1e-3


def dev(x) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def bf16_dev_to_f64(t: torch.Tensor) -> np.ndarray:
    bits = t.detach().view(torch.int16).cpu().numpy().view(np.uint16)
    return bits.view(ml_dtypes.bfloat16).astype(np.float64)


def check_close(d: np.ndarray, ref: np.ndarray, what: str = "") -> dict:
    d = np.asarray(d, np.float64).ravel()
    ref = np.asarray(ref, np.float64).ravel()
    assert d.shape == ref.shape
    assert np.isfinite(ref).all(), f"{what}: non-finite reference"
    assert np.isfinite(d).all(), f"{what}: non-finite output at {np.nonzero(~np.isfinite(d))[0][:8]}"
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = np.abs(d - ref)
    bound = REL_TOL * np.abs(ref) + ABS_TOL_RMS * rms
    bad = np.nonzero(err > bound)[0]
    assert bad.size == 0, (f"{what}: {bad.size} elements out of tolerance, e.g. idx {bad[:5]} "
                           f"d={d[bad[:5]]} ref={ref[bad[:5]]}")
    denom = float(np.sum(d * d) + np.sum(ref * ref))
    glob = 1.0 - 2.0 * float(np.sum(d * ref)) / denom if denom > 0 else 0.0
    assert glob <= GLOBAL_TOL, f"{what}: global difference {glob}"
    rel = err / np.maximum(np.abs(ref), 1e-30)
    return {"max_rel": float(rel.max()) if rel.size else 0.0, "global": glob, "n": int(d.size)}


# ------------------------------------------------------------- input builders

class Dense:
    """A dense problem: e4m3 A (1x128 scales), e4m3 B (128x128 scales) or
    e2m1 B (1x32 scales), optional bf16 C; quantised and packed by the oracle."""

    def __init__(self, seed: int, M: int, N: int, K: int, with_c: bool = True, fp4: bool = False,
                 xa=None, xb=None):
        self.M, self.N, self.K, self.fp4 = M, N, K, fp4
        xa = synth.normal_f32(seed, (M, K)) if xa is None else xa
        xb = synth.normal_f32(seed + 1, (N, K)) if xb is None else xb
        self.qa, self.ea = oracle.quantize_fp8(xa, 1)
        if fp4:
            self.qb, self.eb = oracle.quantize_fp4(xb, 32)
            self.sfb = oracle.pack_sf(self.eb, N)
        else:
            self.qb, self.eb = oracle.quantize_fp8(xb, 128)
            self.sfb = oracle.pack_sf(self.eb, N, row_div=128)
        self.sfa = oracle.pack_sf(self.ea, M)
        self.c = synth.normal_bf16_bits(seed + 2, (M, N)) if with_c else None

    def upload(self):
        self.t_a, self.t_sfa = dev(self.qa), dev(self.sfa)
        self.t_b, self.t_sfb = dev(self.qb), dev(self.sfb)
        self.t_c = dev(self.c.view(np.int16)) if self.c is not None else None
        self.t_d = torch.empty((self.M, self.N), dtype=torch.int16, device="cuda")
        return self

    def run(self, dg):
        fn = dg.dg_fp8_fp4_gemm_nt if self.fp4 else dg.dg_fp8_gemm_nt
        fn(self.t_a, self.t_sfa, self.t_b, self.t_sfb, self.t_c, self.t_d)
        torch.cuda.synchronize()
        return bf16_dev_to_f64(self.t_d)

    def ref(self):
        return oracle.gemm(self.qa, self.ea, self.qb, self.eb, c=self.c, b_fp4=self.fp4)

    def ref_points(self, pm, pn):
        return oracle.gemm_points(self.qa, self.ea, self.qb, self.eb, pm, pn, c=self.c, b_fp4=self.fp4)


def quantize_groups_b(seed: int, G: int, N: int, K: int, fp4: bool = False):
    qs, es, packs = [], [], []
    for g in range(G):
        xb = synth.normal_f32(seed + g, (N, K))
        if fp4:
            q, e = oracle.quantize_fp4(xb, 32)
            p = oracle.pack_sf(e, N)
        else:
            q, e = oracle.quantize_fp8(xb, 128)
            p = oracle.pack_sf(e, N, row_div=128)
        qs.append(q)
        es.append(e)
        packs.append(p.ravel())
    return np.stack(qs), np.stack(es), np.concatenate(packs)
