"""GPU parity of dg_fp8_gemm_nt_promoted (scales applied by per-K-block
promotion in the epilogue instead of inside the block-scaled MMA) against the
CPU oracle, and an accuracy comparison of the two ways of applying the scales
at long K.

The pages' Hopper design promotes every K-block's partial sum into FP32 on
CUDA cores because FP8 tensor-core accumulation is imprecise there ("DeepSeek
开源第三弹 ... DeepGEMM" (app.myzaker.com), section "DeepGEMM": two-level
accumulation).  On sm_100a both paths must meet the same tolerance; the
accuracy test reports, for each, the largest error in units of the bf16 ulp of
the exact result and the share of outputs that are not the correctly rounded
bf16 of the exact value, on inputs chosen to stress the accumulator (K =
16384, all products positive, so nothing cancels)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import Dense, bf16_dev_to_f64, check_close, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from moe_grouped_gemm_06_b200 import build
    build.build()
    import moe_grouped_gemm_06_b200 as dg
    assert dg.dg_get_last_error() == 0
    yield dg
    assert dg.dg_get_last_error() == 0


@pytest.fixture(autouse=True)
def no_device_error_left(dg):
    yield
    assert dg.dg_get_last_error() == 0, "device error recorded during this test"


def run_promoted(dg, p):
    dg.dg_fp8_gemm_nt_promoted(p.t_a, p.t_sfa, p.t_b, p.t_sfb, p.t_c, p.t_d)
    torch.cuda.synchronize()
    return bf16_dev_to_f64(p.t_d)


@pytest.mark.parametrize("M,N,K,with_c", [
    (128, 512, 1024, False),    # the small worked configuration
    (200, 328, 384, True),      # ragged M and N tails, three K-blocks
    (1100, 520, 640, True),     # several m-blocks, K-blocks not a multiple of 4
    (64, 2112, 7168, True),     # small M, the planner may share tiles by K
    (1, 136, 512, True),        # a single row
])
def test_promoted_matches_oracle(dg, M, N, K, with_c):
    p = Dense(12000 + M + N, M, N, K, with_c=with_c).upload()
    check_close(run_promoted(dg, p), p.ref(), f"promoted {M}x{N}x{K}")


@pytest.mark.parametrize("schedule", [2, 3])
def test_promoted_shared_tails_match_oracle(dg, schedule):
    # pieces of shared tiles (per-tile K-slices or stream-K) write FP32 sums
    # from the epilogue's registers; with 7 "SMs" the problem runs whole-tile
    # waves first, as large problems do on 148 SMs
    M, N, K = 1100, 1000, 1536
    dg.dg_set_num_sms(7)
    dg.dg_set_tile_config(128, schedule)
    try:
        assert dg.dg_query_dense_config(M, N, K)["sk_tiles"] > 0
        p = Dense(12100 + schedule, M, N, K, with_c=True).upload()
        got = run_promoted(dg, p)
    finally:
        dg.dg_set_tile_config(0, 0)
        dg.dg_set_num_sms(0)
    check_close(got, p.ref(), f"promoted schedule {schedule}")


def test_promoted_long_k(dg):
    p = Dense(12200, 128, 256, 16384, with_c=False).upload()
    check_close(run_promoted(dg, p), p.ref(), "promoted K=16384")


def test_promoted_scale_doubling_is_bit_exact(dg):
    # C = 0 and one non-zero K-block: raising that block's A scale by one
    # doubles every output exactly
    M, N, K = 256, 256, 512
    p = Dense(12300, M, N, K, with_c=False)
    p.qa[:, :128] = 0
    p.qa[:, 256:] = 0
    p.sfa = oracle.pack_sf(p.ea, M)
    p.upload()
    d1 = run_promoted(dg, p)
    ea2 = p.ea.copy()
    ea2[:, 1] += 1
    p.t_sfa = dev(oracle.pack_sf(ea2, M))
    d2 = run_promoted(dg, p)
    assert np.array_equal(d2, 2.0 * d1)
    assert np.count_nonzero(d1) > 0.9 * d1.size


def test_promoted_full_size_sampled(dg):
    # the dominant sweep shape and a small-M one, in the plans bench.py times
    for (M, N, K) in [(4096, 7168, 16384), (64, 7168, 16384)]:
        xb = synth.normal_f32(12400 + N + K, (N, K))
        p = Dense(12500 + M, M, N, K, with_c=True, xb=xb).upload()
        d = run_promoted(dg, p)
        pm, pn = synth.sample_points(12600 + M, np.arange(M), N, 2048)
        check_close(d[pm, pn], p.ref_points(pm, pn), f"promoted {M}x{N}x{K}")
        del p
        torch.cuda.empty_cache()


def _bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits): 2^(e - 8) for
    |x| in [2^(e-1), 2^e)."""
    _, e = np.frexp(np.abs(x))
    return np.ldexp(1.0, e - 8)


def _accuracy(d, ref):
    err = np.abs(d - ref)
    ulps = err / _bf16_ulp(ref)
    # correctly rounded: within half an ulp of the exact value (a tie can go
    # either way only when the exact value sits on a midpoint)
    return {"max_ulp": float(ulps.max()), "mean_ulp": float(ulps.mean()),
            "not_correctly_rounded": float(np.mean(ulps > 0.5 + 1e-12)),
            "max_rel": float((err / np.abs(ref)).max())}


@pytest.mark.parametrize("inputs", ["normal", "positive"])
def test_accumulation_accuracy_at_long_k(dg, inputs):
    """Both ways of applying the scales at K = 16384 against the exact
    (FP64) result: within the tolerance, and the error statistics printed
    for the record."""
    M, N, K = 256, 256, 16384
    xa = synth.normal_f32(12700, (M, K))
    xb = synth.normal_f32(12701, (N, K))
    if inputs == "positive":
        xa, xb = np.abs(xa), np.abs(xb)
    p = Dense(12702, M, N, K, with_c=False, xa=xa, xb=xb).upload()
    ref = p.ref()
    dg.dg_fp8_gemm_nt(p.t_a, p.t_sfa, p.t_b, p.t_sfb, None, p.t_d)
    torch.cuda.synchronize()
    scaled = bf16_dev_to_f64(p.t_d)
    promoted = run_promoted(dg, p)
    check_close(scaled, ref, f"block-scaled {inputs}")
    check_close(promoted, ref, f"promoted {inputs}")
    a_s, a_p = _accuracy(scaled, ref), _accuracy(promoted, ref)
    print(f"\naccuracy K={K} inputs={inputs}: block-scaled MMA {a_s}; per-K-block promotion {a_p}", flush=True)
