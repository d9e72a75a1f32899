"""dg_fp8_gemm_nt_noalloc: the dense FP8 GEMM for callers that cannot
allocate device memory at call time (a framework that owns all device memory,
a serving loop with memory fixed up front, a hot path where cudaMalloc /
cudaFree are not allowed because they can synchronise the device or fail).
Its split-K partial sums live in the library's fixed device array instead of
a workspace allocated on first use.

Checked through the C ABI against the allocating entry point
dg_fp8_gemm_nt, with the same tolerance as the other GPU tests, on two calls
in a row (the array keeps the previous call's contents).  This file is
collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process."""
import numpy as np
import pytest
import torch

from gpu_util import Dense, bf16_dev_to_f64, check_close

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


@pytest.mark.parametrize("M,N,K", [(64, 2112, 7168), (128, 7168, 2048), (200, 512, 1024), (1100, 520, 512)])
def test_noalloc_matches_allocating_call_twice(dg, M, N, K):
    p = Dense(8000 + M + N, M, N, K, with_c=True).upload()
    cfg = dg.dg_query_dense_config(M, N, K)
    if M <= 200:
        assert cfg["splits"] > 1          # these shapes exercise the scratch array
    need = cfg["splits"] * M * N * 4 if cfg["splits"] > 1 else 0
    assert need <= dg.dg_noalloc_scratch_bytes()

    dg.dg_fp8_gemm_nt(p.t_a, p.t_sfa, p.t_b, p.t_sfb, p.t_c, p.t_d)
    torch.cuda.synchronize()
    want = bf16_dev_to_f64(p.t_d)

    for _ in range(2):                    # two calls in a row on the shared array
        d = torch.full((M, N), 0x7FC1, dtype=torch.int16, device="cuda")
        dg.dg_fp8_gemm_nt_noalloc(p.t_a, p.t_sfa, p.t_b, p.t_sfb, p.t_c, d)
        torch.cuda.synchronize()
        assert dg.dg_get_last_error() == 0
        check_close(bf16_dev_to_f64(d), want, f"noalloc {M}x{N}x{K}")


def test_noalloc_rejects_problems_beyond_its_scratch(dg):
    # Pretend to have 4096 SMs so that the heuristic splits K 8 ways on a
    # 1024 x 8192 output: 8 * 1024 * 8192 * 4 bytes = 256 MiB > 32 MiB.  The
    # call must return DG_ERR_SCRATCH_LIMIT before anything is launched (the
    # pointers below are never dereferenced).
    import ctypes
    dg.dg_set_num_sms(4096)
    try:
        cfg = dg.dg_query_dense_config(1024, 8192, 16384)
        assert cfg["splits"] * 1024 * 8192 * 4 > dg.dg_noalloc_scratch_bytes()
        fake = ctypes.c_void_p(1 << 24)
        launches = dg.dg_launch_count()
        st = dg.lib().dg_fp8_gemm_nt_noalloc(fake, fake, fake, fake, None, fake, 1024, 8192, 16384, None)
        assert st == -6 and dg.status_string(st) == "DG_ERR_SCRATCH_LIMIT"
        assert dg.dg_launch_count() == launches
    finally:
        dg.dg_set_num_sms(0)
