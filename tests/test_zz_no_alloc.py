"""dg_fp8_gemm_nt_noalloc: the dense FP8 GEMM for callers that cannot
allocate device memory at call time (a framework that owns all device memory,
a serving loop with memory fixed up front, a hot path where cudaMalloc /
cudaFree are not allowed because they can synchronise the device or fail).
Its stream-K partial sums live in the library's fixed device array instead of
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


@pytest.fixture
def shared_tiles(request, dg):
    # schedule 2 (per-tile K-slices) makes the small-M shapes keep their
    # partial sums in the scratch array; 0 is the heuristic's own plan
    dg.dg_set_tile_config(0, request.param)
    yield request.param
    dg.dg_set_tile_config(0, 0)


@pytest.mark.parametrize("shared_tiles", [0, 2], indirect=True)
@pytest.mark.parametrize("M,N,K", [(64, 7168, 16384), (128, 7168, 2048), (200, 512, 1024), (1100, 520, 512)])
def test_noalloc_matches_allocating_call_twice(dg, shared_tiles, M, N, K):
    p = Dense(8000 + M + N, M, N, K, with_c=True).upload()
    cfg = dg.dg_query_dense_config(M, N, K, workspace_cap=dg.dg_noalloc_scratch_bytes())
    if M == 64 and shared_tiles == 2:
        assert cfg["sk_tiles"] > 0          # this shape exercises the scratch array
    assert cfg["workspace_bytes"] <= dg.dg_noalloc_scratch_bytes()

    dg.dg_fp8_gemm_nt(p.t_a, p.t_sfa, p.t_b, p.t_sfb, p.t_c, p.t_d)
    torch.cuda.synchronize()
    want = bf16_dev_to_f64(p.t_d)

    for _ in range(2):                    # two calls in a row on the shared array
        d = torch.full((M, N), 0x7FC1, dtype=torch.int16, device="cuda")
        dg.dg_fp8_gemm_nt_noalloc(p.t_a, p.t_sfa, p.t_b, p.t_sfb, p.t_c, d)
        torch.cuda.synchronize()
        assert dg.dg_get_last_error() == 0
        check_close(bf16_dev_to_f64(d), want, f"noalloc {M}x{N}x{K}")
        check_close(bf16_dev_to_f64(d), p.ref(), f"noalloc {M}x{N}x{K} vs oracle")


def test_noalloc_keeps_within_its_scratch(dg):
    # Pretend to have 4096 SMs and force stream-K: sharing a 1024 x 8192 x
    # 16384 problem over them needs more workspace than the fixed array holds,
    # so the no-alloc plan must be a different one that fits.  Query only:
    # with 4096 pretend SMs nothing is launched.
    dg.dg_set_num_sms(4096)
    dg.dg_set_tile_config(0, 3)
    try:
        free = dg.dg_query_dense_config(1024, 8192, 16384)
        capped = dg.dg_query_dense_config(1024, 8192, 16384, workspace_cap=dg.dg_noalloc_scratch_bytes())
    finally:
        dg.dg_set_tile_config(0, 0)
        dg.dg_set_num_sms(0)
    assert free["workspace_bytes"] > dg.dg_noalloc_scratch_bytes()
    assert capped["workspace_bytes"] <= dg.dg_noalloc_scratch_bytes()


def test_noalloc_reserves_no_device_memory(dg):
    # The property the call exists for.  On a stream the library has not used
    # yet, the allocating call must create a new stream-K workspace (device
    # memory reserved), while the no-alloc call on another new stream must
    # leave the device's free memory unchanged.
    M, N, K = 64, 7168, 16384
    dg.dg_set_tile_config(0, 2)             # per-tile K-slices: partial sums in scratch
    try:
        _reserves_nothing(dg, M, N, K)
    finally:
        dg.dg_set_tile_config(0, 0)


def _pool_used_bytes():
    """Bytes in use from the device's default stream-ordered memory pool (the
    one the allocating call's workspace comes from), read through the driver
    API; None where the driver bindings are not importable."""
    try:
        from cuda.bindings import driver as cu
    except ImportError:
        return None
    err, dev = cu.cuDeviceGet(torch.cuda.current_device())
    assert err == cu.CUresult.CUDA_SUCCESS
    err, pool = cu.cuDeviceGetDefaultMemPool(dev)
    assert err == cu.CUresult.CUDA_SUCCESS
    err, used = cu.cuMemPoolGetAttribute(pool, cu.CUmemPool_attribute.CU_MEMPOOL_ATTR_USED_MEM_CURRENT)
    assert err == cu.CUresult.CUDA_SUCCESS
    return int(used)


def _reserves_nothing(dg, M, N, K):
    cfg = dg.dg_query_dense_config(M, N, K, workspace_cap=dg.dg_noalloc_scratch_bytes())
    assert cfg["sk_tiles"] > 0 and cfg["workspace_bytes"] > 0
    p = Dense(8100, M, N, K, with_c=True).upload()
    d = torch.empty((M, N), dtype=torch.int16, device="cuda")
    dg.dg_fp8_gemm_nt_noalloc(p.t_a, p.t_sfa, p.t_b, p.t_sfb, p.t_c, d)   # warm-up (module, address)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    s1 = torch.cuda.Stream()
    free0, _ = torch.cuda.mem_get_info()
    used0 = _pool_used_bytes()
    with torch.cuda.stream(s1):
        dg.dg_fp8_gemm_nt_noalloc(p.t_a, p.t_sfa, p.t_b, p.t_sfb, p.t_c, d, stream=s1)
    s1.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    used1 = _pool_used_bytes()
    assert free1 == free0, f"no-alloc call changed free device memory by {free0 - free1} bytes"
    assert used1 == used0, "no-alloc call took memory from the stream-ordered pool"
    check_close(bf16_dev_to_f64(d), p.ref(), "noalloc on a new stream")

    # control: on another new stream the allocating call takes a workspace
    # from the pool, so the measurement would have seen an allocation
    if used0 is not None:
        s2 = torch.cuda.Stream()
        with torch.cuda.stream(s2):
            dg.dg_fp8_gemm_nt(p.t_a, p.t_sfa, p.t_b, p.t_sfb, p.t_c, d, stream=s2)
        s2.synchronize()
        assert _pool_used_bytes() > used1, "control: no workspace was allocated"
