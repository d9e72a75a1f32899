"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Floating-point outputs are checked under the method's
tolerances (tests/gpu_util.py); integer, byte and index work bit-exactly."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import (Dense, bf16_dev_to_f64, check_close, dev, host, quantize_groups_b)

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
    # every test leaves the device error word clear (tests that provoke an
    # error read and clear it themselves), so a kernel self-check that fires
    # is reported by the test that triggered it
    yield
    assert dg.dg_get_last_error() == 0, "device error recorded during this test"


# ------------------------------------------------------------------ prep

@pytest.mark.parametrize("rows,cols", [(1, 128), (300, 512)])
def test_quantize_fp8_rowwise_bit_exact(dg, rows, cols):
    x = synth.normal_f32(1000 + rows, (rows, cols)) * np.float32(5.0)
    x[0, :128] = 0.0
    if rows > 2:
        x[1, 128:256] = np.float32(3e-39)      # subnormal block
        x[2, :] *= np.float32(1e20)
    q, e = oracle.quantize_fp8(x, 1)
    tq = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    te = torch.empty((rows, cols // 128), dtype=torch.uint8, device="cuda")
    dg.dg_quantize_fp8(dev(x), tq, te, 1)
    torch.cuda.synchronize()
    assert np.array_equal(host(te), e)
    assert np.array_equal(host(tq), q)


def test_quantize_fp8_blockwise_bit_exact(dg):
    rows, cols = 300, 384
    x = synth.normal_f32(1100, (rows, cols))
    q, e = oracle.quantize_fp8(x, 128)
    tq = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    te = torch.empty(e.shape, dtype=torch.uint8, device="cuda")
    dg.dg_quantize_fp8(dev(x), tq, te, 128)
    torch.cuda.synchronize()
    assert np.array_equal(host(te), e)
    assert np.array_equal(host(tq), q)


def test_quantize_fp4_bit_exact(dg):
    rows, cols = 70, 256
    x = synth.normal_f32(1200, (rows, cols))
    x[3, :32] = 0.0
    q, e = oracle.quantize_fp4(x, 32)
    tq = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
    te = torch.empty((rows, cols // 32), dtype=torch.uint8, device="cuda")
    dg.dg_quantize_fp4(dev(x), tq, te)
    torch.cuda.synchronize()
    assert np.array_equal(host(te), e)
    assert np.array_equal(host(tq), q)


@pytest.mark.parametrize("rows,ng,row_div", [(300, 7, 1), (128, 4, 1), (2112, 56, 128), (1, 1, 1)])
def test_pack_sf_bit_exact(dg, rows, ng, row_div):
    e = synth.junk_bytes(1300 + rows, ((rows + row_div - 1) // row_div, ng))
    want = oracle.pack_sf(e, rows, row_div=row_div)
    out = torch.full((dg.dg_packed_sf_words(rows, ng),), -1, dtype=torch.int32, device="cuda")
    dg.dg_pack_sf(dev(e), rows, out, row_div=row_div)
    torch.cuda.synchronize()
    assert np.array_equal(host(out), want.ravel())


# ------------------------------------------------------------------ dense

@pytest.mark.parametrize("M,N,K,with_c", [
    (128, 512, 1024, False),    # the small worked configuration (C = 0)
    (200, 328, 384, True),      # ragged M and N tails, K of three blocks
    (1100, 520, 512, True),     # several m-blocks, no split-K, ragged tails
    (64, 2112, 7168, True),     # stream-K over all SMs (17 tiles)
    (3, 64, 256, True),         # tiny M
    (1, 136, 512, True),        # a single row (one partial 32-row store box)
    (5, 8, 128, True),          # the smallest N and K: one tile, one K-block, 8 of its columns
    (130, 8, 128, False),       # two m-blocks of an 8-column D, full 32-row boxes clipped to 8 columns
])
def test_dense_matches_oracle(dg, M, N, K, with_c):
    p = Dense(2000 + M + N, M, N, K, with_c=with_c).upload()
    d = p.run(dg)
    stats = check_close(d, p.ref(), f"dense {M}x{N}x{K}")
    assert stats["n"] == M * N


@pytest.mark.parametrize("schedule", [2, 3])
@pytest.mark.parametrize("sms", [0, 7])
@pytest.mark.parametrize("bn", [64, 128, 160, 192, 224, 256])
@pytest.mark.parametrize("M,N,K,with_c,fp4", [
    (1100, 520, 512, True, False),     # ragged M and N tails, 4 K-blocks
    (300, 1000, 1536, True, False),    # pieces that start and end inside tiles
    (128, 512, 128, False, False),     # one K-block: every piece is a whole tile
    (200, 904, 1024, True, True),      # FP8 x FP4
])
def test_dense_shared_tail_matches_oracle(dg, schedule, sms, bn, M, N, K, with_c, fp4):
    # Forced per-tile K-slices (2) or stream-K (3).  With 7 "SMs" the small
    # problems run waves of whole tiles before the shared K-blocks of the last
    # tiles, as large problems do on 148 SMs.
    dg.dg_set_num_sms(sms)
    dg.dg_set_tile_config(bn, schedule)
    try:
        cfg = dg.dg_query_dense_config(M, N, K)
        assert cfg["block_n"] == bn
        if cfg["sk_tiles"] == 0:
            pytest.skip(f"no split of this kind: {cfg}")
        assert (cfg["sk_split"] > 0) == (schedule == 2)
        p = Dense(2400 + M + bn + sms, M, N, K, with_c=with_c, fp4=fp4).upload()
        check_close(p.run(dg), p.ref(), f"schedule {schedule} bn={bn} sms={sms} {M}x{N}x{K} {cfg}")
        assert dg.dg_get_last_error() == 0
    finally:
        dg.dg_set_tile_config(0, 0)
        dg.dg_set_num_sms(0)


def test_dense_shared_tail_is_deterministic_and_agrees_with_whole_tiles(dg):
    M, N, K = 1100, 2112, 2048
    p = Dense(2500, M, N, K, with_c=True).upload()
    outs = {}
    dg.dg_set_num_sms(30)          # 153 tiles: 5 waves + 3 shared tiles
    try:
        for sched in (1, 2, 2, 3, 3):
            dg.dg_set_tile_config(128, sched)
            assert (dg.dg_query_dense_config(M, N, K)["sk_tiles"] > 0) == (sched > 1)
            outs.setdefault(sched, []).append(p.run(dg))
    finally:
        dg.dg_set_tile_config(0, 0)
        dg.dg_set_num_sms(0)
    for sched in (2, 3):
        assert np.array_equal(outs[sched][0], outs[sched][1])   # slots summed in K order
        check_close(outs[sched][0], outs[1][0], f"schedule {sched} vs whole tiles")
        check_close(outs[sched][0], p.ref(), f"schedule {sched} vs oracle")


@pytest.mark.parametrize("schedule,S", [(4, 2), (5, 3), (6, 4), (7, 5), (10, 8)])
@pytest.mark.parametrize("bn", [128, 256])
@pytest.mark.parametrize("M,N,K,with_c,fp4", [
    (64, 2112, 7168, True, False),     # small M: the shape these plans are for
    (200, 328, 1024, True, False),     # two m-blocks, ragged M and N tails
    (1, 136, 2048, False, False),      # a single row, no C
    (128, 904, 1024, True, True),      # FP8 x FP4
])
def test_dense_cluster_split_matches_oracle(dg, schedule, S, bn, M, N, K, with_c, fp4):
    # every tile's K-blocks cut into S slices on a cluster of S CTAs, summed
    # through distributed shared memory in slice order
    dg.dg_set_tile_config(bn, schedule)
    try:
        if dg.dg_query_dense_cluster_split(M, N, K) != S:
            pytest.skip(f"no {S}-way split for this shape")
        cfg = dg.dg_query_dense_config(M, N, K)
        assert cfg["block_n"] == bn and cfg["sk_tiles"] == 0 and cfg["workspace_bytes"] == 0
        p = Dense(2650 + M + bn + S, M, N, K, with_c=with_c, fp4=fp4).upload()
        d1 = p.run(dg)
        d2 = p.run(dg)
    finally:
        dg.dg_set_tile_config(0, 0)
    assert np.array_equal(d1, d2)          # fixed summation order
    check_close(d1, p.ref(), f"split S={S} bn={bn} {M}x{N}x{K} fp4={fp4}")


@pytest.mark.parametrize("bn", [64, 160, 224])
@pytest.mark.parametrize("M,N,K,fp4", [(300, 1000, 1024, False), (1100, 2112, 512, False), (200, 904, 512, True)])
def test_dense_forced_widths(dg, bn, M, N, K, fp4):
    # widths the heuristic does not pick by default: 64 (narrow tiles for small
    # M), and 160 / 224, which start tiles 32 or 96 rows into a 128-row scale
    # chunk so the B scale words are re-based in shared memory first
    dg.dg_set_tile_config(bn, 1)
    try:
        assert dg.dg_query_dense_config(M, N, K)["block_n"] == bn
        p = Dense(2600 + M + bn, M, N, K, with_c=True, fp4=fp4).upload()
        check_close(p.run(dg), p.ref(), f"bn={bn} {M}x{N}x{K} fp4={fp4}")
    finally:
        dg.dg_set_tile_config(0, 0)


@pytest.mark.parametrize("bn", [64, 160, 224])
def test_grouped_forced_widths(dg, bn):
    dg.dg_set_tile_config(bn, 1)
    try:
        N, K = 1000, 512
        cs = _contiguous_case(2700 + bn, 3, 60, 200, N, K)
        d = _run_contiguous(dg, cs, N)
        ref = oracle.gemm_contiguous(cs["qa"], cs["ea"], cs["qb"], cs["eb"], cs["mi"], c=cs["c"])
        valid = cs["mi"] >= 0
        check_close(d[valid], ref[valid], f"contiguous bn={bn}")
        G, max_m = 3, 256
        mm = np.array([5, 256, 130], np.int32)
        qa, ea, sfa, qb, eb, sfb = _masked_case(2800 + bn, G, max_m, N, K, mm)
        dm = _run_masked(dg, G, max_m, N, qa, sfa, qb, sfb, mm)
        refm = oracle.gemm_masked(qa, ea, qb, eb, mm)
        ddm = bf16_dev_to_f64(dm)
        for g in range(G):
            check_close(ddm[g, :mm[g]], refm[g, :mm[g]], f"masked bn={bn} g={g}")
            assert np.all(host(dm).view(np.uint16)[g, mm[g]:] == SENTINEL)
    finally:
        dg.dg_set_tile_config(0, 0)


@pytest.mark.parametrize("bn", [64, 160, 224])
def test_grouped_fp4_forced_widths(dg, bn):
    # FP8 x FP4 grouped calls at widths that start tiles 32 or 96 rows into a
    # 128-row scale chunk: the B scale words change every K-block, so the
    # re-base hands every stage over (160 / 224), in both grouped layouts
    dg.dg_set_tile_config(bn, 1)
    try:
        N, K = 1000, 512
        cs = _contiguous_case(2900 + bn, 3, 60, 200, N, K, fp4=True)
        d = _run_contiguous(dg, cs, N, fp4=True)
        ref = oracle.gemm_contiguous(cs["qa"], cs["ea"], cs["qb"], cs["eb"], cs["mi"], c=cs["c"], b_fp4=True)
        valid = cs["mi"] >= 0
        check_close(d[valid], ref[valid], f"contiguous fp4 bn={bn}")
        G, max_m = 3, 256
        mm = np.array([5, 256, 130], np.int32)
        qa, ea, sfa, qb, eb, sfb = _masked_fp4_case(3000 + bn, G, max_m, N, K, mm)
        dm = torch.full((G, max_m, N), SENTINEL, dtype=torch.int16, device="cuda")
        dg.dg_m_grouped_fp8_fp4_gemm_nt_masked(dev(qa), dev(sfa), dev(qb), dev(sfb), dm, dev(mm), expected_m=128)
        torch.cuda.synchronize()
        refm = oracle.gemm_masked(qa, ea, qb, eb, mm, b_fp4=True)
        ddm = bf16_dev_to_f64(dm)
        for g in range(G):
            check_close(ddm[g, :mm[g]], refm[g, :mm[g]], f"masked fp4 bn={bn} g={g}")
            assert np.all(host(dm).view(np.uint16)[g, mm[g]:] == SENTINEL)
        assert dg.dg_get_last_error() == 0
    finally:
        dg.dg_set_tile_config(0, 0)


def test_dense_long_k_accumulation(dg):
    # K = 16384: 128 scaled K-blocks accumulated in FP32 inside TMEM
    p = Dense(2100, 128, 256, 16384, with_c=False).upload()
    check_close(p.run(dg), p.ref(), "dense K=16384")


def test_dense_in_place_c_equals_d(dg):
    p = Dense(2200, 256, 256, 512, with_c=True).upload()
    p.t_d.copy_(p.t_c)
    dg.dg_fp8_gemm_nt(p.t_a, p.t_sfa, p.t_b, p.t_sfb, p.t_d, p.t_d)
    torch.cuda.synchronize()
    check_close(bf16_dev_to_f64(p.t_d), p.ref(), "dense in-place")


@pytest.mark.parametrize("M", [128, 2048])
def test_dense_scale_doubling_is_bit_exact(dg, M):
    # C = 0 and a single non-zero K-block: raising that block's A scale by
    # one must double every output exactly (scaling by 2 commutes with the
    # bf16 rounding away from overflow and underflow).
    N, K = 256, 512
    p = Dense(2300 + M, M, N, K, with_c=False)
    p.qa[:, :128] = 0
    p.qa[:, 256:] = 0
    p.sfa = oracle.pack_sf(p.ea, M)
    p.upload()
    d1 = p.run(dg)
    ea2 = p.ea.copy()
    ea2[:, 1] += 1
    p.t_sfa = dev(oracle.pack_sf(ea2, M))
    d2 = p.run(dg)
    assert np.array_equal(d2, 2.0 * d1)
    assert np.count_nonzero(d1) > 0.9 * d1.size


def test_dense_full_size_sampled(dg):
    # every dense shape of the DeepSeek-V3 projection sweep, sampled outputs
    for (N, K) in synth.DENSE_NK:
        xb = synth.normal_f32(3000 + N + K, (N, K))
        for M in synth.DENSE_M:
            print(f"dense full size {M}x{N}x{K}: {dg.dg_query_dense_config(M, N, K)}", flush=True)
            p = Dense(3100 + M + N + K, M, N, K, with_c=True, xb=xb).upload()
            d = p.run(dg)
            pm, pn = synth.sample_points(3200 + M, np.arange(M), N, 2048)
            check_close(d[pm, pn], p.ref_points(pm, pn), f"dense {M}x{N}x{K}")
            del p
            torch.cuda.empty_cache()


# ------------------------------------------------------------------ bf16

def _bf16_case(seed, M, N, K, with_c):
    import ml_dtypes
    a = synth.normal_f32(seed, (M, K)).astype(ml_dtypes.bfloat16).view(np.uint16)
    b = synth.normal_f32(seed + 1, (N, K)).astype(ml_dtypes.bfloat16).view(np.uint16)
    c = synth.normal_bf16_bits(seed + 2, (M, N)) if with_c else None
    return a, b, c


def _run_bf16(dg, a, b, c):
    M, N = a.shape[0], b.shape[0]
    d = torch.full((M, N), SENTINEL, dtype=torch.int16, device="cuda")
    dg.dg_bf16_gemm_nt(dev(a.view(np.int16)), dev(b.view(np.int16)),
                       dev(c.view(np.int16)) if c is not None else None, d)
    torch.cuda.synchronize()
    return bf16_dev_to_f64(d)


@pytest.mark.parametrize("M,N,K,with_c", [
    (128, 512, 1024, False), (200, 328, 192, True), (1100, 520, 512, True), (64, 2112, 7168, True),
    (3, 64, 64, True)])
def test_bf16_dense_matches_oracle(dg, M, N, K, with_c):
    a, b, c = _bf16_case(6000 + M + N, M, N, K, with_c)
    check_close(_run_bf16(dg, a, b, c), oracle.gemm_bf16(a, b, c), f"bf16 {M}x{N}x{K}")


@pytest.mark.parametrize("bn,schedule", [(64, 1), (128, 1), (192, 1), (256, 1), (128, 2), (256, 3)])
def test_bf16_widths_and_shared_tails(dg, bn, schedule):
    M, N, K = 1100, 1000, 1024
    a, b, c = _bf16_case(6100 + bn + schedule, M, N, K, True)
    dg.dg_set_num_sms(7 if schedule > 1 else 0)
    dg.dg_set_tile_config(bn, schedule)
    try:
        got = _run_bf16(dg, a, b, c)
    finally:
        dg.dg_set_tile_config(0, 0)
        dg.dg_set_num_sms(0)
    check_close(got, oracle.gemm_bf16(a, b, c), f"bf16 bn={bn} schedule={schedule}")


def test_bf16_rejects_k_not_multiple_of_64(dg):
    z = torch.zeros(1024, dtype=torch.int16, device="cuda")
    assert dg.lib().dg_bf16_gemm_nt(_p_(z), _p_(z), None, _p_(z), 8, 8, 96, None) == -1


# ------------------------------------------------------------------ contiguous

def _contiguous_case(seed, G, lo, hi, N, K, fp4=False, with_c=True):
    rows, mi = synth.contiguous_layout(seed, G, lo, hi)
    M = mi.size
    xa = synth.normal_f32(seed + 1, (M, K))
    qa, ea = oracle.quantize_fp8(xa, 1)
    pad = mi < 0
    qa[pad] = synth.junk_bytes(seed + 2, (int(pad.sum()), K))   # junk incl. NaN codes
    qa[pad, ::7] = 0x7F
    ea[pad] = synth.junk_bytes(seed + 3, (int(pad.sum()), K // 128))
    qb, eb, sfb = quantize_groups_b(seed + 10, G, N, K, fp4=fp4)
    c = synth.normal_bf16_bits(seed + 4, (M, N)) if with_c else None
    return dict(rows=rows, mi=mi, M=M, qa=qa, ea=ea, sfa=oracle.pack_sf(ea, M), qb=qb, eb=eb, sfb=sfb, c=c)


def _run_contiguous(dg, cs, N, fp4=False):
    d = torch.empty((cs["M"], N), dtype=torch.int16, device="cuda")
    fn = dg.dg_m_grouped_fp8_fp4_gemm_nt_contiguous if fp4 else dg.dg_m_grouped_fp8_gemm_nt_contiguous
    c = dev(cs["c"].view(np.int16)) if cs["c"] is not None else None
    fn(dev(cs["qa"]), dev(cs["sfa"]), dev(cs["qb"]), dev(cs["sfb"]), c, d, dev(cs["mi"]))
    torch.cuda.synchronize()
    return bf16_dev_to_f64(d)


@pytest.mark.parametrize("fp4", [False, True])
def test_contiguous_matches_oracle(dg, fp4):
    N, K = 384, 512
    cs = _contiguous_case(4000 + fp4, 4, 50, 300, N, K, fp4=fp4)
    d = _run_contiguous(dg, cs, N, fp4=fp4)
    ref = oracle.gemm_contiguous(cs["qa"], cs["ea"], cs["qb"], cs["eb"], cs["mi"], c=cs["c"], b_fp4=fp4)
    valid = cs["mi"] >= 0
    check_close(d[valid], ref[valid], "contiguous")
    # and each group equals the dense call on its own rows
    for g in range(4):
        sel = np.nonzero(cs["mi"] == g)[0]
        assert sel.size == cs["rows"][g]


@pytest.mark.parametrize("N,K", synth.GROUPED_NK)
def test_contiguous_full_size_sampled(dg, N, K):
    cs = _contiguous_case(4100 + N, 8, 6000, 10000, N, K)
    d = _run_contiguous(dg, cs, N)
    valid_rows = np.nonzero(cs["mi"] >= 0)[0]
    pm, pn = synth.sample_points(4200 + N, valid_rows, N, 4096)
    ref = np.empty(pm.size)
    for g in range(8):
        sel = cs["mi"][pm] == g
        ref[sel] = oracle.gemm_points(cs["qa"], cs["ea"], cs["qb"][g], cs["eb"][g], pm[sel], pn[sel], c=cs["c"])
    check_close(d[pm, pn], ref, f"contiguous {N}x{K}")


# ------------------------------------------------------------------ masked

SENTINEL = 0x7FC1  # a bf16 NaN pattern no GEMM result can produce


_B_CACHE = {}


def _grouped_b(seed, G, N, K):
    key = (seed, G, N, K)
    if key not in _B_CACHE:
        _B_CACHE.clear()
        _B_CACHE[key] = quantize_groups_b(seed, G, N, K)
    return _B_CACHE[key]


def _masked_case(seed, G, max_m, N, K, masked_m, b_seed=None):
    xa = synth.normal_f32(seed, (G * max_m, K))
    qa, ea = oracle.quantize_fp8(xa, 1)
    qa = qa.reshape(G, max_m, K)
    ea = ea.reshape(G, max_m, K // 128)
    for g in range(G):                           # junk beyond the valid rows
        v = min(int(masked_m[g]), max_m)
        qa[g, v:] = synth.junk_bytes(seed + 100 + g, (max_m - v, K))
    sfa = np.concatenate([oracle.pack_sf(ea[g], max_m).ravel() for g in range(G)])
    qb, eb, sfb = _grouped_b(seed + 1000 if b_seed is None else b_seed, G, N, K)
    return qa, ea, sfa, qb, eb, sfb


def _run_masked(dg, G, max_m, N, qa, sfa, qb, sfb, masked_m, expected_m=0):
    d = torch.full((G, max_m, N), SENTINEL, dtype=torch.int16, device="cuda")
    dg.dg_m_grouped_fp8_gemm_nt_masked(dev(qa), dev(sfa), dev(qb), dev(sfb), d, dev(masked_m.astype(np.int32)),
                                       expected_m=expected_m)
    torch.cuda.synchronize()
    return d


def test_masked_matches_oracle_and_leaves_rows(dg):
    G, max_m, N, K = 6, 256, 384, 512
    mm = np.array([0, 1, 127, 128, 200, 256], np.int32)
    qa, ea, sfa, qb, eb, sfb = _masked_case(5000, G, max_m, N, K, mm)
    d = _run_masked(dg, G, max_m, N, qa, sfa, qb, sfb, mm)
    bits = host(d).view(np.uint16)
    ref = oracle.gemm_masked(qa, ea, qb, eb, mm)
    dd = bf16_dev_to_f64(d)
    for g in range(G):
        v = int(mm[g])
        assert np.all(bits[g, v:] == SENTINEL), f"group {g}: rows >= masked_m were written"
        if v:
            check_close(dd[g, :v], ref[g, :v], f"masked group {g}")


def _masked_fp4_case(seed, G, max_m, N, K, masked_m):
    qa, ea, sfa, _, _, _ = _masked_case(seed, G, max_m, N, K, masked_m)
    qb, eb, sfb = quantize_groups_b(seed + 2000, G, N, K, fp4=True)
    return qa, ea, sfa, qb, eb, sfb


def test_contiguous_all_padding_rows(dg):
    # every row is padding (m_indices = -1): nothing to compute, no error,
    # and D untouched
    M, N, K, G = 256, 256, 256, 2
    cs = _contiguous_case(6200, G, 60, 200, N, K)
    mi = np.full(M, -1, np.int32)
    d = torch.full((M, N), SENTINEL, dtype=torch.int16, device="cuda")
    assert cs["M"] >= M
    qa = np.ascontiguousarray(cs["qa"][:M])
    sfa = oracle.pack_sf(np.full((M, K // 128), 127, np.uint8), M)
    dg.dg_m_grouped_fp8_gemm_nt_contiguous(dev(qa), dev(sfa), dev(cs["qb"]), dev(cs["sfb"]), None, d, dev(mi))
    torch.cuda.synchronize()
    assert dg.dg_get_last_error() == 0
    assert np.all(host(d).view(np.uint16) == SENTINEL)


def test_masked_at_the_group_limit(dg):
    # 1024 groups (the most the device-side prefix holds), counts from 0 to
    # max_m: valid rows against the oracle, every other row bit-exact
    G, max_m, N, K = 1024, 16, 256, 256
    mm = synth.rng(6100).integers(0, max_m + 1, size=G).astype(np.int32)
    mm[:4] = [0, max_m, 1, 0]
    qa, ea, sfa, qb, eb, sfb = _masked_case(6100, G, max_m, N, K, mm)
    d = _run_masked(dg, G, max_m, N, qa, sfa, qb, sfb, mm, expected_m=8)
    ref = oracle.gemm_masked(qa, ea, qb, eb, mm)
    got = bf16_dev_to_f64(d)
    sent = host(d).view(np.uint16)
    for g in range(G):
        if mm[g] > 0:
            check_close(got[g, :mm[g]], ref[g, :mm[g]], f"masked G=1024 g={g}")
        assert np.all(sent[g, mm[g]:] == SENTINEL)
    assert dg.dg_get_last_error() == 0


def test_masked_fp4_matches_oracle(dg):
    G, max_m, N, K = 3, 256, 384, 512
    mm = np.array([5, 256, 130], np.int32)
    qa, ea, sfa, qb, eb, sfb = _masked_fp4_case(5700, G, max_m, N, K, mm)
    d = torch.full((G, max_m, N), SENTINEL, dtype=torch.int16, device="cuda")
    dg.dg_m_grouped_fp8_fp4_gemm_nt_masked(dev(qa), dev(sfa), dev(qb), dev(sfb), d, dev(mm), expected_m=128)
    torch.cuda.synchronize()
    ref = oracle.gemm_masked(qa, ea, qb, eb, mm, b_fp4=True)
    got = bf16_dev_to_f64(d)
    for g in range(G):
        check_close(got[g, :mm[g]], ref[g, :mm[g]], f"masked fp4 g={g}")
        assert np.all(host(d).view(np.uint16)[g, mm[g]:] == SENTINEL)


@pytest.mark.parametrize("bn", [0, 128, 256])
@pytest.mark.parametrize("fp4", [False, True])
def test_masked_swiglu_matches_oracle(dg, fp4, bn):
    # linear1 with SwiGLU in the epilogue: B rows are gate/up blocks of 64,
    # D has half the GEMM's columns
    G, max_m, N, K = 3, 256, 512, 512
    mm = np.array([0, 200, 256], np.int32)
    if fp4:
        qa, ea, sfa, qb, eb, sfb = _masked_fp4_case(5800, G, max_m, N, K, mm)
        fn = dg.dg_m_grouped_fp8_fp4_gemm_nt_masked_swiglu
    else:
        qa, ea, sfa, qb, eb, sfb = _masked_case(5800, G, max_m, N, K, mm)
        fn = dg.dg_m_grouped_fp8_gemm_nt_masked_swiglu
    d = torch.full((G, max_m, N // 2), SENTINEL, dtype=torch.int16, device="cuda")
    dg.dg_set_tile_config(bn, 0)
    try:
        fn(dev(qa), dev(sfa), dev(qb), dev(sfb), d, dev(mm), expected_m=128)
        torch.cuda.synchronize()
    finally:
        dg.dg_set_tile_config(0, 0)
    ref = oracle.swiglu_interleaved(oracle.gemm_masked(qa, ea, qb, eb, mm, b_fp4=fp4))
    got = bf16_dev_to_f64(d)
    for g in range(G):
        if mm[g]:
            check_close(got[g, :mm[g]], ref[g, :mm[g]], f"swiglu fp4={fp4} bn={bn} g={g}")
        assert np.all(host(d).view(np.uint16)[g, mm[g]:] == SENTINEL)


def test_masked_swiglu_rejects_bad_widths(dg):
    z = torch.zeros(16, dtype=torch.int32, device="cuda")
    # n not a multiple of 128 (whole gate/up block pairs)
    st = dg.lib().dg_m_grouped_fp8_gemm_nt_masked_swiglu(_p_(z), _p_(z), _p_(z), _p_(z), _p_(z), _p_(z), 1, 128,
                                                         192, 128, 0, None)
    assert st == -1
    # a forced tile width that cannot hold whole block pairs
    dg.dg_set_tile_config(192, 0)
    try:
        st = dg.lib().dg_m_grouped_fp8_gemm_nt_masked_swiglu(_p_(z), _p_(z), _p_(z), _p_(z), _p_(z), _p_(z), 1,
                                                             128, 256, 128, 0, None)
    finally:
        dg.dg_set_tile_config(0, 0)
    assert st == -2


def _p_(t):
    import ctypes
    return ctypes.c_void_p(t.data_ptr())


def test_masked_decode_replays_from_a_cuda_graph(dg):
    # The masked call reads masked_m on the device and allocates nothing, so
    # one captured launch serves every step of a decode loop: the counts are
    # rewritten in place between replays.
    G, max_m, N, K = 4, 128, 256, 512
    qa, ea, sfa, qb, eb, sfb = _masked_case(5600, G, max_m, N, K, np.full(G, max_m, np.int32))
    t_a, t_sfa, t_b, t_sfb = dev(qa), dev(sfa), dev(qb), dev(sfb)
    t_mm = torch.zeros(G, dtype=torch.int32, device="cuda")
    d = torch.full((G, max_m, N), SENTINEL, dtype=torch.int16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):            # first call outside the capture (kernel attributes)
        dg.dg_m_grouped_fp8_gemm_nt_masked(t_a, t_sfa, t_b, t_sfb, d, t_mm, expected_m=32)
    s.synchronize()
    graph = torch.cuda.CUDAGraph()
    launches = dg.dg_launch_count()
    with torch.cuda.graph(graph, stream=s):
        dg.dg_m_grouped_fp8_gemm_nt_masked(t_a, t_sfa, t_b, t_sfb, d, t_mm, expected_m=32)
    assert dg.dg_launch_count() == launches + 1
    for counts in ([0, 5, 128, 77], [128, 0, 1, 64], [33, 33, 33, 33]):
        mm = np.array(counts, np.int32)
        d.fill_(SENTINEL)
        t_mm.copy_(torch.from_numpy(mm))
        graph.replay()
        torch.cuda.synchronize()
        assert dg.dg_get_last_error() == 0
        ref = oracle.gemm_masked(qa, ea, qb, eb, mm)
        got = bf16_dev_to_f64(d)
        raw = host(d).view(np.uint16)
        for g in range(G):
            if mm[g] > 0:
                check_close(got[g, :mm[g]], ref[g, :mm[g]], f"graph replay {counts} g={g}")
            assert np.all(raw[g, mm[g]:] == SENTINEL), f"graph replay {counts}: rows >= masked_m written"
    del graph


def test_masked_count_above_max_is_clamped_and_reported(dg):
    G, max_m, N, K = 2, 128, 128, 256
    mm = np.array([300, 5], np.int32)
    qa, ea, sfa, qb, eb, sfb = _masked_case(5100, G, max_m, N, K, np.minimum(mm, max_m))
    d = _run_masked(dg, G, max_m, N, qa, sfa, qb, sfb, mm)
    assert dg.dg_get_last_error() == -5
    ref = oracle.gemm_masked(qa, ea, qb, eb, mm)
    dd = bf16_dev_to_f64(d)
    check_close(dd[0], ref[0], "masked clamped group")
    assert np.all(host(d).view(np.uint16)[1, 5:] == SENTINEL)


@pytest.mark.parametrize("N,K", synth.GROUPED_NK)
@pytest.mark.parametrize("expected_m", [16, 64, 128])
def test_masked_full_size_sampled(dg, expected_m, N, K):
    G, max_m = 32, 256
    mm = synth.masked_counts(5200 + expected_m, G, expected_m, max_m)
    qa, ea, sfa, qb, eb, sfb = _masked_case(5300 + expected_m + N, G, max_m, N, K, mm, b_seed=5500 + N)
    d = _run_masked(dg, G, max_m, N, qa, sfa, qb, sfb, mm, expected_m=expected_m)
    rows_valid = torch.arange(max_m, device="cuda")[None, :] < dev(mm)[:, None]
    untouched = (d == SENTINEL).all(dim=2)
    assert bool(untouched[~rows_valid].all()), "rows >= masked_m were written"
    dd = bf16_dev_to_f64(d)
    valid = [(g, m) for g in range(G) for m in range(int(mm[g]))]
    rng = synth.rng(5400 + expected_m)
    pick = rng.choice(len(valid), size=min(2048, len(valid)), replace=False)
    pn = rng.integers(0, N, size=pick.size)
    ref = np.empty(pick.size)
    got = np.empty(pick.size)
    for i, (j, n) in enumerate(zip(pick, pn)):
        g, m = valid[j]
        got[i] = dd[g, m, n]
    for g in range(G):
        sel = np.array([valid[j][0] == g for j in pick])
        if sel.any():
            ms = np.array([valid[j][1] for j in pick[sel]])
            ref[sel] = oracle.gemm_points(qa[g], ea[g], qb[g], eb[g], ms, pn[sel])
    check_close(got, ref, f"masked {N}x{K} em={expected_m}")


# ------------------------------------------------------------------ FP8 x FP4

@pytest.mark.parametrize("M,N,K", [(256, 384, 512), (200, 136, 256), (64, 2112, 2048)])
def test_fp8_fp4_dense_matches_oracle(dg, M, N, K):
    p = Dense(6000 + M + N, M, N, K, with_c=True, fp4=True).upload()
    check_close(p.run(dg), p.ref(), f"fp8xfp4 {M}x{N}x{K}")


@pytest.mark.parametrize("N,K", synth.GROUPED_NK)
def test_fp8_fp4_full_size_sampled(dg, N, K):
    p = Dense(6100 + N, 4096, N, K, with_c=True, fp4=True).upload()
    d = p.run(dg)
    pm, pn = synth.sample_points(6200 + N, np.arange(4096), N, 2048)
    check_close(d[pm, pn], p.ref_points(pm, pn), f"fp8xfp4 4096x{N}x{K}")


@pytest.mark.parametrize("N,K", synth.GROUPED_NK)
def test_fp8_fp4_contiguous_full_size_sampled(dg, N, K):
    # the FP8 x FP4 MoE prefill at full size: 8 experts of U[6000, 10000]
    # tokens each padded to 128 (padding rows of A full of junk and NaN
    # codes), e2m1 weights with 1x32 scales, in the plan the bench times
    cs = _contiguous_case(6300 + N, 8, 6000, 10000, N, K, fp4=True)
    cfg = dg.dg_query_config("contiguous", cs["M"], N, K, groups=8, fp4=True)
    print(f"fp8xfp4 contiguous {cs['M']}x{N}x{K}: {cfg}", flush=True)
    assert cfg["grid"] == dg.dg_get_num_sms() and cfg["units"] > 4 * cfg["grid"]
    d = _run_contiguous(dg, cs, N, fp4=True)
    valid_rows = np.nonzero(cs["mi"] >= 0)[0]
    pm, pn = synth.sample_points(6400 + N, valid_rows, N, 4096)
    ref = np.empty(pm.size)
    for g in range(8):
        sel = cs["mi"][pm] == g
        assert sel.any()
        ref[sel] = oracle.gemm_points(cs["qa"], cs["ea"], cs["qb"][g], cs["eb"][g], pm[sel], pn[sel], c=cs["c"],
                                      b_fp4=True)
    check_close(d[pm, pn], ref, f"fp8xfp4 contiguous {N}x{K}")
    # the rows after the padding rows of every group are that group's
    pad_end = np.nonzero(np.diff((cs["mi"] < 0).astype(np.int8)) == -1)[0] + 1
    edge = pad_end[pad_end < cs["M"]]
    for m in edge[:4]:
        g = int(cs["mi"][m])
        pn_e = np.arange(0, N, 97)
        check_close(d[m, pn_e], oracle.gemm_points(cs["qa"], cs["ea"], cs["qb"][g], cs["eb"][g], np.full(pn_e.size, m),
                                                    pn_e, c=cs["c"], b_fp4=True), f"first row of group {g}")


_FP4_B_CACHE = {}


def _fp4_grouped_b(seed, G, N, K):
    key = (seed, G, N, K)
    if key not in _FP4_B_CACHE:
        _FP4_B_CACHE.clear()
        _FP4_B_CACHE[key] = quantize_groups_b(seed, G, N, K, fp4=True)
    return _FP4_B_CACHE[key]


@pytest.mark.parametrize("swiglu", [False, True])
def test_masked_fp4_full_size_sampled(dg, swiglu):
    # the FP8 x FP4 MoE decode at full size: 32 experts, max_m = 256,
    # masked_m ~ U[0, 2 x 128], linear1 shape (N, K) = (4096, 7168), plain or
    # with SwiGLU fused (gate / up rows interleaved in blocks of 64, D has
    # N / 2 columns); rows >= masked_m must stay untouched bit for bit
    G, max_m, N, K, em = 32, 256, 4096, 7168, 128
    mm = synth.masked_counts(5900, G, em, max_m)
    xa = synth.normal_f32(5901, (G * max_m, K))
    qa, ea = oracle.quantize_fp8(xa, 1)
    del xa
    qa = qa.reshape(G, max_m, K)
    ea = ea.reshape(G, max_m, K // 128)
    for g in range(G):
        v = int(mm[g])
        qa[g, v:] = synth.junk_bytes(5902 + g, (max_m - v, K))
    sfa = np.concatenate([oracle.pack_sf(ea[g], max_m).ravel() for g in range(G)])
    qb, eb, sfb = _fp4_grouped_b(5950, G, N, K)
    cols = N // 2 if swiglu else N
    cfg = dg.dg_query_config("masked", max_m, N, K, groups=G, fp4=True, expected_m=em, swiglu=swiglu)
    print(f"fp8xfp4 masked swiglu={swiglu}: {cfg}", flush=True)
    assert cfg["grid"] == dg.dg_get_num_sms()
    d = torch.full((G, max_m, cols), SENTINEL, dtype=torch.int16, device="cuda")
    fn = dg.dg_m_grouped_fp8_fp4_gemm_nt_masked_swiglu if swiglu else dg.dg_m_grouped_fp8_fp4_gemm_nt_masked
    fn(dev(qa), dev(sfa), dev(qb), dev(sfb), d, dev(mm), expected_m=em)
    torch.cuda.synchronize()
    rows_valid = torch.arange(max_m, device="cuda")[None, :] < dev(mm)[:, None]
    assert bool((d == SENTINEL).all(dim=2)[~rows_valid].all()), "rows >= masked_m were written"
    dd = bf16_dev_to_f64(d)
    r = synth.rng(5960 + swiglu)
    valid = [(g, m) for g in range(G) for m in range(int(mm[g]))]
    pick = r.choice(len(valid), size=2048, replace=False)
    pj = r.integers(0, cols, size=pick.size)
    pg = np.array([valid[j][0] for j in pick])
    pm = np.array([valid[j][1] for j in pick])
    got = dd[pg, pm, pj]
    ref = np.empty(pick.size)
    for g in range(G):
        sel = pg == g
        if not sel.any():
            continue
        if swiglu:
            # output column j = 64 p + i reads gate column 128 p + i and up
            # column 128 p + 64 + i; the oracle's SwiGLU with blocks of one
            # column applied to the (gate, up) pair of each point
            p_, i_ = pj[sel] // 64, pj[sel] % 64
            gate = oracle.gemm_points(qa[g], ea[g], qb[g], eb[g], pm[sel], 128 * p_ + i_, b_fp4=True)
            up = oracle.gemm_points(qa[g], ea[g], qb[g], eb[g], pm[sel], 128 * p_ + 64 + i_, b_fp4=True)
            ref[sel] = oracle.swiglu_interleaved(np.stack([gate, up], axis=-1), block=1)[:, 0]
        else:
            ref[sel] = oracle.gemm_points(qa[g], ea[g], qb[g], eb[g], pm[sel], pj[sel], b_fp4=True)
    check_close(got, ref, f"fp8xfp4 masked full size swiglu={swiglu}")


# ------------------------------------------------------------------ failure paths

def test_starved_wait_times_out_and_context_survives(dg):
    dg.dg_debug_starved_wait(20000)   # 20 ms
    assert dg.dg_get_last_error() == -4
    assert dg.dg_get_last_error() == 0
    p = Dense(7000, 128, 128, 256).upload()
    check_close(p.run(dg), p.ref(), "after timeout")


def test_contiguous_group_index_out_of_range_is_reported(dg):
    N, K = 128, 256
    cs = _contiguous_case(7100, 2, 100, 120, N, K)
    mi = cs["mi"].copy()
    mi[128:256][mi[128:256] >= 0] = 7      # second block claims group 7 of 2
    cs["mi"] = mi
    _run_contiguous(dg, cs, N)
    assert dg.dg_get_last_error() == -5


@pytest.mark.parametrize("kind", ["two_groups_in_a_block", "valid_row_after_padding", "padding_then_valid_warp"])
def test_contiguous_block_precondition_is_reported(dg, kind):
    # every 128-row block holds one group's rows, then padding (-1): a block
    # that mixes groups or has a valid row after a padding row is reported
    N, K = 128, 256
    cs = _contiguous_case(7200, 2, 100, 120, N, K)
    mi = cs["mi"].copy()
    r0 = int(cs["rows"][0])                  # first padding row of block 0
    assert 100 <= r0 < 128 and mi[r0] == -1
    if kind == "two_groups_in_a_block":
        mi[40] = 1                           # a row of group 1 inside group 0's block
    elif kind == "valid_row_after_padding":
        mi[127] = 0                          # group 0 again after its padding
    else:
        mi[32:64] = -1                       # a padding warp-row group, then valid rows
    cs["mi"] = mi
    _run_contiguous(dg, cs, N)
    assert dg.dg_get_last_error() == -5
    # the untouched layout reports nothing
    cs["mi"] = _contiguous_case(7200, 2, 100, 120, N, K)["mi"]
    _run_contiguous(dg, cs, N)
    assert dg.dg_get_last_error() == 0


# ------------------------------------------------- NN contiguous (B [G, K, N])

def _nn_case(seed, G, lo, hi, N, K):
    cs = _contiguous_case(seed, G, lo, hi, N, K)
    cs["qb_kn"] = np.ascontiguousarray(cs["qb"].transpose(0, 2, 1))   # the same weights, stored [K][N]
    return cs


def _run_nn(dg, cs, N, c_given=True):
    d = torch.empty((cs["M"], N), dtype=torch.int16, device="cuda")
    c = dev(cs["c"].view(np.int16)) if (c_given and cs["c"] is not None) else None
    dg.dg_m_grouped_fp8_gemm_nn_contiguous(dev(cs["qa"]), dev(cs["sfa"]), dev(cs["qb_kn"]), dev(cs["sfb"]), c, d,
                                           dev(cs["mi"]))
    torch.cuda.synchronize()
    return bf16_dev_to_f64(d)


@pytest.mark.parametrize("bn", [0, 128, 256])
@pytest.mark.parametrize("N", [384, 208, 112])
def test_nn_contiguous_matches_oracle(dg, bn, N):
    # N = 208: the second 128-column block of a 256-wide tile is partly past
    # N; N = 112: wholly past it (not loaded)
    K = 512
    cs = _nn_case(8000 + N, 3, 50, 300, N, K)
    dg.dg_set_tile_config(bn, 0)
    try:
        d = _run_nn(dg, cs, N)
    finally:
        dg.dg_set_tile_config(0, 0)
    ref = oracle.gemm_nn_contiguous(cs["qa"], cs["ea"], cs["qb_kn"], cs["eb"], cs["mi"], c=cs["c"])
    valid = cs["mi"] >= 0
    check_close(d[valid], ref[valid], f"nn contiguous N={N} bn={bn}")


def test_nn_contiguous_equals_nt_contiguous_on_the_same_weights(dg):
    N, K = 256, 768
    cs = _nn_case(8100, 2, 100, 260, N, K)
    nn = _run_nn(dg, cs, N)
    nt = _run_contiguous(dg, cs, N)
    valid = cs["mi"] >= 0
    check_close(nn[valid], nt[valid], "nn vs nt")


@pytest.mark.parametrize("N,K", synth.GROUPED_NK)
def test_nn_contiguous_full_size_sampled(dg, N, K):
    cs = _nn_case(8200 + N, 8, 6000, 10000, N, K)
    d = _run_nn(dg, cs, N)
    valid_rows = np.nonzero(cs["mi"] >= 0)[0]
    pm, pn = synth.sample_points(8300 + N, valid_rows, N, 4096)
    ref = np.empty(pm.size)
    for g in range(8):
        sel = cs["mi"][pm] == g
        # the oracle's NN call equals its NT call on the transposed weights
        ref[sel] = oracle.gemm_points(cs["qa"], cs["ea"], cs["qb"][g], cs["eb"][g], pm[sel], pn[sel], c=cs["c"])
    check_close(d[pm, pn], ref, f"nn contiguous {N}x{K}")


# --------------------------------------- K-grouped TN (weight gradient)

def _tn_case(seed, M, N, ks, with_c=True, tail=0):
    """A [Kt, M], B [Kt, N] e4m3, each quantised 1x128 along K (per column),
    Kt = sum(ks) + tail."""
    ks = np.asarray(ks, np.int32)
    Kt = int(ks.sum()) + tail
    qaT, ea = oracle.quantize_fp8(synth.normal_f32(seed, (M, Kt)), 1) if Kt else (np.zeros((M, 0), np.uint8),
                                                                                  np.zeros((M, 0), np.uint8))
    qbT, eb = oracle.quantize_fp8(synth.normal_f32(seed + 1, (N, Kt)), 1) if Kt else (np.zeros((N, 0), np.uint8),
                                                                                      np.zeros((N, 0), np.uint8))
    G = ks.size
    return dict(ks=ks, Kt=Kt, M=M, N=N, G=G, qa=np.ascontiguousarray(qaT.T), ea=ea,
                qb=np.ascontiguousarray(qbT.T), eb=eb,
                sfa=oracle.pack_sf(ea, M) if Kt else np.zeros(128, np.int32),
                sfb=oracle.pack_sf(eb, N) if Kt else np.zeros(128, np.int32),
                c=synth.normal_bf16_bits(seed + 2, (G, M, N)) if with_c else None)


def _run_tn(dg, cs, in_place=False):
    G, M, N = cs["G"], cs["M"], cs["N"]
    a = dev(cs["qa"]) if cs["Kt"] else torch.zeros((1, M), dtype=torch.uint8, device="cuda")
    b = dev(cs["qb"]) if cs["Kt"] else torch.zeros((1, N), dtype=torch.uint8, device="cuda")
    if in_place:
        d = dev(cs["c"].view(np.int16))
        c = d
    else:
        d = torch.full((G, M, N), 0x7FC1, dtype=torch.int16, device="cuda")
        c = dev(cs["c"].view(np.int16)) if cs["c"] is not None else None
    fn = dg.dg_k_grouped_fp8_gemm_tn_contiguous
    if cs["Kt"]:
        fn(a, dev(cs["sfa"]), b, dev(cs["sfb"]), c, d, dev(cs["ks"]))
    else:  # k_total = 0: the binding reads it from a's rows, so call the C ABI directly
        import ctypes
        st = dg.lib().dg_k_grouped_fp8_gemm_tn_contiguous(
            ctypes.c_void_p(a.data_ptr()), ctypes.c_void_p(dev(cs["sfa"]).data_ptr()), ctypes.c_void_p(b.data_ptr()),
            ctypes.c_void_p(dev(cs["sfb"]).data_ptr()), ctypes.c_void_p(c.data_ptr()) if c is not None else None,
            ctypes.c_void_p(d.data_ptr()), ctypes.c_void_p(dev(cs["ks"]).data_ptr()), G, M, N, 0, None)
        assert st == 0
    torch.cuda.synchronize()
    return bf16_dev_to_f64(d)


def _tn_ref(cs):
    return oracle.gemm_k_grouped_tn(cs["qa"], cs["ea"], cs["qb"], cs["eb"], cs["ks"], c=cs["c"])


@pytest.mark.parametrize("bn", [0, 128, 256])
@pytest.mark.parametrize("M,N", [(256, 384), (144, 208), (128, 112)])
def test_k_grouped_tn_matches_oracle(dg, bn, M, N):
    cs = _tn_case(9000 + M + N, M, N, [256, 0, 384, 128, 640], tail=128)
    dg.dg_set_tile_config(bn, 0)
    try:
        d = _run_tn(dg, cs)
    finally:
        dg.dg_set_tile_config(0, 0)
    check_close(d, _tn_ref(cs), f"k-grouped tn {M}x{N} bn={bn}")


def test_k_grouped_tn_without_c_and_in_place(dg):
    cs = _tn_case(9100, 160, 256, [128, 512, 0])
    ref = _tn_ref(cs)
    check_close(_run_tn(dg, cs, in_place=True), ref, "tn in place")
    cs0 = dict(cs, c=None)
    d = _run_tn(dg, cs0)
    check_close(d, _tn_ref(cs0), "tn C = 0")
    assert np.all(d[2] == 0.0)                       # empty group, no C: zeros


def test_k_grouped_tn_all_groups_empty(dg):
    cs = _tn_case(9200, 128, 128, [0, 0])
    d = _run_tn(dg, cs)
    assert np.array_equal(d, cs["c"].view(ml_dtypes_bf16()).astype(np.float64))


def ml_dtypes_bf16():
    import ml_dtypes
    return ml_dtypes.bfloat16


def test_k_grouped_tn_bad_sizes_are_reported(dg):
    cs = _tn_case(9300, 128, 128, [256, 128])
    bad = dict(cs, ks=np.array([256, 64], np.int32))     # 64 is not a multiple of 128
    _run_tn(dg, bad)
    assert dg.dg_get_last_error() == -5
    over = dict(cs, ks=np.array([256, 256], np.int32))   # sum beyond k_total
    _run_tn(dg, over)
    assert dg.dg_get_last_error() == -5


def test_k_grouped_tn_full_size_sampled(dg):
    # weight gradient of the (N, K) = (4096, 7168) projection over 8 experts
    # of ~6000-10000 tokens each: D[g] [4096, 7168]
    M, N = 4096, 7168
    ks = synth.k_grouped_sizes(9400, 8, 6000, 10000)
    cs = _tn_case(9401, M, N, ks)
    d = _run_tn(dg, cs)
    r = synth.rng(9402)
    pg, pi, pj = r.integers(0, 8, 2048), r.integers(0, M, 2048), r.integers(0, N, 2048)
    ref = oracle.gemm_k_grouped_tn_points(cs["qa"], cs["ea"], cs["qb"], cs["eb"], cs["ks"], pg, pi, pj, c=cs["c"])
    check_close(d[pg, pi, pj], ref, "k-grouped tn full size")


# ------------------------------------- dense NN / TN / TT storage layouts

def _run_dense_layout(dg, p, layout):
    a = p.qa.T if layout[0] == "t" else p.qa          # A stored [K, M] for "t"
    b = p.qb.T if layout[1] == "n" else p.qb          # B stored [K, N] for "n"
    d = torch.empty((p.M, p.N), dtype=torch.int16, device="cuda")
    c = dev(p.c.view(np.int16)) if p.c is not None else None
    getattr(dg, f"dg_fp8_gemm_{layout}")(dev(a), dev(p.sfa), dev(b), dev(p.sfb), c, d)
    torch.cuda.synchronize()
    return bf16_dev_to_f64(d), a, b


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
@pytest.mark.parametrize("bn,schedule,sms", [(0, 0, 0), (128, 1, 0), (256, 1, 0), (128, 2, 7), (256, 3, 7)])
@pytest.mark.parametrize("M,N,K,with_c", [
    (1104, 528, 512, True),     # ragged M and N tails
    (304, 1008, 1536, True),    # shared pieces that start and end inside tiles
    (128, 512, 128, False),     # one K-block
])
def test_dense_layouts_match_oracle(dg, layout, bn, schedule, sms, M, N, K, with_c):
    dg.dg_set_num_sms(sms)
    dg.dg_set_tile_config(bn, schedule)
    try:
        p = Dense(2800 + M + bn + schedule, M, N, K, with_c=with_c)
        d, a, b = _run_dense_layout(dg, p, layout)
        assert dg.dg_get_last_error() == 0
    finally:
        dg.dg_set_tile_config(0, 0)
        dg.dg_set_num_sms(0)
    ref = oracle.gemm_layout(np.ascontiguousarray(a), p.ea, np.ascontiguousarray(b), p.eb, layout, c=p.c)
    check_close(d, ref, f"{layout} bn={bn} schedule={schedule} {M}x{N}x{K}")


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
def test_dense_layouts_full_size_sampled(dg, layout):
    M, N, K = 4096, 7168, 2048
    p = Dense(2900, M, N, K, with_c=True)
    d, _, _ = _run_dense_layout(dg, p, layout)
    pm, pn = synth.sample_points(2901, np.arange(M), N, 2048)
    # the oracle's layout calls equal its NT call on the logical operands
    check_close(d[pm, pn], p.ref_points(pm, pn), f"{layout} {M}x{N}x{K}")


# ------------------------------------------------------------------ tensor probe

@pytest.mark.parametrize("kind", ["fp8_block_scaled", "fp8_plain", "bf16"])
def test_tensor_probe_runs_and_reports_a_rate(dg, kind):
    # the throughput probe the bench divides by: it must finish, leave no
    # device error, and land between a tenth of and twice the nominal dense
    # peak of its kind (FP8 4.5, bf16 2.25 PFLOP/s)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dg.dg_probe_mma_peak(kind, 256, 64)
    e0.record()
    f = dg.dg_probe_mma_peak(kind, 256, 2048)
    e1.record()
    torch.cuda.synchronize()
    tflops = f / (e0.elapsed_time(e1) * 1e-3) / 1e12
    nominal = 2250.0 if kind == "bf16" else 4500.0
    print(f"{kind}: {tflops:.0f} TFLOP/s", flush=True)
    assert 0.1 * nominal < tflops < 2.0 * nominal
