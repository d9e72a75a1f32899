"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: ml_dtypes'
code tables and casts, numpy float64 matmul on operands decoded through
ml_dtypes, closed forms, exact power-of-two invariants, index-placement
probes, and per-group slicing of the dense definition.
"""
import ml_dtypes
import numpy as np
import pytest

import oracle
import synth

E4M3_DT = ml_dtypes.float8_e4m3fn
E2M1_DT = ml_dtypes.float4_e2m1fn
E8M0_DT = ml_dtypes.float8_e8m0fnu


def same_or_nan(x, y):
    x, y = np.asarray(x, np.float64), np.asarray(y, np.float64)
    return np.array_equal(np.isnan(x), np.isnan(y)) and np.array_equal(x[~np.isnan(x)], y[~np.isnan(y)])


# --- code tables ----------------------------------------------------------

def test_e4m3_table_all_codes():
    e4, _, _ = oracle.tables()
    lib = np.arange(256, dtype=np.uint8).view(E4M3_DT).astype(np.float64)
    assert same_or_nan(e4, lib)
    assert np.isnan(e4[0x7F]) and np.isnan(e4[0xFF])
    assert int(np.isnan(e4).sum()) == 2
    assert e4[0x7E] == 448.0 and e4[0xFE] == -448.0
    assert e4[0x01] == 2.0 ** -9 and e4[0x08] == 2.0 ** -6 and e4[0x38] == 1.0
    assert e4[0x00] == 0.0 and np.signbit(e4[0x80])
    finite = e4[~np.isnan(e4)]
    assert finite.size == 254 and np.abs(finite).max() == 448.0


def test_e2m1_table_all_codes():
    _, e2, _ = oracle.tables()
    # ml_dtypes stores float4 one code per byte: decode codes 0..15 directly.
    lib = np.arange(16, dtype=np.uint8).view(E2M1_DT).astype(np.float64)
    assert np.array_equal(e2, lib)
    assert list(e2[:8]) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert list(e2[8:]) == [-0.0, -0.5, -1, -1.5, -2, -3, -4, -6]


def test_ue8m0_table_all_codes():
    _, _, ue = oracle.tables()
    lib = np.arange(256, dtype=np.uint8).view(E8M0_DT).astype(np.float64)
    assert same_or_nan(ue, lib)
    assert ue[127] == 1.0 and ue[0] == 2.0 ** -127 and ue[254] == 2.0 ** 127 and np.isnan(ue[255])


# --- encoders ---------------------------------------------------------------

def _e4m3_probe_values():
    e4, _, _ = oracle.tables()
    pos = np.sort(e4[:0x7F])
    mids = (pos[:-1] + pos[1:]) / 2            # exact ties
    r = synth.rng(1)
    rand = np.concatenate([r.uniform(-448, 448, 4000), r.standard_normal(4000) * 2.0 ** r.integers(-12, 8, 4000)])
    return np.concatenate([pos, -pos, mids, -mids, rand, [0.0, -0.0, 448.0, -448.0]])


def test_encode_e4m3_matches_ml_dtypes_rne():
    v = _e4m3_probe_values()
    got = oracle.encode_e4m3(v)
    want = v.astype(E4M3_DT).view(np.uint8)
    assert np.array_equal(got, want)


def test_encode_e4m3_ties_go_to_even_mantissa():
    e4, _, _ = oracle.tables()
    # 1.0 (0x38) and 1.125 (0x39): the tie 1.0625 goes to the even code 0x38;
    # 1.125 and 1.25 (0x3A): the tie 1.1875 goes to 0x3A.
    assert list(oracle.encode_e4m3([1.0625, 1.1875, -1.0625])) == [0x38, 0x3A, 0xB8]
    # saturation at +-448 (the recipe never reaches it, but it is defined)
    assert list(oracle.encode_e4m3([1000.0, -1000.0])) == [0x7E, 0xFE]


def test_encode_e2m1_matches_ml_dtypes_rne():
    _, e2, _ = oracle.tables()
    pos = e2[:8]
    mids = (pos[:-1] + pos[1:]) / 2
    r = synth.rng(2)
    v = np.concatenate([pos, -pos, mids, -mids, r.uniform(-6, 6, 3000)])
    got = oracle.encode_e2m1(v)
    want = v.astype(E2M1_DT).view(np.uint8) & 0xF
    assert np.array_equal(got, want)
    assert list(oracle.encode_e2m1([0.25, 0.75, 2.5, 5.0])) == [0, 2, 4, 6]


def test_scale_exponent_definition():
    # i = ceil(log2(amax / qmax)) as the least i with qmax * 2^i >= amax
    cases = {448.0: 0, 448.0 * (1 + 2 ** -40): 1, 224.0: -1, 224.0 * (1 + 2 ** -40): 0,
             0.0: 0, 1.0: -8, 3.5: -7, 3.5 * (1 + 2 ** -30): -6}
    got = oracle.scale_exponents(list(cases), 448.0)
    assert list(got) == list(cases.values())
    assert list(oracle.scale_exponents([6.0, 3.0, 3.0001, 0.75], 6.0)) == [0, -1, 0, -3]
    r = synth.rng(3)
    amax = np.abs(r.standard_normal(2000)) * 2.0 ** r.integers(-30, 30, 2000)
    i = oracle.scale_exponents(amax, 448.0).astype(np.float64)
    assert np.all(448.0 * 2.0 ** i >= amax) and np.all(448.0 * 2.0 ** (i - 1) < amax)


# --- quantisers ---------------------------------------------------------------

@pytest.mark.parametrize("rows,cols,gr", [(5, 256, 1), (300, 384, 128), (128, 128, 128)])
def test_quantize_fp8_recipe(rows, cols, gr):
    x = synth.normal_f32(10 + rows, (rows, cols)) * np.float32(3.0)
    q, e = oracle.quantize_fp8(x, gr)
    assert e.shape == ((rows + gr - 1) // gr, cols // 128)
    i = e.astype(np.int64) - 127
    # the scale of each block is the least power of two that maps amax into 448
    for br in range(e.shape[0]):
        for bc in range(e.shape[1]):
            blk = np.abs(x[br * gr:(br + 1) * gr, bc * 128:(bc + 1) * 128].astype(np.float64))
            amax = blk.max()
            s = 2.0 ** i[br, bc]
            assert 448.0 * s >= amax and 448.0 * s / 2 < amax
            assert amax / s > 224.0
    # codes are the RNE image of x / 2^i (library cast as the independent route)
    srow = np.repeat(np.repeat(2.0 ** i, gr, axis=0)[:rows], 128, axis=1)
    want = (x.astype(np.float64) / srow).astype(E4M3_DT).view(np.uint8)
    assert np.array_equal(q, want)


def test_quantize_fp8_zero_block_and_tiny_block():
    x = np.zeros((2, 256), np.float32)
    x[1, 128:] = np.float32(1e-30)
    q, e = oracle.quantize_fp8(x, 1)
    assert e[0, 0] == 127 and e[0, 1] == 127 and np.all(q[0] == 0)
    assert e[1, 0] == 127
    # 1e-30 / 448 -> 2^-109 < 1e-30 / 448 <= 2^-108: i = -108
    assert e[1, 1] == 127 - 108 and np.all(q[1, 128:] != 0)


def test_quantize_fp4_recipe_and_nibble_order():
    x = synth.normal_f32(20, (7, 128))
    q, e = oracle.quantize_fp4(x, 32)
    assert q.shape == (7, 64) and e.shape == (7, 4)
    i = e.astype(np.int64) - 127
    s = np.repeat(2.0 ** i, 32, axis=1)
    codes = (x.astype(np.float64) / s).astype(E2M1_DT).view(np.uint8) & 0xF
    assert np.array_equal(q & 0xF, codes[:, 0::2]) and np.array_equal(q >> 4, codes[:, 1::2])
    amax = np.abs(x.astype(np.float64)).reshape(7, 4, 32).max(axis=2)
    assert np.all(6.0 * 2.0 ** i >= amax) and np.all(3.0 * 2.0 ** i < amax)


# --- scale packing ------------------------------------------------------------

def _unpack_by_reshape(packed, rows):
    """Inverse of the packed layout by array reshapes (no index formula)."""
    Q, Cr, _ = packed.shape
    by = packed.view(np.uint8).reshape(Q, Cr, 32, 4, 4)       # [q, chunk, lane, word, byte]
    by = by.transpose(1, 3, 2, 0, 4).reshape(Cr * 128, Q * 4)  # row = chunk*128 + word*32 + lane
    return by[:rows]


def test_pack_sf_layout_by_reshape():
    rows, ng = 300, 7
    e = synth.junk_bytes(5, (rows, ng))
    p = oracle.pack_sf(e, rows)
    assert p.shape == (2, 3, 128)
    un = _unpack_by_reshape(p, rows)
    assert np.array_equal(un[:, :ng], e)
    assert np.all(un[:, ng:] == 127)
    full = p.view(np.uint8).reshape(2, 3, 32, 4, 4).transpose(1, 3, 2, 0, 4).reshape(384, 8)
    assert np.all(full[rows:] == 127)


def test_pack_sf_hand_example():
    # row 33, scale column 5 -> group q = 1, byte 1, chunk 0, lane 1, word 1:
    # int32 index within the chunk = lane*4 + word = 5.
    e = np.full((40, 6), 127, np.uint8)
    e[33, 5] = 0xAB
    e[33, 4] = 0x11
    p = oracle.pack_sf(e, 40)
    assert p.shape == (2, 1, 128)
    assert int(np.uint32(p[1, 0, 5])) == 0x7F7FAB11
    assert int(np.uint32(p[0, 0, 0])) == 0x7F7F7F7F


def test_pack_sf_block_rows_expand():
    eb = synth.junk_bytes(6, (3, 5))          # 128x128 block scales of a 300-row matrix
    p = oracle.pack_sf(eb, 300, row_div=128)
    un = _unpack_by_reshape(p, 300)
    assert np.array_equal(un[:, :5], np.repeat(eb, 128, axis=0)[:300])


# --- contraction --------------------------------------------------------------

def _finite_codes(seed, shape):
    c = synth.junk_bytes(seed, shape)
    c[(c & 0x7F) == 0x7F] = 0x38
    return c


def _deq_a(a, sfa):
    v = a.view(E4M3_DT).astype(np.float64)
    s = sfa.view(E8M0_DT).astype(np.float64)
    return v * np.repeat(s, 128, axis=1)


def _deq_b(b, sfb, N):
    v = b.view(E4M3_DT).astype(np.float64)
    s = sfb.view(E8M0_DT).astype(np.float64)
    return v * np.repeat(np.repeat(s, 128, axis=0)[:N], 128, axis=1)


def _deq_b_fp4(b, sfb):
    lo = (b & 0xF).view(E2M1_DT)
    hi = (b >> 4).view(E2M1_DT)
    N, K2 = b.shape
    v = np.empty((N, 2 * K2))
    v[:, 0::2] = lo.astype(np.float64)
    v[:, 1::2] = hi.astype(np.float64)
    s = sfb.view(E8M0_DT).astype(np.float64)
    return v * np.repeat(s, 32, axis=1)


def _scales(seed, shape):
    return (synth.rng(seed).integers(120, 134, size=shape)).astype(np.uint8)


@pytest.mark.parametrize("M,N,K", [(m, n, k) for m in (1, 2, 3) for n in (1, 2, 3) for k in (128, 256)])
def test_gemm_brute_force_tiny(M, N, K):
    seed = 100 * M + 10 * N + K
    a, b = _finite_codes(seed, (M, K)), _finite_codes(seed + 1, (N, K))
    sfa, sfb = _scales(seed + 2, (M, K // 128)), _scales(seed + 3, (1, K // 128))
    c = synth.normal_bf16_bits(seed + 4, (M, N))
    got = oracle.gemm(a, sfa, b, sfb, c)
    cd = c.view(ml_dtypes.bfloat16).astype(np.float64)
    want = cd + _deq_a(a, sfa) @ _deq_b(b, sfb, N).T
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=0)


def test_gemm_ragged_blocks_vs_numpy():
    M, N, K = 130, 200, 384                    # N is not a multiple of 128
    a, b = _finite_codes(7, (M, K)), _finite_codes(8, (N, K))
    sfa, sfb = _scales(9, (M, 3)), _scales(10, (2, 3))
    got = oracle.gemm(a, sfa, b, sfb)
    want = _deq_a(a, sfa) @ _deq_b(b, sfb, N).T
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-300)
    pm, pn = synth.sample_points(11, np.arange(M), N, 50)
    assert np.array_equal(oracle.gemm_points(a, sfa, b, sfb, pm, pn), got[pm, pn])


def test_gemm_closed_form_all_ones():
    for K in (128, 1024, 4096):
        a = np.full((3, K), 0x38, np.uint8)           # 1.0
        b = np.full((5, K), 0x38, np.uint8)
        sfa = np.full((3, K // 128), 127, np.uint8)   # 2^0
        sfb = np.full((1, K // 128), 127, np.uint8)
        assert np.all(oracle.gemm(a, sfa, b, sfb) == K)


def test_gemm_single_nonzero_lands_at_its_index():
    # catches transposed operands and wrong scale indexing
    M, N, K = 4, 260, 512
    a = np.zeros((M, K), np.uint8)
    b = np.zeros((N, K), np.uint8)
    a[2, 300] = 0x40      # 2.0
    b[257, 300] = 0xC4    # -3.0
    sfa = np.full((M, 4), 127, np.uint8)
    sfb = np.full((3, 4), 127, np.uint8)
    sfa[2, 2] = 130       # 2^3 on the K-block that holds k = 300
    sfb[2, 2] = 125       # 2^-2 on B's block (rows 256.., K-block 2)
    d = oracle.gemm(a, sfa, b, sfb)
    want = np.zeros((M, N))
    want[2, 257] = 2.0 * -3.0 * 8.0 * 0.25
    assert np.array_equal(d, want)


def test_gemm_scale_bump_adds_exactly_one_block():
    # raising ea[m, kb] by one adds exactly the old contribution of block kb
    M, N, K = 3, 140, 512
    a, b = _finite_codes(20, (M, K)), _finite_codes(21, (N, K))
    a[:, :] = np.where(synth.junk_bytes(22, (M, K)) < 128, 0x38, 0xB0)   # +-1, +-0.5: sums stay exact
    b[:, :] = np.where(synth.junk_bytes(23, (N, K)) < 128, 0x40, 0xA8)   # +2, -0.25
    sfa, sfb = _scales(24, (M, 4)), _scales(25, (2, 4))
    base = oracle.gemm(a, sfa, b, sfb)
    for kb in range(4):
        only = np.zeros_like(a)
        only[:, kb * 128:(kb + 1) * 128] = a[:, kb * 128:(kb + 1) * 128]
        block = oracle.gemm(only, sfa, b, sfb)
        bumped = sfa.copy()
        bumped[1, kb] += 1
        d = oracle.gemm(a, bumped, b, sfb)
        assert np.array_equal(d[1], base[1] + block[1])
        assert np.array_equal(d[[0, 2]], base[[0, 2]])


def test_gemm_fp4_closed_form_row_sums():
    M, N, K = 4, 6, 256
    a, sfa = _finite_codes(30, (M, K)), _scales(31, (M, 2))
    b = np.full((N, K // 2), 0x22, np.uint8)           # every e2m1 code = 1.0
    sfb = np.full((N, K // 32), 127, np.uint8)
    d = oracle.gemm(a, sfa, b, sfb, b_fp4=True)
    rows = _deq_a(a, sfa).sum(axis=1)
    assert np.array_equal(d, np.repeat(rows[:, None], N, axis=1))


def test_gemm_fp4_vs_numpy():
    M, N, K = 5, 70, 256
    a, sfa = _finite_codes(32, (M, K)), _scales(33, (M, 2))
    b = synth.junk_bytes(34, (N, K // 2))
    sfb = _scales(35, (N, K // 32))
    c = synth.normal_bf16_bits(36, (M, N))
    d = oracle.gemm(a, sfa, b, sfb, c=c, b_fp4=True)
    want = c.view(ml_dtypes.bfloat16).astype(np.float64) + _deq_a(a, sfa) @ _deq_b_fp4(b, sfb).T
    np.testing.assert_allclose(d, want, rtol=1e-13, atol=1e-300)


# --- grouped layouts --------------------------------------------------------------

def test_contiguous_equals_per_group_dense_and_skips_padding():
    G, N, K = 3, 136, 256
    rows, mi = synth.contiguous_layout(40, G, 20, 150)
    M = mi.size
    a = _finite_codes(41, (M, K))
    a[mi < 0] = 0x7F                                   # NaN codes in padding rows
    sfa = _scales(42, (M, 2))
    b = np.stack([_finite_codes(43 + g, (N, K)) for g in range(G)])
    sfb = np.stack([_scales(50 + g, (2, 2)) for g in range(G)])
    c = synth.normal_bf16_bits(60, (M, N))
    prior = np.full((M, N), -7.0)
    d = oracle.gemm_contiguous(a, sfa, b, sfb, mi, c=c, out=prior)
    assert np.all(d[mi < 0] == -7.0)
    for g in range(G):
        sel = np.nonzero(mi == g)[0]
        assert sel.size == rows[g]
        ref = oracle.gemm(a[sel], sfa[sel], b[g], sfb[g], c=c[sel])
        assert np.array_equal(d[sel], ref)
    assert not np.isnan(d[mi >= 0]).any()


def test_masked_equals_per_group_dense_and_leaves_rest():
    G, max_m, N, K = 4, 40, 72, 256
    mm = np.array([0, 40, 17, 99], np.int32)           # 99 > max_m is clipped to 40
    a = _finite_codes(70, (G, max_m, K))
    sfa = _scales(71, (G, max_m, 2))
    b = np.stack([_finite_codes(72 + g, (N, K)) for g in range(G)])
    sfb = np.stack([_scales(80 + g, (1, 2)) for g in range(G)])
    prior = np.full((G, max_m, N), 5.5)
    d = oracle.gemm_masked(a, sfa, b, sfb, mm, out=prior)
    for g in range(G):
        v = min(int(mm[g]), max_m)
        assert np.all(d[g, v:] == 5.5)
        if v:
            assert np.array_equal(d[g, :v], oracle.gemm(a[g, :v], sfa[g, :v], b[g], sfb[g]))


def test_contiguous_fp4_equals_per_group_dense():
    G, N, K = 2, 64, 256
    _, mi = synth.contiguous_layout(90, G, 10, 60)
    M = mi.size
    a, sfa = _finite_codes(91, (M, K)), _scales(92, (M, 2))
    b = synth.junk_bytes(93, (G, N, K // 2))
    sfb = _scales(94, (G, N, K // 32))
    d = oracle.gemm_contiguous(a, sfa, b, sfb, mi, b_fp4=True)
    for g in range(G):
        sel = np.nonzero(mi == g)[0]
        assert np.array_equal(d[sel], oracle.gemm(a[sel], sfa[sel], b[g], sfb[g], b_fp4=True))


# ------------------------------------------------------------------ SwiGLU

def test_silu_closed_forms():
    # silu(x) = x * sigmoid(x): silu(0) = 0, silu(+-1) = +-1 / (1 + e^-+1),
    # silu(x) -> x for large x and -> 0 from below for very negative x
    e = 2.718281828459045
    got = oracle.silu(np.array([0.0, 1.0, -1.0, 40.0, -40.0, -800.0]))
    assert got[0] == 0.0
    assert abs(got[1] - 1.0 / (1.0 + 1.0 / e)) < 1e-15
    assert abs(got[2] + 1.0 / (1.0 + e)) < 1e-15
    assert abs(got[3] - 40.0) < 1e-12
    assert -1e-15 < got[4] < 0.0
    assert got[5] == 0.0 or (got[5] < 0.0 and got[5] > -1e-300)


def test_swiglu_interleaved_picks_gate_and_up_columns():
    # columns 0..255 hold their own index: gate blocks are columns 0-63 and
    # 128-191, up blocks 64-127 and 192-255, so output j < 64 is
    # silu(j) * (j + 64) and output 64 + i is silu(128 + i) * (192 + i)
    g = np.arange(256, dtype=np.float64)[None, :] / 64.0
    out = oracle.swiglu_interleaved(g)
    assert out.shape == (1, 128)
    for j in (0, 5, 63):
        x, u = j / 64.0, (j + 64) / 64.0
        assert abs(out[0, j] - x / (1 + np.exp(-x)) * u) < 1e-15
    for i in (0, 6, 63):
        x, u = (128 + i) / 64.0, (192 + i) / 64.0
        assert abs(out[0, 64 + i] - x / (1 + np.exp(-x)) * u) < 1e-15
    with pytest.raises(ValueError):
        oracle.swiglu_interleaved(np.zeros((2, 96)))


def test_swiglu_of_a_gemm_equals_gemm_of_the_deinterleaved_halves():
    # the interleaving is a row permutation of B: computing the gate and up
    # products as two separate GEMMs and combining them gives the same result
    rng = np.random.default_rng(3)
    qa, ea = oracle.quantize_fp8(rng.standard_normal((5, 256)).astype(np.float32), 1)
    qb, eb = oracle.quantize_fp8(rng.standard_normal((256, 256)).astype(np.float32), 128)
    g = oracle.gemm(qa, ea, qb, eb)
    gate = np.concatenate([g[:, 0:64], g[:, 128:192]], axis=1)
    up = np.concatenate([g[:, 64:128], g[:, 192:256]], axis=1)
    assert np.array_equal(oracle.swiglu_interleaved(g), gate / (1 + np.exp(-gate)) * up)


# ------------------------------------------------------------------ BF16

def test_bf16_decode_matches_ml_dtypes_on_every_code():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_f64(codes)
    want = codes.view(ml_dtypes.bfloat16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


def test_bf16_gemm_brute_force():
    rng = np.random.default_rng(11)
    a = rng.standard_normal((3, 70)).astype(ml_dtypes.bfloat16).view(np.uint16)
    b = rng.standard_normal((4, 70)).astype(ml_dtypes.bfloat16).view(np.uint16)
    c = rng.standard_normal((3, 4)).astype(ml_dtypes.bfloat16).view(np.uint16)
    got = oracle.gemm_bf16(a, b, c)
    av = a.view(ml_dtypes.bfloat16).astype(float)
    bv = b.view(ml_dtypes.bfloat16).astype(float)
    cv = c.view(ml_dtypes.bfloat16).astype(float)
    for i in range(3):
        for j in range(4):
            s = float(cv[i, j])
            for kk in range(70):
                s += float(av[i, kk]) * float(bv[j, kk])
            assert abs(got[i, j] - s) <= 1e-12 * (1 + abs(s))


# ---- NN contiguous and K-grouped TN (the layouts whose B, or A and B, are
# stored with K as the row index)

def _deq_b_nn(bkn, sfb):
    """B stored [K][N] with 128x128 block codes sfb [ceil(N/128)][K/128],
    dequantised as a [K][N] array (independent of the oracle)."""
    K, N = bkn.shape
    v = bkn.view(E4M3_DT).astype(np.float64)
    s = sfb.view(E8M0_DT).astype(np.float64)          # [n-block][k-block]
    return v * np.repeat(np.repeat(s.T, 128, axis=0), 128, axis=1)[:K, :N]


def test_nn_contiguous_vs_numpy_and_skips_padding():
    G, N, K = 3, 200, 384                              # N is not a multiple of 128
    rows, mi = synth.contiguous_layout(70, G, 20, 150)
    M = mi.size
    a = _finite_codes(71, (M, K))
    a[mi < 0] = 0x7F
    sfa = _scales(72, (M, 3))
    b = np.stack([_finite_codes(73 + g, (K, N)) for g in range(G)])
    sfb = np.stack([_scales(80 + g, (2, 3)) for g in range(G)])
    c = synth.normal_bf16_bits(90, (M, N))
    prior = np.full((M, N), -7.0)
    d = oracle.gemm_nn_contiguous(a, sfa, b, sfb, mi, c=c, out=prior)
    assert np.all(d[mi < 0] == -7.0)
    cd = c.view(ml_dtypes.bfloat16).astype(np.float64)
    for g in range(G):
        sel = np.nonzero(mi == g)[0]
        assert sel.size == rows[g]
        want = cd[sel] + _deq_a(a[sel], sfa[sel]) @ _deq_b_nn(b[g], sfb[g])
        np.testing.assert_allclose(d[sel], want, rtol=1e-12, atol=1e-300)


def test_nn_contiguous_equals_nt_on_the_transposed_weights():
    # the same products in the same order: bit-identical
    G, N, K = 2, 136, 256
    rows, mi = synth.contiguous_layout(91, G, 10, 140)
    M = mi.size
    a, sfa = _finite_codes(92, (M, K)), _scales(93, (M, 2))
    b_nk = np.stack([_finite_codes(94 + g, (N, K)) for g in range(G)])
    sfb = np.stack([_scales(96 + g, (2, 2)) for g in range(G)])
    nt = oracle.gemm_contiguous(a, sfa, b_nk, sfb, mi)
    nn = oracle.gemm_nn_contiguous(a, sfa, np.ascontiguousarray(b_nk.transpose(0, 2, 1)), sfb, mi)
    assert np.array_equal(np.isnan(nt), np.isnan(nn))
    assert np.array_equal(nt[mi >= 0], nn[mi >= 0])


def test_nn_single_nonzero_lands_at_its_index():
    M, N, K = 128, 260, 512
    mi = np.zeros(M, np.int32)
    a = np.zeros((M, K), np.uint8)
    b = np.zeros((1, K, N), np.uint8)
    a[2, 300] = 0x40      # 2.0
    b[0, 300, 257] = 0xC4  # -3.0 at k = 300, n = 257
    sfa = np.full((M, 4), 127, np.uint8)
    sfb = np.full((1, 3, 4), 127, np.uint8)
    sfa[2, 2] = 130       # 2^3 on K-block 2
    sfb[0, 2, 2] = 125    # 2^-2 on B's block (n-block 2, K-block 2)
    d = oracle.gemm_nn_contiguous(a, sfa, b, sfb, mi)
    want = np.zeros((M, N))
    want[2, 257] = 2.0 * -3.0 * 8.0 * 0.25
    assert np.array_equal(d, want)


def _deq_kmajor_cols(x, sf):
    """x [Kt][R] codes with one code per (column r, 128-row block of K):
    sf [R][Kt/128]; dequantised [Kt][R]."""
    v = x.view(E4M3_DT).astype(np.float64)
    s = sf.view(E8M0_DT).astype(np.float64)
    return v * np.repeat(s.T, 128, axis=0)


def test_k_grouped_tn_vs_numpy_with_an_empty_group():
    M, N = 136, 200
    ks = np.array([256, 0, 128, 384], np.int32)
    Kt = int(ks.sum()) + 128                            # unused tail rows
    a, b = _finite_codes(100, (Kt, M)), _finite_codes(101, (Kt, N))
    sfa, sfb = _scales(102, (M, Kt // 128)), _scales(103, (N, Kt // 128))
    c = synth.normal_bf16_bits(104, (ks.size, M, N))
    d = oracle.gemm_k_grouped_tn(a, sfa, b, sfb, ks, c=c)
    cd = c.view(ml_dtypes.bfloat16).astype(np.float64)
    da, db = _deq_kmajor_cols(a, sfa), _deq_kmajor_cols(b, sfb)
    k0 = 0
    for g, kk in enumerate(ks):
        want = cd[g] + da[k0:k0 + kk].T @ db[k0:k0 + kk]
        np.testing.assert_allclose(d[g], want, rtol=1e-12, atol=1e-300)
        k0 += kk
    assert np.array_equal(d[1], cd[1])                 # empty group: C exactly
    assert np.array_equal(oracle.gemm_k_grouped_tn(a, sfa, b, sfb, ks)[1], np.zeros((M, N)))


def test_k_grouped_tn_single_nonzero_lands_in_its_group():
    M, N = 40, 150
    ks = np.array([256, 384], np.int32)                 # k = 300 is group 1, its K-block 2
    Kt = 640
    a = np.zeros((Kt, M), np.uint8)
    b = np.zeros((Kt, N), np.uint8)
    a[300, 5] = 0x40       # 2.0
    b[300, 130] = 0xC4     # -3.0
    sfa = np.full((M, 5), 127, np.uint8)
    sfb = np.full((N, 5), 127, np.uint8)
    sfa[5, 2] = 131        # 2^4
    sfb[130, 2] = 124      # 2^-3
    sfb[131, 2] = 140      # a neighbour's scale must not leak
    d = oracle.gemm_k_grouped_tn(a, sfa, b, sfb, ks)
    want = np.zeros((2, M, N))
    want[1, 5, 130] = 2.0 * -3.0 * 16.0 * 0.125
    assert np.array_equal(d, want)


def test_k_grouped_tn_scale_bump_adds_exactly_one_block():
    M, N = 6, 130
    ks = np.array([128, 384], np.int32)
    Kt = 512
    a = np.where(synth.junk_bytes(110, (Kt, M)) < 128, 0x38, 0xB0).astype(np.uint8)   # +-1, -0.5
    b = np.where(synth.junk_bytes(111, (Kt, N)) < 128, 0x40, 0xA8).astype(np.uint8)   # 2, -0.25
    sfa, sfb = _scales(112, (M, 4)), _scales(113, (N, 4))
    base = oracle.gemm_k_grouped_tn(a, sfa, b, sfb, ks)
    for kb in range(4):
        g = 0 if kb == 0 else 1
        only = np.zeros_like(a)
        only[kb * 128:(kb + 1) * 128] = a[kb * 128:(kb + 1) * 128]
        block = oracle.gemm_k_grouped_tn(only, sfa, b, sfb, ks)
        bumped = sfa.copy()
        bumped[3, kb] += 1
        d = oracle.gemm_k_grouped_tn(a, bumped, b, sfb, ks)
        assert np.array_equal(d[g, 3], base[g, 3] + block[g, 3])
        assert np.array_equal(d[1 - g], base[1 - g])
        assert np.array_equal(np.delete(d[g], 3, axis=0), np.delete(base[g], 3, axis=0))


def test_k_grouped_tn_points_match_the_full_reference():
    M, N = 48, 160
    ks = np.array([128, 256, 0, 128], np.int32)
    Kt = 512
    a, b = _finite_codes(120, (Kt, M)), _finite_codes(121, (Kt, N))
    sfa, sfb = _scales(122, (M, 4)), _scales(123, (N, 4))
    c = synth.normal_bf16_bits(124, (4, M, N))
    full = oracle.gemm_k_grouped_tn(a, sfa, b, sfb, ks, c=c)
    r = synth.rng(125)
    pg, pi, pj = r.integers(0, 4, 300), r.integers(0, M, 300), r.integers(0, N, 300)
    pts = oracle.gemm_k_grouped_tn_points(a, sfa, b, sfb, ks, pg, pi, pj, c=c)
    assert np.array_equal(pts, full[pg, pi, pj])


# ---- dense NT / NN / TN / TT storage layouts

@pytest.mark.parametrize("layout", ["nt", "nn", "tn", "tt"])
def test_gemm_layout_vs_numpy_and_nt_identity(layout):
    M, N, K = 48, 200, 384
    a, b = _finite_codes(130, (M, K)), _finite_codes(131, (N, K))   # logical [M, K], [N, K]
    sfa, sfb = _scales(132, (M, 3)), _scales(133, (2, 3))
    c = synth.normal_bf16_bits(134, (M, N))
    sa = np.ascontiguousarray(a.T) if layout[0] == "t" else a
    sb = np.ascontiguousarray(b.T) if layout[1] == "n" else b
    d = oracle.gemm_layout(sa, sfa, sb, sfb, layout, c=c)
    # the same products in the same order as the NT call on the logical operands
    assert np.array_equal(d, oracle.gemm(a, sfa, b, sfb, c=c))
    want = c.view(ml_dtypes.bfloat16).astype(np.float64) + _deq_a(a, sfa) @ _deq_b(b, sfb, N).T
    np.testing.assert_allclose(d, want, rtol=1e-12, atol=1e-300)


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
def test_gemm_layout_single_nonzero_lands_at_its_index(layout):
    M, N, K = 20, 260, 512
    a = np.zeros((M, K), np.uint8)
    b = np.zeros((N, K), np.uint8)
    a[7, 300] = 0x40       # 2.0
    b[257, 300] = 0xC4     # -3.0
    sfa = np.full((M, 4), 127, np.uint8)
    sfb = np.full((3, 4), 127, np.uint8)
    sfa[7, 2] = 130        # 2^3
    sfb[2, 2] = 125        # 2^-2
    sa = np.ascontiguousarray(a.T) if layout[0] == "t" else a
    sb = np.ascontiguousarray(b.T) if layout[1] == "n" else b
    d = oracle.gemm_layout(sa, sfa, sb, sfb, layout)
    want = np.zeros((M, N))
    want[7, 257] = 2.0 * -3.0 * 8.0 * 0.25
    assert np.array_equal(d, want)
