"""The C-ABI library builds, loads and exports every entry point that
include/dg.h declares; host-side argument checks and host heuristics work
without a GPU (no compute call is made here)."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dg():
    from moe_grouped_gemm_06_b200 import build
    build.build()
    import moe_grouped_gemm_06_b200 as dg
    return dg


def header_functions():
    text = open(os.path.join(ROOT, "include", "dg.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dg_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = header_functions()
    for required in ("dg_fp8_gemm_nt", "dg_m_grouped_fp8_gemm_nt_contiguous", "dg_m_grouped_fp8_gemm_nt_masked",
                     "dg_fp8_fp4_gemm_nt", "dg_m_grouped_fp8_fp4_gemm_nt_contiguous", "dg_pack_sf",
                     "dg_get_num_sms", "dg_set_num_sms", "dg_get_mk_alignment_for_contiguous_layout"):
        assert required in names


def test_library_exports_every_declared_symbol(dg):
    lib = dg.lib()
    names = header_functions()
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(dg.SYMBOLS) == names


def test_nm_shows_exports(dg):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", dg.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (dg_[a-z0-9_]+)", out))
    assert set(header_functions()) <= exported


def test_status_strings_and_alignment(dg):
    assert dg.status_string(0) == "DG_OK"
    assert dg.status_string(-1) == "DG_ERR_INVALID_ARG"
    assert dg.status_string(-4) == "DG_ERR_TIMEOUT"
    assert dg.dg_get_mk_alignment_for_contiguous_layout() == 128


def test_invalid_arguments_rejected_on_host(dg):
    lib = dg.lib()
    fake = 1 << 20  # never dereferenced: every call below fails its host checks
    p = lambda v: None if v is None else __import__("ctypes").c_void_p(v)
    # null pointer
    assert lib.dg_fp8_gemm_nt(None, p(fake), p(fake), p(fake), None, p(fake), 128, 128, 128, None) == -1
    # K not a multiple of 128
    assert lib.dg_fp8_gemm_nt(p(fake), p(fake), p(fake), p(fake), None, p(fake), 128, 128, 100, None) == -1
    # N not a multiple of 8
    assert lib.dg_fp8_gemm_nt(p(fake), p(fake), p(fake), p(fake), None, p(fake), 128, 100, 128, None) == -1
    # misaligned pointer
    assert lib.dg_fp8_gemm_nt(p(fake + 4), p(fake), p(fake), p(fake), None, p(fake), 128, 128, 128, None) == -1
    # negative M
    assert lib.dg_fp8_gemm_nt(p(fake), p(fake), p(fake), p(fake), None, p(fake), -1, 128, 128, None) == -1
    # m == 0 is a no-op
    assert lib.dg_fp8_gemm_nt(p(fake), p(fake), p(fake), p(fake), None, p(fake), 0, 128, 128, None) == 0
    # contiguous: m_total must be a multiple of 128, groups > 0
    assert lib.dg_m_grouped_fp8_gemm_nt_contiguous(p(fake), p(fake), p(fake), p(fake), None, p(fake), p(fake),
                                                   100, 128, 128, 2, None) == -1
    assert lib.dg_m_grouped_fp8_gemm_nt_contiguous(p(fake), p(fake), p(fake), p(fake), None, p(fake), p(fake),
                                                   128, 128, 128, 0, None) == -1
    # masked: at most 1024 groups, max_m > 0
    assert lib.dg_m_grouped_fp8_gemm_nt_masked(p(fake), p(fake), p(fake), p(fake), p(fake), p(fake), 1025, 256,
                                               128, 128, 0, None) == -1
    assert lib.dg_m_grouped_fp8_gemm_nt_masked(p(fake), p(fake), p(fake), p(fake), p(fake), p(fake), 4, 0,
                                               128, 128, 0, None) == -1
    # quantiser: cols % 128, block_rows in {1, 128}
    assert lib.dg_quantize_fp8(p(fake), 4, 100, 1, p(fake), p(fake), None) == -1
    assert lib.dg_quantize_fp8(p(fake), 4, 128, 64, p(fake), p(fake), None) == -1
    assert lib.dg_quantize_fp4(p(fake), 4, 48, p(fake), p(fake), None) == -1


def test_packed_sf_words(dg):
    assert dg.dg_packed_sf_words(128, 4) == 128
    assert dg.dg_packed_sf_words(129, 5) == 2 * 2 * 128
    assert dg.dg_packed_sf_words(300, 7) == 2 * 3 * 128
    assert dg.dg_packed_sf_words(0, 7) == 0


def _golden_rows():
    path = os.path.join(ROOT, "tests", "golden", "nonaligned_block_n.txt")
    rows = []
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append([int(v) for v in line.split()])
    return rows


def test_tile_count_matches_pages_worked_example(dg):
    for m, n, bm, bn, tiles, _sms in _golden_rows():
        assert dg.dg_num_tiles(m, n, bm, bn) == tiles


def test_heuristic_in_the_pages_example(dg):
    # The page's unaligned BLOCK_N=112 keeps 128 of 132 SMs busy for M=256,
    # N=7168 where 128x128 tiles keep 112.  Block widths here are multiples of
    # 64 (the scale-factor operand's TMEM address must be even), so the
    # heuristic has {128, 192, 256} x split-K; it must never do worse than the
    # page's aligned baseline and must fill whole waves.
    (m, n, _, _, base, sms), _ = _golden_rows()
    dg.dg_set_num_sms(sms)
    try:
        cfg = dg.dg_query_dense_config(m, n, 7168)
    finally:
        dg.dg_set_num_sms(0)
    assert cfg["block_n"] % 64 == 0
    assert cfg["grid"] >= base
    assert cfg["units"] <= sms or cfg["units"] % cfg["grid"] == 0


def test_heuristic_large_m_has_no_split(dg):
    dg.dg_set_num_sms(148)
    try:
        cfg = dg.dg_query_dense_config(4096, 7168, 16384)
        small = dg.dg_query_dense_config(64, 2112, 7168)
    finally:
        dg.dg_set_num_sms(0)
    assert cfg["splits"] == 1 and cfg["grid"] == 148
    assert small["splits"] > 1 and small["units"] <= 148


def test_tile_config_override_and_pairs_refused(dg):
    assert dg.lib().dg_set_tile_config(96, 0) == -1          # not an instantiated width
    assert dg.lib().dg_set_tile_config(0, 2) == -2           # CTA pairs are not launched
    dg.dg_set_num_sms(148)
    try:
        dg.dg_set_tile_config(256, 1)
        assert dg.dg_query_dense_config(4096, 7168, 16384)["block_n"] == 256
        dg.dg_set_tile_config(0, 0)
        for shape in [(4096, 7168, 16384), (4096, 2112, 7168), (256, 7168, 7168)]:
            assert dg.dg_query_dense_config(*shape)["ctas"] == 1
    finally:
        dg.dg_set_tile_config(0, 0)
        dg.dg_set_num_sms(0)
