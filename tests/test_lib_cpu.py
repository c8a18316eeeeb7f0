"""Host-side tests of the C ABI (no GPU needed): the library loads, exports every
symbol include/dg.h declares, its utilities and launch plan follow the pages'
rules, and bad arguments are rejected synchronously before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

import moe_grouped_gemm_weight_b200 as dg
from moe_grouped_gemm_weight_b200 import build as dgbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dg.h")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    dgbuild.build()
    yield


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^DG_API\s+[\w\s\*]+?\b(dg_\w+)\s*\(", text, re.M)))


def test_header_declares_the_three_gemms_and_utilities():
    names = declared_functions()
    for n in ["dg_fp8_gemm_nt", "dg_grouped_contiguous_nt", "dg_grouped_masked_nt", "dg_set_num_sms",
              "dg_get_num_sms", "dg_get_m_alignment_for_contiguous_layout", "dg_get_tma_aligned_size",
              "dg_get_device_error", "dg_status_string", "dg_last_error_message", "dg_make_plan"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(dg.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_library_exports_nothing_undeclared():
    out = os.popen(f"nm -D --defined-only {dg.LIB_PATH}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l and l.split()[-1].startswith("dg")}
    assert exported == set(declared_functions())


def test_library_does_not_link_the_oracle():
    out = os.popen(f"ldd {dg.LIB_PATH}").read() + os.popen(f"nm -D {dg.LIB_PATH}").read()
    assert "oracle" not in out and "dgo_" not in out


def test_utilities():
    assert dg.dg_get_m_alignment_for_contiguous_layout() == 128
    assert dg.dg_get_tma_aligned_size(64, 4) == 64
    assert dg.dg_get_tma_aligned_size(65, 4) == 68
    assert dg.dg_get_tma_aligned_size(1, 4) == 4
    assert dg.dg_get_tma_aligned_size(3, 2) == 8
    assert dg.dg_get_tma_aligned_size(17, 1) == 32
    assert dg.dg_get_tma_aligned_size(0, 4) == 0
    assert dg.dg_status_string(0) == "ok"
    assert "invalid" in dg.dg_status_string(1)


def test_plan_reproduces_the_pages_block_count_arithmetic():
    # README page, section "非对齐的块大小": M=256, N=7168 with 128x128 blocks
    # gives (256/128)*(7168/128) = 112 tiles, which leaves SMs of a 132-SM part
    # idle.  The plan keeps the tile arithmetic exact.
    p = dg.dg_make_plan(0, 256, 7168, 7168, 1, 132)
    assert p["block_m"] == 128
    assert p["m_blocks"] == 2
    assert p["tiles"] == p["m_blocks"] * p["n_blocks"]
    assert p["n_blocks"] == -(-7168 // p["block_n"])
    if p["block_n"] == 128:
        assert p["tiles"] == 112


@pytest.mark.parametrize("mode,rows,N,K,G", [(0, 64, 2112, 7168, 1), (0, 4096, 7168, 16384, 1),
                                            (1, 32768, 4096, 7168, 4), (2, 256, 4096, 7168, 4),
                                            (2, 1024, 4096, 7168, 1), (0, 129, 512, 1024, 1)])
def test_plan_is_consistent(mode, rows, N, K, G):
    p = dg.dg_make_plan(mode, rows, N, K, G, 148)
    assert p["n_blocks"] == -(-N // p["block_n"])
    mb = -(-rows // p["block_m"]) * (G if mode == 2 else 1)
    assert p["m_blocks"] == mb
    assert p["tiles"] == mb * p["n_blocks"]
    assert p["stages"] >= 2
    if p["swap_ab"]:
        # Few-row kernel: 128 weight rows per tile, one CTA per SM; K split
        # over a cluster of split_k CTAs per tile only when the tiles do not
        # fill the SMs, else single CTAs walk the tiles.
        assert rows <= (256 if mode == 2 else 128)
        assert p["block_n"] == 128 and p["block_m"] in (32, 64, 128)
        assert 1 <= p["split_k"] <= 8 and (p["split_k"] == 1 or K // 128 // p["split_k"] >= 4)
        if p["split_k"] > 1:
            assert p["grid"] == p["tiles"] * p["split_k"] and p["tiles"] < 148
        else:
            assert p["grid"] == min(p["tiles"], 148)
        assert 113 * 1024 < p["smem_bytes"] <= 227 * 1024
    else:
        assert p["block_m"] == 128 and p["block_n"] in (64, 128, 256)
        assert p["split_k"] == 1
        assert 1 <= p["grid"] <= 148
        assert p["smem_bytes"] <= 227 * 1024


@pytest.mark.parametrize("M,N,K,tn,split", [
    # the planner's cost model (fitted to measured decode timings) on the sweep
    (1, 2112, 7168, 32, 6), (32, 2112, 7168, 32, 6), (64, 2112, 7168, 64, 6), (128, 2112, 7168, 64, 3),
    (64, 4096, 7168, 64, 4), (128, 4096, 7168, 128, 4), (64, 7168, 2048, 32, 1), (128, 7168, 2048, 64, 1),
    (64, 7168, 16384, 64, 2), (128, 7168, 16384, 128, 2),
    (64, 24576, 1536, 64, 1), (128, 24576, 1536, 128, 1), (64, 32768, 512, 64, 1), (128, 32768, 512, 128, 1),
])
def test_few_row_plan_tile_and_split(M, N, K, tn, split):
    p = dg.dg_make_plan(0, M, N, K, 1, 148)
    assert p["swap_ab"] == 1 and p["block_m"] == tn and p["split_k"] == split, p
    assert p["m_blocks"] == -(-M // tn) and p["n_blocks"] == -(-N // 128)
    assert dg.dg_make_plan(0, 129, N, K, 1, 148)["swap_ab"] == 0


def test_few_row_plan_tile_never_taller_than_the_rows_need():
    for M in range(1, 129):
        p = dg.dg_make_plan(0, M, 520, 4480, 1, 148)
        assert p["block_m"] <= (32 if M <= 32 else 64 if M <= 64 else 128)
        assert p["m_blocks"] == -(-M // p["block_m"]) and p["grid"] == p["tiles"] * p["split_k"]


@pytest.mark.parametrize("args,expect", [
    ((0, 64, 2112, 7100, 1), dg.DG_ERR_UNSUPPORTED),  # K % 128
    ((0, 64, 2110, 7168, 1), dg.DG_ERR_UNSUPPORTED),  # N % 8
    ((0, -1, 64, 128, 1), dg.DG_ERR_INVALID_ARG),
    ((1, 130, 64, 128, 2), dg.DG_ERR_INVALID_ARG),    # contiguous M_total % 128
    ((2, 64, 64, 128, 5000), dg.DG_ERR_UNSUPPORTED),  # too many masked groups
    ((3, 64, 64, 128, 1), dg.DG_ERR_INVALID_ARG),     # bad mode
])
def test_plan_rejects_bad_sizes(args, expect):
    with pytest.raises(dg.DGError) as ei:
        dg.dg_make_plan(*args, 148)
    assert ei.value.status == expect


def test_gemm_calls_reject_bad_arguments_without_touching_the_gpu():
    L = dg.lib()
    fake = 1 << 20  # never dereferenced: every call below fails validation first
    st = L.dg_fp8_gemm_nt(fake, fake, fake, 64, fake, fake, 64, 64, 100, 0)
    assert st == dg.DG_ERR_UNSUPPORTED and b"K=100" in L.dg_last_error_message()
    assert L.dg_fp8_gemm_nt(0, fake, fake, 64, fake, fake, 64, 64, 128, 0) == dg.DG_ERR_INVALID_ARG
    assert L.dg_fp8_gemm_nt(fake + 4, fake, fake, 64, fake, fake, 64, 64, 128, 0) == dg.DG_ERR_MISALIGNED
    assert L.dg_fp8_gemm_nt(fake, fake, fake, 62, fake, fake, 64, 64, 128, 0) == dg.DG_ERR_INVALID_ARG
    assert L.dg_fp8_gemm_nt(fake, fake, fake, 66, fake, fake, 64, 64, 128, 0) == dg.DG_ERR_INVALID_ARG
    assert L.dg_grouped_contiguous_nt(fake, fake, fake, 128, fake, fake, 0, 128, 64, 128, 2, 0) == \
        dg.DG_ERR_INVALID_ARG
    assert L.dg_grouped_contiguous_nt(fake, fake, fake, 200, fake, fake, fake, 200, 64, 128, 2, 0) == \
        dg.DG_ERR_INVALID_ARG
    assert L.dg_grouped_masked_nt(fake, fake, fake, 64, fake, fake, 0, 2, 64, 64, 128, 0, 0) == \
        dg.DG_ERR_INVALID_ARG
    assert L.dg_grouped_masked_nt(fake, fake, fake, 64, fake, fake, fake, 2, 64, 64, 128, 0, 0) != dg.DG_OK or \
        dg.dg_get_num_sms() > 0


def test_cast_calls_reject_bad_arguments_without_touching_the_gpu():
    L = dg.lib()
    fake = 1 << 20  # never dereferenced: every call below fails validation first
    st = L.dg_to_fp8_1x128(fake, fake, 64, fake, 64, 100, 0)
    assert st == dg.DG_ERR_UNSUPPORTED and b"K=100" in L.dg_last_error_message()
    assert L.dg_to_fp8_1x128(0, fake, 64, fake, 64, 128, 0) == dg.DG_ERR_INVALID_ARG
    assert L.dg_to_fp8_1x128(fake, fake, 64, fake + 8, 64, 128, 0) == dg.DG_ERR_MISALIGNED
    assert L.dg_to_fp8_1x128(fake, fake + 2, 64, fake, 64, 128, 0) == dg.DG_ERR_MISALIGNED
    assert L.dg_to_fp8_1x128(fake, fake, 63, fake, 64, 128, 0) == dg.DG_ERR_INVALID_ARG
    assert L.dg_to_fp8_1x128(fake, fake, 64, fake, -1, 128, 0) == dg.DG_ERR_INVALID_ARG
    assert L.dg_to_fp8_1x128(fake, fake, 0, fake, 0, 128, 0) == dg.DG_OK  # empty: nothing launched
    assert L.dg_to_fp8_128x128(fake, fake, fake, 64, 130, 0) == dg.DG_ERR_UNSUPPORTED
    assert L.dg_to_fp8_128x128(fake, 0, fake, 64, 128, 0) == dg.DG_ERR_INVALID_ARG
    assert L.dg_to_fp8_128x128(fake + 4, fake, fake, 64, 128, 0) == dg.DG_ERR_MISALIGNED
    assert L.dg_to_fp8_128x128(fake, fake, fake, 0, 128, 0) == dg.DG_OK


def test_empty_problem_is_a_no_op():
    L = dg.lib()
    fake = 1 << 20
    assert L.dg_fp8_gemm_nt(fake, fake, fake, 0, fake, fake, 0, 64, 128, 0) == dg.DG_OK


def test_binding_fails_loudly_when_library_missing(tmp_path, monkeypatch):
    import importlib
    mod = importlib.import_module("moe_grouped_gemm_weight_b200")
    monkeypatch.setattr(mod, "_lib", None)
    monkeypatch.setattr(mod, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        mod.dg_get_num_sms()


def test_pdl_switch_defaults_to_the_environment(monkeypatch):
    try:
        dg.dg_set_pdl(None)
        monkeypatch.delenv("DG_PDL", raising=False)
        assert dg.dg_get_pdl() is True  # on unless DG_PDL=0
        monkeypatch.setenv("DG_PDL", "1")
        assert dg.dg_get_pdl() is True
        monkeypatch.setenv("DG_PDL", "0")
        assert dg.dg_get_pdl() is False
        dg.dg_set_pdl(True)
        assert dg.dg_get_pdl() is True
        dg.dg_set_pdl(False)
        monkeypatch.setenv("DG_PDL", "1")
        assert dg.dg_get_pdl() is False
    finally:
        dg.dg_set_pdl(None)


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "dg.h"

int main(void) {
    dg_plan p;
    dg_status s = dg_make_plan(0, 4096, 7168, 16384, 1, 148, &p);
    if (s != DG_OK) return 1;
    printf("plan %d %d %d %d %d\n", p.block_m, p.block_n, p.tiles, p.grid, p.tail_split);
    s = dg_make_plan_ue8m0(4096, 7168, 16384, 148, &p);
    if (s != DG_OK) return 2;
    printf("ue8m0 %d %d %d\n", p.block_n, p.tiles, p.tail_split);
    printf("align %d %d\n", dg_get_m_alignment_for_contiguous_layout(), dg_get_tma_aligned_size(65, 4));
    s = dg_make_plan(0, 64, 2112, 100, 1, 148, &p);
    printf("bad %d %s|%s\n", (int)s, dg_status_string(s), strstr(dg_last_error_message(), "K=100") ? "K" : "?");
    /* a GEMM call with a null output is refused before any device work */
    s = dg_fp8_gemm_nt(NULL, NULL, NULL, 64, NULL, NULL, 64, 64, 128, NULL);
    printf("null %d\n", (int)s);
    return 0;
}
"""


def test_header_compiles_as_c99_and_links(tmp_path):
    """include/dg.h is a C ABI: a plain C99 client (-pedantic -Werror) compiles
    against it, links libdg.so and calls the host-only functions."""
    src, exe = tmp_path / "client.c", tmp_path / "client"
    src.write_text(C_CLIENT)
    libdir = os.path.dirname(dg.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", libdir, "-ldg", f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    lines = dict(l.split(" ", 1) for l in r.stdout.strip().splitlines())
    assert lines["plan"].split()[:2] == ["128", "256"]
    assert lines["ue8m0"] == "256 896 8"
    assert lines["align"] == "128 68"
    assert lines["bad"] == f"{dg.DG_ERR_UNSUPPORTED} {dg.dg_status_string(dg.DG_ERR_UNSUPPORTED)}|K"
    assert lines["null"] == str(dg.DG_ERR_INVALID_ARG)
