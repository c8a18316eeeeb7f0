"""Host-side property tests of the launch plan (no GPU needed).

For random dense, contiguous and masked problems on 1..148 SMs, dg_make_plan
must return a plan whose tile arithmetic is exact and whose kernel choice
respects the limits the kernels are built for:
  * few-row problems (dense M <= 128, masked M_max <= 256) take the swap-AB
    split-K kernel: 128 weight rows per tile, TN in {32, 64, 128} activation
    rows (masked: the smallest that holds min(M_max, 128); dense: that size or
    a half / quarter of it, at least 32), 1..4 K slices of at least 8 K blocks
    (or one slice), one cluster per tile, <= 113 KiB of shared memory so that
    two CTAs share an SM;
  * everything else takes the persistent 128 x BN kernel (BN in {64, 128,
    256}) with at most one CTA per SM, and dense calls may split the tiles of a
    partial last wave into 2..8 K slices of at least 16 K blocks that the idle
    CTAs of that wave can hold.
"""
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import moe_grouped_gemm_weight_b200 as dg
from moe_grouped_gemm_weight_b200 import build as dgbuild


@pytest.fixture(scope="module", autouse=True)
def built_library():
    dgbuild.build()
    yield


def cdiv(a, b):
    return -(-a // b)


def smallest_tn(rows):
    return 32 if rows <= 32 else 64 if rows <= 64 else 128


@st.composite
def problems(draw):
    mode = draw(st.sampled_from([0, 1, 2]))
    if mode == 0:
        rows, G = draw(st.one_of(st.integers(1, 128), st.integers(129, 20000))), 1
    elif mode == 1:
        rows, G = 128 * draw(st.integers(1, 512)), draw(st.integers(1, 16))
    else:
        rows, G = draw(st.one_of(st.integers(1, 256), st.integers(257, 4096))), draw(st.integers(1, 64))
    N = 8 * draw(st.integers(1, 8192))
    K = 128 * draw(st.integers(1, 256))
    sms = draw(st.integers(1, 148))
    return mode, rows, N, K, G, sms


@settings(max_examples=600, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(problems())
def test_plan_invariants(problem):
    mode, rows, N, K, G, sms = problem
    p = dg.dg_make_plan(mode, rows, N, K, G, sms)
    nkb = K // 128
    groups = G if mode == 2 else 1
    assert p["n_blocks"] == cdiv(N, p["block_n"])
    assert p["m_blocks"] == groups * cdiv(rows, p["block_m"])
    assert p["tiles"] == p["m_blocks"] * p["n_blocks"]
    assert p["stages"] >= 2 and p["smem_bytes"] <= 227 * 1024
    assert p["cta_pair"] == 0  # CTA pairs are opt-in only
    few_rows = (mode == 0 and rows <= 128) or (mode == 2 and rows <= 256)
    assert p["swap_ab"] == int(few_rows)
    if few_rows:
        assert p["block_n"] == 128
        t0 = smallest_tn(min(rows, 128))
        if mode == 2:
            assert p["block_m"] == t0
        else:
            assert p["block_m"] in (t0, t0 // 2, t0 // 4) and p["block_m"] >= 32
        assert 1 <= p["split_k"] <= max(1, min(4, nkb // 8))
        assert p["grid"] == p["tiles"] * p["split_k"]
        assert p["smem_bytes"] <= 113 * 1024
        assert p["tail_split"] == 1
    else:
        assert p["block_m"] == 128 and p["block_n"] in (64, 128, 256)
        assert p["split_k"] == 1
        assert p["grid"] == (sms if mode == 2 else min(p["tiles"], sms))
        S = p["tail_split"]
        if S > 1:
            waves, rest = divmod(p["tiles"], p["grid"])
            assert mode == 0 and waves >= 1 and rest > 0
            assert 2 <= S <= 8 and rest * S <= p["grid"] and nkb // S >= 16
        else:
            assert S == 1


def test_few_row_split_grows_with_k_until_four_slices():
    # One weight tile (N = 128), so SMs never cap the split: the K-block count does.
    got = [dg.dg_make_plan(0, 64, 128, 128 * nkb, 1, 148)["split_k"] for nkb in (4, 8, 15, 16, 24, 32, 64, 256)]
    assert got == [1, 1, 1, 2, 3, 4, 4, 4]
