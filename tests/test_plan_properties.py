"""Host-side property tests of the launch plan (no GPU needed).

For random dense, contiguous and masked problems on 1..148 SMs, dg_make_plan
must return a plan whose tile arithmetic is exact and whose kernel choice
respects the limits the kernels are built for:
  * few-row problems (dense M <= 128, masked M_max <= 256) take the swap-AB
    kernel: 128 weight rows per tile, TN in {32, 64, 128} activation rows (no
    taller than min(rows, 128) needs), one CTA per SM; K is split into S
    slices of at least 4 K blocks only when the tiles do not fill the SMs, with
    one cluster of S CTAs per tile and every cluster resident at once;
    otherwise single-CTA clusters walk the tiles (grid = min(tiles, SMs));
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


# CTAs of one-CTA-per-SM clusters of size S resident at once on a 148-SM B200
# (cudaOccupancyMaxActiveClusters x S).
CLUSTER_CAPACITY = {1: 148, 2: 148, 3: 135, 4: 132, 5: 130, 6: 132, 7: 105, 8: 120}


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
    few_rows = (mode == 0 and rows <= 128) or (mode == 2 and rows <= 256)
    assert p["swap_ab"] == int(few_rows)
    if few_rows:
        assert p["block_n"] == 128
        assert p["block_m"] in (32, 64, 128) and p["block_m"] <= smallest_tn(min(rows, 128))
        S = p["split_k"]
        assert 1 <= S <= (4 if p["block_m"] == 128 else 8)
        if S > 1:
            # split only when the tiles do not fill the SMs, slices of >= 4
            # K blocks, one cluster per tile, all clusters resident at once
            assert p["tiles"] < sms and nkb // S >= 4
            assert p["grid"] == p["tiles"] * S <= CLUSTER_CAPACITY[S] * sms // 148
        else:
            assert p["grid"] == min(p["tiles"], sms)
        assert p["smem_bytes"] > 113 * 1024  # one CTA per SM
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


def test_few_row_split_grows_with_k_until_the_cluster_cap():
    # One weight tile (N = 128), so SMs never cap the split: the K-block count
    # (slices of >= 4 blocks, and long enough to repay the reduction) and the
    # cluster size cap (8 for TN <= 64) do.
    got = [dg.dg_make_plan(0, 64, 128, 128 * nkb, 1, 148)["split_k"] for nkb in (4, 8, 15, 16, 24, 32, 64, 256)]
    assert got == [1, 1, 3, 4, 6, 8, 8, 8]
    assert all(a <= b for a, b in zip(got, got[1:]))


@st.composite
def block_scaled_problems(draw):
    M = draw(st.one_of(st.integers(0, 256), st.integers(257, 20000)))
    N = 8 * draw(st.integers(1, 8192))
    K = 128 * draw(st.integers(1, 256))
    return M, N, K, draw(st.integers(1, 148))


@settings(max_examples=600, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(block_scaled_problems())
def test_block_scaled_plan_invariants(problem):
    """The block-scaled kernel: 128 x 256 tiles, persistent on at most one CTA
    per SM, and a K-split of the partial last wave (of every tile, when there
    are fewer tiles than SMs) into 2..8 slices of >= 16 K blocks whose
    partials fit the workspace's one partial per SM."""
    M, N, K, sms = problem
    p = dg.dg_make_plan_ue8m0(M, N, K, sms)
    nkb = K // 128
    assert (p["block_m"], p["block_n"]) == (128, 256)
    assert p["m_blocks"] == cdiv(M, 128) and p["n_blocks"] == cdiv(N, 256)
    assert p["tiles"] == p["m_blocks"] * p["n_blocks"]
    assert p["stages"] >= 2 and 113 * 1024 < p["smem_bytes"] <= 227 * 1024
    assert p["swap_ab"] == 0 and p["split_k"] == 1
    S = p["tail_split"]
    tiles = p["tiles"]
    if S == 1:
        assert p["grid"] == min(tiles, sms)
        return
    rest = tiles % sms
    assert rest > 0 and 2 <= S <= 8 and nkb // S >= 16 and rest * S <= sms
    if tiles < sms:
        assert p["grid"] == tiles * S
        partials = tiles * (S - 1)
    else:
        assert p["grid"] == sms
        partials = rest * (S - 1)
    assert partials < sms


def test_block_scaled_split_follows_the_tail_rule():
    # 300 x 520: 3 x 3 tiles.  S ~ sqrt(nkb / 1.5) rounded, capped by 8, by
    # SMs / leftover tiles and by nkb / 16.
    assert dg.dg_make_plan_ue8m0(300, 520, 6400, 148)["tail_split"] == 3   # nkb 50: 16/17/17
    assert dg.dg_make_plan_ue8m0(300, 520, 6400, 148)["grid"] == 27
    assert dg.dg_make_plan_ue8m0(300, 520, 2048, 148)["tail_split"] == 1   # nkb 16: no room
    assert dg.dg_make_plan_ue8m0(300, 520, 16384, 148)["tail_split"] == 8  # nkb 128: the cap
    assert dg.dg_make_plan_ue8m0(300, 520, 16384, 20)["tail_split"] == 2   # 9 tiles on 20 SMs
    # 4096 x 7168: 32 x 28 = 896 tiles, 6 full waves and 8 left over.
    p = dg.dg_make_plan_ue8m0(4096, 7168, 16384, 148)
    assert (p["tiles"], p["grid"], p["tail_split"]) == (896, 148, 8)
    # A whole number of waves needs no split.
    assert dg.dg_make_plan_ue8m0(128 * 148, 256, 16384, 148)["tail_split"] == 1


def test_block_scaled_plan_rejects_what_the_call_rejects():
    for args in [(64, 512, 1000, 148), (64, 500, 1024, 148), (-1, 512, 1024, 148), (64, 512, 1024, 0)]:
        with pytest.raises(RuntimeError):
            dg.dg_make_plan_ue8m0(*args)
    assert dg.dg_make_plan_ue8m0(0, 512, 1024, 148)["tiles"] == 0
