"""GPU: the power-of-two-scale dense GEMM (block-scaled tensor-core MMA) against
the CPU oracle.

With every scale a power of two, tcgen05.mma kind::mxf8f6f4.block_scale
applies sa*sb to each K=32 partial product before the FP32 accumulation; the
result is the method's sum up to FP32 order, checked with the same per-element
tolerance as the other GEMMs:
    |D_gpu - D_ref| <= 2^-7 * |D_ref| + 1e-4 * MAG.
Inputs are the stress generator's (Student-t activations with outlier
channels, scales 2^ceil(log2(amax/448))).  Bytes around D are compared
bit-exactly against a sentinel.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FBF
GUARD = 256


@pytest.fixture(autouse=True)
def force_block_scaled(monkeypatch):
    # Every test here runs the block-scaled kernel, whatever the shape routing.
    monkeypatch.setenv("DG_FORCE_BLOCK_SCALED", "1")
    yield


@pytest.fixture(scope="module")
def dgm():
    from moe_grouped_gemm_weight_b200 import build
    build.build()
    import moe_grouped_gemm_weight_b200 as dg
    dg.dg_set_num_sms(0)
    dg.dg_get_device_error()
    return dg


def _run(dg, c):
    cg = c.to("cuda")
    buf = torch.full((c.M * c.N + 2 * GUARD,), SENTINEL, dtype=torch.int16, device="cuda")
    D = buf[GUARD:GUARD + c.M * c.N].view(torch.bfloat16).view(c.M, c.N)
    dg.dg_fp8_gemm_nt_ue8m0(D, cg.A, cg.sa, cg.sa_stride, cg.B, cg.sb)
    torch.cuda.synchronize()
    b = buf.cpu().numpy().view(np.uint16)
    assert np.all(b[:GUARD] == SENTINEL) and np.all(b[-GUARD:] == SENTINEL), "write outside D"
    return b[GUARD:GUARD + c.M * c.N].reshape(c.M, c.N)


def _check(got, c, rows, what):
    ref, _, mag = oracle.gemm_nt(c.A.numpy(), c.sa.numpy(), c.sa_stride, c.B.numpy(), c.sb.numpy(),
                                 c.M, c.N, c.K, rows=rows, want_d64=False)
    idx = np.arange(c.M) if rows is None else rows
    g = (got[idx].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = (ref[idx].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    tol = 2.0 ** -7 * np.abs(r) + 1e-4 * mag[idx]
    bad = ~(np.abs(g - r) <= tol)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance; got {g[bad][:4]} ref {r[bad][:4]}"


@pytest.mark.parametrize("M,N,K", [(1, 256, 128), (128, 256, 256), (300, 520, 640), (129, 136, 512),
                                   (513, 1032, 1024)])
def test_ue8m0_matches_oracle_full(dgm, M, N, K):
    c = wl.dense_case(M, N, K, seed=M + N + K, stress=True)
    got = _run(dgm, c)
    assert dgm.dg_get_device_error() == 0
    _check(got, c, None, f"ue8m0 {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", wl.STRESS_SHAPES)
def test_ue8m0_stress_shapes_sampled(dgm, M, N, K):
    c = wl.dense_case(M, N, K, seed=0, stress=True, device="cuda").to("cpu")
    got = _run(dgm, c)
    assert dgm.dg_get_device_error() == 0
    rows = np.unique(np.concatenate([np.arange(0, M, 97), [0, 1, 127, 128, M - 1]]))
    _check(got, c, rows, f"ue8m0 stress {M}x{N}x{K}")


def test_scales_that_are_not_powers_of_two_are_flagged(dgm):
    c = wl.dense_case(128, 256, 256, seed=5)  # amax/448 scales
    _run(dgm, c)
    assert dgm.dg_get_device_error() & dgm.DG_DEVERR_NOT_POW2
    assert dgm.dg_get_device_error() == 0


@pytest.mark.parametrize("sms", [148, 7, 4])
def test_ue8m0_k_split(dgm, sms):
    # 300 x 520 x 6144: 3 x 3 tiles of 128 x 256 and 48 K blocks.  On 148 SMs
    # all nine tiles are split into 3 K slices (27 CTAs); on 7 SMs the two
    # tiles after one full wave are, on 4 SMs the one tile after two waves.
    c = wl.dense_case(300, 520, 6144, seed=11, stress=True)
    assert dgm.dg_make_plan_ue8m0(300, 520, 6144, sms)["tail_split"] == 3
    dgm.dg_set_num_sms(sms)
    try:
        got = _run(dgm, c)
        again = _run(dgm, c)
    finally:
        dgm.dg_set_num_sms(0)
    assert dgm.dg_get_device_error() == 0
    assert dgm.dg_get_workspace_count() >= 1, "the split ran without its workspace"
    assert np.array_equal(got, again), "split result differs between runs"
    _check(got, c, None, f"ue8m0 split on {sms} SMs")


def test_ue8m0_uneven_k_split(dgm):
    # 300 x 520 x 6400: 9 tiles of 50 K blocks, split 3 ways on 148 SMs into
    # slices of 16, 17 and 17 K blocks: the second and third slices start at
    # K blocks 16 and 33, so their groups of four scale bytes start off the
    # multiples of four.
    c = wl.dense_case(300, 520, 6400, seed=23, stress=True)
    assert dgm.dg_make_plan_ue8m0(300, 520, 6400, dgm.dg_get_num_sms())["tail_split"] == 3
    got = _run(dgm, c)
    again = _run(dgm, c)
    assert dgm.dg_get_device_error() == 0
    assert np.array_equal(got, again), "split result differs between runs"
    _check(got, c, None, "ue8m0 uneven split")


@pytest.mark.parametrize("sms", [4, 3])
def test_ue8m0_odd_k_blocks_over_many_work_items(dgm, sms):
    # 513 x 1032 x 640: 5 x 5 tiles of 5 K blocks each, too short to split.
    # On 4 (3) SMs each CTA walks 6-7 (8-9) work items, so the two MMA warps'
    # turn -- alternate K blocks, counted over the CTA's work items -- falls
    # on the other warp at every new tile.
    c = wl.dense_case(513, 1032, 640, seed=17, stress=True)
    assert dgm.dg_make_plan_ue8m0(513, 1032, 640, sms)["tail_split"] == 1
    dgm.dg_set_num_sms(sms)
    try:
        got = _run(dgm, c)
    finally:
        dgm.dg_set_num_sms(0)
    assert dgm.dg_get_device_error() == 0
    _check(got, c, None, f"ue8m0 odd K blocks on {sms} SMs")


@pytest.mark.parametrize("M", [128, 256, 384])
def test_routing_keeps_the_result(monkeypatch, dgm, M):
    # Unforced, up to 256 rows take the promotion path and more the
    # block-scaled kernel: the same sum either way.
    monkeypatch.delenv("DG_FORCE_BLOCK_SCALED", raising=False)
    c = wl.dense_case(M, 512, 4096, seed=9, stress=True)
    got = _run(dgm, c)
    assert dgm.dg_get_device_error() == 0
    _check(got, c, None, f"routed ue8m0 call, M={M}")
