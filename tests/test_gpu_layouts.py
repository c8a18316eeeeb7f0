"""GPU: the NN, TN and TT storage orders against the CPU oracle.

Each case is generated in the NT order the oracle takes (A [M][K], B [N][K]);
the GPU call gets the same values stored the other way ([K][M] and / or
[K][N], a transposed copy made on the GPU), so the result must be the NT
result.  Tolerance as for the other GEMMs:
    |D_gpu - D_ref| <= 2^-7 * |D_ref| + 1e-4 * MAG.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FBF
GUARD = 256
CALLS = {"nn": ("dg_fp8_gemm_nn", False, True), "tn": ("dg_fp8_gemm_tn", True, True),
         "tt": ("dg_fp8_gemm_tt", True, False)}


@pytest.fixture(scope="module")
def dgm():
    from moe_grouped_gemm_weight_b200 import build
    build.build()
    import moe_grouped_gemm_weight_b200 as dg
    dg.dg_set_num_sms(0)
    return dg


def _run(dg, layout, c, sms=0):
    name, a_t, b_t = CALLS[layout]
    cg = c.to("cuda")
    A = cg.A.t().contiguous() if a_t else cg.A
    B = cg.B.t().contiguous() if b_t else cg.B
    buf = torch.full((c.M * c.N + 2 * GUARD,), SENTINEL, dtype=torch.int16, device="cuda")
    D = buf[GUARD:GUARD + c.M * c.N].view(torch.bfloat16).view(c.M, c.N)
    try:
        dg.dg_set_num_sms(sms)
        getattr(dg, name)(D, A, cg.sa, cg.sa_stride, B, cg.sb)
        torch.cuda.synchronize()
    finally:
        dg.dg_set_num_sms(0)
    b = buf.cpu().numpy().view(np.uint16)
    assert np.all(b[:GUARD] == SENTINEL) and np.all(b[-GUARD:] == SENTINEL), "write outside D"
    return b[GUARD:GUARD + c.M * c.N].reshape(c.M, c.N)


def _check(got, c, rows, what):
    ref, _, mag = oracle.gemm_nt(c.A.numpy(), c.sa.numpy(), c.sa_stride, c.B.numpy(), c.sb.numpy(),
                                 c.M, c.N, c.K, rows=rows, want_d64=False)
    idx = np.arange(c.M) if rows is None else rows
    g = (got[idx].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = (ref[idx].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    bad = ~(np.abs(g - r) <= 2.0 ** -7 * np.abs(r) + 1e-4 * mag[idx])
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance; got {g[bad][:4]} ref {r[bad][:4]}"


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (64, 256, 256), (256, 512, 384), (1008, 528, 640),
                                   (384, 1792, 1024)])
def test_layouts_match_oracle_full(dgm, layout, M, N, K):
    c = wl.dense_case(M, N, K, seed=M + 2 * N + K)
    got = _run(dgm, layout, c)
    _check(got, c, None, f"{layout} {M}x{N}x{K}")


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
def test_layouts_with_k_split_tail(dgm, layout):
    # 3 x 7 = 21 tiles on 20 SMs: the last tile is split along K.
    c = wl.dense_case(384, 1792, 8192, seed=77)
    got = _run(dgm, layout, c, sms=20)
    assert dgm.dg_make_plan(0, 384, 1792, 8192, 1, 20)["tail_split"] > 1
    _check(got, c, None, f"{layout} tail split")
    assert dgm.dg_get_device_error() == 0


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
def test_layouts_full_size_sampled(dgm, layout):
    c = wl.dense_case(4096, 7168, 2048, seed=0, device="cuda").to("cpu")
    got = _run(dgm, layout, c)
    rows = np.unique(np.concatenate([np.arange(0, 4096, 131), [0, 127, 128, 4095]]))
    _check(got, c, rows, f"{layout} 4096x7168x2048")


def test_layout_alignment_is_checked(dgm):
    c = wl.dense_case(120, 128, 128, seed=1).to("cuda")  # M % 16 != 0 for an [K][M] A
    D = torch.empty(120, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dgm.DGError):
        dgm.dg_fp8_gemm_tn(D, c.A.t().contiguous(), c.sa, c.sa_stride, c.B.t().contiguous(), c.sb)
