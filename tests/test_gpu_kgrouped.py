"""GPU: the K-grouped GEMM (weight-gradient form) against the CPU oracle.

Group g owns the K rows [k_offsets[g], k_offsets[g+1]); its output is the dense
GEMM restricted to those K blocks, so the reference for D[g] is the oracle's
dense GEMM on the group's slice of A, B, sa and sb (a selection of the data,
no arithmetic).  An empty group gives zeros.  A and B reach the GPU stored
[K][M] and [K][N] (transposed copies of the NT case).  Tolerance:
    |D_gpu - D_ref| <= 2^-7 * |D_ref| + 1e-4 * MAG.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FBF


@pytest.fixture(scope="module")
def dgm():
    from moe_grouped_gemm_weight_b200 import build
    build.build()
    import moe_grouped_gemm_weight_b200 as dg
    dg.dg_set_num_sms(0)
    dg.dg_get_device_error()
    return dg


def _run(dg, c, offsets):
    G = len(offsets) - 1
    cg = c.to("cuda")
    D = torch.full((G, c.M, c.N), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    ko = torch.tensor(offsets, dtype=torch.int32, device="cuda")
    dg.dg_k_grouped_fp8_gemm_tn(D, cg.A.t().contiguous(), cg.sa, cg.sa_stride, cg.B.t().contiguous(), cg.sb, ko)
    torch.cuda.synchronize()
    return D.view(torch.int16).cpu().numpy().view(np.uint16)


def _check_group(got_g, c, k0, k1, rows, what):
    if k1 == k0:
        assert np.all(got_g == 0), f"{what}: empty group not zero"
        return
    kb0, kb1 = k0 // 128, k1 // 128
    A = np.ascontiguousarray(c.A.numpy()[:, k0:k1])
    B = np.ascontiguousarray(c.B.numpy()[:, k0:k1])
    sa = np.ascontiguousarray(c.sa.numpy().reshape(-1, c.sa_stride)[kb0:kb1]).reshape(-1)
    sb = np.ascontiguousarray(c.sb.numpy()[:, kb0:kb1])
    ref, _, mag = oracle.gemm_nt(A, sa, c.sa_stride, B, sb, c.M, c.N, k1 - k0, rows=rows, want_d64=False)
    idx = np.arange(c.M) if rows is None else rows
    g = (got_g[idx].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = (ref[idx].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    bad = ~(np.abs(g - r) <= 2.0 ** -7 * np.abs(r) + 1e-4 * mag[idx])
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance; got {g[bad][:4]} ref {r[bad][:4]}"


@pytest.mark.parametrize("M,N,counts", [(256, 512, [256, 0, 128, 384]), (1008, 528, [640, 1024]),
                                        (128, 256, [128]), (384, 1792, [1024, 2048, 0, 512, 128])])
def test_k_grouped_matches_oracle(dgm, M, N, counts):
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(int).tolist()
    c = wl.dense_case(M, N, offsets[-1], seed=M + N + len(counts))
    got = _run(dgm, c, offsets)
    assert dgm.dg_get_device_error() == 0
    for g in range(len(counts)):
        _check_group(got[g], c, offsets[g], offsets[g + 1], None, f"group {g} of {M}x{N}")


def test_k_grouped_weight_gradient_size_sampled(dgm):
    # 4 experts, 2048 input x 7168 output features, 1024..4096 tokens each.
    M, N, counts = 7168, 2048, [2048, 4096, 1024, 3072]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(int).tolist()
    c = wl.dense_case(M, N, offsets[-1], seed=3, device="cuda").to("cpu")
    got = _run(dgm, c, offsets)
    rows = np.unique(np.concatenate([np.arange(0, M, 397), [0, 127, 128, M - 1]]))
    for g in range(len(counts)):
        _check_group(got[g], c, offsets[g], offsets[g + 1], rows, f"wgrad group {g}")


def test_bad_k_offsets_are_flagged_and_zeroed(dgm):
    M, N = 128, 256
    c = wl.dense_case(M, N, 512, seed=4)
    got = _run(dgm, c, [0, 200, 512])  # 200 is not a multiple of 128
    assert dgm.dg_get_device_error() & dgm.DG_DEVERR_BAD_K_OFFSET
    assert dgm.dg_get_device_error() == 0
    assert np.all(got[0] == 0) and np.all(got[1] == 0)
