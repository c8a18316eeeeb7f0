"""GPU: the FP8 cast kernels (through the C ABI) against the CPU oracle.

The cast takes every decision in IEEE single precision on both sides (amax,
s = amax/448, r = 448/amax, x*r, e4m3 round to nearest even with saturation),
so the e4m3 codes and the scales are compared bit for bit.  Bytes around Q and
the padding of each sa_stride run are compared against a sentinel.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

GUARD = 512


@pytest.fixture(scope="module")
def dgm():
    from moe_grouped_gemm_weight_b200 import build
    build.build()
    import moe_grouped_gemm_weight_b200 as dg
    dg.dg_set_num_sms(0)
    return dg


def _bf16_bits_np(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _inputs(R, K, seed, specials=False):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((R, K)) * np.exp(rng.uniform(-8, 8, (R, 1)))
    x[0, :128] = 0.0                           # all-zero tile
    if R > 1:
        x[R - 1, -128:] *= 1e-9                # below the 1e-4 floor
    x[R // 2, K // 2] = 2.5e5                  # outlier
    x[(R * 3) // 4, 3] = -1e-3
    if specials:
        x[R // 2, 7] = np.nan
        x[0, 129] = np.inf
        x[R - 1, 0] = -np.inf
    return _bf16_bits_np(x)


def _run_1x128(dg, X, M, K, sa_stride):
    Xg = torch.from_numpy(X.view(np.int16)).cuda()
    qbuf = torch.full((M * K + 2 * GUARD,), 0x5A, dtype=torch.uint8, device="cuda")
    Q = qbuf[GUARD:GUARD + M * K].view(M, K)
    sa = torch.full(((K // 128) * sa_stride,), -7.0, dtype=torch.float32, device="cuda")
    dg.dg_to_fp8_1x128(Q, sa, sa_stride, Xg.view(torch.bfloat16).view(M, K))
    torch.cuda.synchronize()
    qb = qbuf.cpu().numpy()
    assert np.all(qb[:GUARD] == 0x5A) and np.all(qb[-GUARD:] == 0x5A), "write outside Q"
    return qb[GUARD:GUARD + M * K].reshape(M, K), sa.cpu().numpy()


@pytest.mark.parametrize("M,K,sa_stride", [(1, 128, 4), (16, 256, 16), (37, 384, 40), (100, 640, 100),
                                           (257, 7168, 260), (4096, 7168, 4096)])
def test_cast_1x128_is_bit_exact(dgm, M, K, sa_stride):
    X = _inputs(M, K, seed=M + K)
    Q, sa = _run_1x128(dgm, X, M, K, sa_stride)
    Qr, sar = oracle.cast_1x128(X, M, K, sa_stride)
    for kb in range(K // 128):
        run = sa[kb * sa_stride:(kb + 1) * sa_stride]
        assert np.array_equal(run[:M].view(np.uint32), sar[kb * sa_stride:kb * sa_stride + M].view(np.uint32))
        assert np.all(run[M:] == -7.0), "sa padding was written"
    bad = np.argwhere(Q != Qr)
    assert bad.size == 0, f"{len(bad)} codes differ, first {bad[:4].tolist()}: {Q[tuple(bad[0])]:#x} vs {Qr[tuple(bad[0])]:#x}"


def test_cast_1x128_nan_and_inf(dgm):
    M, K = 8, 256
    X = _inputs(M, K, seed=3, specials=True)
    Q, sa = _run_1x128(dgm, X, M, K, M)
    Qr, sar = oracle.cast_1x128(X, M, K, M)
    assert np.array_equal(sa.view(np.uint32), sar.view(np.uint32))
    assert np.array_equal(Q, Qr)


@pytest.mark.parametrize("N,K", [(1, 128), (128, 128), (200, 256), (1000, 1024), (7168, 2048)])
def test_cast_128x128_is_bit_exact(dgm, N, K):
    W = _inputs(N, K, seed=N * 3 + K)
    Wg = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16).view(N, K)
    qbuf = torch.full((N * K + 2 * GUARD,), 0x5A, dtype=torch.uint8, device="cuda")
    Q = qbuf[GUARD:GUARD + N * K].view(N, K)
    sb = torch.full(((N + 127) // 128, K // 128), -7.0, dtype=torch.float32, device="cuda")
    dgm.dg_to_fp8_128x128(Q, sb, Wg)
    torch.cuda.synchronize()
    qb = qbuf.cpu().numpy()
    assert np.all(qb[:GUARD] == 0x5A) and np.all(qb[-GUARD:] == 0x5A), "write outside Q"
    Qr, sbr = oracle.cast_128x128(W, N, K)
    assert np.array_equal(sb.cpu().numpy().view(np.uint32), sbr.view(np.uint32))
    assert np.array_equal(qb[GUARD:GUARD + N * K].reshape(N, K), Qr)


def test_cast_then_gemm_on_the_gpu(dgm):
    # bf16 activations and weights -> GPU casts -> GPU GEMM; the GEMM inputs
    # equal the oracle's cast (bit-exact), so the product matches the oracle
    # GEMM of the oracle cast within the GEMM tolerance.
    M, N, K = 100, 1000, 1024
    X, W = _inputs(M, K, seed=8), _inputs(N, K, seed=9)
    sa_stride = dgm.dg_get_tma_aligned_size(M, 4)
    A, sa = _run_1x128(dgm, X, M, K, sa_stride)
    Wg = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16).view(N, K)
    Bq = torch.empty(N, K, dtype=torch.uint8, device="cuda")
    sb = torch.empty((N + 127) // 128, K // 128, dtype=torch.float32, device="cuda")
    dgm.dg_to_fp8_128x128(Bq, sb, Wg)
    D = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    dgm.dg_fp8_gemm_nt(D, torch.from_numpy(A).cuda(), torch.from_numpy(sa).cuda(), sa_stride, Bq, sb)
    torch.cuda.synchronize()
    Ar, sar = oracle.cast_1x128(X, M, K, sa_stride)
    Br, sbr = oracle.cast_128x128(W, N, K)
    ref, _, mag = oracle.gemm_nt(Ar, sar, sa_stride, Br, sbr, M, N, K, want_d64=False)
    got = D.view(torch.int16).cpu().numpy().view(np.uint16)
    g = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = (ref.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.abs(g - r) <= 2.0 ** -7 * np.abs(r) + 1e-4 * mag)
