"""GPU: the allocation-free dense entry point against the oracle.

dg_fp8_gemm_nt_noalloc exists for callers that must not allocate device
memory once running (a serving loop that reserved HBM for its own pool, code
that cannot take the synchronisation cudaMalloc/cudaFree may bring): it keeps
the K-split scratch in a static device array that every call shares.  Each case
runs it twice in a row, after other cases have left their partials and flags
there, and compares both results with the CPU oracle's D within the parity
tolerance
    |D_new - D_ref| <= 2^-7 * |D_ref| + 1e-4 * MAG,   MAG = sum_k |sa*sb*a_k*b_k|
on one row of every 128-row block plus the edges.  The ordinary entry point's
result is compared the same way, and the cases that are meant to use the
scratch are checked to plan a K split.  Bytes around D are compared
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

# (M, N, K, SM cap or 0 for all, uses the scratch): K-split tails of 3, 68 and
# 56 partials, a ragged shape and a few-row shape that take no scratch, then
# the first again.
CASES = [(384, 1792, 8192, 20, True), (4096, 4096, 7168, 0, True), (1000, 1000, 1024, 0, False),
         (64, 2112, 7168, 0, False), (4096, 7168, 16384, 0, True), (384, 1792, 8192, 20, True)]


@pytest.fixture(scope="module")
def dgm():
    from moe_grouped_gemm_weight_b200 import build
    build.build()
    import moe_grouped_gemm_weight_b200 as dg
    dg.dg_set_num_sms(0)
    assert dg.dg_get_device_error() == 0
    return dg


def _call(fn, c):
    buf = torch.full((c.M * c.N + 2 * GUARD,), SENTINEL, dtype=torch.int16, device="cuda")
    D = buf[GUARD:GUARD + c.M * c.N].view(torch.bfloat16).view(c.M, c.N)
    fn(D, c.A, c.sa, c.sa_stride, c.B, c.sb)
    torch.cuda.synchronize()
    b = buf.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.all(b[:GUARD] == SENTINEL) and np.all(b[-GUARD:] == SENTINEL), "write outside D"
    return b[GUARD:GUARD + c.M * c.N].reshape(c.M, c.N)


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_noalloc_matches_oracle_on_consecutive_calls(dgm):
    import torch as _t
    sms_all = _t.cuda.get_device_properties(0).multi_processor_count
    for i, (M, N, K, sms, split) in enumerate(CASES):
        plan = dgm.dg_make_plan(0, M, N, K, 1, sms or sms_all)
        assert (plan["tail_split"] > 1) == split, (M, N, K, sms, plan)
        c = wl.dense_case(M, N, K, seed=100 + i, device="cuda")
        try:
            dgm.dg_set_num_sms(sms)
            ref_entry = _call(dgm.dg_fp8_gemm_nt, c)
            first = _call(dgm.dg_fp8_gemm_nt_noalloc, c)
            second = _call(dgm.dg_fp8_gemm_nt_noalloc, c)
        finally:
            dgm.dg_set_num_sms(0)
        rows = np.array(sorted({0, M - 1} | set(range(min(M - 1, 77), M, 128))), dtype=np.int64)
        cc = c.to("cpu")
        d_bits, _, mag = oracle.gemm_nt(cc.A.numpy(), cc.sa.numpy(), cc.sa_stride, cc.B.numpy(), cc.sb.numpy(),
                                        M, N, K, rows=rows, want_d64=False)
        r = _f64(d_bits[rows])
        tol = 2.0 ** -7 * np.abs(r) + 1e-4 * mag[rows]
        for name, got in (("dg_fp8_gemm_nt", ref_entry), ("first noalloc", first), ("second noalloc", second)):
            g = _f64(got[rows])
            bad = ~(np.abs(g - r) <= tol)
            assert not bad.any(), (f"{M}x{N}x{K} sms={sms} {name} call: {bad.sum()} of {bad.size} outside "
                                   f"tolerance; got={g[bad][:4]} oracle={r[bad][:4]}")
        assert dgm.dg_get_device_error() == 0
