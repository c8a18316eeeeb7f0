"""Failure detection on the GPU without a fault: a bounded wait runs out.

The self-test kernel waits on an mbarrier that nothing completes.  The wait
gives up after about a second, records DG_DEVERR_TIMEOUT in the device error
word and returns; the context must stay usable afterwards (a GEMM still runs
and matches the oracle)."""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    import moe_grouped_gemm_weight_b200 as dg
    assert dg.dg_get_device_error() == 0
    t0 = time.perf_counter()
    dg.dg_selftest_bounded_wait()
    code = dg.dg_get_device_error()
    dt = time.perf_counter() - t0
    assert code & dg.DG_DEVERR_TIMEOUT
    assert 0.5 < dt < 30.0
    assert dg.dg_get_device_error() == 0  # cleared by the read

    # The context is still usable.
    c = wl.dense_case(64, 136, 256, seed=1)
    cg = c.to("cuda")
    D = torch.empty(c.M, c.N, dtype=torch.bfloat16, device="cuda")
    dg.dg_fp8_gemm_nt(D, cg.A, cg.sa, cg.sa_stride, cg.B, cg.sb)
    torch.cuda.synchronize()
    ref, _, mag = oracle.gemm_nt(c.A.numpy(), c.sa.numpy(), c.sa_stride, c.B.numpy(), c.sb.numpy(),
                                 c.M, c.N, c.K, want_d64=False)
    got = D.view(torch.int16).cpu().numpy().view(np.uint16)
    g = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = (ref.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.abs(g - r) <= 2.0 ** -7 * np.abs(r) + 1e-4 * mag)
    assert dg.dg_get_device_error() == 0
