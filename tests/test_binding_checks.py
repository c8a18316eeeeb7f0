"""Host-side checks of the Python binding's tensor arguments (no GPU needed).

The C ABI takes plain device pointers, so the binding checks every tensor's
element size, contiguity, extent (the elements the call reads or writes, per
the layouts include/dg.h fixes) and device before a pointer crosses the
boundary.  On this host every valid argument set must get through the size
checks and stop only at the device check; each kind of bad argument must be
refused with DG_ERR_INVALID_ARG naming the tensor.
"""
import pytest
import torch

import moe_grouped_gemm_weight_b200 as dg
import workloads as wl


def bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def refused(fn, *args, match):
    with pytest.raises(dg.DGError) as ei:
        fn(*args)
    assert ei.value.status == dg.DG_ERR_INVALID_ARG
    assert match in str(ei.value), str(ei.value)


def reaches_device_check(fn, *args):
    refused(fn, *args, match="is not on a CUDA device")


@pytest.mark.parametrize("M,N,K", [(1, 8, 128), (100, 520, 640), (300, 1032, 6144)])
def test_valid_dense_arguments_pass_every_size_check(M, N, K):
    c = wl.dense_case(M, N, K, seed=0)
    for fn in (dg.dg_fp8_gemm_nt, dg.dg_fp8_gemm_nt_ue8m0, dg.dg_fp8_gemm_nt_noalloc):
        reaches_device_check(fn, bf16(M, N), c.A, c.sa, c.sa_stride, c.B, c.sb)
    At, Bt = c.A.t().contiguous(), c.B.t().contiguous()
    reaches_device_check(dg.dg_fp8_gemm_nn, bf16(M, N), c.A, c.sa, c.sa_stride, Bt, c.sb)
    reaches_device_check(dg.dg_fp8_gemm_tn, bf16(M, N), At, c.sa, c.sa_stride, Bt, c.sb)
    reaches_device_check(dg.dg_fp8_gemm_tt, bf16(M, N), At, c.sa, c.sa_stride, c.B, c.sb)
    ko = torch.tensor([0, 128, K], dtype=torch.int32)
    reaches_device_check(dg.dg_k_grouped_fp8_gemm_tn, bf16(2, M, N), At, c.sa, c.sa_stride, Bt, c.sb, ko)


def test_valid_grouped_and_cast_arguments_pass_every_size_check():
    c = wl.contiguous_case([100, 0, 300], 264, 256, seed=0)
    reaches_device_check(dg.dg_grouped_contiguous_nt, bf16(c.M, c.N), c.A, c.sa, c.sa_stride, c.B, c.sb,
                         c.m_indices)
    m = wl.masked_case(3, 40, 264, 256, seed=0)
    reaches_device_check(dg.dg_grouped_masked_nt, bf16(3, 40, 264), m.A, m.sa, m.sa_stride, m.B, m.sb,
                         m.masked_m)
    M, K = 100, 1024
    st = dg.dg_get_tma_aligned_size(M, 4)
    reaches_device_check(dg.dg_to_fp8_1x128, torch.empty(M, K, dtype=torch.uint8),
                         torch.empty(K // 128 * st), st, bf16(M, K))
    N = 200
    reaches_device_check(dg.dg_to_fp8_128x128, torch.empty(N, K, dtype=torch.uint8),
                         torch.empty(2, K // 128), bf16(N, K))


def test_the_minimal_transposed_scale_extent_is_enough():
    # sa[kb*sa_stride + m] for kb < K/128 and m < M: the last K block needs
    # only M entries past its start, not a whole stride.
    M, N, K = 100, 256, 512
    c = wl.dense_case(M, N, K, seed=0)
    st = c.sa_stride + 28
    sa = torch.zeros((K // 128 - 1) * st + M)
    reaches_device_check(dg.dg_fp8_gemm_nt, bf16(M, N), c.A, sa, st, c.B, c.sb)
    refused(dg.dg_fp8_gemm_nt, bf16(M, N), c.A, sa[:-1], st, c.B, c.sb, match="sa holds")


def test_bad_dense_arguments_are_refused():
    M, N, K = 100, 264, 512
    c = wl.dense_case(M, N, K, seed=0)
    D = bf16(M, N)
    f = dg.dg_fp8_gemm_nt
    refused(f, bf16(M, N - 8), c.A, c.sa, c.sa_stride, c.B, c.sb, match="D holds")
    refused(f, torch.zeros(M, N), c.A, c.sa, c.sa_stride, c.B, c.sb, match="D has 4-byte elements")
    refused(f, bf16(N, M).t(), c.A, c.sa, c.sa_stride, c.B, c.sb, match="D is not contiguous")
    refused(f, D, c.A, c.sa[:-1], c.sa_stride, c.B, c.sb, match="sa holds")
    refused(f, D, c.A, c.sa.double(), c.sa_stride, c.B, c.sb, match="sa has 8-byte elements")
    refused(f, D, c.A, c.sa, c.sa_stride, c.B, c.sb[:-1], match="sb holds")
    refused(f, D, c.A, c.sa, c.sa_stride, c.B[:, :K - 128], c.sb, match="K of B is")
    refused(f, D, c.A[:, :K - 128].contiguous(), c.sa, c.sa_stride, c.B, c.sb, match="K of B is")
    At = c.A.t()  # a transposed view is not the [M][K] storage the call reads
    refused(dg.dg_fp8_gemm_tt, D, At, c.sa, c.sa_stride, c.B, c.sb, match="A is not contiguous")
    refused(dg.dg_fp8_gemm_nn, D, c.A, c.sa, c.sa_stride, c.B, c.sb, match="K of B is")


def test_bad_grouped_arguments_are_refused():
    c = wl.contiguous_case([128, 256], 264, 256, seed=0)
    f = dg.dg_grouped_contiguous_nt
    D = bf16(c.M, c.N)
    refused(f, D, c.A, c.sa, c.sa_stride, c.B, c.sb, c.m_indices.long(), match="m_indices has 8-byte")
    refused(f, D, c.A, c.sa, c.sa_stride, c.B, c.sb, c.m_indices[:-1], match="m_indices holds")
    refused(f, D, c.A, c.sa, c.sa_stride, c.B[0], c.sb, c.m_indices, match="rank of B")
    refused(f, D, c.A, c.sa, c.sa_stride, c.B, c.sb[:1], c.m_indices, match="sb holds")
    m = wl.masked_case(3, 40, 264, 256, seed=0)
    g = dg.dg_grouped_masked_nt
    D = bf16(3, 40, 264)
    refused(g, D, m.A, m.sa, m.sa_stride, m.B[:2].contiguous(), m.sb, m.masked_m, match="group count of B")
    refused(g, D, m.A, m.sa, m.sa_stride, m.B, m.sb, m.masked_m[:2], match="masked_m holds")
    refused(g, bf16(3, 39, 264), m.A, m.sa, m.sa_stride, m.B, m.sb, m.masked_m, match="D holds")
    refused(g, D, m.A, m.sa[:-1], m.sa_stride, m.B, m.sb, m.masked_m, match="sa holds")
    refused(g, D, m.A[0], m.sa, m.sa_stride, m.B, m.sb, m.masked_m, match="rank of A")


def test_null_pointers_pass_through_to_the_library():
    # None becomes a null pointer, which the library reports itself; the
    # binding checks only the tensors it is given (here host tensors, so the
    # first of them stops at the device check).
    c = wl.dense_case(64, 64, 128, seed=0)
    refused(dg.dg_fp8_gemm_nt, None, c.A, c.sa, c.sa_stride, c.B, c.sb, match="A is not on a CUDA device")
