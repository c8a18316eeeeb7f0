"""GPU parity: the sm_100a kernels (through the C ABI) against the CPU oracle.

Tolerance (per element, from the definition of the method): the GPU keeps FP32
accumulators and rounds to bf16 once, the oracle is exact up to its single
bf16 rounding, so
    |D_gpu - D_ref| <= 2^-7 * |D_ref| + 1e-4 * MAG,   MAG = sum_k |sa*sb*a_k*b_k|.
2^-7 covers one bf16 rounding on each side (2^-9 each) plus FP32 rounding of
the scaled partial sums; 1e-4*MAG bounds the FP32 accumulation error relative
to the magnitudes that cancel.  Rows and columns the call must not write
(padding rows, rows past masked_m, bytes around D) are compared bit-exactly
against their sentinel.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FBF  # a NaN pattern the kernels never produce


@pytest.fixture(scope="module")
def dgm():
    from moe_grouped_gemm_weight_b200 import build
    build.build()
    import moe_grouped_gemm_weight_b200 as dg
    dg.dg_set_num_sms(0)
    assert dg.dg_get_device_error() == 0
    return dg


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_close(gpu_bits, ref_bits, mag, what=""):
    g = bf16_bits_to_f64(gpu_bits)
    r = bf16_bits_to_f64(ref_bits)
    tol = 2.0 ** -7 * np.abs(r) + 1e-4 * mag
    bad = ~(np.abs(g - r) <= tol)
    if bad.any():
        i = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first {i.tolist()}: "
                             f"gpu={g[bad][:5]} ref={r[bad][:5]} mag={mag[bad][:5]}")


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def sample_rows(M, n_random=24, seed=0, extra=()):
    rng = np.random.default_rng(seed)
    base = {0, 1, 63, 64, 127, 128, 129, M - 1, M - 2} | set(extra)
    base |= set(rng.integers(0, M, n_random).tolist())
    return np.array(sorted(r for r in base if 0 <= r < M), dtype=np.int64)


def run_dense(dg, c: wl.Case, guard=256):
    cg = c.to("cuda")
    buf = torch.full((c.M * c.N + 2 * guard,), SENTINEL, dtype=torch.int16, device="cuda")
    D = buf[guard:guard + c.M * c.N].view(torch.bfloat16).view(c.M, c.N)
    dg.dg_fp8_gemm_nt(D, cg.A, cg.sa, cg.sa_stride, cg.B, cg.sb)
    torch.cuda.synchronize()
    b = _bits(buf)
    assert np.all(b[:guard] == SENTINEL) and np.all(b[-guard:] == SENTINEL), "write outside D"
    return b[guard:guard + c.M * c.N].reshape(c.M, c.N)


def oracle_dense(c: wl.Case, rows=None):
    D, _, MAG = oracle.gemm_nt(c.A.numpy(), c.sa.numpy(), c.sa_stride, c.B.numpy(), c.sb.numpy(),
                               c.M, c.N, c.K, rows=rows, want_d64=False)
    return D, MAG


# --------------------------------------------------------------- dense -----

# ... plus the narrowest output the layout allows (N = 8: one 16-byte row of
# D) on the few-row kernel and on the 128-row tile kernel.
DENSE_SMALL = [(1, 64, 128), (64, 64, 256), (127, 200, 384), (128, 128, 128), (129, 136, 512),
               (300, 264, 1024), (256, 520, 640), (513, 1032, 256), (64, 2112, 7168), (1, 8, 128),
               (300, 8, 256)]


@pytest.mark.parametrize("M,N,K", DENSE_SMALL)
def test_dense_small_full(dgm, M, N, K):
    c = wl.dense_case(M, N, K, seed=M * 7 + N + K)
    got = run_dense(dgm, c)
    ref, mag = oracle_dense(c)
    assert_close(got, ref, mag, f"dense {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", wl.DENSE_SWEEP)
def test_dense_sweep_sampled(dgm, M, N, K):
    c = wl.dense_case(M, N, K, seed=0, device="cuda").to("cpu")
    got = run_dense(dgm, c)
    rows = sample_rows(M, seed=M + N)
    ref, mag = oracle_dense(c, rows=rows)
    assert_close(got[rows], ref[rows], mag[rows], f"dense sweep {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", wl.STRESS_SHAPES)
def test_stress_sampled(dgm, M, N, K):
    c = wl.dense_case(M, N, K, seed=0, stress=True, device="cuda").to("cpu")
    got = run_dense(dgm, c)
    rows = sample_rows(M, n_random=16, seed=3)
    ref, mag = oracle_dense(c, rows=rows)
    assert_close(got[rows], ref[rows], mag[rows], f"stress {M}x{N}x{K}")


def test_dense_is_deterministic(dgm):
    c = wl.dense_case(300, 264, 1024, seed=2)
    a = run_dense(dgm, c)
    b = run_dense(dgm, c)
    assert np.array_equal(a, b)


def test_dense_with_few_sms(dgm):
    c = wl.dense_case(300, 520, 512, seed=4)
    try:
        dgm.dg_set_num_sms(3)
        got = run_dense(dgm, c)
    finally:
        dgm.dg_set_num_sms(0)
    ref, mag = oracle_dense(c)
    assert_close(got, ref, mag, "dense, 3 SMs")


# ---------------------------------------------------------- contiguous -----

def run_contiguous(dg, c: wl.Case):
    cg = c.to("cuda")
    D = torch.full((c.M, c.N), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    dg.dg_grouped_contiguous_nt(D, cg.A, cg.sa, cg.sa_stride, cg.B, cg.sb, cg.m_indices)
    torch.cuda.synchronize()
    return _bits(D)


def oracle_contiguous(c: wl.Case, rows=None):
    D, _, MAG = oracle.grouped_contiguous(c.A.numpy(), c.sa.numpy(), c.sa_stride, c.B.numpy(), c.sb.numpy(),
                                          c.m_indices.numpy(), c.M, c.N, c.K, c.G, rows=rows, want_d64=False)
    return D, MAG


@pytest.mark.parametrize("group_rows,N,K", [([3, 130, 0, 5, 256], 264, 384), ([128], 64, 128),
                                            ([1, 1, 1], 136, 256)])
def test_contiguous_small_full(dgm, group_rows, N, K):
    c = wl.contiguous_case(group_rows, N, K, seed=len(group_rows) + N)
    got = run_contiguous(dgm, c)
    idx = c.m_indices.numpy()
    assert np.all(got[idx < 0] == SENTINEL), "padding rows were written"
    ref, mag = oracle_contiguous(c)
    v = idx >= 0
    assert_close(got[v], ref[v], mag[v], "contiguous small")


@pytest.mark.parametrize("group_rows", [[8192] * 4, [1000, 3000, 37, 4155]])
def test_contiguous_full_size_sampled(dgm, group_rows):
    c = wl.contiguous_case(group_rows, 4096, 7168, seed=0, device="cuda").to("cpu")
    got = run_contiguous(dgm, c)
    idx = c.m_indices.numpy()
    assert np.all(got[idx < 0] == SENTINEL), "padding rows were written"
    bounds = np.cumsum([0] + [-(-r // 128) * 128 for r in group_rows])
    extra = [b for b in bounds[:-1]] + [b - 1 for b in bounds[1:]]
    rows = sample_rows(c.M, seed=5, extra=extra)
    ref, mag = oracle_contiguous(c, rows=rows)
    v = rows[idx[rows] >= 0]
    assert_close(got[v], ref[v], mag[v], "contiguous full size")


def test_contiguous_bad_index_is_flagged_and_skipped(dgm):
    c = wl.contiguous_case([128, 128], 64, 128, seed=9)
    c.m_indices[5] = 7  # outside [-1, G)
    got = run_contiguous(dgm, c)
    assert dgm.dg_get_device_error() & dgm.DG_DEVERR_BAD_M_INDEX
    assert np.all(got[5] == SENTINEL)
    assert dgm.dg_get_device_error() == 0  # reading clears it


# -------------------------------------------------------------- masked -----

def run_masked(dg, c: wl.Case, expected_m=0):
    cg = c.to("cuda")
    D = torch.full((c.G, c.M, c.N), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    dg.dg_grouped_masked_nt(D, cg.A, cg.sa, cg.sa_stride, cg.B, cg.sb, cg.masked_m, expected_m)
    torch.cuda.synchronize()
    return _bits(D)


def oracle_masked(c: wl.Case, rows=None):
    D, _, MAG = oracle.grouped_masked(c.A.numpy(), c.sa.numpy(), c.sa_stride, c.B.numpy(), c.sb.numpy(),
                                      c.masked_m.numpy(), c.G, c.M, c.N, c.K, rows=rows, want_d64=False)
    return D, MAG


def check_masked_untouched(got, masked_m):
    for g, mm in enumerate(masked_m):
        assert np.all(got[g, mm:] == SENTINEL), f"group {g}: rows past masked_m were written"


# The last two: every group empty on the 128-row tile kernel (M_max > 256;
# D must stay untouched), and N = 8 on the few-row kernel.
@pytest.mark.parametrize("G,Mmax,N,K,mm", [(3, 200, 136, 256, [0, 200, 65]), (1, 5, 64, 128, [5]),
                                           (5, 130, 264, 384, [129, 1, 130, 0, 128]),
                                           (2, 300, 136, 256, [0, 0]), (2, 40, 8, 128, [40, 0])])
def test_masked_small_full(dgm, G, Mmax, N, K, mm):
    c = wl.masked_case(G, Mmax, N, K, masked_m=mm, seed=G + Mmax)
    got = run_masked(dgm, c)
    check_masked_untouched(got, mm)
    ref, mag = oracle_masked(c)
    for g in range(G):
        assert_close(got[g, :mm[g]], ref[g, :mm[g]], mag[g, :mm[g]], f"masked g={g}")


@pytest.mark.parametrize("cfg", [wl.MASKED_MAIN, wl.MASKED_SINGLE])
def test_masked_full_size_sampled(dgm, cfg):
    c = wl.masked_case(seed=0, device="cuda", **cfg).to("cpu")
    got = run_masked(dgm, c)
    mm = c.masked_m.numpy().tolist()
    check_masked_untouched(got, mm)
    rows = []
    rng = np.random.default_rng(7)
    for g, m in enumerate(mm):
        cand = {0, m - 1, 127, 128} | set(rng.integers(0, max(m, 1), 6).tolist())
        rows += [g * c.M + r for r in cand if 0 <= r < m]
    rows = np.array(sorted(rows), dtype=np.int64)
    ref, mag = oracle_masked(c, rows=rows)
    flat_g, flat_r = got.reshape(-1, c.N), ref.reshape(-1, c.N)
    assert_close(flat_g[rows], flat_r[rows], mag.reshape(-1, c.N)[rows], "masked full size")


@pytest.mark.parametrize("hint", [1, 40, 100, 200, 1000])
def test_masked_expected_m_hint_never_changes_the_result(dgm, hint):
    # expected_m only steers the planner's tile shape; D must match the
    # unhinted call bit for bit (no K split is planned at these sizes, so
    # every element is summed in the same order), and the oracle.
    c = wl.masked_case(3, 200, 264, 512, masked_m=[0, 200, 65], seed=21)
    base = run_masked(dgm, c, 0)
    got = run_masked(dgm, c, hint)
    assert dgm.dg_get_device_error() == 0
    assert np.array_equal(got, base), f"expected_m={hint} changed D"
    ref, mag = oracle_masked(c)
    check_masked_untouched(got, [0, 200, 65])
    for g, mm in enumerate([0, 200, 65]):
        assert_close(got[g, :mm], ref[g, :mm], mag[g, :mm], f"masked hint {hint}, group {g}")


def test_masked_count_beyond_mmax_is_clamped_and_flagged(dgm):
    c = wl.masked_case(2, 64, 64, 128, masked_m=[3, 64], seed=11)
    c.masked_m[1] = 1000
    got = run_masked(dgm, c)
    assert dgm.dg_get_device_error() & dgm.DG_DEVERR_BAD_MASKED_M
    c.masked_m[1] = 64
    ref, mag = oracle_masked(c)
    assert_close(got[1], ref[1], mag[1], "clamped group")
    check_masked_untouched(got, [3, 64])


def test_masked_under_cuda_graph_follows_device_counts(dgm):
    c = wl.masked_case(4, 256, 256, 512, masked_m=[10, 0, 256, 129], seed=12)
    cg = c.to("cuda")
    D = torch.full((c.G, c.M, c.N), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dgm.dg_grouped_masked_nt(D, cg.A, cg.sa, cg.sa_stride, cg.B, cg.sb, cg.masked_m, 128)  # warm-up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dgm.dg_grouped_masked_nt(D, cg.A, cg.sa, cg.sa_stride, cg.B, cg.sb, cg.masked_m, 128)
    for counts in ([1, 2, 3, 4], [256, 0, 0, 200], [0, 0, 0, 0]):
        D.view(torch.int16).fill_(SENTINEL)
        cg.masked_m.copy_(torch.tensor(counts, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        got = _bits(D)
        check_masked_untouched(got, counts)
        c.masked_m = torch.tensor(counts, dtype=torch.int32)
        ref, mag = oracle_masked(c)
        for gi, m in enumerate(counts):
            assert_close(got[gi, :m], ref[gi, :m], mag[gi, :m], f"graph replay g={gi}")
    assert dgm.dg_get_device_error() == 0


# ------------------------------------------------- few-row (swap-AB) kernel --

@pytest.mark.parametrize("M", [1, 17, 32, 33, 64, 100, 128])
@pytest.mark.parametrize("sms", [148, 16, 3])
def test_few_rows_split_k_variants(dgm, M, sms):
    # 35 K blocks, 5 weight tiles: clusters of 7 on 148 SMs (TN = 32 or 64),
    # of 2 on 16 SMs for M <= 64, unsplit where the tiles fill the SMs.
    N, K = 520, 4480
    c = wl.dense_case(M, N, K, seed=M * 3 + sms)
    try:
        dgm.dg_set_num_sms(sms)
        plan = dgm.dg_make_plan(0, M, N, K, 1, sms)
        assert plan["swap_ab"] == 1
        want = {148: 7, 16: 2 if M <= 64 else 1, 3: 1}[sms]
        assert plan["split_k"] == want, plan
        got = run_dense(dgm, c)
    finally:
        dgm.dg_set_num_sms(0)
    ref, mag = oracle_dense(c)
    assert_close(got, ref, mag, f"few rows M={M} split={plan['split_k']}")


@pytest.mark.parametrize("K,split", [(512, 1), (1024, 1), (2048, 4), (3072, 6), (3968, 6)])
def test_few_rows_split_count_follows_k(dgm, K, split):
    # 17 weight tiles: below 16 K blocks the split does not repay its
    # reduction; above, at most 6 CTAs per cluster keep all 17 clusters
    # resident: 16, 24 and 31 blocks give 4, 6 and 6 slices (31 = 5 + 5 + 5 +
    # 5 + 5 + 6).
    c = wl.dense_case(64, 2112, K, seed=K)
    assert dgm.dg_make_plan(0, 64, 2112, K, 1, 148)["split_k"] == split
    got = run_dense(dgm, c)
    ref, mag = oracle_dense(c)
    assert_close(got, ref, mag, f"few rows K={K} split={split}")


def test_few_rows_k_split_uneven(dgm):
    # 35 K blocks over a cluster of 6 CTAs (slices of 5 and 6 blocks) and
    # 64 activation rows in slices of 10 and 11 rows per CTA: the fixed-order
    # sum must still match, and repeat bit for bit.
    c = wl.dense_case(64, 2112, 4480, seed=21)
    assert dgm.dg_make_plan(0, 64, 2112, 4480, 1, 148)["split_k"] == 6
    got = run_dense(dgm, c)
    assert np.array_equal(run_dense(dgm, c), got)
    ref, mag = oracle_dense(c)
    assert_close(got, ref, mag, "uneven split")


@pytest.mark.parametrize("M,N,K,sms", [(64, 24576, 1536, 148), (128, 4224, 1024, 20), (7, 1040, 512, 3)])
def test_few_rows_persistent_tiles(dgm, M, N, K, sms):
    # More weight tiles than SMs: single-CTA clusters walk several tiles each
    # with one operand ring across them.
    c = wl.dense_case(M, N, K, seed=M + N + sms)
    try:
        dgm.dg_set_num_sms(sms)
        plan = dgm.dg_make_plan(0, M, N, K, 1, sms)
        assert plan["split_k"] == 1 and plan["tiles"] > plan["grid"] == sms
        rows = sample_rows(M, n_random=8, seed=2)
        got = run_dense(dgm, c)
    finally:
        dgm.dg_set_num_sms(0)
    ref, mag = oracle_dense(c, rows=rows)
    assert_close(got[rows], ref[rows], mag[rows], f"persistent few rows {M}x{N}x{K} on {sms} SMs")


# ------------------------------------------- K-split of the last partial wave --

@pytest.mark.parametrize("M,N,K,sms,split", [(256, 1536, 4096, 5, 2), (384, 1792, 6144, 20, 3),
                                             (384, 1792, 8192, 20, 4)])
def test_tail_split_matches_oracle_and_is_deterministic(dgm, M, N, K, sms, split):
    c = wl.dense_case(M, N, K, seed=M + N + K + sms)
    try:
        dgm.dg_set_num_sms(sms)
        plan = dgm.dg_make_plan(0, M, N, K, 1, sms)
        assert plan["tail_split"] == split and plan["tiles"] % plan["grid"] != 0
        a = run_dense(dgm, c)
        b = run_dense(dgm, c)
    finally:
        dgm.dg_set_num_sms(0)
    assert np.array_equal(a, b)
    ref, mag = oracle_dense(c)
    assert_close(a, ref, mag, f"tail split {split}")
    assert dgm.dg_get_device_error() == 0


def test_tail_split_workspaces_stay_bounded_over_many_streams(dgm):
    # One split call on each of six fresh streams: at most four per device
    # keep a workspace (the least recently used is freed), and every stream's
    # result is the same bits as the default stream's.
    M, N, K, sms = 384, 1792, 8192, 20
    c = wl.dense_case(M, N, K, seed=77).to("cuda")
    try:
        dgm.dg_set_num_sms(sms)
        assert dgm.dg_make_plan(0, M, N, K, 1, sms)["tail_split"] > 1
        D0 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        dgm.dg_fp8_gemm_nt(D0, c.A, c.sa, c.sa_stride, c.B, c.sb)
        torch.cuda.synchronize()
        for i in range(6):
            st = torch.cuda.Stream()
            D = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
            torch.cuda.synchronize()
            with torch.cuda.stream(st):
                dgm.dg_fp8_gemm_nt(D, c.A, c.sa, c.sa_stride, c.B, c.sb)
            st.synchronize()
            assert torch.equal(D.view(torch.int16), D0.view(torch.int16)), f"stream {i}"
            assert dgm.dg_get_workspace_count() <= 4
    finally:
        dgm.dg_set_num_sms(0)
    assert dgm.dg_get_device_error() == 0


# ------------------------------------- back-to-back launches (PDL) --------
# With PDL on (the default; DG_PDL=0 turns it off) GEMM launches allow
# programmatic dependent launch: a kernel may
# start its set-up while the previous kernel in the stream finishes.  It must
# still read the inputs that kernel wrote, write D after it, and use the
# K-split workspace only after it.  Each test runs with PDL on and off.

@pytest.fixture(params=["pdl", "serial"])
def pdl_mode(request, monkeypatch):
    monkeypatch.setenv("DG_PDL", "1" if request.param == "pdl" else "0")
    yield request.param

def _fill_from(dst: wl.Case, src: wl.Case):
    for k in ("A", "sa", "B", "sb"):
        getattr(dst, k).copy_(getattr(src, k))


@pytest.mark.parametrize("M,N,K", [(64, 2112, 1024), (4096, 1024, 1024)])
def test_inputs_written_just_before_the_gemm_are_seen(dgm, pdl_mode, M, N, K):
    c1, c2 = wl.dense_case(M, N, K, seed=11), wl.dense_case(M, N, K, seed=12)
    g1, g2 = c1.to("cuda"), c2.to("cuda")
    work = wl.dense_case(M, N, K, seed=13).to("cuda")  # operand buffers rewritten before each call
    D = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    for _ in range(3):  # no synchronisation between the kernels
        _fill_from(work, g1)
        dgm.dg_fp8_gemm_nt(D, work.A, work.sa, work.sa_stride, work.B, work.sb)
        _fill_from(work, g2)
        dgm.dg_fp8_gemm_nt(D, work.A, work.sa, work.sa_stride, work.B, work.sb)
    torch.cuda.synchronize()
    rows = sample_rows(M, n_random=8, seed=4)
    ref, mag = oracle_dense(c2, rows=rows)
    assert_close(_bits(D)[rows], ref[rows], mag[rows], f"last of back-to-back GEMMs {M}x{N}x{K}")


def test_back_to_back_k_split_gemms_share_the_workspace(dgm, pdl_mode):
    # Tail-split launches back to back on one stream (distinct inputs and
    # outputs): each publishes partials to the same workspace only after the
    # previous launch has finished with it.
    M, N, K, sms = 384, 1792, 8192, 20
    cases = [wl.dense_case(M, N, K, seed=40 + i) for i in range(3)]
    gs = [c.to("cuda") for c in cases]
    Ds = [torch.empty(M, N, dtype=torch.bfloat16, device="cuda") for _ in cases]
    try:
        dgm.dg_set_num_sms(sms)
        assert dgm.dg_make_plan(0, M, N, K, 1, sms)["tail_split"] > 1
        for _ in range(2):
            for g, D in zip(gs, Ds):
                dgm.dg_fp8_gemm_nt(D, g.A, g.sa, g.sa_stride, g.B, g.sb)
        torch.cuda.synchronize()
    finally:
        dgm.dg_set_num_sms(0)
    for c, D in zip(cases, Ds):
        ref, mag = oracle_dense(c)
        assert_close(_bits(D), ref, mag, "back-to-back tail split")
    assert dgm.dg_get_device_error() == 0


def test_back_to_back_launches_in_a_cuda_graph(dgm, pdl_mode):
    M, N, K = 64, 2112, 1024
    c1, c2 = wl.dense_case(M, N, K, seed=21), wl.dense_case(M, N, K, seed=22)
    g1, g2 = c1.to("cuda"), c2.to("cuda")
    work = wl.dense_case(M, N, K, seed=23).to("cuda")
    D1 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    D2 = torch.empty_like(D1)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dgm.dg_fp8_gemm_nt(D1, work.A, work.sa, work.sa_stride, work.B, work.sb)  # first call on s
    s.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        _fill_from(work, g1)
        dgm.dg_fp8_gemm_nt(D1, work.A, work.sa, work.sa_stride, work.B, work.sb)
        _fill_from(work, g2)
        dgm.dg_fp8_gemm_nt(D2, work.A, work.sa, work.sa_stride, work.B, work.sb)
    for _ in range(2):
        with torch.cuda.stream(s):
            graph.replay()
    torch.cuda.synchronize()
    for c, D in ((c1, D1), (c2, D2)):
        ref, mag = oracle_dense(c)
        assert_close(_bits(D), ref, mag, "graph back-to-back")
