"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test fixes the oracle to something the pages or the mathematics settle:
the e4m3 bit definition and torch's float8_e4m3fn decoder, torch's float->bf16
rounding plus the nearest/ties-to-even property, a brute-force
dequantise-then-matmul in numpy, exact integer results, linearity in one scale
block, and the grouped layouts reduced to dense GEMMs.  The shapes are chosen
so that a transposed operand, a wrong scale index (sb[kb][nb], n/128 vs m/128),
a dropped K tail or a truncating bf16 conversion each fail at least one test.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

HERE = os.path.dirname(os.path.abspath(__file__))


# ------------------------------------------------------------------ helpers --

def dequant_torch(codes) -> np.ndarray:
    """e4m3 codes -> float64 through torch's own float8_e4m3fn decoder."""
    t = torch.as_tensor(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def brute_force(case: wl.Case, g: int = 0, rows=None, with_mag: bool = False):
    """D64 by dequantising A and B (with their scales) to float64 and one matmul.

    With ``with_mag`` it also returns |A_s| @ |B_s|^T, the sum over k of the
    magnitudes of the scaled products: the tolerance term the oracle reports
    as MAG, computed here from the dequantised operands instead of per block."""
    K, N = case.K, case.N
    nkb = case.nkb
    A = case.A.numpy().reshape(-1, K)
    sa = case.sa.numpy()
    if case.mode == "masked":
        A = case.A.numpy()[g]
        sa = sa.reshape(case.G, nkb, case.sa_stride)[g].reshape(-1)
    M = A.shape[0]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    sa_mk = sa.reshape(nkb, case.sa_stride)[:, :M].T.astype(np.float64)      # [M, nkb]
    kblk = np.arange(K) // 128
    A_s = dequant_torch(A[rows]) * sa_mk[rows][:, kblk]
    B = case.B.numpy().reshape(-1, N, K)[g]
    sb = case.sb.numpy().reshape(-1, case.nbn, nkb)[g].astype(np.float64)
    nblk = np.arange(N) // 128
    B_s = dequant_torch(B) * sb[nblk][:, kblk]
    if with_mag:
        return A_s @ B_s.T, np.abs(A_s) @ np.abs(B_s).T
    return A_s @ B_s.T


def assert_mag_matches(mag, mag_ref):
    """MAG is a sum of non-negative terms in another order: equal to 1e-12 relative."""
    assert np.all(np.abs(mag - mag_ref) <= 1e-12 * mag_ref), "MAG differs from |A_s| @ |B_s|^T"


def run_dense(case: wl.Case, **kw):
    return oracle.gemm_nt(case.A.numpy(), case.sa.numpy(), case.sa_stride, case.B.numpy(),
                          case.sb.numpy(), case.M, case.N, case.K, **kw)


def assert_bf16_of(d_bits, d64_expected, rel=1e-12):
    """d_bits must be the RNE bf16 of d64_expected, allowing a one-ulp flip only
    where d64_expected sits within ``rel`` of a rounding midpoint."""
    exp_bits = oracle.bf16_rne(d64_expected)
    bad = d_bits != exp_bits
    if bad.any():
        x = d64_expected[bad]
        lo = oracle.bf16_to_f64(np.minimum(d_bits[bad], exp_bits[bad]))
        hi = oracle.bf16_to_f64(np.maximum(d_bits[bad], exp_bits[bad]))
        mid = 0.5 * (lo + hi)
        assert np.all(np.abs(x - mid) <= rel * np.abs(x) + 1e-300), "bf16 mismatch away from a tie"


# ------------------------------------------------------------------- e4m3 ----

def test_e4m3_anchor_values():
    # OCP E4M3FN: sign | 4-bit exponent, bias 7 | 3-bit mantissa; no Inf; max 448.
    d = oracle.e4m3_decode
    assert d(0x38) == 1.0            # 0 0111 000
    assert d(0x7E) == 448.0          # 0 1111 110: largest finite
    assert d(0xFE) == -448.0
    assert d(0x01) == 2.0 ** -9      # smallest subnormal
    assert d(0x07) == 7 * 2.0 ** -9  # largest subnormal
    assert d(0x08) == 2.0 ** -6      # smallest normal
    assert d(0x78) == 256.0          # 0 1111 000
    assert d(0x3F) == 1.875          # 0 0111 111
    assert d(0x00) == 0.0 and not math.copysign(1.0, d(0x00)) < 0
    assert d(0x80) == 0.0 and math.copysign(1.0, d(0x80)) < 0
    assert math.isnan(d(0x7F)) and math.isnan(d(0xFF))


def test_e4m3_table_matches_torch_float8_e4m3fn():
    table = oracle.e4m3_table()
    ref = dequant_torch(np.arange(256, dtype=np.uint8))
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(table), nan)
    assert nan.sum() == 2
    assert np.array_equal(table[~nan], ref[~nan])
    assert np.array_equal(np.signbit(table[~nan]), np.signbit(ref[~nan]))


def test_e4m3_positive_codes_strictly_increase():
    t = oracle.e4m3_table()
    assert np.all(np.diff(t[0x00:0x7F]) > 0)
    assert np.array_equal(t[0x80:0xFF], -t[0x00:0x7F])


# ------------------------------------------------------------------- bf16 ----

def test_bf16_rne_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2 ** 32, size=1_000_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    ours = oracle.bf16_rne(f.astype(np.float64))
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rne_is_nearest_with_ties_to_even_on_doubles():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(200_000) * np.exp2(rng.integers(-140, 120, 200_000))
    bits = oracle.bf16_rne(x)
    v = oracle.bf16_to_f64(bits)
    sgn = np.where(np.signbit(x), 0x8000, 0).astype(np.uint32)
    mag = bits.astype(np.uint32) & 0x7FFF
    up = oracle.bf16_to_f64((sgn | np.minimum(mag + 1, 0x7F80)).astype(np.uint16))
    dn = oracle.bf16_to_f64((sgn | np.maximum(mag.astype(np.int64) - 1, 0).astype(np.uint32)).astype(np.uint16))
    err = np.abs(x - v)
    assert np.all(err <= np.abs(x - up)) and np.all(err <= np.abs(x - dn))
    tie = (err == np.abs(x - up)) | ((err == np.abs(x - dn)) & (mag > 0))
    assert np.all((mag[tie] & 1) == 0)


def test_bf16_rne_edges():
    r = lambda x: int(oracle.bf16_rne(np.array([x]))[0])
    assert r(1.0) == 0x3F80
    assert r(1.0 + 2 ** -8) == 0x3F80                 # tie -> even (down)
    assert r(1.0 + 3 * 2 ** -8) == 0x3F82             # tie -> even (up)
    assert r(1.0 + 2 ** -8 + 2 ** -40) == 0x3F81      # just above the tie: no double rounding
    assert r(2.0 ** 128) == 0x7F80
    assert r(-(2.0 ** 128)) == 0xFF80
    maxbf = (2 - 2 ** -7) * 2.0 ** 127
    assert r(maxbf) == 0x7F7F
    assert r(maxbf + 2.0 ** 119) == 0x7F80            # halfway to 2^128, odd -> rounds up
    assert r(2.0 ** -133) == 0x0001                   # smallest subnormal
    assert r(2.0 ** -134) == 0x0000                   # tie to even (zero)
    assert r(1.5 * 2.0 ** -133) == 0x0002             # tie to even (2)
    assert (r(float("nan")) & 0x7FFF) > 0x7F80
    assert r(-0.0) == 0x8000


# ---------------------------------------------------- brute-force shapes -----

# (M, K, N): the README's 3x5 by 5x2 shape example (section on M, N and K,
# "矩阵乘法回顾"), a single-block case, and shapes with K and N tails.
BRUTE_SHAPES = [(3, 5, 2), (1, 128, 1), (2, 256, 3), (5, 384, 129), (65, 257, 130), (9, 640, 300)]


@pytest.mark.parametrize("M,K,N", BRUTE_SHAPES)
@pytest.mark.parametrize("stress", [False, True])
def test_dense_matches_bruteforce_dequantised_matmul(M, K, N, stress):
    case = wl.dense_case(M, N, K, seed=11 + M + K + N, stress=stress)
    D, D64, MAG = run_dense(case)
    ref, mag_ref = brute_force(case, with_mag=True)
    # MAG must be the scaled magnitude sum itself, pinned from both sides:
    # a MAG that lost its scales or a factor would make every tolerance
    # built on it wrong.
    assert_mag_matches(MAG, mag_ref)
    # Two FP64 summation orders differ by at most ~K*eps*sum|terms|.
    assert np.all(np.abs(D64 - ref) <= 1e-12 * MAG)
    assert_bf16_of(D, ref, rel=1e-9)
    # MAG is the sum of |scaled products|: it bounds |D64| and equals it when
    # every product has one sign.
    assert np.all(MAG >= np.abs(D64) * (1 - 1e-12))


def test_dense_distinct_scale_blocks_are_not_interchangeable():
    # One nonzero block per operand: only A block kb=2 and B rows of block nb=1.
    M, N, K = 4, 300, 384
    case = wl.dense_case(M, N, K, seed=5)
    A = case.A.clone()
    A[:, :256] = 0
    B = case.B.clone()
    B[:128] = 0
    B[256:] = 0
    sa = case.sa.clone().view(3, case.sa_stride)
    sa[2, :M] = torch.tensor([1.0, 2.0, 4.0, 8.0])
    sb = torch.tensor([[1, 1, 16.0], [1, 1, 0.5], [1, 1, 64.0]], dtype=torch.float32)
    c = wl.Case("dense", M, N, K, 1, A, sa.reshape(-1).contiguous(), case.sa_stride, B, sb)
    D, D64, _ = run_dense(c)
    ref = brute_force(c)
    np.testing.assert_allclose(D64, ref, rtol=1e-12, atol=0)
    assert np.all(D64[:, :128] == 0) and np.all(D64[:, 256:] == 0)
    assert np.any(D64[:, 128:256] != 0)


def test_integer_results_are_exact():
    rng = np.random.default_rng(3)
    M, N, K = 7, 300, 300
    ia = rng.integers(-3, 4, (M, K)) * (rng.random((M, K)) < 0.3)
    ib = rng.integers(-3, 4, (N, K)) * (rng.random((N, K)) < 0.3)
    A = torch.from_numpy(ia.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    B = torch.from_numpy(ib.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    st = wl.sa_stride_for(M)
    sa = torch.ones(3 * st, dtype=torch.float32)
    sb = torch.ones(3, 3, dtype=torch.float32)
    c = wl.Case("dense", M, N, K, 1, A, sa, st, B, sb)
    D, D64, _ = run_dense(c)
    exact = (ia @ ib.T).astype(np.int64)
    assert np.array_equal(D64, exact.astype(np.float64))
    ref_bits = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(D, ref_bits)


def test_power_of_two_scales_give_exact_sums():
    rng = np.random.default_rng(4)
    M, N, K = 5, 260, 384
    ia = rng.integers(-4, 5, (M, K))
    ib = rng.integers(-4, 5, (N, K))
    A = torch.from_numpy(ia.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    B = torch.from_numpy(ib.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    ja = rng.integers(-3, 4, (M, 3))
    jb = rng.integers(-3, 4, (3, 3))
    st = wl.sa_stride_for(M)
    sa = wl.transpose_scales(torch.from_numpy(np.exp2(ja).astype(np.float32)), st)
    sb = torch.from_numpy(np.exp2(jb).astype(np.float32))
    c = wl.Case("dense", M, N, K, 1, A, sa, st, B, sb)
    _, D64, _ = run_dense(c)
    exp = np.zeros((M, N))
    for kb in range(3):
        blk = (ia[:, kb * 128:(kb + 1) * 128] @ ib[:, kb * 128:(kb + 1) * 128].T).astype(np.float64)
        exp += np.exp2(ja[:, kb][:, None] + jb[np.arange(N) // 128, kb][None, :]) * blk
    assert np.array_equal(D64, exp)


@pytest.mark.parametrize("which", ["sa", "sb"])
def test_linearity_in_one_scale_block(which):
    rng = np.random.default_rng(6)
    M, N, K = 6, 384, 512
    ia = rng.integers(-6, 7, (M, K))
    ib = rng.integers(-6, 7, (N, K))
    A = torch.from_numpy(ia.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    B = torch.from_numpy(ib.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    st = wl.sa_stride_for(M)
    sa_mk = np.exp2(rng.integers(-2, 3, (M, 4))).astype(np.float32)
    sb = np.exp2(rng.integers(-2, 3, (3, 4))).astype(np.float32)
    base = wl.Case("dense", M, N, K, 1, A, wl.transpose_scales(torch.from_numpy(sa_mk), st), st,
                   B, torch.from_numpy(sb))
    _, D0, _ = run_dense(base)
    m, nb, kb = 4, 1, 2
    sa2, sb2 = sa_mk.copy(), sb.copy()
    if which == "sa":
        sa2[m, kb] *= 2
    else:
        sb2[nb, kb] *= 2
    c2 = wl.Case("dense", M, N, K, 1, A, wl.transpose_scales(torch.from_numpy(sa2), st), st,
                 B, torch.from_numpy(sb2))
    _, D1, _ = run_dense(c2)
    blk = (ia[:, kb * 128:(kb + 1) * 128] @ ib[:, kb * 128:(kb + 1) * 128].T).astype(np.float64)
    contrib = sa_mk[:, kb][:, None].astype(np.float64) * sb[np.arange(N) // 128, kb][None, :] * blk
    expect = np.zeros((M, N))
    if which == "sa":
        expect[m] = contrib[m]
    else:
        expect[:, nb * 128:(nb + 1) * 128] = contrib[:, nb * 128:(nb + 1) * 128]
    assert np.array_equal(D1 - D0, expect)


def test_k_tail_is_zero_extended():
    case = wl.dense_case(3, 2, 5, seed=9)
    D, D64, _ = run_dense(case)
    A = torch.zeros(3, 128, dtype=torch.uint8)
    A[:, :5] = case.A
    B = torch.zeros(2, 128, dtype=torch.uint8)
    B[:, :5] = case.B
    c = wl.Case("dense", 3, 2, 128, 1, A, case.sa, case.sa_stride, B, case.sb)
    D2, D642, _ = run_dense(c)
    assert np.array_equal(D64, D642) and np.array_equal(D, D2)


def test_nan_code_propagates_to_its_row_only():
    case = wl.dense_case(3, 4, 128, seed=10)
    case.A[1, 7] = 0x7F
    D, D64, _ = run_dense(case)
    assert np.all(np.isnan(D64[1])) and not np.any(np.isnan(D64[[0, 2]]))
    assert np.all((D[1] & 0x7FFF) > 0x7F80)


def test_row_subset_matches_full():
    case = wl.dense_case(40, 200, 256, seed=12)
    D, D64, _ = run_dense(case)
    rows = [0, 5, 39, 17]
    sentinel = np.full((40, 200), 0xBEEF, dtype=np.uint16)
    Ds, D64s, _ = run_dense(case, rows=rows, D=sentinel.copy())
    assert np.array_equal(Ds[rows], D[rows]) and np.array_equal(D64s[rows], D64[rows])
    others = np.setdiff1d(np.arange(40), rows)
    assert np.all(Ds[others] == 0xBEEF)


# ------------------------------------------------------------ grouped -------

SENT = 0xDEAD


def test_contiguous_equals_dense_per_segment_and_leaves_padding():
    case = wl.contiguous_case([3, 130, 0, 5], N=136, K=256, seed=13)
    M = case.M
    D0 = np.full((M, case.N), SENT, dtype=np.uint16)
    D, D64, MAG = oracle.grouped_contiguous(case.A.numpy(), case.sa.numpy(), case.sa_stride,
                                          case.B.numpy(), case.sb.numpy(), case.m_indices.numpy(),
                                          M, case.N, case.K, case.G, D=D0)
    idx = case.m_indices.numpy()
    assert np.all(D[idx < 0] == SENT)
    for g in range(case.G):
        rows = np.nonzero(idx == g)[0]
        if rows.size == 0:
            continue
        ref, mag_ref = brute_force(case, g=g, rows=rows, with_mag=True)
        assert_mag_matches(MAG[rows], mag_ref)
        assert np.all(np.abs(D64[rows] - ref) <= 1e-12 * MAG[rows])
        assert_bf16_of(D[rows], ref, rel=1e-9)


def test_contiguous_rejects_bad_group_index():
    case = wl.contiguous_case([2, 2], N=8, K=128, seed=14, align=4)
    mi = case.m_indices.numpy().copy()
    mi[1] = case.G
    with pytest.raises(ValueError):
        oracle.grouped_contiguous(case.A.numpy(), case.sa.numpy(), case.sa_stride, case.B.numpy(),
                                  case.sb.numpy(), mi, case.M, case.N, case.K, case.G)


def test_masked_equals_dense_on_valid_rows_and_leaves_the_rest():
    case = wl.masked_case(3, 70, 136, 256, masked_m=[0, 70, 33], seed=15)
    D0 = np.full((3, 70, case.N), SENT, dtype=np.uint16)
    D, D64, MAG = oracle.grouped_masked(case.A.numpy(), case.sa.numpy(), case.sa_stride,
                                      case.B.numpy(), case.sb.numpy(), case.masked_m.numpy(),
                                      3, 70, case.N, case.K, D=D0)
    for g, mm in enumerate([0, 70, 33]):
        assert np.all(D[g, mm:] == SENT)
        if mm:
            ref, mag_ref = brute_force(case, g=g, rows=np.arange(mm), with_mag=True)
            assert_mag_matches(MAG[g, :mm], mag_ref)
            assert np.all(np.abs(D64[g, :mm] - ref) <= 1e-12 * MAG[g, :mm])
            assert_bf16_of(D[g, :mm], ref, rel=1e-9)


def test_masked_rejects_count_beyond_mmax():
    case = wl.masked_case(2, 8, 8, 128, masked_m=[1, 9], seed=16)
    with pytest.raises(ValueError):
        oracle.grouped_masked(case.A.numpy(), case.sa.numpy(), case.sa_stride, case.B.numpy(),
                              case.sb.numpy(), case.masked_m.numpy(), 2, 8, 8, 128)


# -------------------------------------------------- measurement convention --

def _load_perf_rows():
    rows = []
    with open(os.path.join(HERE, "golden", "perf_tables.tsv")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            kind, g, m, n, k, tf, gbs, sp = line.split()
            rows.append((kind, int(g), int(m), int(n), int(k), float(tf), float(gbs)))
    return rows


def test_pages_gbps_convention_is_A_plus_B_plus_D_bytes():
    rows = _load_perf_rows()
    assert len(rows) == 28
    for kind, g, m, n, k, tf, gbs in rows:
        mt = g * m
        flops = 2.0 * mt * n * k
        byts = mt * k + g * n * k + 2 * mt * n
        pred = tf * 1e12 / flops * byts / 1e9
        assert abs(pred - gbs) <= 0.01 * gbs + 1.0, (kind, m, n, k, pred, gbs)


def test_case_bytes_adds_only_scales_and_indices():
    c = wl.dense_case(64, 256, 256, seed=0)
    base = 64 * 256 + 256 * 256 + 2 * 64 * 256
    assert base < c.bytes() <= base * 1.02


# ------------------------------------------------------------- FP8 cast --
# The cast ahead of the GEMM (activations per 1x128 tile, weights per 128x128
# block): amax = max(max|x|, 1e-4), s = amax/448, q = e4m3_rne_satfinite(x*(448/amax)).

def _finite_codes():
    return [c for c in range(256) if c not in (0x7F, 0xFF)]


def test_e4m3_encode_inverts_decode_on_every_finite_code():
    codes = np.array(_finite_codes(), dtype=np.uint8)
    vals = dequant_torch(codes).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


def test_e4m3_encode_matches_torch_cast_including_ties():
    pos = np.array(sorted(set(np.abs(dequant_torch(np.arange(0, 0x7F, dtype=np.uint8))))))
    mids = (pos[:-1] + pos[1:]) / 2  # exact ties, representable in float32
    rng = np.random.default_rng(7)
    rand = rng.uniform(-448, 448, 20000)
    small = rng.uniform(-2 ** -5, 2 ** -5, 5000)  # subnormal range
    x = np.concatenate([mids, -mids, rand, small, pos, -pos]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x), ref)


def test_e4m3_encode_saturates_and_keeps_nan():
    x = np.array([448.0, 449.0, 464.0, 1e6, np.inf, -np.inf, -1e30, np.nan], dtype=np.float32)
    assert oracle.e4m3_encode(x).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F]


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_vals(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _cast_inputs(M, K, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)) * np.exp(rng.uniform(-6, 6, (M, 1)))
    x[0, :128] = 0.0                    # an all-zero tile
    x[M - 1, 128:256] *= 1e-7           # a tile below the 1e-4 floor
    x[M // 2, 5] = 3e4                  # an outlier dominating one tile
    return _bf16_bits(x)


def _check_cast(X, Q, s_tile, tiles):
    """tiles: list of (row slice, col slice) with scale s_tile[i]."""
    xv = _bf16_vals(X)
    qv = dequant_torch(Q)
    for (rs, cs), s in zip(tiles, s_tile):
        x, q = xv[rs, cs], qv[rs, cs]
        amax = max(np.abs(x).max(), 1e-4)
        assert s == np.float32(np.float32(amax) / np.float32(448.0))
        if np.abs(x).max() >= 1e-4:
            assert np.abs(q).max() == 448.0          # the largest |x| maps to 448
        err = np.abs(s * q - x)
        assert np.all(err <= 2.0 ** -4 * np.abs(x) * (1 + 2.0 ** -20) + s * 2.0 ** -10 + np.abs(x) * 2.0 ** -20)


def test_cast_1x128_tiles_scales_and_layout():
    M, K, stride = 37, 384, 40
    X = _cast_inputs(M, K, 1)
    Q, sa = oracle.cast_1x128(X, M, K, stride)
    tiles = [(slice(m, m + 1), slice(kb * 128, kb * 128 + 128)) for m in range(M) for kb in range(K // 128)]
    scales = [sa[kb * stride + m] for m in range(M) for kb in range(K // 128)]
    _check_cast(X, Q, scales, tiles)
    pad = np.concatenate([sa[kb * stride + M:(kb + 1) * stride] for kb in range(K // 128)])
    assert np.all(pad == 0)                           # padding of sa_stride untouched


def test_cast_128x128_tiles_and_ragged_rows():
    N, K = 200, 256
    W = _cast_inputs(N, K, 2)
    Q, sb = oracle.cast_128x128(W, N, K)
    assert sb.shape == (2, 2)
    tiles = [(slice(nb * 128, min(N, nb * 128 + 128)), slice(kb * 128, kb * 128 + 128))
             for nb in range(2) for kb in range(2)]
    _check_cast(W, Q, sb.reshape(-1), tiles)


@pytest.mark.parametrize("k", [-3, 5])
def test_cast_is_invariant_under_power_of_two_scaling(k):
    M, K = 9, 256
    X = _cast_inputs(M, K, 3)
    X2 = _bf16_bits(_bf16_vals(X) * 2.0 ** k)
    assert np.array_equal(_bf16_vals(X2), _bf16_vals(X) * 2.0 ** k)  # exact in bf16
    Q, sa = oracle.cast_1x128(X, M, K, M)
    Q2, sa2 = oracle.cast_1x128(X2, M, K, M)
    keep = np.repeat((np.abs(_bf16_vals(X)).reshape(M, -1, 128).max(axis=2) * 2.0 ** min(k, 0) >= 1e-4)
                     .T.reshape(-1), 1)
    assert np.array_equal(sa2[keep], sa[keep] * np.float32(2.0 ** k))
    rows = np.repeat(keep.reshape(K // 128, M).T, 128, axis=1)
    assert np.array_equal(Q2[rows], Q[rows])


def test_cast_sign_symmetry_and_tile_independence():
    M, K = 6, 384
    X = _cast_inputs(M, K, 4)
    Q, sa = oracle.cast_1x128(X, M, K, M)
    Qn, san = oracle.cast_1x128(X ^ np.uint16(0x8000), M, K, M)
    assert np.array_equal(san, sa)
    assert np.array_equal(Qn[Q != 0], Q[Q != 0] ^ np.uint8(0x80))
    X3 = X.copy()
    X3[2, 130] = _bf16_bits(np.array([_bf16_vals(X[2:3, 130])[0] * 64 + 1.0]))[0]
    Q3, sa3 = oracle.cast_1x128(X3, M, K, M)
    changed = np.argwhere(Q3 != Q)
    assert len(changed) and np.all(changed[:, 0] == 2) and np.all((changed[:, 1] >= 128) & (changed[:, 1] < 256))
    assert [i for i in range(sa.size) if sa3[i] != sa[i]] == [1 * M + 2]


def test_cast_then_gemm_tracks_the_bf16_product():
    # The cast's sa / sb layouts must be the ones the GEMM reads: the GEMM of
    # the cast operands stays close to the FP64 product of the bf16 inputs.
    rng = np.random.default_rng(5)
    M, N, K = 24, 260, 384
    Xb = _bf16_bits(rng.standard_normal((M, K)) * np.exp(rng.uniform(-3, 3, (M, 1))))
    Wb = _bf16_bits(0.02 * rng.standard_normal((N, K)) * np.exp(rng.uniform(-2, 2, (1, K))))
    A, sa = oracle.cast_1x128(Xb, M, K, M)
    B, sb = oracle.cast_128x128(Wb, N, K)
    _, D64, _ = oracle.gemm_nt(A, sa, M, B, sb, M, N, K)
    ref = _bf16_vals(Xb) @ _bf16_vals(Wb).T
    rel = np.linalg.norm(D64 - ref) / np.linalg.norm(ref)
    assert rel < 0.05
