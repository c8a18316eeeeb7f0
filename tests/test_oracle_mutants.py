"""Plant plausible mistakes in a copy of the oracle and check the pins catch them.

Each mutant is one textual change to oracle/dg_oracle.c, compiled on the CPU
into a temporary library; the pin suite (tests/test_oracle_pins.py) is then
run against it in a subprocess and must fail.  The real oracle is untouched.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dg_oracle.c")

MUTANTS = {
    "sb_index_transposed": ("sb[(int64_t)nb * nkb + kb]", "sb[(int64_t)kb * nkb + nb]"),
    "sb_block_ignored": ("int nb = n / 128;", "int nb = 0;"),
    "k_tail_dropped": ("int k1 = k0 + 128 < K ? k0 + 128 : K;", "int k1 = k0 + 128 < K ? k0 + 128 : k0;"),
    "b_transposed": ("double t = g_e4m3[a[k]] * g_e4m3[bn[k]];",
                     "double t = g_e4m3[a[k]] * g_e4m3[b[(int64_t)k * N + n]];"),
    "bf16_truncates": ("if (frac > 0.5)", "if (frac > 2.0)"),
    "e4m3_bias_8": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "sa_not_transposed": ("sa_m[(int64_t)kb * sa_stride]", "sa_m[kb]"),
    "products_lose_sign": ("p += t;", "p += fabs(t);"),
    "contiguous_ignores_group": ("B + (int64_t)g * N * K, sb + (int64_t)g * nbn * nkb, N, K,\n                 D + m * N",
                                 "B, sb, N, K,\n                 D + m * N"),
    "mag_unscaled": ("acc_mag += fabs(s) * pmag;", "acc_mag += pmag;"),
    "mag_doubled": ("acc_mag += fabs(s) * pmag;", "acc_mag += 2.0 * fabs(s) * pmag;"),
    "mag_signed_products": ("pmag += fabs(t);", "pmag += t;"),
    "masked_off_by_one": ("if (m >= masked_m[g]) continue;", "if (m > masked_m[g]) continue;"),
    "cast_ties_away": ("if (rem > 0.5 || (rem == 0.5 && fmod(f, 2.0) == 1.0)) f += 1.0;", "if (rem >= 0.5) f += 1.0;"),
    "cast_sign_lost": ("const uint8_t sign = signbit(x) ? 0x80 : 0x00;", "const uint8_t sign = 0x00;"),
    "cast_no_floor": ("amax = fmaxf(amax, 1e-4f);", "amax = fmaxf(amax, 0.0f);"),
    "cast_no_saturation": ("if (a >= 448.0) return sign | 0x7E;", "if (a >= 1e30) return sign | 0x7E;"),
    "cast_half_tile_amax": ("for (int k = c0; k < c0 + 128; ++k) amax = fmaxf",
                            "for (int k = c0; k < c0 + 64; ++k) amax = fmaxf"),
    "e4m3_subnormal_scale": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "bf16_ties_away": ("r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;", "r = fl + 1.0;"),
    "bf16_no_subnormal_spacing": ("if (q < -133) q = -133;", "if (q < -126) q = -126;"),
    "masked_sa_ignores_group": ("const float* sa_m = sa + (int64_t)g * nkb * sa_stride + m;",
                                "const float* sa_m = sa + m;"),
    "masked_b_ignores_group": ("B + (int64_t)g * N * K, sb + (int64_t)g * nbn * nkb, N, K,\n                 D + flat * N",
                               "B, sb, N, K,\n                 D + flat * N"),
    "cast_subnormal_scale": ("return sign | (uint8_t)(v / ldexp(1.0, -9));", "return sign | (uint8_t)(v / ldexp(1.0, -10));"),
    "cast_exponent_bias": ("return sign | (uint8_t)(((E2 + 7) << 3) | mant);", "return sign | (uint8_t)(((E2 + 8) << 3) | mant);"),
    "cast_sa_not_transposed": ("cast_tile(X, K, m, m + 1, kb * 128, Q, sa + (int64_t)kb * sa_stride + m);",
                               "cast_tile(X, K, m, m + 1, kb * 128, Q, sa + (int64_t)m * nkb + kb);"),
}


def _run_mutant(name: str, workdir: str):
    """Compile mutant `name` and run the pin suite against it; returns
    (pin suite exit code, tail of its output)."""
    old, new = MUTANTS[name]
    src = open(SRC).read()
    if src.count(old) != 1:
        return None, f"mutation site for {name} not found exactly once"
    mut = os.path.join(workdir, f"{name}.c")
    so = os.path.join(workdir, f"lib{name}.so")
    with open(mut, "w") as f:
        f.write(src.replace(old, new))
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
                    mut, "-o", so, "-lm"], check=True)
    env = dict(os.environ, DG_ORACLE_SO=so, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    """Every mutant's pin-suite run, four at a time (each run is its own
    process with two OpenMP threads)."""
    workdir = str(tmp_path_factory.mktemp("mutants"))
    with ThreadPoolExecutor(max_workers=4) as ex:
        futs = {n: ex.submit(_run_mutant, n, workdir) for n in sorted(MUTANTS)}
        return {n: f.result() for n, f in futs.items()}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, mutant_results):
    code, out = mutant_results[name]
    assert code is not None, out
    assert code != 0, f"mutant {name} passed every pin:\n{out}"
