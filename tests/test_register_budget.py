"""Host-side check of the kernels' setmaxnreg splits against their compiled
register counts (no GPU needed).

`setmaxnreg.inc` takes registers from the pool a CTA was launched with: its
threads times the kernel's compiled registers per thread.  A split whose sum
exceeds that pool waits forever, so every kernel that rebalances registers must
be compiled with enough of them.  This test compiles the library with
`-Xptxas -v`, reads each such kernel's register count from ptxas's report, and
compares it with the split budgets, which a small host program reads from the
kernel headers themselves.  The library refuses such a build at run time as
well (DG_ERR_UNSUPPORTED before the first launch); this catches it at build
time.
"""
import os
import re
import subprocess

import pytest

from moe_grouped_gemm_weight_b200 import build as dgbuild

CSRC = os.path.join(dgbuild.ROOT, "moe_grouped_gemm_weight_b200", "csrc")

PROBE = r"""
#include <cstdio>
#include "dg_kernel.cuh"
#include "dg_kernel_ue8m0.cuh"
template <int BN> void large() {
    using C = dg::Cfg<BN>;
    std::printf("large %d %d %d %d %d %d\n", BN, int(C::kSplitRegs), C::kThreadsC, C::kRegsLow, C::kEpiWGs,
                C::kRegsHigh);
}
int main() {
    large<64>();
    large<128>();
    large<256>();
    std::printf("ue8m0 %d %d %d %d %d\n", dg::kUeThreads, dg::kUeFirstEpiWarp, dg::kUeEpiWarps, dg::kUeRegsLow,
                dg::kUeRegsHigh);
    return 0;
}
"""


@pytest.fixture(scope="module")
def budgets(tmp_path_factory):
    d = tmp_path_factory.mktemp("regprobe")
    src, exe = d / "probe.cu", d / "probe"
    src.write_text(PROBE)
    cmd = [dgbuild.nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17",
           "-I", CSRC, "-I", os.path.join(dgbuild.ROOT, "include"), str(src), "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    large, ue = {}, None
    for line in out.splitlines():
        f = line.split()
        if f[0] == "large":
            bn, split, threads, low, wgs, high = map(int, f[1:])
            large[bn] = dict(split=bool(split), threads=threads, need=128 * low + 128 * wgs * high)
        else:
            threads, first, epi, low, high = map(int, f[1:])
            assert first % 4 == 0 and epi % 4 == 0  # setmaxnreg acts on whole warpgroups
            ue = dict(threads=threads, need=32 * (first * low + epi * high))
    return large, ue


@pytest.fixture(scope="module")
def compiled_registers(tmp_path_factory):
    """{mangled kernel name: registers per thread} from a verbose build."""
    out = tmp_path_factory.mktemp("regbuild") / "libdg_probe.so"
    r = subprocess.run(dgbuild.command(out=str(out), verbose_ptxas=True), capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    regs, name = {}, None
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '(\w+)'", line)
        if m:
            name = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and name:
            regs[name] = int(m.group(1))
            name = None
    assert regs, "no ptxas register report"
    return regs


def test_large_kernel_splits_fit_the_launch_pool(budgets, compiled_registers):
    large, _ = budgets
    assert large[256]["split"] and not large[128]["split"] and not large[64]["split"]
    seen = 0
    for name, n in compiled_registers.items():
        m = re.match(r"_ZN2dg15fp8_gemm_kernelILi(\d+)E", name)
        if not m:
            continue
        b = large[int(m.group(1))]
        assert n * b["threads"] <= 65536, (name, n)
        if b["split"]:
            seen += 1
            assert n * b["threads"] >= b["need"], (name, n, b)
    assert seen >= 4  # every BN = 256 instance (dense, grouped, layouts) was checked


def test_block_scaled_kernel_split_fits_the_launch_pool(budgets, compiled_registers):
    _, ue = budgets
    names = [k for k in compiled_registers if "fp8_gemm_ue8m0_kernel" in k]
    assert len(names) == 1, names
    n = compiled_registers[names[0]]
    assert ue["need"] <= 65536
    assert n * ue["threads"] >= ue["need"], (n, ue)
