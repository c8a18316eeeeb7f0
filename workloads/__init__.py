"""Seeded synthetic inputs for the FP8 block-scaled NT GEMM.

This module is the one piece that both the CUDA path's tests/benchmarks and the
CPU oracle consume: it draws random activations and weights and quantises them
to e4m3 codes with FP32 scales, 1x128 per activation row tile and 128x128 per
weight block (the granularity the DeepGEMM pages fix; casting itself is left to
the caller by the README's "Interface" section, so this quantiser is an input
recipe, not part of the method).  It holds none of the GEMM's arithmetic.

Recipes (seed 0 unless stated):
  normal   A = randn(M,K); B = 0.02*randn(N,K); scale = max(amax, 1e-4)/448.
  stress   A = Student-t(nu=3) with round(1% of K) channels x100, scales are
           powers of two 2^ceil(log2(amax/448)) (UE8M0-representable).
Codes are produced by clamping x/scale to [-448, 448] and casting with
torch.float8_e4m3fn (round to nearest even), so no NaN code is ever emitted.

Layouts (the library's and the oracle's common input contract):
  A   uint8 [M,K] (or [G,Mmax,K]), K contiguous
  sa  float32, transposed: sa[kb*sa_stride + m] (masked: per group
      [nkb][sa_stride]); sa_stride = M rounded up to 4 floats (16 bytes),
      padding entries are zero
  B   uint8 [N,K] (grouped: [G,N,K])
  sb  float32 [nbn, nkb] (grouped: [G, nbn, nkb])
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch

FP8_MAX = 448.0


def cdiv(a: int, b: int) -> int:
    return (a + b - 1) // b


def sa_stride_for(m: int) -> int:
    """Row stride of the transposed sa: m rounded up to a multiple of 4 floats."""
    return cdiv(m, 4) * 4


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _scale_from_amax(amax: torch.Tensor, pow2: bool) -> torch.Tensor:
    amax = amax.clamp_min(1e-4)
    if pow2:
        return torch.exp2(torch.ceil(torch.log2(amax / FP8_MAX)))
    return amax / FP8_MAX


def _to_codes(x: torch.Tensor) -> torch.Tensor:
    q = x.clamp(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn)
    return q.view(torch.uint8)


def quantize_1x128(x: torch.Tensor, pow2: bool = False):
    """Per-row, per-128-column quantisation of x [R,K] (K % 128 == 0 or not).

    Returns (codes uint8 [R,K], scales float32 [R, ceil(K/128)])."""
    R, K = x.shape
    nkb = cdiv(K, 128)
    pad = nkb * 128 - K
    xp = torch.nn.functional.pad(x, (0, pad)) if pad else x
    xb = xp.view(R, nkb, 128)
    s = _scale_from_amax(xb.abs().amax(dim=2), pow2)
    q = _to_codes(xb / s[:, :, None]).view(R, nkb * 128)[:, :K]
    return q.contiguous(), s.float().contiguous()


def quantize_128x128(w: torch.Tensor, pow2: bool = False):
    """Per-128x128-block quantisation of w [N,K].

    Returns (codes uint8 [N,K], scales float32 [ceil(N/128), ceil(K/128)])."""
    N, K = w.shape
    nbn, nkb = cdiv(N, 128), cdiv(K, 128)
    wp = torch.nn.functional.pad(w, (0, nkb * 128 - K, 0, nbn * 128 - N))
    wb = wp.view(nbn, 128, nkb, 128)
    s = _scale_from_amax(wb.abs().amax(dim=(1, 3)), pow2)
    q = _to_codes(wb / s[:, None, :, None]).view(nbn * 128, nkb * 128)[:N, :K]
    return q.contiguous(), s.float().contiguous()


def transpose_scales(s: torch.Tensor, stride: Optional[int] = None) -> torch.Tensor:
    """[M, nkb] scales -> flat transposed layout s_t[kb*stride + m] (zero padded)."""
    M, nkb = s.shape
    stride = sa_stride_for(M) if stride is None else stride
    out = torch.zeros(nkb, stride, dtype=torch.float32, device=s.device)
    out[:, :M] = s.t()
    return out.reshape(-1).contiguous()


def _activations(M, K, g, device, stress: bool):
    if not stress:
        return torch.randn(M, K, generator=g, device=device)
    nu = 3
    z = torch.randn(M, K, generator=g, device=device)
    chi2 = (torch.randn(nu, M, K, generator=g, device=device) ** 2).sum(0)
    a = z / torch.sqrt(chi2 / nu)
    n_out = round(0.01 * K)
    ch = torch.randperm(K, generator=g, device=device)[:n_out]
    a[:, ch] *= 100.0
    return a


@dataclass
class Case:
    """One synthetic problem.  Tensors live on ``device`` given at creation."""
    mode: str                      # "dense" | "contiguous" | "masked"
    M: int                         # dense/contiguous: rows of A; masked: Mmax
    N: int
    K: int
    G: int
    A: torch.Tensor                # uint8
    sa: torch.Tensor               # float32 flat, transposed
    sa_stride: int
    B: torch.Tensor                # uint8 [G,N,K] (dense: [N,K])
    sb: torch.Tensor               # float32 [G,nbn,nkb] (dense: [nbn,nkb])
    m_indices: Optional[torch.Tensor] = None   # int32 [M] (contiguous)
    masked_m: Optional[torch.Tensor] = None    # int32 [G] (masked)
    meta: dict = field(default_factory=dict)

    @property
    def nkb(self) -> int:
        return cdiv(self.K, 128)

    @property
    def nbn(self) -> int:
        return cdiv(self.N, 128)

    def rows_computed(self) -> int:
        if self.mode == "dense":
            return self.M
        if self.mode == "contiguous":
            return int((self.m_indices >= 0).sum().item())
        return int(self.masked_m.clamp(0, self.M).sum().item())

    def groups_active(self) -> int:
        if self.mode == "dense":
            return 1
        if self.mode == "contiguous":
            return int(torch.unique(self.m_indices[self.m_indices >= 0]).numel())
        return int((self.masked_m > 0).sum().item())

    def flops(self) -> int:
        return 2 * self.rows_computed() * self.N * self.K

    def bytes(self) -> int:
        """Algorithmic bytes: A rows + active B + D + scales (+ index array)."""
        r, ga = self.rows_computed(), self.groups_active()
        b = r * self.K + ga * self.N * self.K + 2 * r * self.N
        b += 4 * r * self.nkb + 4 * ga * self.nbn * self.nkb
        if self.mode == "contiguous":
            b += 4 * self.M
        elif self.mode == "masked":
            b += 4 * self.G
        return b

    def to(self, device):
        kw = {}
        for name in ("A", "sa", "B", "sb", "m_indices", "masked_m"):
            t = getattr(self, name)
            kw[name] = None if t is None else t.to(device)
        return Case(self.mode, self.M, self.N, self.K, self.G, kw["A"], kw["sa"], self.sa_stride,
                    kw["B"], kw["sb"], kw["m_indices"], kw["masked_m"], dict(self.meta))


def dense_case(M: int, N: int, K: int, seed: int = 0, stress: bool = False,
               device="cpu") -> Case:
    g = _gen(seed, device)
    a = _activations(M, K, g, device, stress)
    w = 0.02 * torch.randn(N, K, generator=g, device=device)
    A, sa = quantize_1x128(a, pow2=stress)
    B, sb = quantize_128x128(w, pow2=stress)
    st = sa_stride_for(M)
    return Case("dense", M, N, K, 1, A, transpose_scales(sa, st), st, B, sb,
                meta={"seed": seed, "stress": stress})


def contiguous_case(group_rows: List[int], N: int, K: int, seed: int = 0, align: int = 128,
                    device="cpu") -> Case:
    """Segments of group_rows[g] real rows, each padded with -1 rows to ``align``."""
    G = len(group_rows)
    g = _gen(seed, device)
    idx = []
    for gi, r in enumerate(group_rows):
        padded = cdiv(r, align) * align
        idx += [gi] * r + [-1] * (padded - r)
    M = len(idx)
    a = torch.randn(M, K, generator=g, device=device)
    A, sa = quantize_1x128(a)
    Bs, sbs = [], []
    for _ in range(G):
        w = 0.02 * torch.randn(N, K, generator=g, device=device)
        q, s = quantize_128x128(w)
        Bs.append(q)
        sbs.append(s)
    st = sa_stride_for(M)
    mi = torch.tensor(idx, dtype=torch.int32, device=device)
    return Case("contiguous", M, N, K, G, A, transpose_scales(sa, st), st,
                torch.stack(Bs).contiguous(), torch.stack(sbs).contiguous(), m_indices=mi,
                meta={"seed": seed, "group_rows": list(group_rows), "align": align})


def masked_case(G: int, Mmax: int, N: int, K: int, masked_m=None, seed: int = 0,
                device="cpu") -> Case:
    """masked_m: list of G counts, or None to draw uniform ints in [1, Mmax]."""
    g = _gen(seed, device)
    if masked_m is None:
        mm = torch.randint(1, Mmax + 1, (G,), generator=g, device=device).to(torch.int32)
    else:
        mm = torch.tensor(list(masked_m), dtype=torch.int32, device=device)
    a = torch.randn(G * Mmax, K, generator=g, device=device)
    A, sa = quantize_1x128(a)
    st = sa_stride_for(Mmax)
    sa_t = torch.cat([transpose_scales(sa[i * Mmax:(i + 1) * Mmax], st) for i in range(G)])
    Bs, sbs = [], []
    for _ in range(G):
        w = 0.02 * torch.randn(N, K, generator=g, device=device)
        q, s = quantize_128x128(w)
        Bs.append(q)
        sbs.append(s)
    return Case("masked", Mmax, N, K, G, A.view(G, Mmax, K).contiguous(), sa_t.contiguous(), st,
                torch.stack(Bs).contiguous(), torch.stack(sbs).contiguous(), masked_m=mm,
                meta={"seed": seed})


# ---------------------------------------------------------------- configs ----

# The dense shapes of the DeepGEMM performance table (M x (N, K)).
DENSE_NK = [(2112, 7168), (24576, 1536), (32768, 512), (7168, 16384), (4096, 7168), (7168, 2048)]
DENSE_SWEEP = [(m, n, k) for m in (64, 128, 4096) for (n, k) in DENSE_NK]

# Grouped contiguous workload: 4 groups x 8192 rows, N=4096, K=7168.
CONTIGUOUS_MAIN = dict(group_rows=[8192] * 4, N=4096, K=7168)
# Masked decode workload: G=4, Mmax=256, masked_m ~ U[1,256]; and G=1, 1024 rows.
MASKED_MAIN = dict(G=4, Mmax=256, N=4096, K=7168)
MASKED_SINGLE = dict(G=1, Mmax=1024, N=4096, K=7168, masked_m=[1024])
# Stress shapes (heavy-tailed activations, power-of-two scales).
STRESS_SHAPES = [(256, 7168, 7168), (4096, 7168, 16384)]
