"""Multi-GPU partitions of the GEMM: which slice of one problem each rank owns.

The GEMM needs no exchange while it runs.  A dense problem is split along N:
every rank holds all of A and sa, its own rows of B with the matching rows of
sb, and writes its own columns of D.  The boundaries fall on multiples of 128
so that each rank's columns use whole 128 x 128 scale blocks of B (column n
uses sb[n // 128]).  The grouped forms are split by expert: each rank owns a
contiguous range of groups (B[g] and sb[g] of those groups, and the rows of A
and D that belong to them), balanced by rows.  Only a caller that needs the
whole of D on one rank adds a collective, after the GEMMs: an all-gather.

This module is host logic only: index ranges, views and the reassembly after
the all-gather.  The arithmetic is the library's (or whatever ``gemm`` callable
a caller passes, e.g. a test's reference).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence, Tuple

import torch

BLOCK = 128  # scale block of B along N (and of A along K)


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


def n_shards(N: int, world: int) -> List[Tuple[int, int]]:
    """Column ranges [n0, n1) of D for each rank: whole 128-column blocks,
    as even as the blocks allow (the first ranks take one block more); the
    last nonempty range ends at N.  Ranks beyond the number of blocks get an
    empty range."""
    if N <= 0 or world <= 0:
        raise ValueError(f"N={N} and world={world} must be positive")
    blocks = _cdiv(N, BLOCK)
    out, b0 = [], 0
    for r in range(world):
        nb = blocks // world + (1 if r < blocks % world else 0)
        n0, n1 = min(b0 * BLOCK, N), min((b0 + nb) * BLOCK, N)
        out.append((n0, n1))
        b0 += nb
    return out


def expert_shards(group_rows: Sequence[int], world: int) -> List[Tuple[int, int]]:
    """Contiguous group ranges [g0, g1) per rank, balanced by rows: rank r
    takes groups until the running row count reaches (r+1)/world of the total.
    Every group goes to exactly one rank; ranks may be empty."""
    G = len(group_rows)
    if world <= 0:
        raise ValueError("world must be positive")
    if any(r < 0 for r in group_rows):
        raise ValueError("group row counts must be non-negative")
    total = sum(group_rows)
    out, g, acc = [], 0, 0
    for r in range(world):
        g0 = g
        target = total * (r + 1) / world
        if r == world - 1:
            g = G
        else:
            while g < G and (acc + group_rows[g] <= target or g == g0 and acc < target):
                acc += group_rows[g]
                g += 1
        out.append((g0, g))
    return out


@dataclass
class DenseShard:
    """Rank's part of a dense problem D[M, N] = A . B^T (scaled)."""
    n0: int
    n1: int
    B: torch.Tensor    # rows [n0, n1) of B
    sb: torch.Tensor   # rows [n0 // 128, ceil(n1 / 128)) of sb

    @property
    def N(self) -> int:
        return self.n1 - self.n0


def dense_shard(B: torch.Tensor, sb: torch.Tensor, rank: int, world: int) -> DenseShard:
    """Views of this rank's rows of B [N, K] and sb [ceil(N/128), K/128]."""
    N = B.shape[0]
    n0, n1 = n_shards(N, world)[rank]
    return DenseShard(n0, n1, B[n0:n1], sb[n0 // BLOCK:_cdiv(n1, BLOCK)])


def gather_columns(d_local: torch.Tensor, N: int, world: int, group=None) -> torch.Tensor:
    """All-gather every rank's column slice D[:, n0:n1] and reassemble D [M, N].

    Slices have different widths when N is not a multiple of 128 * world; each
    is padded to the widest before the all-gather and cut back after."""
    import torch.distributed as dist
    shards = n_shards(N, world)
    width = max(n1 - n0 for n0, n1 in shards)
    M = d_local.shape[0]
    pad = torch.zeros(M, width, dtype=d_local.dtype, device=d_local.device)
    pad[:, :d_local.shape[1]] = d_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:, :n1 - n0] for p, (n0, n1) in zip(parts, shards)], dim=1)


def sharded_gemm_nt(A: torch.Tensor, sa: torch.Tensor, sa_stride: int, B: torch.Tensor, sb: torch.Tensor,
                    rank: int, world: int, gemm: Optional[Callable] = None, gather: bool = False, group=None):
    """This rank's columns of the dense GEMM (A, sa replicated; B, sb split
    along N).  ``gemm(D, A, sa, sa_stride, B, sb)`` computes one dense GEMM;
    the default is the library's dg_fp8_gemm_nt.  Returns (D_local [M, n1-n0],
    (n0, n1)), or the whole D [M, N] after an all-gather when ``gather``."""
    if gemm is None:
        from . import dg_fp8_gemm_nt as gemm
    M, N = A.shape[0], B.shape[0]
    sh = dense_shard(B, sb, rank, world)
    D = torch.empty(M, sh.N, dtype=torch.bfloat16, device=A.device)
    if sh.N > 0:
        gemm(D, A, sa, sa_stride, sh.B, sh.sb)
    if gather:
        return gather_columns(D, N, world, group=group), (sh.n0, sh.n1)
    return D, (sh.n0, sh.n1)


@dataclass
class ContiguousShard:
    """Rank's part of a contiguous-layout grouped problem: groups [g0, g1),
    which own the rows [r0, r1) of A and D (segments are consecutive)."""
    g0: int
    g1: int
    r0: int
    r1: int
    m_indices: torch.Tensor  # rows [r0, r1), group ids shifted by -g0 (-1 stays -1)


def contiguous_shard(m_indices: torch.Tensor, G: int, rank: int, world: int) -> ContiguousShard:
    """Split by expert.  m_indices (int32 [M_total], on any device) must hold
    each group's rows as one consecutive segment in group order, with padding
    rows (-1) after a segment; a padding row goes with the segment before it.
    Raises ValueError otherwise."""
    idx = m_indices.to("cpu").tolist()
    M = len(idx)
    owner = []  # group each row belongs to, padding counted with the segment before it
    cur = -1
    starts = [None] * G
    for r, g in enumerate(idx):
        if g >= G or g < -1:
            raise ValueError(f"m_indices[{r}] = {g} outside [-1, {G})")
        if g >= 0:
            if g < cur:
                raise ValueError("groups must appear in order, each as one segment")
            if g != cur:
                if starts[g] is not None:
                    raise ValueError(f"group {g} appears in two segments")
                starts[g] = r
            cur = g
        owner.append(cur)
    rows_per_group = [0] * G
    for r, g in enumerate(idx):
        if g >= 0:
            rows_per_group[g] += 1
    g0, g1 = expert_shards(rows_per_group, world)[rank]
    sel = [r for r in range(M) if (g0 <= owner[r] < g1) or (owner[r] == -1 and g0 == 0 and g1 > 0)]
    r0, r1 = (sel[0], sel[-1] + 1) if sel else (0, 0)
    local = torch.tensor([g - g0 if g >= 0 else -1 for g in idx[r0:r1]], dtype=torch.int32)
    return ContiguousShard(g0, g1, r0, r1, local.to(m_indices.device))


@dataclass
class MaskedShard:
    """Rank's groups [g0, g1) of a masked-layout grouped problem."""
    g0: int
    g1: int


def masked_shard(expected_rows: Sequence[int], rank: int, world: int) -> MaskedShard:
    """Split the G groups of a masked problem by expert, balanced by the
    expected rows per group (e.g. masked_m read on the host, or M_max each)."""
    g0, g1 = expert_shards(list(expected_rows), world)[rank]
    return MaskedShard(g0, g1)


def gather_rows(d_local: torch.Tensor, counts: Sequence[int], group=None) -> torch.Tensor:
    """All-gather every rank's block of rows (rank r holds counts[r] rows) and
    concatenate them in rank order."""
    import torch.distributed as dist
    width = max(counts) if counts else 0
    tail = tuple(d_local.shape[1:])
    pad = torch.zeros((width,) + tail, dtype=d_local.dtype, device=d_local.device)
    pad[:d_local.shape[0]] = d_local
    parts = [torch.empty_like(pad) for _ in counts]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:c] for p, c in zip(parts, counts)], dim=0)
