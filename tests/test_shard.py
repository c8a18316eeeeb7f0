"""Multi-GPU partitions (moe_grouped_gemm_weight_b200.shard) on CPU.

The planner's ranges are checked for the properties the split relies on
(whole 128-column scale blocks, every column / group owned once, balance), and
world-size 2 and 3 gloo ranks each compute their part with the CPU oracle,
all-gather it and must reassemble exactly the single-process oracle result:
bit for bit, since every output element depends only on its own row of A, its
own row of B and one scale block of each."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads as wl
from moe_grouped_gemm_weight_b200 import shard


# ----------------------------------------------------------- planner -----

@pytest.mark.parametrize("N,world", [(2112, 2), (2112, 8), (128, 4), (7168, 3), (24576, 8), (200, 2), (8, 1)])
def test_n_shards_are_whole_scale_blocks_covering_n_once(N, world):
    sh = shard.n_shards(N, world)
    assert len(sh) == world
    assert sh[0][0] == 0
    for (a0, a1), (b0, b1) in zip(sh, sh[1:]):
        assert a1 == b0
    assert max(n1 for _, n1 in sh) == N
    for n0, n1 in sh:
        assert n0 % 128 == 0 and n0 <= n1
        assert n1 % 128 == 0 or n1 == N
    widths = [-(-(n1 - n0) // 128) for n0, n1 in sh]
    assert max(widths) - min(widths) <= 1


@pytest.mark.parametrize("rows,world", [([8192] * 4, 2), ([8192] * 4, 4), ([1000, 3000, 37, 4155], 2),
                                        ([5, 0, 0, 9, 1], 3), ([7], 4), ([0, 0], 2)])
def test_expert_shards_cover_groups_once_in_order(rows, world):
    sh = shard.expert_shards(rows, world)
    assert len(sh) == world and sh[0][0] == 0 and sh[-1][1] == len(rows)
    for (a0, a1), (b0, b1) in zip(sh, sh[1:]):
        assert a1 == b0 and a0 <= a1
    total = sum(rows)
    if total and world <= len(rows):
        # no rank holds more than its share plus one group
        for g0, g1 in sh:
            assert sum(rows[g0:g1]) <= total / world + max(rows)


def test_contiguous_shard_shifts_group_ids_and_keeps_padding():
    c = wl.contiguous_case([130, 3, 0, 260], N=8, K=128, seed=1)
    idx = c.m_indices
    s0 = shard.contiguous_shard(idx, c.G, 0, 2)
    s1 = shard.contiguous_shard(idx, c.G, 1, 2)
    assert s0.r0 == 0 and s0.r1 == s1.r0 and s1.r1 == c.M
    glob = idx.tolist()
    for s in (s0, s1):
        loc = s.m_indices.tolist()
        assert loc == [g - s.g0 if g >= 0 else -1 for g in glob[s.r0:s.r1]]
        assert all(-1 <= g < s.g1 - s.g0 for g in loc)


def test_contiguous_shard_rejects_interleaved_groups():
    with pytest.raises(ValueError):
        shard.contiguous_shard(torch.tensor([0, 1, 0], dtype=torch.int32), 2, 0, 2)


# -------------------------------------------- gloo ranks with the oracle --

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_gemm(D, A, sa, sa_stride, B, sb):
    bits, _, _ = oracle.gemm_nt(A.numpy(), sa.numpy(), sa_stride, B.contiguous().numpy(), sb.contiguous().numpy(),
                                A.shape[0], B.shape[0], A.shape[1], want_d64=False, want_mag=False)
    D.view(torch.int16).copy_(torch.from_numpy(bits.view(np.int16)))


def _i32(d_bf16: torch.Tensor) -> torch.Tensor:
    return d_bf16.view(torch.int16).to(torch.int32) & 0xFFFF


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), OMP_NUM_THREADS="1")
    import torch.distributed as dist
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        out = {}
        # dense: N split in whole 128-column blocks, A and sa replicated
        c = wl.dense_case(5, 2112, 256, seed=3)
        d_local, (n0, n1) = shard.sharded_gemm_nt(c.A, c.sa, c.sa_stride, c.B, c.sb, rank, world,
                                                  gemm=_oracle_gemm)
        # gloo has no 16-bit integer all-gather: move the bf16 bit patterns as int32
        out["dense"] = shard.gather_columns(_i32(d_local), c.N, world).numpy().astype(np.uint16)
        # contiguous: split by expert, each rank its groups' rows
        cc = wl.contiguous_case([200, 3, 0, 390], N=136, K=256, seed=4)
        s = shard.contiguous_shard(cc.m_indices, cc.G, rank, world)
        nkb = cc.K // 128
        rows = s.r1 - s.r0
        sa_full = cc.sa.view(nkb, cc.sa_stride)
        sa_loc = torch.zeros(nkb, max(4, -(-rows // 4) * 4), dtype=torch.float32)
        sa_loc[:, :rows] = sa_full[:, s.r0:s.r1]
        Bg = cc.B.view(cc.G, cc.N, cc.K)[s.g0:s.g1].contiguous()
        sbg = cc.sb.view(cc.G, -1)[s.g0:s.g1].contiguous()
        D0 = np.full((rows, cc.N), 0x7FBF, dtype=np.uint16)
        if rows and s.g1 > s.g0:
            D0, _, _ = oracle.grouped_contiguous(cc.A[s.r0:s.r1].numpy(), sa_loc.reshape(-1).numpy(), sa_loc.shape[1],
                                                 Bg.numpy(), sbg.numpy(), s.m_indices.numpy(), rows, cc.N, cc.K,
                                                 s.g1 - s.g0, D=D0, want_d64=False, want_mag=False)
        counts = [shard.contiguous_shard(cc.m_indices, cc.G, r, world) for r in range(world)]
        out["contiguous"] = shard.gather_rows(torch.from_numpy(D0.astype(np.int32)),
                                              [x.r1 - x.r0 for x in counts]).numpy().astype(np.uint16)
        # masked: split by expert over the groups
        mc = wl.masked_case(5, 40, 136, 256, masked_m=[40, 0, 17, 33, 1], seed=5)
        ms = shard.masked_shard(mc.masked_m.tolist(), rank, world)
        G_l = ms.g1 - ms.g0
        Dm = np.full((G_l, mc.M, mc.N), 0x7FBF, dtype=np.uint16)
        if G_l:
            sa_g = mc.sa.view(mc.G, -1)[ms.g0:ms.g1].contiguous()
            Dm, _, _ = oracle.grouped_masked(mc.A.view(mc.G, mc.M, mc.K)[ms.g0:ms.g1].contiguous().numpy(),
                                             sa_g.reshape(-1).numpy(), mc.sa_stride,
                                             mc.B.view(mc.G, mc.N, mc.K)[ms.g0:ms.g1].contiguous().numpy(),
                                             mc.sb.view(mc.G, -1)[ms.g0:ms.g1].contiguous().numpy(),
                                             mc.masked_m[ms.g0:ms.g1].numpy(), G_l, mc.M, mc.N, mc.K, D=Dm,
                                             want_d64=False, want_mag=False)
        gcounts = [shard.masked_shard(mc.masked_m.tolist(), r, world) for r in range(world)]
        out["masked"] = shard.gather_rows(torch.from_numpy(Dm.astype(np.int32)),
                                          [x.g1 - x.g0 for x in gcounts]).numpy().astype(np.uint16)
        q.put((rank, out))
    except Exception as e:  # report instead of leaving the parent waiting
        q.put((rank, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_results_reassemble_to_the_single_process_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=240) for _ in range(world))
    bad = {r: v for r, v in res.items() if isinstance(v, str)}
    assert not bad, bad
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    c = wl.dense_case(5, 2112, 256, seed=3)
    ref, _, _ = oracle.gemm_nt(c.A.numpy(), c.sa.numpy(), c.sa_stride, c.B.numpy(), c.sb.numpy(), c.M, c.N, c.K,
                               want_d64=False, want_mag=False)
    cc = wl.contiguous_case([200, 3, 0, 390], N=136, K=256, seed=4)
    D0 = np.full((cc.M, cc.N), 0x7FBF, dtype=np.uint16)
    ref_c, _, _ = oracle.grouped_contiguous(cc.A.numpy(), cc.sa.numpy(), cc.sa_stride, cc.B.numpy(), cc.sb.numpy(),
                                            cc.m_indices.numpy(), cc.M, cc.N, cc.K, cc.G, D=D0, want_d64=False,
                                            want_mag=False)
    mc = wl.masked_case(5, 40, 136, 256, masked_m=[40, 0, 17, 33, 1], seed=5)
    Dm = np.full((mc.G, mc.M, mc.N), 0x7FBF, dtype=np.uint16)
    ref_m, _, _ = oracle.grouped_masked(mc.A.numpy(), mc.sa.numpy(), mc.sa_stride, mc.B.numpy(), mc.sb.numpy(),
                                        mc.masked_m.numpy(), mc.G, mc.M, mc.N, mc.K, D=Dm, want_d64=False,
                                        want_mag=False)
    for r in range(world):
        assert np.array_equal(res[r]["dense"], ref)
        assert np.array_equal(res[r]["contiguous"], ref_c)
        assert np.array_equal(res[r]["masked"], ref_m)
