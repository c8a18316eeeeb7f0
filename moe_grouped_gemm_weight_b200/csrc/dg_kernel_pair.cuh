// dg_kernel_pair.cuh -- the large-M kernel on CTA pairs (tcgen05 cta_group::2).
//
// A thread-block cluster of two CTAs on two SMs computes a 256 x 256 output
// tile: CTA r holds rows [128r, 128r+128) of the tile's A block and of its
// FP32 results, and columns [128r, 128r+128) of the tile's B block.  The
// leader CTA (rank 0) issues tcgen05.mma.cta_group::2 with M = 256: each SM's
// tensor core multiplies its own A rows by both halves of B.  Per K block an
// SM therefore streams 16 KiB of A and 16 KiB of B (32 KiB) for a 128 x 256
// slice of work, where a single CTA needs 48 KiB -- a third less L2->SMEM and
// shared-memory operand traffic per FLOP.
//
// Everything else follows the single-CTA kernel (dg_kernel.cuh): warp 0 loads,
// warp 1 of the leader issues MMAs into one of two 256-column TMEM buffers per
// K block, warp 2 stages sa/sb, warps 4..11 of each CTA promote their 128 rows
// in FP32 registers and store bf16.  Synchronisation across the pair:
//   * both CTAs' loads complete on the leader's `full` barrier (the leader
//     arms it with the pair's byte count);
//   * the leader's MMA completion is multicast-committed to `empty` and
//     `tfull` in both CTAs;
//   * both CTAs' promotion warps release a TMEM buffer by arriving on the
//     leader's `tempty` barrier.
// No TMA load multicasts: every CTA loads only its own tiles.
#pragma once

#include "dg_kernel.cuh"

namespace dg {

constexpr int kPairBM = 256;  // rows per pair tile (128 per CTA)

// Pair tile 256 x BN: each CTA loads BN/2 rows of B.  BN = 128 keeps the
// operand bytes per FLOP of a single-CTA 128 x 256 tile but leaves four
// 128-column TMEM buffers per CTA (the MMA runs up to three K blocks ahead of
// the promotion) and 64 columns per promotion warp (one TMEM read round trip
// per K block); BN = 256 streams a third fewer bytes per FLOP with two buffers.
template <int BN>
struct PairCfg {
    static_assert(BN == 128 || BN == 256, "pair tiles are 256 x 128 or 256 x 256");
    static constexpr int kTileBBytes = (BN / 2) * kBK;               // this CTA's half of B
    static constexpr int kStageBytes = kTileABytes + kTileBBytes;
    static constexpr int kNBuf = 512 / BN;                           // TMEM buffers of BN columns
    static constexpr int kTmemCols = 512;
    static constexpr int kColsPerWarp = BN / 2;                      // two warpgroups split the columns
    static constexpr int kChunks = kColsPerWarp / 32;
    static constexpr int kBatch = 2;
    static constexpr int kReleases = 2 * kEpiWarps;                  // promotion warps of both CTAs
};

template <int BN, int STAGES>
constexpr int pair_smem_bytes() {
    return 1024 + STAGES * PairCfg<BN>::kStageBytes + kEpiWarps * kStageOutBytes + 512 +
           kScaleSlots * kScaleSlotFloats * 4 + 4 * (kMaxMaskedGroups + 1);
}

template <int BN, int MODE>
__device__ __forceinline__ Tile decode_pair_tile(const Params& p, int t, int m_blocks, const int* mb_prefix,
                                                 int rank) {
    int mb, nb;
    raster_tile(t, m_blocks, p.n_blocks, p.raster, mb, nb);
    Tile tl;
    tl.n0 = nb * BN;
    tl.valid = true;
    if (MODE == kMasked) {
        int lo = 0, hi = p.G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (mb_prefix[mid] <= mb) lo = mid; else hi = mid - 1;
        }
        tl.g = lo;
        tl.m0 = (mb - mb_prefix[lo]) * kPairBM + rank * kBM;
    } else {
        tl.g = 0;
        tl.m0 = mb * kPairBM + rank * kBM;
    }
    return tl;
}

template <int BN, int STAGES, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
fp8_gemm_pair_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmD) {
    static_assert(MODE == kDense || MODE == kMasked, "pairs need one group per 256-row tile");
    using C = PairCfg<BN>;
    constexpr int kNBuf = C::kNBuf;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + STAGES * kTileABytes;
    uint8_t* sOut = sB + STAGES * C::kTileBBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + kEpiWarps * kStageOutBytes);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + kNBuf;
    uint64_t* sfull = tempty + kNBuf;
    uint64_t* sempty = sfull + kScaleSlots;
    uint64_t* done = sempty + kScaleSlots;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* sring = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 512);
    int* mb_prefix = reinterpret_cast<int*>(sring + kScaleSlots * kScaleSlotFloats);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rank = static_cast<int>(cluster_ctarank());
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);   // leader: its producer's arrival + both CTAs' bytes
            mbar_init(empty + s, 1);  // one multicast commit per use
        }
        for (int b = 0; b < kNBuf; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, C::kReleases);  // leader: 8 promotion warps per CTA
        }
        for (int s = 0; s < kScaleSlots; ++s) {
            mbar_init(sfull + s, 32);
            mbar_init(sempty + s, kEpiWarps);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmD);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::kTmemCols);
        tmem_relinquish_pair();
    }
    // Nothing above reads or writes global data (see the single-CTA kernel).
    griddep_wait();
    griddep_launch_dependents();
    int m_blocks = p.m_blocks;
    if (MODE == kMasked) {
        for (int g = threadIdx.x; g < p.G; g += kThreads) {
            int mm = __ldg(p.masked_m + g);
            if (mm < 0 || mm > p.M) {
                if (leader) atomicOr(&g_dg_error, 4u);
                mm = min(max(mm, 0), p.M);
            }
            mb_prefix[g + 1] = (mm + kPairBM - 1) / kPairBM;
        }
        __syncthreads();
        if (warp == 0) {
            int carry = 0;
            for (int base = 0; base < p.G; base += 32) {
                const int i = base + lane;
                int v = (i < p.G) ? mb_prefix[i + 1] : 0;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, v, off);
                    if (lane >= off) v += u;
                }
                if (i < p.G) mb_prefix[i + 1] = v + carry;
                carry += __shfl_sync(0xffffffffu, v, 31);
            }
            if (lane == 0) mb_prefix[0] = 0;
        }
    }
    // Both CTAs' barriers must be initialised before either touches the other's.
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    if (MODE == kMasked) m_blocks = mb_prefix[p.G];
    const int tiles = m_blocks * p.n_blocks;
    const int nkb = p.nkb;

    if (warp < kFirstEpiWarp) {
        regs_dec<64>();
        if (warp == 0) {
            // -------------------------------------------------- producer ----
            const uint64_t pol_a = l2_policy_evict_last();
            const uint64_t pol_b = l2_policy_evict_last();
            const uint32_t full_leader = dsmem_addr(smem_u32(full), 0);
            int stage = 0, fills = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = pair; t < tiles && ok; t += num_pairs) {
                const Tile tl = decode_pair_tile<BN, MODE>(p, t, m_blocks, mb_prefix, rank);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag)) { ok = false; break; }
                    if (lane == 0) {
                        if (leader) mbar_arrive_expect_tx(full + stage, 2 * C::kStageBytes);
                        const uint32_t fb = full_leader + stage * 8;
                        if (MODE == kMasked)
                            tma_load_3d_pair(sA + stage * kTileABytes, &tmA, fb, kb * kBK, tl.m0, tl.g, pol_a);
                        else
                            tma_load_2d_pair(sA + stage * kTileABytes, &tmA, fb, kb * kBK, tl.m0, pol_a);
                        tma_load_3d_pair(sB + stage * C::kTileBBytes, &tmB, fb, kb * kBK, tl.n0 + rank * (BN / 2),
                                         tl.g, pol_b);
                    }
                    __syncwarp();
                    ++fills;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // The leader's `full` barriers count both CTAs' copies: once the
            // last phases have completed nothing is in flight for either CTA.
            if (lane == 0 && leader) {
                const int first = fills > STAGES ? fills - STAGES : 0;
                for (int i = first; i < fills; ++i)
                    mbar_wait_drain(full + (i % STAGES), static_cast<uint32_t>((i / STAGES) & 1));
            }
            __syncwarp();
        } else if (warp == 1 && leader) {
            // ---------------------------------------------- MMA (leader) ----
            constexpr uint32_t idesc = idesc_e4m3_f32(kPairBM, BN);
            int stage = 0, buf = 0;
            uint32_t phase = 0, bphase = 0;
            bool ok = true;
            for (int t = pair; t < tiles && ok; t += num_pairs) {
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(tempty + buf, bphase ^ 1u, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(full + stage, phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t a_addr = smem_u32(sA + stage * kTileABytes);
                        const uint32_t b_addr = smem_u32(sB + stage * C::kTileBBytes);
                        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
#pragma unroll
                        for (int k = 0; k < kBK / 32; ++k)
                            umma_f8_pair(d_tmem, sdesc_kmajor_sw128(a_addr + k * 32),
                                         sdesc_kmajor_sw128(b_addr + k * 32), idesc, k > 0 ? 1u : 0u);
                        umma_commit_pair_mc(empty + stage, 0x3);
                        umma_commit_pair_mc(tfull + buf, 0x3);
                    }
                    __syncwarp();
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    if (++buf == kNBuf) { buf = 0; bphase ^= 1u; }
                }
            }
            if (lane == 0) {
                umma_commit_pair(done);
                mbar_wait_drain(done, 0);
            }
            __syncwarp();
        } else if (warp == 2) {
            // -------------------------------------------- scale producer ----
            int slot = 0;
            uint32_t sphase = 0;
            const int row_limit = p.M;
            for (int t = pair; t < tiles; t += num_pairs) {
                const Tile tl = decode_pair_tile<BN, MODE>(p, t, m_blocks, mb_prefix, rank);
                const float* sa_base = p.sa + (MODE == kMasked ? static_cast<int64_t>(tl.g) * nkb * p.sa_stride : 0);
                const float* sb_g = p.sb + static_cast<int64_t>(tl.g) * p.nbn * nkb;
                const int nb = tl.n0 / 128 + (lane & 3);
                const bool nb_ok = nb < p.nbn;
                const int r4 = tl.m0 + lane * 4;
                const int left = row_limit - r4;
                const uint32_t sa_bytes = left >= 4 ? 16u : (left > 0 ? static_cast<uint32_t>(left) * 4u : 0u);
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(sempty + slot, sphase ^ 1u, abort_flag)) { ok = false; break; }
                    const uint32_t dst = smem_u32(sring + slot * kScaleSlotFloats);
                    const float* src = sa_bytes ? sa_base + static_cast<int64_t>(kb) * p.sa_stride + r4 : p.sa;
                    cp_async_16(dst + lane * 16, src, sa_bytes);
                    if (lane < 4)
                        cp_async_4(dst + (kBM + lane) * 4, nb_ok ? sb_g + static_cast<int64_t>(nb) * nkb + kb : p.sb,
                                   nb_ok ? 4u : 0u);
                    cp_async_arrive(sfull + slot);
                    if (++slot == kScaleSlots) { slot = 0; sphase ^= 1u; }
                }
                if (!ok) break;
            }
            asm volatile("cp.async.wait_all;" ::: "memory");
        }
    } else {
        // ------------------------------------------ promotion + epilogue ----
        regs_inc<216>();
        const int ew = warp - kFirstEpiWarp;
        const int half = ew >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int col0 = half * C::kColsPerWarp;
        const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        int buf = 0, slot = 0;
        uint32_t bphase = 0, sphase = 0;
        bool ok = true;
        for (int t = pair; t < tiles && ok; t += num_pairs) {
            const Tile tl = decode_pair_tile<BN, MODE>(p, t, m_blocks, mb_prefix, rank);
            const int g = tl.g;
            const uint32_t tempty_leader = dsmem_addr(smem_u32(tempty), 0);
            const int row = tl.m0 + r;
            bool row_ok;
            int64_t d_row;
            if (MODE == kMasked) {
                const int mm = min(max(__ldg(p.masked_m + g), 0), p.M);
                row_ok = row < mm;
                d_row = static_cast<int64_t>(g) * p.M + row;
            } else {
                row_ok = row < p.M;
                d_row = row;
            }
            int sb_sel[C::kChunks];
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c) sb_sel[c] = (tl.n0 + col0 + c * 32) / 128 - tl.n0 / 128;

            float2 acc[C::kColsPerWarp / 2];
#pragma unroll
            for (int j = 0; j < C::kColsPerWarp / 2; ++j) acc[j] = make_float2(0.f, 0.f);

            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(sfull + slot, sphase, abort_flag)) { ok = false; break; }
                const float* sc = sring + slot * kScaleSlotFloats;
                const float s_a = sc[r];
                float2 s2[C::kChunks];
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c) {
                    const float s = s_a * sc[kBM + sb_sel[c]];
                    s2[c] = make_float2(s, s);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(sempty + slot);
                if (++slot == kScaleSlots) { slot = 0; sphase ^= 1u; }

                if (!mbar_wait(tfull + buf, bphase, abort_flag)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int cb = 0; cb < C::kChunks; cb += C::kBatch) {
                    uint32_t v[C::kBatch][32];
#pragma unroll
                    for (int c = 0; c < C::kBatch; ++c)
                        tmem_ld_32x32b_x32(t_lane + static_cast<uint32_t>(buf * BN + col0 + (cb + c) * 32), v[c]);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < C::kBatch; ++c) reg_fence(v[c]);
                    if (cb + C::kBatch == C::kChunks) {
                        // Last TMEM read of this buffer: release it to the leader's MMA warp.
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_remote(tempty_leader + buf * 8);
                    }
#pragma unroll
                    for (int c = 0; c < C::kBatch; ++c)
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float2 pv = make_float2(__uint_as_float(v[c][2 * j]), __uint_as_float(v[c][2 * j + 1]));
                            acc[(cb + c) * 16 + j] = __ffma2_rn(pv, s2[cb + c], acc[(cb + c) * 16 + j]);
                        }
                }
                if (++buf == kNBuf) { buf = 0; bphase ^= 1u; }
            }
            if (!ok) break;

            // Epilogue (as in the single-CTA kernel).
            const bool clip_ok = row_ok || MODE == kDense || (MODE == kMasked && row >= p.M);
            if (__all_sync(0xffffffffu, clip_ok)) {
                const uint32_t stg = smem_u32(sOut + ew * kStageOutBytes);
#pragma unroll
                for (int pc = 0; pc < C::kColsPerWarp / 32; ++pc) {
                    if (lane == 0) bulk_wait_read<0>();
                    __syncwarp();
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        __nv_bfloat162 h0 = __float22bfloat162_rn(acc[pc * 16 + q * 4 + 0]);
                        __nv_bfloat162 h1 = __float22bfloat162_rn(acc[pc * 16 + q * 4 + 1]);
                        __nv_bfloat162 h2 = __float22bfloat162_rn(acc[pc * 16 + q * 4 + 2]);
                        __nv_bfloat162 h3 = __float22bfloat162_rn(acc[pc * 16 + q * 4 + 3]);
                        const uint32_t off = lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4);
                        st_shared_v4(stg + off, *reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                                     *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    const int x = tl.n0 + col0 + pc * 32;
                    if (lane == 0 && x < p.N) {
                        if (MODE == kMasked)
                            tma_store_3d(&tmD, sOut + ew * kStageOutBytes, x, tl.m0 + quarter * 32, g);
                        else
                            tma_store_2d(&tmD, sOut + ew * kStageOutBytes, x, tl.m0 + quarter * 32);
                        bulk_commit();
                    }
                }
            } else if (row_ok) {
                uint16_t* drow = p.D + d_row * p.N;
#pragma unroll
                for (int q = 0; q < C::kColsPerWarp / 8; ++q) {
                    const int col = tl.n0 + col0 + q * 8;
                    if (col < p.N) {
                        uint4 pk;
                        __nv_bfloat162 h0 = __float22bfloat162_rn(acc[q * 4 + 0]);
                        __nv_bfloat162 h1 = __float22bfloat162_rn(acc[q * 4 + 1]);
                        __nv_bfloat162 h2 = __float22bfloat162_rn(acc[q * 4 + 2]);
                        __nv_bfloat162 h3 = __float22bfloat162_rn(acc[q * 4 + 3]);
                        pk.x = *reinterpret_cast<uint32_t*>(&h0);
                        pk.y = *reinterpret_cast<uint32_t*>(&h1);
                        pk.z = *reinterpret_cast<uint32_t*>(&h2);
                        pk.w = *reinterpret_cast<uint32_t*>(&h3);
                        *reinterpret_cast<uint4*>(drow + col) = pk;
                    }
                }
            }
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    // Neither CTA may leave while the other can still signal its barriers or
    // its tensor core can still write this CTA's TMEM.
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::kTmemCols);
    }
}

}  // namespace dg
