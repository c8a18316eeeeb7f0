// dg_kernel_ue8m0.cuh -- sm_100a dense GEMM for power-of-two scales, scaled
// inside the tensor core.
//
// When every scale is a power of two (UE8M0-representable: the FP32 value is
// 2^e, its exponent field is the UE8M0 code), the scaled sum of the method
//   D[m,n] = sum_kb sa[m,kb] * sb[n/128,kb] * sum_{k in kb} A[m,k] * B[n,k]
// is what tcgen05.mma kind::mxf8f6f4.block_scale computes when it is given
// one scale per row of A and one per column of B for every 32-wide K step:
// the product of the two scales multiplies the step's partial sum before it
// enters the FP32 accumulator in TMEM.  The 1x128 / 128x128 scales are simply
// repeated over the four K=32 steps of each 128-wide K block.  No promotion
// through registers is needed, so the accumulator stays in TMEM for a whole
// tile and the epilogue reads it once.
//
// The pages' Hopper design promotes on CUDA cores because Hopper's FP8
// tensor-core accumulation is not FP32 ("Deepseek DeepGEMM 技术原理的深入分析",
// section "技术背景与核心原理"); the later-version article on DeepGEMM
// (section 3.1) notes that on SM100 the scales are UE8M0.  This kernel is the
// SM100 path for such scales; the general FP32-scale kernels stay the default.
//
// Tiles 128 x 256, persistent CTAs of 512 threads (four warpgroups, so that
// every warpgroup executes one setmaxnreg: 56 registers for the first two,
// 200 for the epilogue's two).  The work items are those
// of the promotion kernel: whole tiles round-robin, and, when the planner asks
// for it, the tiles of the last partial wave (or all tiles, when there are
// fewer than CTAs) split into K slices whose FP32 partials slice 0 adds up.
//   warp 0      TMA producer (A 128x128 and B 256x128 per K block, 4 stages)
//   warps 1-2   MMA issuers, taking alternate K blocks (warp 1 also owns
//               TMEM); the K block that starts a group of four first copies
//               the group's scale factors from shared memory to TMEM
//               (tcgen05.cp); each K block is 4 MMAs into the one accumulator
//   warps 4-5   scale converters, taking alternate groups of four K blocks:
//               FP32 sa (128 rows) and sb (2 blocks) read from global memory,
//               UE8M0 codes written in the scale-factor layout, 8-slot ring;
//               a scale that is not a positive normal power of two sets
//               DG_DEVERR_NOT_POW2 (its code is still its exponent field, so
//               the result is wrong for it)
//   warps 8-15  epilogue: TMEM -> bf16 -> TMA store (two warpgroups of 128
//               columns; warp w reads TMEM lanes 32 * (w % 4) onwards)
//   warps 3, 6, 7 have no role.
// Scale-factor layout in shared memory (one 512-byte block per 128 rows or
// columns): the 32-bit word for row r sits at byte (r % 32) * 16 + (r / 32) * 4.
// tcgen05.cp .32x128b.warpx4 places it in TMEM column (r / 32) of lane r % 32,
// repeated in every 32-lane quarter.  Each MMA picks one byte of the word
// (sf_id); since a scale is constant over a 128-wide K block, byte j holds
// the code of the j-th K block of a group of four, and the four MMAs of that K
// block all use sf_id = j: one copy to TMEM serves four K blocks.
#pragma once

#include "dg_kernel.cuh"

namespace dg {

constexpr int kUeBN = 256;
constexpr int kUeStages = 4;
constexpr int kUeSfSlots = 8;
constexpr int kUeSfaBytes = 512;                       // 128 rows of A
constexpr int kUeSfbBytes = 1024;                      // 256 columns of B
constexpr int kUeSfSlotBytes = kUeSfaBytes + kUeSfbBytes;
constexpr int kUeSfColsPerSlot = 12;                   // TMEM: 4 (A) + 8 (B)
constexpr int kUeSfGroup = 4;                          // K blocks per scale-factor slot (one byte each)
constexpr int kUeAccCols = kUeBN;                      // one FP32 accumulator
constexpr int kUeTmemCols = 512;
constexpr int kUeFirstEpiWarp = 8;                     // warpgroups 0-1: producer, MMA, converters
constexpr int kUeEpiWarps = 8;
constexpr int kUeThreads = 32 * (kUeFirstEpiWarp + kUeEpiWarps);
static_assert(kUeFirstEpiWarp % 4 == 0 && kUeEpiWarps % 4 == 0, "setmaxnreg works on whole warpgroups");
// setmaxnreg budgets: the first two warpgroups give registers to the
// epilogue's two.  Their sum over all threads must stay within the registers
// the CTA is launched with (kUeThreads x the kernel's register count); the
// host checks the compiled count against kUeLaunchRegsNeeded before the first
// launch.
constexpr int kUeRegsLow = 56;
constexpr int kUeRegsHigh = 200;
constexpr int kUeRegsTotal = 32 * (kUeFirstEpiWarp * kUeRegsLow + kUeEpiWarps * kUeRegsHigh);
constexpr int kUeLaunchRegsNeeded = (kUeRegsTotal + kUeThreads - 1) / kUeThreads;
static_assert(kUeRegsTotal <= 65536, "register split exceeds the file");
constexpr int kUeTileBBytes = kUeBN * kBK;
static_assert(kUeAccCols + kUeSfSlots * kUeSfColsPerSlot <= kUeTmemCols, "TMEM budget");

constexpr int ue8m0_smem_bytes() {
    return 1024 + kUeStages * (kTileABytes + kUeTileBBytes) + kUeEpiWarps * kStageOutBytes +
           kUeSfSlots * kUeSfSlotBytes + 512;
}

// UE8M0 code of a positive normal power of two; anything else raises the
// error bit (and keeps its exponent field).
__device__ __forceinline__ uint32_t ue8m0_code(float v) {
    const uint32_t bits = __float_as_uint(v);
    const uint32_t e = (bits >> 23) & 0xFFu;
    if ((bits & 0x807FFFFFu) != 0u || e == 0u || e == 0xFFu) atomicOr(&g_dg_error, 8u);
    return e;
}

// Copies ring slot `slot` of the scale factors (A's 128 rows, B's two
// 128-column blocks) from shared memory to its TMEM columns.  One thread.
__device__ __forceinline__ void copy_sf_slot(const uint8_t* sSF, uint32_t tmem_base, int slot) {
    const uint32_t sf_col = tmem_base + static_cast<uint32_t>(kUeAccCols + slot * kUeSfColsPerSlot);
    const uint32_t sf_smem = smem_u32(sSF + slot * kUeSfSlotBytes);
    tmem_cp_sf_block(sf_col, sdesc_sf_block(sf_smem));
    tmem_cp_sf_block(sf_col + 4, sdesc_sf_block(sf_smem + kUeSfaBytes));
    tmem_cp_sf_block(sf_col + 8, sdesc_sf_block(sf_smem + kUeSfaBytes + 512));
}

__global__ void __launch_bounds__(kUeThreads, 1)
fp8_gemm_ue8m0_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmD) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + kUeStages * kTileABytes;
    uint8_t* sOut = sB + kUeStages * kUeTileBBytes;
    uint8_t* sSF = sOut + kUeEpiWarps * kStageOutBytes;  // 512-byte aligned
    uint64_t* full = reinterpret_cast<uint64_t*>(sSF + kUeSfSlots * kUeSfSlotBytes);
    uint64_t* empty = full + kUeStages;
    uint64_t* sf_full = empty + kUeStages;
    uint64_t* sf_empty = sf_full + kUeSfSlots;
    uint64_t* acc_full = sf_empty + kUeSfSlots;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* done = acc_empty + 1;   // [2], one per MMA warp
    uint64_t* hand = done + 2;        // [2]: MMA warp w has issued its latest K block
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(hand + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kUeStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int s = 0; s < kUeSfSlots; ++s) {
            mbar_init(sf_full + s, 1);
            mbar_init(sf_empty + s, 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kUeEpiWarps);
        for (int w2 = 0; w2 < 2; ++w2) {
            mbar_init(done + w2, 1);
            mbar_init(hand + w2, 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmD);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kUeTmemCols);
        tmem_relinquish();
    }
    griddep_wait();
    griddep_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int tiles = p.m_blocks * p.n_blocks;
    const int nkb = p.nkb;

    if (warp < kUeFirstEpiWarp) {
        regs_dec<kUeRegsLow>();
        if (warp == 0) {
            // ------------------------------------------------------ producer ----
            const uint64_t pol_a = l2_policy_evict_last();
            const uint64_t pol_b = p.b_stream ? l2_policy_evict_first() : l2_policy_evict_last();
            int stage = 0, fills = 0;
            uint32_t phase = 0;
            bool ok = true;
            Work w;
            for (int it = 0; ok && next_work(p, tiles, it, w); ++it) {
                int mb, nb;
                raster_tile(w.t, p.m_blocks, p.n_blocks, p.raster, mb, nb);
                for (int kb = w.kb0; kb < w.kb1; ++kb) {
                    if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag)) { ok = false; break; }
                    if (lane == 0) {
                        mbar_arrive_expect_tx(full + stage, kTileABytes + kUeTileBBytes);
                        tma_load_2d(sA + stage * kTileABytes, &tmA, full + stage, kb * kBK, mb * kBM, pol_a);
                        tma_load_3d(sB + stage * kUeTileBBytes, &tmB, full + stage, kb * kBK, nb * kUeBN, 0, pol_b);
                    }
                    __syncwarp();
                    ++fills;
                    if (++stage == kUeStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (lane == 0) {
                const int first = fills > kUeStages ? fills - kUeStages : 0;
                for (int i = first; i < fills; ++i)
                    mbar_wait_drain(full + (i % kUeStages), static_cast<uint32_t>((i / kUeStages) & 1));
            }
            __syncwarp();
        } else if (warp == 1 || warp == 2) {
            // ----------------------------------------------------------- MMA ----
            // Two warps issue the MMAs of alternate K blocks (the CTA's i-th K
            // block, counted over its work items, goes to warp 1 + i % 2).  A
            // warp waits for its operand stage (and, at a group start, copies
            // the scale factors) while the other issues; the hand-over keeps
            // the MMAs into the one accumulator in K order: the issuer of
            // block i fences and arrives on hand[its warp] once its MMAs and
            // commits are issued, and block i+1's issuer waits for that
            // arrival and fences before its first MMA.
            const int mw = warp - 1;
            int stage = 0, slot = 0, items = 0, i = 0;
            uint32_t phase = 0, sphase = 0;
            bool ok = true;
            Work w;
            for (int it = 0; ok && next_work(p, tiles, it, w); ++it, ++items) {
                for (int kb = w.kb0; kb < w.kb1; ++kb, ++i) {
                    const int j = (kb - w.kb0) % kUeSfGroup;  // byte of the scale words this K block uses
                    const bool group_end = j == kUeSfGroup - 1 || kb == w.kb1 - 1;
                    if ((i & 1) == mw) {
                        const uint32_t sf_col = static_cast<uint32_t>(kUeAccCols + slot * kUeSfColsPerSlot);
                        if (kb == w.kb0) {
                            // The accumulator is free once the epilogue has read the previous work item.
                            if (!mbar_wait(acc_empty, (items & 1) ^ 1u, abort_flag)) { ok = false; break; }
                        }
                        if (!mbar_wait(full + stage, phase, abort_flag)) { ok = false; break; }
                        if (j == 0 && !mbar_wait(sf_full + slot, sphase, abort_flag)) { ok = false; break; }
                        if (i > 0) {
                            // Block i-1 was the other warp's: its ((i + mw) / 2)-th hand-over.
                            const uint32_t hp = static_cast<uint32_t>((i + mw) / 2 - 1) & 1u;
                            if (!mbar_wait(hand + (1 - mw), hp, abort_flag)) { ok = false; break; }
                        }
                        tc_fence_after();
                        if (lane == 0) {
                            if (j == 0) copy_sf_slot(sSF, tmem_base, slot);
                            const uint32_t a_addr = smem_u32(sA + stage * kTileABytes);
                            const uint32_t b_addr = smem_u32(sB + stage * kUeTileBBytes);
                            const uint32_t idesc = idesc_e4m3_ue8m0(kBM, kUeBN, j, j);
#pragma unroll
                            for (int k = 0; k < kBK / 32; ++k)
                                umma_f8_block_scaled(tmem_base, sdesc_kmajor_sw128(a_addr + k * 32),
                                                     sdesc_kmajor_sw128(b_addr + k * 32), idesc, tmem_base + sf_col,
                                                     tmem_base + sf_col + 4, (kb > w.kb0 || k > 0) ? 1u : 0u);
                            umma_commit(empty + stage);
                            if (group_end) umma_commit(sf_empty + slot);
                            if (kb == w.kb1 - 1) umma_commit(acc_full);
                        }
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(hand + mw);
                    }
                    if (++stage == kUeStages) { stage = 0; phase ^= 1u; }
                    if (group_end) {
                        if (++slot == kUeSfSlots) { slot = 0; sphase ^= 1u; }
                    }
                }
            }
            // All MMAs of this warp must have finished before TMEM is released.
            if (lane == 0) {
                umma_commit(done + mw);
                mbar_wait_drain(done + mw, 0);
            }
            __syncwarp();
        } else if (warp == 4 || warp == 5) {
            // ------------------------------------------ scale converters ----
            // The CTA's g-th group of kUeSfGroup K blocks, counted over its
            // work items in order, goes to warp 4 + g % 2 and to ring slot
            // g % kUeSfSlots.  For its group a warp reads the FP32 scales from
            // global memory -- lane l the sa of rows m0 + l + 32c (c < 4) and
            // the sb of the tile's two 128-column blocks, for each K block of
            // the group -- and writes their UE8M0 codes in the scale-factor
            // layout, lane l line l of each block.  Byte j of a word is the
            // code of K block kb0 + j.  Entries past the data (rows past M,
            // blocks past N, K blocks past the end) read as 1.0, code 127, and
            // only meet zero-filled operands or unused bytes.  The loads of
            // two K blocks are in flight at a time (the warp runs in 56
            // registers); the first pair is issued before the wait for the
            // slot.
            const int cw = warp - 4;
            int g = 0;
            bool ok = true;
            Work w;
            for (int it = 0; ok && next_work(p, tiles, it, w); ++it) {
                int mb, nb;
                raster_tile(w.t, p.m_blocks, p.n_blocks, p.raster, mb, nb);
                const int m0 = mb * kBM;
                const int nb0 = nb * (kUeBN / 128);
                for (int kb0 = w.kb0; kb0 < w.kb1; kb0 += kUeSfGroup, ++g) {
                    if ((g & 1) != cw) continue;
                    const int sslot = g % kUeSfSlots;
                    const uint32_t sphase = static_cast<uint32_t>(g / kUeSfSlots) & 1u;
                    uint32_t a[4] = {0u, 0u, 0u, 0u}, b0 = 0u, b1 = 0u;
#pragma unroll
                    for (int jp = 0; jp < kUeSfGroup; jp += 2) {
                        float fa[2][4], fb[2][2];
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int kb = kb0 + jp + jj;
                            const bool kb_ok = kb < w.kb1;
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const int row = m0 + lane + 32 * c;
                                fa[jj][c] = (kb_ok && row < p.M)
                                                ? __ldg(p.sa + static_cast<int64_t>(kb) * p.sa_stride + row)
                                                : 1.0f;
                            }
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                fb[jj][h] = (kb_ok && nb0 + h < p.nbn)
                                                ? __ldg(p.sb + static_cast<int64_t>(nb0 + h) * nkb + kb)
                                                : 1.0f;
                        }
                        if (jp == 0 && !mbar_wait(sf_empty + sslot, sphase ^ 1u, abort_flag)) { ok = false; break; }
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int sh = 8 * (jp + jj);
#pragma unroll
                            for (int c = 0; c < 4; ++c) a[c] |= ue8m0_code(fa[jj][c]) << sh;
                            b0 |= ue8m0_code(fb[jj][0]) << sh;
                            b1 |= ue8m0_code(fb[jj][1]) << sh;
                        }
                    }
                    if (!ok) break;
                    const uint32_t base = smem_u32(sSF + sslot * kUeSfSlotBytes);
                    st_shared_v4(base + lane * 16, a[0], a[1], a[2], a[3]);
                    st_shared_v4(base + kUeSfaBytes + lane * 16, b0, b0, b0, b0);
                    st_shared_v4(base + kUeSfaBytes + 512 + lane * 16, b1, b1, b1, b1);
                    fence_proxy_async_smem();  // the copy to TMEM reads through the async proxy
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sf_full + sslot);
                }
            }
        }
    } else {
        // ------------------------------------------------------- epilogue ----
        regs_inc<kUeRegsHigh>();
        const int ew = warp - kUeFirstEpiWarp;
        const int half = ew >> 2;  // 128-column half of the tile
        const int quarter = warp & 3;
        const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        int items = 0;
        bool ok = true;
        Work w;
        for (int it = 0; ok && next_work(p, tiles, it, w); ++it, ++items) {
            int mb, nb;
            raster_tile(w.t, p.m_blocks, p.n_blocks, p.raster, mb, nb);
            if (!mbar_wait(acc_full, items & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t v[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_lane + static_cast<uint32_t>(half * 128 + c * 32), v[c]);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 4; ++c) reg_fence(v[c]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);  // the MMA may start the next work item
            if (w.slice >= 0) {
                // K slice of a split tile.  Partial (r, s) for slices s >= 1
                // lives at ws + (r*(S-1) + s-1) * 128*256 floats in the layout
                // [epilogue warp][float4 j][lane] (float4 j = columns 4j..4j+3
                // of the warp's 128).  Slice s >= 1 writes its partial and
                // raises its flag; slice 0 waits for every flag, adds the
                // partials in slice order (so the result does not depend on
                // timing), clears the flags and stores D.
                const int S = p.tail_split;
                const int rt = w.t - p.full_tiles;
                const bool leader = (warp == kUeFirstEpiWarp && lane == 0);
                if (w.slice > 0) {
                    float4* dst = reinterpret_cast<float4*>(p.ws + static_cast<int64_t>(rt * (S - 1) + w.slice - 1) * kBM * kUeBN);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const uint32_t* q = &v[j >> 3][(j & 7) * 4];
                        __stcg(dst + (ew * 32 + j) * 32 + lane, make_float4(__uint_as_float(q[0]), __uint_as_float(q[1]),
                                                                            __uint_as_float(q[2]), __uint_as_float(q[3])));
                    }
                    __threadfence();
                    named_barrier_sync(1, 32 * kUeEpiWarps);
                    if (leader) st_release_gpu(p.ws_flags + rt * (S - 1) + w.slice - 1, 1u);
                    continue;  // slice 0 stores the tile
                }
                bool got = true;
                if (leader) {
                    for (int s2 = 1; s2 < S && got; ++s2) got = wait_flag_gpu(p.ws_flags + rt * (S - 1) + s2 - 1);
                    for (int s2 = 1; s2 < S; ++s2) p.ws_flags[rt * (S - 1) + s2 - 1] = 0u;
                    if (!got) atomicOr(&g_dg_error, 1u);
                }
                named_barrier_sync(1, 32 * kUeEpiWarps);
                for (int s2 = 1; s2 < S; ++s2) {
                    const float4* src = reinterpret_cast<const float4*>(p.ws + static_cast<int64_t>(rt * (S - 1) + s2 - 1) * kBM * kUeBN);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float4 a = __ldcg(src + (ew * 32 + j) * 32 + lane);
                        uint32_t* q = &v[j >> 3][(j & 7) * 4];
                        q[0] = __float_as_uint(__uint_as_float(q[0]) + a.x);
                        q[1] = __float_as_uint(__uint_as_float(q[1]) + a.y);
                        q[2] = __float_as_uint(__uint_as_float(q[2]) + a.z);
                        q[3] = __float_as_uint(__uint_as_float(q[3]) + a.w);
                    }
                }
            }
            // bf16, staged 32 rows x 32 columns at a time with the 64-byte
            // swizzle of the output map, one TMA store per piece.
            const uint32_t stg = smem_u32(sOut + ew * kStageOutBytes);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (lane == 0) bulk_wait_read<0>();
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t w4[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(v[c][q * 8 + 2 * h]),
                                                                 __uint_as_float(v[c][q * 8 + 2 * h + 1]));
                        w4[h] = *reinterpret_cast<uint32_t*>(&b);
                    }
                    const uint32_t off = lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4);
                    st_shared_v4(stg + off, w4[0], w4[1], w4[2], w4[3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                const int x = nb * kUeBN + half * 128 + c * 32;
                if (lane == 0 && x < p.N) {
                    tma_store_2d(&tmD, sOut + ew * kStageOutBytes, x, mb * kBM + quarter * 32);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kUeTmemCols);
    }
}

}  // namespace dg
