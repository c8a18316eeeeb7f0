// dg_kernel_small.cuh -- sm_100a kernel for few rows per group (decode-sized M).
//
// With M <= 128 rows the output has too few 128-row tiles to keep 148 SMs
// streaming the weights, so this kernel swaps the operands and splits K:
//   * the MMA's 128-row side runs over N (the weights B), its N side over the
//     TN (32, 64 or 128) rows of A:  P_kb^T[n, m] = sum_k B[n,k] * A[m,k];
//   * a thread-block cluster of S CTAs shares one 128 x TN output tile; CTA r
//     of the cluster handles K blocks [r*nkb/S, (r+1)*nkb/S);
//   * each CTA promotes its blocks into FP32 registers exactly as the large
//     kernel does, acc[n,m] += (sa[m,kb] * sb[n/128,kb]) * P_kb[n,m] (the
//     128-row weight tile lies inside one 128x128 scale block, so sb is one
//     value per kb), with sa*sb formed once per kb by the scale warp;
//   * the S partial tiles are added in a fixed order (CTA 0 first) through
//     distributed shared memory -- no global scratch -- and the sum is rounded
//     to bf16 once and stored.
// Per CTA: 256 threads, <= 113 KiB shared memory and 256 TMEM columns, so two
// CTAs share an SM and every SM keeps up to 2 x STAGES K blocks in flight.
// Warp roles: 0 TMA producer, 1 TMEM owner + MMA issuer, 2 scale producer,
// 3 idle, 4..7 promotion (TMEM lane quarter = warp % 4, lane = output column).
#pragma once

#include "dg_kernel.cuh"

namespace dg {

constexpr int kSmallThreads = 256;
constexpr int kSmallFirstEpiWarp = 4;
constexpr int kSmallEpiWarps = 4;
constexpr int kSmallScaleSlots = 16;  // depth of the scale ring, in K blocks
// The scale ring is filled and released kSmallScaleGroup K blocks at a time,
// so the promotion waits on a scale barrier once per group.
constexpr int kSmallScaleGroup = 4;
constexpr int kSmallScaleGroups = kSmallScaleSlots / kSmallScaleGroup;
constexpr int kSmallTmemCols = 256;
// Largest cluster (K splits per tile).  Measured on the M = 64 / 128 shapes of
// the dense sweep, clusters of 6 and 8 CTAs were never faster than 4: at two
// CTAs per SM an 8-CTA cluster lands on four SMs, and per slice the set-up and
// the DSMEM reduction cost more than the shorter K loop saves.
constexpr int kSmallMaxSplit = 4;

template <int TN>
struct SmallCfg {
    static_assert(TN == 32 || TN == 64 || TN == 128, "TN must be 32, 64 or 128");
    static constexpr int kTileBBytes = 128 * kBK;   // 128 weight rows
    static constexpr int kTileABytes = TN * kBK;    // TN activation rows
    static constexpr int kStageBytes = kTileBBytes + kTileABytes;
    static constexpr int kStages = (96 * 1024) / kStageBytes;  // 4, 4 or 3 stages: ~96 KiB of ring
    static constexpr int kNBuf = kSmallTmemCols / TN > 4 ? 4 : kSmallTmemCols / TN;
    static constexpr int kChunks = TN / 32;
    static constexpr int kBatch = TN == 128 ? 1 : (kChunks < 2 ? kChunks : 2);
    static constexpr int kRedBytes = TN * 128 * 4;  // FP32 partial tile, aliases the ring
    static_assert(kRedBytes <= kStages * kStageBytes, "partial tile must fit in the ring");
    static_assert(kNBuf * TN <= kSmallTmemCols, "TMEM buffers overflow the allocation");
};

template <int TN>
constexpr int small_smem_bytes() {
    return 1024 + SmallCfg<TN>::kStages * SmallCfg<TN>::kStageBytes + 512 + kSmallScaleSlots * (TN + 4) * 4;
}

// Grid: x = split index (the cluster spans x), y = 128-wide block of N,
// z = TN-row block of M (masked: g * m_blocks + block inside the group;
// Params::m_blocks holds the blocks per group).
template <int TN, int MODE>
__global__ void __launch_bounds__(kSmallThreads, 2)
fp8_gemm_swapab_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB) {
    using C = SmallCfg<TN>;
    constexpr int STAGES = C::kStages;
    constexpr int kNBuf = C::kNBuf;

    const int S = gridDim.x;
    const int rank = blockIdx.x;
    const int n0 = blockIdx.y * 128;
    int g = 0, m0;
    if (MODE == kMasked) {
        g = blockIdx.z / p.m_blocks;
        m0 = (blockIdx.z % p.m_blocks) * TN;
    } else {
        m0 = blockIdx.z * TN;
    }
    int rows_valid = p.M;
    if (MODE == kMasked) {
        // masked_m may come from the previous kernel in the stream.
        griddep_wait();
        const int mm = __ldg(p.masked_m + g);
        if ((mm < 0 || mm > p.M) && rank == 0 && blockIdx.y == 0 && m0 == 0) atomicOr(&g_dg_error, 4u);
        rows_valid = min(max(mm, 0), p.M);
    }
    // Every CTA of a cluster shares (y, z), so the whole cluster leaves together.
    if (m0 >= rows_valid) return;

    const int nkb = p.nkb;
    const int kb0 = static_cast<int>(static_cast<int64_t>(rank) * nkb / S);
    const int kb1 = static_cast<int>(static_cast<int64_t>(rank + 1) * nkb / S);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + STAGES * C::kStageBytes);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + kNBuf;
    uint64_t* sfull = tempty + kNBuf;
    uint64_t* sempty = sfull + kSmallScaleSlots;
    uint64_t* done = sempty + kSmallScaleSlots;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* sring = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 512);
    float* red = reinterpret_cast<float*>(ring);  // [TN][128] FP32 partial, after the main loop
    // Scale ring: kSmallScaleSlots slots of TN sa values followed by sb (TN + 4 floats, 16-byte aligned).

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Stage `stage` <- the weight tile and the activation tile of K block kb.
    auto issue_stage = [&](int stage, int kb) {
        uint8_t* st = ring + stage * C::kStageBytes;
        const uint64_t pol_w = l2_policy_evict_first();  // weights stream through once
        const uint64_t pol_a = l2_policy_evict_last();   // activations are re-read by every n-block
        mbar_arrive_expect_tx(full + stage, C::kStageBytes);
        tma_load_3d(st, &tmB, full + stage, kb * kBK, n0, g, pol_w);
        if (MODE == kMasked)
            tma_load_3d(st + C::kTileBBytes, &tmA, full + stage, kb * kBK, m0, g, pol_a);
        else
            tma_load_2d(st + C::kTileBBytes, &tmA, full + stage, kb * kBK, m0, pol_a);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int b = 0; b < kNBuf; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, kSmallEpiWarps);
        }
        for (int s = 0; s < kSmallScaleSlots; ++s) {
            mbar_init(sfull + s, 32);
            mbar_init(sempty + s, kSmallEpiWarps);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_mbar_init();
        // The ring starts empty: pull its first weight tiles into L2 while the
        // previous kernel may still run, then (once its data is visible)
        // issue the first loads, so that their latency overlaps the rest of
        // the set-up.
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        for (int i = 0; i < STAGES && kb0 + i < kb1; ++i) tma_prefetch_3d(&tmB, (kb0 + i) * kBK, n0, g);
        griddep_wait();
        for (int i = 0; i < STAGES && kb0 + i < kb1; ++i) issue_stage(i, kb0 + i);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kSmallTmemCols);
        tmem_relinquish();
    }
    griddep_wait();
    griddep_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp < kSmallFirstEpiWarp) {
        regs_dec<56>();
        if (warp == 0) {
            // -------------------------------------------------- producer ----
            // The first STAGES blocks were issued during set-up.
            int stage = 0, fills = 0;
            uint32_t phase = 0;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (fills >= STAGES) {
                    if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag)) break;
                    if (lane == 0) issue_stage(stage, kb);
                    __syncwarp();
                }
                ++fills;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (lane == 0) {
                const int first = fills > STAGES ? fills - STAGES : 0;
                for (int i = first; i < fills; ++i)
                    mbar_wait_drain(full + (i % STAGES), static_cast<uint32_t>((i / STAGES) & 1));
            }
            __syncwarp();
        } else if (warp == 1) {
            // ------------------------------------------------------- MMA ----
            constexpr uint32_t idesc = idesc_e4m3_f32(128, TN);
            int stage = 0, buf = 0;
            uint32_t phase = 0, bphase = 0;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!mbar_wait(tempty + buf, bphase ^ 1u, abort_flag)) break;
                if (!mbar_wait(full + stage, phase, abort_flag)) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t w_addr = smem_u32(ring + stage * C::kStageBytes);
                    const uint32_t a_addr = w_addr + C::kTileBBytes;
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * TN);
#pragma unroll
                    for (int k = 0; k < kBK / 32; ++k)
                        umma_f8(d_tmem, sdesc_kmajor_sw128(w_addr + k * 32), sdesc_kmajor_sw128(a_addr + k * 32),
                                idesc, k > 0 ? 1u : 0u);
                    umma_commit(empty + stage);
                    umma_commit(tfull + buf);
                }
                __syncwarp();
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                if (++buf == kNBuf) { buf = 0; bphase ^= 1u; }
            }
            if (lane == 0) {
                umma_commit(done);
                mbar_wait_drain(done, 0);
            }
            __syncwarp();
        } else if (warp == 2) {
            // ------------------------------------------- scale producer ----
            // Per K block: sa[m0 .. m0+TN) (lane l copies TN/32 consecutive
            // rows) and sb[n0/128] (lane 0), copied asynchronously.  Up to
            // kSmallScaleGroup consecutive K blocks share a ring slot whose
            // barrier completes when all of their copies land.  Rows past the
            // data are zero-filled and never read.
            constexpr int kPer = TN / 32;  // floats per lane
            const float* sa_base = p.sa + (MODE == kMasked ? static_cast<int64_t>(g) * nkb * p.sa_stride : 0);
            const float* sb_row = p.sb + (static_cast<int64_t>(g) * p.nbn + n0 / 128) * nkb;
            const int r = m0 + lane * kPer;
            const int left = p.M - r;
            const uint32_t sa_bytes = left >= kPer ? 4u * kPer : (left > 0 ? 4u * static_cast<uint32_t>(left) : 0u);
            int slot = 0;
            uint32_t sphase = 0;
            for (int kg = kb0; kg < kb1; kg += kSmallScaleGroup) {
                if (!mbar_wait(sempty + slot, sphase ^ 1u, abort_flag)) break;
                const int n = min(kSmallScaleGroup, kb1 - kg);
                for (int j = 0; j < n; ++j) {
                    const int kb = kg + j;
                    const uint32_t dst = smem_u32(sring + (slot * kSmallScaleGroup + j) * (TN + 4));
                    const float* src = sa_bytes ? sa_base + static_cast<int64_t>(kb) * p.sa_stride + r : p.sa;
                    if (kPer == 4)
                        cp_async_16(dst + lane * 16, src, sa_bytes);
                    else if (kPer == 2)
                        cp_async_8(dst + lane * 8, src, sa_bytes);
                    else
                        cp_async_4(dst + lane * 4, src, sa_bytes);
                    if (lane == 0) cp_async_4(dst + TN * 4, sb_row + kb, 4u);
                }
                cp_async_arrive(sfull + slot);
                if (++slot == kSmallScaleGroups) { slot = 0; sphase ^= 1u; }
            }
            asm volatile("cp.async.wait_all;" ::: "memory");
        }
    } else {
        // ------------------------------------------------------ promotion ----
        regs_inc<192>();
        float2 acc[TN / 2];
#pragma unroll
        for (int j = 0; j < TN / 2; ++j) acc[j] = make_float2(0.f, 0.f);
        const int quarter = warp & 3;
        const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        int buf = 0, slot = 0;
        uint32_t bphase = 0, sphase = 0;
        for (int kb = kb0; kb < kb1; ++kb) {
            const int jg = (kb - kb0) % kSmallScaleGroup;  // K block inside its scale group
            if (jg == 0 && !mbar_wait(sfull + slot, sphase, abort_flag)) break;
            if (!mbar_wait(tfull + buf, bphase, abort_flag)) break;
            tc_fence_after();
            // Scales of this K block: s[j] = sa[m0 + j] * sb, formed here.
            const float* slot_f = sring + (slot * kSmallScaleGroup + jg) * (TN + 4);
            const float2* sc = reinterpret_cast<const float2*>(slot_f);
            const float s_b = slot_f[TN];
            const float2 sb2 = make_float2(s_b, s_b);
#pragma unroll
            for (int cb = 0; cb < C::kChunks; cb += C::kBatch) {
                uint32_t v[C::kBatch][32];
#pragma unroll
                for (int c = 0; c < C::kBatch; ++c)
                    tmem_ld_32x32b_x32(t_lane + static_cast<uint32_t>(buf * TN + (cb + c) * 32), v[c]);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < C::kBatch; ++c) reg_fence(v[c]);
                if (cb + C::kBatch == C::kChunks) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tempty + buf);
                }
#pragma unroll
                for (int c = 0; c < C::kBatch; ++c)
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float2 pv = make_float2(__uint_as_float(v[c][2 * j]), __uint_as_float(v[c][2 * j + 1]));
                        const int q = (cb + c) * 16 + j;
                        acc[q] = __ffma2_rn(pv, __fmul2_rn(sc[q], sb2), acc[q]);
                    }
            }
            if (jg == kSmallScaleGroup - 1 || kb == kb1 - 1) {
                // The group's last K block is done with its scales: release the slot.
                __syncwarp();
                if (lane == 0) mbar_arrive(sempty + slot);
                if (++slot == kSmallScaleGroups) { slot = 0; sphase ^= 1u; }
            }
            if (++buf == kNBuf) { buf = 0; bphase ^= 1u; }
        }
        // The ring is idle once this CTA's last partial has been read out of
        // TMEM (every load was consumed by an MMA that has completed): it
        // becomes this CTA's FP32 partial tile red[j][n] (n contiguous).
        const int n = quarter * 32 + lane;
#pragma unroll
        for (int q = 0; q < TN / 2; ++q) {
            red[(2 * q) * 128 + n] = acc[q].x;
            red[(2 * q + 1) * 128 + n] = acc[q].y;
        }
    }

    // -------------------------------------------- split-K reduction ----
    // CTA `rank` owns float4 groups [rank*E/S, (rank+1)*E/S) of the tile and
    // adds the S partials in rank order (all loads first, then the sums).
    constexpr int E4 = TN * 128 / 4;
    const int e_begin = static_cast<int>(static_cast<int64_t>(rank) * E4 / S);
    const int e_end = static_cast<int>(static_cast<int64_t>(rank + 1) * E4 / S);
    const uint32_t red_local = smem_u32(red);
    auto store4 = [&](int e, float4 sum) {
        const int j = (e * 4) / 128;
        const int nn = (e * 4) % 128;
        const int row = m0 + j, col = n0 + nn;
        if (row < rows_valid && col < p.N) {
            const int64_t d_row = (MODE == kMasked ? static_cast<int64_t>(g) * p.M : 0) + row;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(sum.x, sum.y);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(sum.z, sum.w);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t*>(&h0);
            pk.y = *reinterpret_cast<uint32_t*>(&h1);
            *reinterpret_cast<uint2*>(p.D + d_row * p.N + col) = pk;
        }
    };
    if (S == 1) {
        __syncthreads();
        for (int e = static_cast<int>(threadIdx.x); e < E4; e += kSmallThreads)
            store4(e, reinterpret_cast<const float4*>(red)[e]);
    } else {
        cluster_sync();  // every partial tile written and visible cluster-wide
        for (int e = e_begin + static_cast<int>(threadIdx.x); e < e_end; e += kSmallThreads) {
            float4 v[kSmallMaxSplit];
#pragma unroll
            for (int r = 0; r < kSmallMaxSplit; ++r)
                if (r < S) v[r] = ld_dsmem_f4(dsmem_addr(red_local + e * 16, r));
            float4 sum = v[0];
#pragma unroll
            for (int r = 1; r < kSmallMaxSplit; ++r)
                if (r < S) {
                    sum.x += v[r].x; sum.y += v[r].y; sum.z += v[r].z; sum.w += v[r].w;
                }
            store4(e, sum);
        }
        // No CTA may leave while others still read its partial tile.
        cluster_sync_relaxed();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kSmallTmemCols);
    }
}

}  // namespace dg
