// dg_kernel_small.cuh -- sm_100a kernel for few rows per group (decode-sized M).
//
// With M <= 128 rows the GEMM streams the weights B once from HBM and the
// activations are a small, L2-resident operand.  The kernel is built around
// keeping every SM's TMA queue full of weight tiles from the first
// microsecond to the last:
//   * operands swapped: the MMA's 128-row side runs over 128 weight rows,
//     its N side over the TN (32, 64 or 128) activation rows, so one tile
//     covers all rows of a group and B is read exactly once;
//   * one CTA per SM with a deep operand ring (5 to 10 stages, up to ~200
//     KiB in flight), so few round trips to HBM cover a CTA's share;
//   * tiles (group, TN-row block, 128-wide block of N) are spread over
//     clusters of S CTAs; CTA r of a cluster handles K blocks
//     [r*nkb/S, (r+1)*nkb/S) of its cluster's tile.  S = 1 clusters are
//     persistent (a CTA walks tiles cid, cid + C, ... with one ring across
//     them); S > 1 is used only when every cluster has one tile, and the host
//     sizes S so that all clusters are resident at once;
//   * each CTA promotes its K blocks in FP32 registers,
//         acc[n, m] += (sa[m, kb] * sb[n/128, kb]) * P_kb[n, m],
//     with two promotion warpgroups splitting the activation rows (the
//     128-row weight tile lies inside one 128 x 128 scale block, so sb is one
//     value per K block);
//   * split tiles are reduced through distributed shared memory without a
//     barrier on the critical path: each CTA writes its FP32 partial tile into
//     its (now idle) ring and bulk-copies slice r of it into CTA r's receive
//     area, counted on CTA r's mbarrier; CTA r then adds the S slices in rank
//     order (a fixed order, so results are deterministic), rounds to bf16 once
//     and stores its rows.  Unsplit tiles are rounded to bf16, staged in
//     shared memory and stored with 16-byte writes.
// Warp roles: 0 TMA producer, 1 TMEM owner + MMA issuer, 2 scale producer,
// 3 second MMA issuer, 4..11 promotion (warpgroup h = activation rows [h*TN/2, (h+1)*TN/2),
// TMEM lane quarter = warp % 4, lane = weight row).
#pragma once

#include "dg_kernel.cuh"

namespace dg {

// Cluster-barrier arrive without release semantics: for a barrier that only
// keeps the CTAs of a cluster alive until their peers are done, where nothing
// written before the arrive is read after the wait because of it.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

constexpr int kSmallThreads = 384;
constexpr int kSmallFirstEpiWarp = 4;
constexpr int kSmallEpiWarps = 8;
constexpr int kSmallEpiThreads = 32 * kSmallEpiWarps;
constexpr int kSmallScaleSlots = 16;  // depth of the scale ring, in K blocks
// The scale ring is filled and released kSmallScaleGroup K blocks at a time,
// so the promotion waits on a scale barrier once per group.
constexpr int kSmallScaleGroup = 4;
constexpr int kSmallScaleGroups = kSmallScaleSlots / kSmallScaleGroup;
constexpr int kSmallSmemLimit = 232448;  // 227 KiB: one CTA per SM
constexpr int kSmallBarrierBytes = 1024;
constexpr int kSmallGroupTableBytes = 8 * (kMaxMaskedGroups + 1);  // masked: tile prefix + clamped counts

// Largest receive area over the cluster sizes a TN allows: S - 1 slices of
// ceil(TN / S) rows of 128 FP32 values.
constexpr int small_recv_bytes(int tn, int max_split) {
    int best = 0;
    for (int s = 2; s <= max_split; ++s) {
        const int b = (s - 1) * ((tn + s - 1) / s) * 128 * 4;
        best = b > best ? b : best;
    }
    return best;
}

template <int TN>
struct SmallCfg {
    static_assert(TN == 32 || TN == 64 || TN == 128, "TN must be 32, 64 or 128");
    static constexpr int kMaxSplit = TN == 128 ? 4 : 8;  // cluster size (K slices per tile)
    static constexpr int kTileBBytes = 128 * kBK;        // 128 weight rows
    static constexpr int kTileABytes = TN * kBK;         // TN activation rows
    static constexpr int kStageBytes = kTileBBytes + kTileABytes;
    static constexpr int kTileF32Bytes = TN * 128 * 4;   // FP32 partial tile
    static constexpr int kRecvBytes = small_recv_bytes(TN, kMaxSplit);
    static constexpr int kStageOutBytes = TN * 128 * 2;  // bf16 tile staged for the store
    static constexpr int kAuxBytes = kRecvBytes > kStageOutBytes ? kRecvBytes : kStageOutBytes;
    static constexpr int kScaleBytes = kSmallScaleSlots * (TN + 4) * 4;
    static constexpr int kFixedBytes = 1024 + kAuxBytes + kScaleBytes + kSmallBarrierBytes + kSmallGroupTableBytes;
    static constexpr int kStagesFit = (kSmallSmemLimit - kFixedBytes) / kStageBytes;
    static constexpr int kStages = kStagesFit > 12 ? 12 : kStagesFit;
    static constexpr int kNBuf = 4;                       // TMEM partial buffers
    static constexpr int kTmemCols = kNBuf * TN <= 128 ? 128 : (kNBuf * TN <= 256 ? 256 : 512);
    static constexpr int kCols = TN / 2;                  // activation rows per promotion warpgroup
    static constexpr int kChunk = kCols < 32 ? kCols : 32;  // columns per tcgen05.ld
    static constexpr int kChunks = kCols / kChunk;
    static_assert(kTileF32Bytes <= kStages * kStageBytes, "partial tile must fit in the ring");
    static_assert(kStages >= 4, "ring too shallow");
    static_assert(kStages * kStageBytes + kFixedBytes <= kSmallSmemLimit, "shared memory overflow");
};

template <int TN>
constexpr int small_smem_bytes() {
    return SmallCfg<TN>::kStages * SmallCfg<TN>::kStageBytes + SmallCfg<TN>::kFixedBytes;
}

// One tile of the few-row kernel.
struct SmallTile {
    int g;     // group
    int m0;    // first activation row inside the group
    int n0;    // first weight row (output column)
    int rows;  // rows of the group that exist (dense M, masked masked_m[g])
};

// Tile t in the order (group, n-block, m-block), m-block fastest: tiles that
// run on neighbouring clusters share their weight tiles in L2.
template <int TN, int MODE>
__device__ __forceinline__ SmallTile small_tile(const Params& p, int t, const int* prefix, const int* counts) {
    SmallTile tl;
    if (MODE == kMasked) {
        int lo = 0, hi = p.G - 1;  // largest g with prefix[g] <= t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
        }
        const int local = t - prefix[lo];
        const int mbg = (counts[lo] + TN - 1) / TN;
        tl.g = lo;
        tl.n0 = (local / mbg) * 128;
        tl.m0 = (local % mbg) * TN;
        tl.rows = counts[lo];
    } else {
        tl.g = 0;
        tl.n0 = (t / p.m_blocks) * 128;
        tl.m0 = (t % p.m_blocks) * TN;
        tl.rows = p.M;
    }
    return tl;
}

// Grid: 1-D, clusters of S CTAs along x (S = cluster size).  Params::m_blocks
// holds the TN-row blocks per group; Params::n_blocks the 128-wide blocks of N.
template <int TN, int MODE>
__global__ void __launch_bounds__(kSmallThreads, 1)
fp8_gemm_swapab_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB) {
    using C = SmallCfg<TN>;
    constexpr int STAGES = C::kStages;
    constexpr int kNBuf = C::kNBuf;
    // The tensor maps live in parameter space: start fetching them first.
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }

    const int S = static_cast<int>(cluster_nctarank());
    const int rank = static_cast<int>(cluster_ctarank());
    const int cid = static_cast<int>(blockIdx.x) / S;
    const int nclusters = static_cast<int>(gridDim.x) / S;
    // Split clusters own one tile each (the host launches one cluster per
    // tile); single-CTA clusters walk tiles cid, cid + nclusters, ...
    const int tstep = S > 1 ? (1 << 30) : nclusters;
    const int nkb = p.nkb;
    const int kb0 = static_cast<int>(static_cast<int64_t>(rank) * nkb / S);
    const int kb1 = static_cast<int>(static_cast<int64_t>(rank + 1) * nkb / S);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    uint8_t* aux = ring + STAGES * C::kStageBytes;  // receive area (split) / bf16 staging (unsplit)
    float* sring = reinterpret_cast<float*>(aux + C::kAuxBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sring) + C::kScaleBytes);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + kNBuf;
    uint64_t* sfull = tempty + kNBuf;
    uint64_t* sempty = sfull + kSmallScaleSlots;
    uint64_t* done = sempty + kSmallScaleSlots;  // one per MMA warp
    uint64_t* rbar = done + 2;  // the split partials this CTA receives
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rbar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* prefix = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + kSmallBarrierBytes);
    int* counts = prefix + kMaxMaskedGroups + 1;
    // A split tile's FP32 partial [TN][128] (weight row fastest) goes into the
    // ring once the main loop is done; CTA r owns activation rows
    // [r*TN/S, (r+1)*TN/S) of it.
    float* red = reinterpret_cast<float*>(ring);
    const int my_j0 = rank * TN / S, my_j1 = (rank + 1) * TN / S;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

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
        mbar_init(done + 1, 1);
        mbar_init(rbar, 1);
        // The whole receive area arrives in one phase: S - 1 slices of this
        // CTA's rows from the other CTAs of the cluster.
        if (S > 1) mbar_arrive_expect_tx(rbar, static_cast<uint32_t>((S - 1) * (my_j1 - my_j0) * 128 * 4));
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // Every CTA's receive barrier is initialised before any peer copies into it.
    if (S > 1) cluster_arrive();
    const uint32_t tmem_base = *tmem_slot;
    // Nothing above touched global memory: with programmatic dependent launch
    // all of it overlaps the end of the previous kernel in the stream.
    griddep_launch_dependents();
    if (MODE != kMasked && threadIdx.x == 0 && cid < p.m_blocks * p.n_blocks) {
        // Pull this CTA's first weight tiles into L2 while the previous kernel
        // may still run.  L2 is the point of coherence, so a prefetch issued
        // before the dependency wait never makes a later read return data
        // older than the wait exposes.  (Masked tiles depend on masked_m,
        // which the previous kernel may write.)
        const int n0 = (cid / p.m_blocks) * 128;
        for (int i = 0; i < STAGES && kb0 + i < kb1; ++i) tma_prefetch_3d(&tmB, (kb0 + i) * kBK, n0, 0);
    }
    griddep_wait();

    int tiles;
    if (MODE == kMasked) {
        // Tiles per group from the device-resident masked_m (clamped to
        // [0, M_max] and flagged when outside), then an exclusive prefix.
        for (int g = threadIdx.x; g < p.G; g += kSmallThreads) {
            int mm = __ldg(p.masked_m + g);
            if (mm < 0 || mm > p.M) {
                if (blockIdx.x == 0) atomicOr(&g_dg_error, 4u);
                mm = min(max(mm, 0), p.M);
            }
            counts[g] = mm;
            prefix[g + 1] = ((mm + TN - 1) / TN) * p.n_blocks;
        }
        __syncthreads();
        if (warp == 0) {
            int carry = 0;
            for (int base = 0; base < p.G; base += 32) {
                const int i = base + lane;
                int v = (i < p.G) ? prefix[i + 1] : 0;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, v, off);
                    if (lane >= off) v += u;
                }
                if (i < p.G) prefix[i + 1] = v + carry;
                carry += __shfl_sync(0xffffffffu, v, 31);
            }
            if (lane == 0) prefix[0] = 0;
        }
        __syncthreads();
        tiles = prefix[p.G];
    } else {
        tiles = p.m_blocks * p.n_blocks;
    }

    if (warp < kSmallFirstEpiWarp) {
        if (warp == 0) {
            // -------------------------------------------------- producer ----
            // Weights are read once when a group has one TN-row block; with
            // more, neighbouring clusters re-read each weight tile from L2.
            const uint64_t pol_w = p.b_stream ? l2_policy_evict_first() : l2_policy_evict_normal();
            const uint64_t pol_a = l2_policy_evict_last();  // activations are re-read by every n-block
            int stage = 0, fills = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = cid; ok && t < tiles; t += tstep) {
                const SmallTile tl = small_tile<TN, MODE>(p, t, prefix, counts);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag)) { ok = false; break; }
                    if (lane == 0) {
                        uint8_t* st = ring + stage * C::kStageBytes;
                        mbar_arrive_expect_tx(full + stage, C::kStageBytes);
                        tma_load_3d(st, &tmB, full + stage, kb * kBK, tl.n0, tl.g, pol_w);
                        if (MODE == kMasked)
                            tma_load_3d(st + C::kTileBBytes, &tmA, full + stage, kb * kBK, tl.m0, tl.g, pol_a);
                        else
                            tma_load_2d(st + C::kTileBBytes, &tmA, full + stage, kb * kBK, tl.m0, pol_a);
                    }
                    __syncwarp();
                    ++fills;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // No copy into this CTA's shared memory may still be in flight
            // when it exits (matters only after an abort).
            if (lane == 0) {
                const int first = fills > STAGES ? fills - STAGES : 0;
                for (int i = first; i < fills; ++i)
                    mbar_wait_drain(full + (i % STAGES), static_cast<uint32_t>((i / STAGES) & 1));
            }
            __syncwarp();
        } else if (warp == 1 || warp == 3) {
            // ------------------------------------------------------- MMA ----
            // Two warps take alternate K blocks (the CTA's i-th K block goes
            // to warp 1 for even i, to warp 3 for odd i): issuing four
            // tcgen05.mma and two commits costs a warp several hundred
            // cycles, more than the tensor core needs for a 128 x TN x 128
            // block.  Each block has its own stage and TMEM buffer, so the
            // two instruction streams never touch the same data.
            constexpr uint32_t idesc = idesc_e4m3_f32(128, TN);
            const int mw = warp == 1 ? 0 : 1;
            int i = 0;  // K blocks of this CTA so far, over all its tiles
            bool ok = true;
            for (int t = cid; ok && t < tiles; t += tstep) {
                for (int kb = kb0; kb < kb1; ++kb, ++i) {
                    if ((i & 1) != mw) continue;
                    const int stage = i % STAGES, buf = i % kNBuf;
                    const uint32_t phase = static_cast<uint32_t>(i / STAGES) & 1u;
                    const uint32_t bphase = static_cast<uint32_t>(i / kNBuf) & 1u;
                    if (!mbar_wait(tempty + buf, bphase ^ 1u, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(full + stage, phase, abort_flag)) { ok = false; break; }
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
                }
            }
            if (lane == 0) {
                umma_commit(done + mw);
                mbar_wait_drain(done + mw, 0);
            }
            __syncwarp();
        } else if (warp == 2) {
            // ------------------------------------------- scale producer ----
            // Per K block: the products sa[m0 + j] * sb for the tile's TN
            // activation rows (lane l forms TN/32 consecutive rows) and its
            // 128-row weight block, so that promotion is one FMA per value.
            // Up to kSmallScaleGroup consecutive K blocks share a ring slot
            // whose barrier completes when all 32 lanes have written theirs.
            // Rows past the data get zero scales and are never stored.
            constexpr int kPer = TN / 32;  // floats per lane
            int slot = 0;
            uint32_t sphase = 0;
            bool ok = true;
            for (int t = cid; ok && t < tiles; t += tstep) {
                const SmallTile tl = small_tile<TN, MODE>(p, t, prefix, counts);
                const float* sa_base = p.sa + (MODE == kMasked ? static_cast<int64_t>(tl.g) * nkb * p.sa_stride : 0);
                const float* sb_row = p.sb + (static_cast<int64_t>(tl.g) * p.nbn + tl.n0 / 128) * nkb;
                const int r = tl.m0 + lane * kPer;
                const int left = p.M - r;
                const int nvalid = left >= kPer ? kPer : (left > 0 ? left : 0);
                for (int kg = kb0; kg < kb1; kg += kSmallScaleGroup) {
                    if (!mbar_wait(sempty + slot, sphase ^ 1u, abort_flag)) { ok = false; break; }
                    const int n = min(kSmallScaleGroup, kb1 - kg);
                    float sav[kSmallScaleGroup][kPer];
                    float sbv[kSmallScaleGroup];
#pragma unroll
                    for (int j = 0; j < kSmallScaleGroup; ++j) {
                        sbv[j] = j < n ? __ldg(sb_row + kg + j) : 0.f;
#pragma unroll
                        for (int e = 0; e < kPer; ++e)
                            sav[j][e] = (j < n && e < nvalid) ? __ldg(sa_base + static_cast<int64_t>(kg + j) * p.sa_stride + r + e) : 0.f;
                    }
#pragma unroll
                    for (int j = 0; j < kSmallScaleGroup; ++j)
                        if (j < n) {
                            float* dstf = sring + (slot * kSmallScaleGroup + j) * (TN + 4);
#pragma unroll
                            for (int e = 0; e < kPer; ++e) dstf[lane * kPer + e] = sav[j][e] * sbv[j];
                        }
                    mbar_arrive(sfull + slot);
                    if (++slot == kSmallScaleGroups) { slot = 0; sphase ^= 1u; }
                }
            }
        }
        if (S > 1) {
            // These warps take part in the cluster barriers only.
            cluster_wait();
            cluster_arrive();
        }
    } else {
        // ------------------------------------------------------ promotion ----
        // Warpgroup h promotes activation rows [h*TN/2, (h+1)*TN/2) of every
        // K block; its four warps cover the 128 weight rows (TMEM lane
        // quarter = warp % 4).
        const int ew = warp - kSmallFirstEpiWarp;
        const int half = ew >> 2;
        const int quarter = warp & 3;
        const int n = quarter * 32 + lane;              // weight row inside the tile
        const int j_base = half * C::kCols;
        const int ptid = threadIdx.x - kSmallFirstEpiWarp * 32;  // 0..255
        const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        int buf = 0, slot = 0;
        uint32_t bphase = 0, sphase = 0;
        bool ok = true;
        float2 acc[C::kCols / 2];
        for (int t = cid; t < tiles; t += tstep) {
            const SmallTile tl = small_tile<TN, MODE>(p, t, prefix, counts);
#pragma unroll
            for (int q = 0; q < C::kCols / 2; ++q) acc[q] = make_float2(0.f, 0.f);
            for (int kb = kb0; ok && kb < kb1; ++kb) {
                const int jg = (kb - kb0) % kSmallScaleGroup;  // K block inside its scale group
                if (jg == 0 && !mbar_wait(sfull + slot, sphase, abort_flag)) { ok = false; break; }
                if (!mbar_wait(tfull + buf, bphase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                uint32_t v[C::kChunks][C::kChunk];
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c) {
                    const uint32_t ta = t_lane + static_cast<uint32_t>(buf * TN + j_base + c * C::kChunk);
                    if constexpr (C::kChunk == 32)
                        tmem_ld_32x32b_x32(ta, reinterpret_cast<uint32_t(&)[32]>(v[c]));
                    else
                        tmem_ld_32x32b_x16(ta, reinterpret_cast<uint32_t(&)[16]>(v[c]));
                }
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c) reg_fence(v[c]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty + buf);
                // Scales of this K block: s[j] = sa[m0 + j] * sb, formed by the
                // scale warp.
                const float* slot_f = sring + (slot * kSmallScaleGroup + jg) * (TN + 4);
                const float2* sc = reinterpret_cast<const float2*>(slot_f + j_base);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
#pragma unroll
                    for (int j = 0; j < C::kChunk / 2; ++j) {
                        const float2 pv = make_float2(__uint_as_float(v[c][2 * j]), __uint_as_float(v[c][2 * j + 1]));
                        const int q = c * (C::kChunk / 2) + j;
                        acc[q] = __ffma2_rn(pv, sc[q], acc[q]);
                    }
                if (jg == kSmallScaleGroup - 1 || kb == kb1 - 1) {
                    // The group's last K block is done with its scales: release the slot.
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sempty + slot);
                    if (++slot == kSmallScaleGroups) { slot = 0; sphase ^= 1u; }
                }
                if (++buf == kNBuf) { buf = 0; bphase ^= 1u; }
            }
            const int64_t d_base = (MODE == kMasked ? static_cast<int64_t>(tl.g) * p.M : 0);
            if (S == 1) {
                // ---------------------------- unsplit tile: bf16 store ----
                // Stage the tile as bf16 [TN][128] (weight row fastest) and
                // write each row's 128 columns with 16-byte stores.  The first
                // barrier keeps this tile's staging off the previous tile's
                // reads.
                uint16_t* stg = reinterpret_cast<uint16_t*>(aux);
                named_barrier_sync(1, kSmallEpiThreads);
#pragma unroll
                for (int q = 0; q < C::kCols / 2; ++q) {
                    const __nv_bfloat162 h = __float22bfloat162_rn(acc[q]);
                    stg[(j_base + 2 * q) * 128 + n] = *reinterpret_cast<const uint16_t*>(&h.x);
                    stg[(j_base + 2 * q + 1) * 128 + n] = *reinterpret_cast<const uint16_t*>(&h.y);
                }
                named_barrier_sync(1, kSmallEpiThreads);
                for (int c = ptid; c < TN * 16; c += kSmallEpiThreads) {
                    const int j = c >> 4, col = tl.n0 + (c & 15) * 8;
                    const int row = tl.m0 + j;
                    if (row < tl.rows && col < p.N)
                        *reinterpret_cast<uint4*>(p.D + (d_base + row) * p.N + col) =
                            *reinterpret_cast<const uint4*>(stg + j * 128 + (c & 15) * 8);
                }
            } else {
                // ------------------------------ split tile: reduction ----
                // The ring is idle once this CTA's last partial has been read
                // out of TMEM (every load was consumed by an MMA that has
                // completed): it takes the FP32 partial.
#pragma unroll
                for (int q = 0; q < C::kCols / 2; ++q) {
                    red[(j_base + 2 * q) * 128 + n] = acc[q].x;
                    red[(j_base + 2 * q + 1) * 128 + n] = acc[q].y;
                }
                fence_proxy_async_smem();
                named_barrier_sync(1, kSmallEpiThreads);
                cluster_wait();  // every peer's receive barrier is initialised
                if (ptid == 0) {
                    for (int r = 0; r < S; ++r) {
                        if (r == rank) continue;
                        const int j0 = r * TN / S, j1 = (r + 1) * TN / S;
                        const uint32_t bytes = static_cast<uint32_t>((j1 - j0) * 128 * 4);
                        const int slot_in_r = rank < r ? rank : rank - 1;
                        bulk_copy_to_peer(dsmem_addr(smem_u32(aux) + static_cast<uint32_t>(slot_in_r) * bytes, r),
                                          red + j0 * 128, bytes, dsmem_addr(smem_u32(rbar), r));
                    }
                }
                // This CTA's rows: its own partial plus S - 1 received slices,
                // added in rank order.
                if (!mbar_wait(rbar, 0, abort_flag)) {
                    // Another role gave up: still let copies already on their
                    // way into this CTA land before it can exit.
                    ok = false;
                    mbar_wait_drain(rbar, 0);
                }
                // Everything this CTA receives has landed: arrive now, so the
                // barrier that keeps each CTA alive until every copy out of it
                // has completed overlaps the sums below.  The arrive needs no
                // release: a peer arrives only once its own receive barrier has
                // counted our copies in, and what this CTA reads after the
                // final wait is only its own shared memory.  (A release arrive
                // cost ~860 cycles here, on the critical path.)
                cluster_arrive_relaxed();
                const float* rcv = reinterpret_cast<const float*>(aux);
                const int rows_mine = my_j1 - my_j0;
                // One 8-column chunk per thread and step: a single pass for
                // the rows a CTA owns at TN <= 64, and one 16-byte store
                // (N % 8 == 0, so a chunk is wholly inside D or wholly past N).
                for (int e = ptid; e < rows_mine * 16; e += kSmallEpiThreads) {
                    const int jj = e >> 4, c8 = (e & 15) * 8;
                    float4 sa4 = make_float4(0.f, 0.f, 0.f, 0.f), sb4 = sa4;
#pragma unroll
                    for (int r = 0; r < C::kMaxSplit; ++r)
                        if (r < S) {
                            const float* src = r == rank ? red + (my_j0 + jj) * 128 + c8
                                                         : rcv + ((r < rank ? r : r - 1) * rows_mine + jj) * 128 + c8;
                            const float4 a4 = *reinterpret_cast<const float4*>(src);
                            const float4 b4 = *reinterpret_cast<const float4*>(src + 4);
                            if (r == 0) {
                                sa4 = a4; sb4 = b4;
                            } else {
                                sa4.x += a4.x; sa4.y += a4.y; sa4.z += a4.z; sa4.w += a4.w;
                                sb4.x += b4.x; sb4.y += b4.y; sb4.z += b4.z; sb4.w += b4.w;
                            }
                        }
                    const int row = tl.m0 + my_j0 + jj, col = tl.n0 + c8;
                    if (row < tl.rows && col < p.N) {
                        __nv_bfloat162 h0 = __floats2bfloat162_rn(sa4.x, sa4.y);
                        __nv_bfloat162 h1 = __floats2bfloat162_rn(sa4.z, sa4.w);
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(sb4.x, sb4.y);
                        __nv_bfloat162 h3 = __floats2bfloat162_rn(sb4.z, sb4.w);
                        uint4 pk;
                        pk.x = *reinterpret_cast<uint32_t*>(&h0);
                        pk.y = *reinterpret_cast<uint32_t*>(&h1);
                        pk.z = *reinterpret_cast<uint32_t*>(&h2);
                        pk.w = *reinterpret_cast<uint32_t*>(&h3);
                        *reinterpret_cast<uint4*>(p.D + (d_base + row) * p.N + col) = pk;
                    }
                }
            }
        }
        if (S > 1 && tiles <= cid) {
            // A cluster without a tile still completes both cluster barriers.
            cluster_wait();
            cluster_arrive();
        }
    }

    if (S > 1) cluster_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

}  // namespace dg
