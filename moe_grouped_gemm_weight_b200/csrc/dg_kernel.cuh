// dg_kernel.cuh -- persistent, warp-specialised sm_100a kernel for the FP8
// block-scaled NT GEMM (dense, grouped-contiguous and grouped-masked forms).
//
// Per output tile of 128 x BN:
//   * warp 0 (operand producer): TMA-loads, for every 128-wide K block kb,
//     the A tile [128 rows x 128 K] and the B tile [BN rows x 128 K]
//     (128-byte swizzle) into a STAGES-deep shared-memory ring.
//   * warps 1 and 3 (MMA, alternate K blocks): issue four tcgen05.mma
//     kind::f8f6f4 (K = 32 each) that write P_kb = A_kb . B_kb^T into a FRESH
//     TMEM buffer (one of NBUF), then commit to the ring's "empty" barrier and
//     the buffer's "full" barrier.
//   * warp 2 (scale producer): copies sa[m0..m0+127, kb] and the one or two
//     sb[n/128, kb] the tile needs into a 16-deep shared-memory scale ring,
//     running ahead of the promotion so that no global-memory latency sits on
//     its critical path.
//   * warps 4..11 (promotion + epilogue, two warpgroups splitting the tile's
//     columns): pull P_kb out of TMEM with tcgen05.ld, release the buffer,
//     and accumulate
//         acc[m,n] += (sa[m,kb] * sb[n/128,kb]) * P_kb[m,n]
//     in FP32 registers with packed FP32x2 FMAs -- the two-level accumulation
//     with promotion interval 128 described on the page "Deepseek DeepGEMM
//     技术原理的深入分析" (section "技术背景与核心原理").  After the last kb
//     they round to bf16 and store the valid rows and columns.
// TMEM buffers let the tensor core run up to NBUF-1 blocks ahead of the
// promotion, and the next tile's MMAs overlap the previous tile's epilogue.
// Tiles are handed out round-robin over a rasterised order (groups of
// `raster` m-blocks, m fastest) so CTAs running together share A and B in L2.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "dg_ptx.cuh"

namespace dg {

enum Mode : int { kDense = 0, kContiguous = 1, kMasked = 2, kKGrouped = 3 };

constexpr int kBM = 128;                 // tile rows = tcgen05 M
constexpr int kBK = 128;                 // K per block = scale granularity
constexpr int kThreads = 384;            // 12 warps
constexpr int kFirstEpiWarp = 4;         // warps 4..11: promotion/epilogue
constexpr int kEpiWarps = 8;
constexpr int kTileABytes = kBM * kBK;   // 16 KiB of e4m3
constexpr int kMaxMaskedGroups = 1024;   // masked mode: prefix table in smem
constexpr int kScaleSlots = 16;          // depth of the scale ring, in K blocks
constexpr int kScaleSlotFloats = kBM + 4;  // sa for 128 rows + up to 4 sb values
// fp8_gemm_kernel fills and releases the scale ring kScaleGroup K blocks at a
// time: its promotion waits on a scale barrier once per group instead of once
// per K block.
constexpr int kScaleGroup = 4;
constexpr int kScaleGroups = kScaleSlots / kScaleGroup;
constexpr int kStageOutBytes = 32 * 32 * 2;  // per promotion warp: 32 rows x 32 bf16 columns

struct Params {
    uint16_t* D;
    const float* sa;
    const float* sb;
    const int32_t* m_indices;  // contiguous mode
    const int32_t* masked_m;   // masked mode
    const int32_t* k_offsets;  // K-grouped mode: group g owns K [k_offsets[g], k_offsets[g+1])
    int sa_stride;
    int M;          // dense: M; contiguous: M_total; masked: M_max
    int N, K, G;
    int nkb;        // K / 128
    int nbn;        // ceil(N / 128): rows of sb per group
    int n_blocks;   // ceil(N / BN)
    int m_blocks;   // dense/contiguous: ceil(M / 128); masked: unused (device prefix)
    int raster;     // m-blocks per raster group
    int b_stream;   // 1: B is read once (evict-first in L2), 0: B is reused
    // K-split of the last partial wave (dense only; tail_split = 1: off).
    // Tiles [0, full_tiles) go round-robin, whole K; each of the remaining
    // tiles is split into tail_split K slices run by otherwise idle CTAs.
    int full_tiles;
    int tail_split;
    float* ws;            // FP32 partials of slices 1..tail_split-1
    unsigned int* ws_flags;  // one ready flag per partial
};

// One unit of work of this CTA: a tile (index t) over K blocks [kb0, kb1);
// slice = -1 for a whole tile, else the K slice of a split tail tile.
struct Work {
    int t, kb0, kb1, slice;
};

// The CTA's i-th unit of work (all roles walk the same sequence).
__device__ __forceinline__ bool next_work(const Params& p, int tiles, int i, Work& w) {
    const int full = p.tail_split > 1 ? p.full_tiles : tiles;
    const int t = blockIdx.x + i * gridDim.x;
    if (t < full) {
        w = {t, 0, p.nkb, -1};
        return true;
    }
    if (p.tail_split > 1 && i == p.full_tiles / static_cast<int>(gridDim.x)) {
        const int u = blockIdx.x;
        if (u < (tiles - full) * p.tail_split) {
            const int sl = u % p.tail_split;
            w = {full + u / p.tail_split, sl * p.nkb / p.tail_split, (sl + 1) * p.nkb / p.tail_split, sl};
            return true;
        }
    }
    return false;
}

// Tile configuration.  The promotion warpgroups split the tile's columns.
// BN = 192 uses three of them (64 columns per warp): every warp then reads its
// whole share of a K block's partial in one TMEM round trip and hands the
// buffer back before its FMAs, which keeps the FMAs off the path that frees
// TMEM for the next MMA.  BN = 256 uses two (128 columns per warp, read in two
// halves with FMAs in between -- accumulators plus a whole share would not fit
// in the register file).
template <int BN>
struct Cfg {
    static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN must be 64, 128, 192 or 256");
    static constexpr int kTileBBytes = BN * kBK;
    static constexpr int kNBuf = (BN <= 128) ? 4 : 2;
    static constexpr int kTmemCols = (kNBuf * BN <= 256) ? 256 : 512;
    static constexpr int kEpiWGs = (BN == 192) ? 3 : 2;     // promotion warpgroups
    static constexpr int kEpiWarpsC = 4 * kEpiWGs;
    static constexpr int kThreadsC = 32 * (kFirstEpiWarp + kEpiWarpsC);
    static constexpr int kColsPerWarp = BN / kEpiWGs;
    static constexpr int kChunks = kColsPerWarp / 32;  // tcgen05.ld 32x32b.x32 chunks
    static constexpr int kBatch = kChunks < 2 ? kChunks : 2;  // chunks loaded per wait
    static constexpr bool kSplitRegs = BN > 128;       // needs setmaxnreg rebalancing
    // setmaxnreg budgets (multiples of 8) for the producer/MMA/scale warpgroup
    // and the promotion warpgroups; their sum over all threads stays within
    // the 64 K registers the CTA launches with.
    static constexpr int kRegsLow = kEpiWGs == 3 ? 40 : 56;
    static constexpr int kRegsHigh = kEpiWGs == 3 ? 152 : 224;
    static_assert(128 * kRegsLow + 128 * kEpiWGs * kRegsHigh <= 65536, "register split exceeds the file");
    static_assert(kNBuf * BN <= kTmemCols, "TMEM buffers overflow the allocation");
    static_assert(kChunks % kBatch == 0, "chunk batching");
};

template <int BN, int STAGES, int SP = 1>
constexpr int smem_bytes() {
    // 1 KiB alignment slack + operand ring + output staging (SP pieces of
    // 32 x 32 bf16 per promotion warp) + barriers and bookkeeping (512 B) +
    // scale ring + masked prefix table.
    return 1024 + STAGES * (kTileABytes + Cfg<BN>::kTileBBytes) + Cfg<BN>::kEpiWarpsC * SP * kStageOutBytes + 512 +
           kScaleSlots * kScaleSlotFloats * 4 + 4 * (kMaxMaskedGroups + 1);
}

struct Tile {
    int g;        // group
    int m0;       // first output row (dense/contiguous: global; masked: inside group g)
    int n0;       // first output column
    bool valid;
};

// Linear tile index -> (m-block, n-block) in a rasterised order: the m-blocks
// are taken in groups of `raster`; inside a group m runs fastest.
__device__ __forceinline__ void raster_tile(int t, int m_blocks, int n_blocks, int raster, int& mb, int& nb) {
    const int per_group = raster * n_blocks;
    const int sg = t / per_group;
    const int within = t - sg * per_group;
    const int first = sg * raster;
    const int gm = min(raster, m_blocks - first);
    mb = first + within % gm;
    nb = within / gm;
}

template <int BN, int MODE>
__device__ __forceinline__ Tile decode_tile(const Params& p, int t, int m_blocks, const int* mb_prefix) {
    int mb, nb;
    if (MODE == kKGrouped) {
        // Groups outermost: tiles of one group share its K range of A and B.
        const int per_group = m_blocks * p.n_blocks;
        raster_tile(t % per_group, m_blocks, p.n_blocks, p.raster, mb, nb);
        Tile tl;
        tl.g = t / per_group;
        tl.m0 = mb * kBM;
        tl.n0 = nb * BN;
        tl.valid = true;
        return tl;
    }
    raster_tile(t, m_blocks, p.n_blocks, p.raster, mb, nb);
    Tile tl;
    tl.n0 = nb * BN;
    tl.valid = true;
    if (MODE == kDense) {
        tl.g = 0;
        tl.m0 = mb * kBM;
    } else if (MODE == kContiguous) {
        tl.m0 = mb * kBM;
        const int g = __ldg(p.m_indices + tl.m0);
        // A tile whose first row is padding holds only padding (segments are
        // aligned to 128 rows and padded at their end); out-of-range group
        // ids are bad data and are skipped (the epilogue flags them).
        tl.g = g;
        tl.valid = (g >= 0 && g < p.G);
    } else {
        // Largest g with mb_prefix[g] <= mb: the group owning global m-block mb.
        int lo = 0, hi = p.G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (mb_prefix[mid] <= mb) lo = mid; else hi = mid - 1;
        }
        tl.g = lo;
        tl.m0 = (mb - mb_prefix[lo]) * kBM;
    }
    return tl;
}

// K-grouped mode: the tile's K blocks are its group's [k_offsets[g], k_offsets[g+1]).
// Offsets that are not multiples of 128, decrease, or leave [0, K] are bad
// data: flagged (DG_DEVERR_BAD_K_OFFSET) and the group treated as empty, so
// its D is written as zeros.
template <int MODE>
__device__ __forceinline__ void group_k_range(const Params& p, const Tile& tl, Work& w) {
    if (MODE != kKGrouped) return;
    const int k0 = __ldg(p.k_offsets + tl.g), k1 = __ldg(p.k_offsets + tl.g + 1);
    if (k0 < 0 || k1 < k0 || k1 > p.K || (k0 | k1) % kBK != 0) {
        if (threadIdx.x == 0 && tl.m0 == 0 && tl.n0 == 0) atomicOr(&g_dg_error, 16u);
        w.kb0 = w.kb1 = 0;
        return;
    }
    w.kb0 = k0 / kBK;
    w.kb1 = k1 / kBK;
}

// LAYOUT (dense only) gives the operands' storage: bit 0 set = A stored
// [K][M] (M-major, the "T" of TN / TT), bit 1 set = B stored [K][N] (N-major,
// the "N" of NN / TN); clear = K-major as in NT.  An MN-major operand is loaded
// as 128 x 128 TMA boxes (MN inner) and described to the MMA as MN-major.
// SP: staging pieces per promotion warp.  With one, each 32 x 32 piece of
// the epilogue waits until the previous piece's TMA store has read the
// buffer; with one per piece of the warp's columns, a tile's whole epilogue
// is staged and stored without waiting (the next tile's epilogue waits once),
// which pays on short K where the epilogue is a large share of a tile.
template <int BN, int STAGES, int MODE, int LAYOUT = 0, int SP = 1>
__global__ void __launch_bounds__(Cfg<BN>::kThreadsC, 1)
fp8_gemm_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmA,
                const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmD) {
    using C = Cfg<BN>;
    constexpr int kNBuf = C::kNBuf;
    constexpr bool kAmn = (LAYOUT & 1) != 0;
    constexpr bool kBmn = (LAYOUT & 2) != 0;
    static_assert(LAYOUT == 0 || ((MODE == kDense || MODE == kKGrouped) && BN % 128 == 0),
                  "MN-major operands: dense or K-grouped, BN 128 or 256");
    static_assert(MODE != kKGrouped || LAYOUT == 3, "K-grouped: A stored [K][M], B stored [K][N]");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + STAGES * kTileABytes;
    uint8_t* sOut = sB + STAGES * C::kTileBBytes;  // 1 KiB aligned, SP x kStageOutBytes per promotion warp
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + C::kEpiWarpsC * SP * kStageOutBytes);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + kNBuf;
    uint64_t* sfull = tempty + kNBuf;
    uint64_t* sempty = sfull + kScaleSlots;
    uint64_t* done = sempty + kScaleSlots;  // one per MMA warp
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* sring = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 512);
    int* mb_prefix = reinterpret_cast<int*>(sring + kScaleSlots * kScaleSlotFloats);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int b = 0; b < kNBuf; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, C::kEpiWarpsC);
        }
        for (int s = 0; s < kScaleSlots; ++s) {
            mbar_init(sfull + s, 32);
            mbar_init(sempty + s, C::kEpiWarpsC);
        }
        mbar_init(done, 1);
        mbar_init(done + 1, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmD);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    // Nothing above reads or writes global data: with programmatic dependent
    // launch it overlaps the end of the previous kernel in the stream.
    griddep_wait();
    griddep_launch_dependents();
    int m_blocks = p.m_blocks;
    if (MODE == kMasked) {
        // Per-group m-block counts from the device-resident masked_m, then an
        // exclusive prefix over groups.  Counts outside [0, M_max] are clamped
        // and flagged.
        for (int g = threadIdx.x; g < p.G; g += C::kThreadsC) {
            int mm = __ldg(p.masked_m + g);
            if (mm < 0 || mm > p.M) {
                atomicOr(&g_dg_error, 4u);
                mm = min(max(mm, 0), p.M);
            }
            mb_prefix[g + 1] = (mm + kBM - 1) / kBM;
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
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    if (MODE == kMasked) m_blocks = mb_prefix[p.G];
    const int tiles = (MODE == kKGrouped ? p.G : 1) * m_blocks * p.n_blocks;
    const int nkb = p.nkb;

    // Register budget: the producer / MMA / scale warps need few registers,
    // the promotion warps hold BN/2 FP32 accumulators each.  Each branch sets
    // its own budget so that the compiler allocates every role against it.
    if (warp < kFirstEpiWarp) {
    if (C::kSplitRegs) regs_dec<C::kRegsLow>();
    if (warp == 0) {
        // ------------------------------------------------------ producer ----
        const uint64_t pol_a = l2_policy_evict_last();
        const uint64_t pol_b = p.b_stream ? l2_policy_evict_first() : l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        int fills = 0;
        bool ok = true;
        Work w;
        for (int it = 0; ok && next_work(p, tiles, it, w); ++it) {
            const Tile tl = decode_tile<BN, MODE>(p, w.t, m_blocks, mb_prefix);
            if (!tl.valid) continue;
            group_k_range<MODE>(p, tl, w);
            for (int kb = w.kb0; kb < w.kb1; ++kb) {
                if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(full + stage, kTileABytes + C::kTileBBytes);
                    if (kAmn)
                        tma_load_2d(sA + stage * kTileABytes, &tmA, full + stage, tl.m0, kb * kBK, pol_a);
                    else if (MODE == kMasked)
                        tma_load_3d(sA + stage * kTileABytes, &tmA, full + stage, kb * kBK, tl.m0, tl.g, pol_a);
                    else
                        tma_load_2d(sA + stage * kTileABytes, &tmA, full + stage, kb * kBK, tl.m0, pol_a);
                    if (kBmn) {
#pragma unroll
                        for (int h = 0; h < BN / 128; ++h)
                            tma_load_2d(sB + stage * C::kTileBBytes + h * 128 * kBK, &tmB, full + stage, tl.n0 + h * 128,
                                        kb * kBK, pol_b);
                    } else {
                        tma_load_3d(sB + stage * C::kTileBBytes, &tmB, full + stage, kb * kBK, tl.n0, tl.g, pol_b);
                    }
                }
                __syncwarp();
                ++fills;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        // Make sure no copy into this CTA's shared memory is still in flight
        // before the CTA can exit (matters only after an abort).
        if (lane == 0) {
            const int first = fills > STAGES ? fills - STAGES : 0;
            for (int i = first; i < fills; ++i)
                mbar_wait_drain(full + (i % STAGES), static_cast<uint32_t>((i / STAGES) & 1));
        }
        __syncwarp();
    } else if (warp == 1 || warp == 3) {
        // ----------------------------------------------------------- MMA ----
        // Two warps issue the MMAs of alternate K blocks (the CTA's i-th K
        // block goes to warp 1 for even i, to warp 3 for odd i).  Issuing a
        // block's four tcgen05.mma and two commits keeps a warp busy for
        // several hundred cycles; with two issuers one of them is always
        // already waiting for the next free TMEM buffer, so the tensor core
        // gets the next block as soon as the promotion releases it.
        constexpr uint32_t idesc = idesc_e4m3_f32_major(kBM, BN, kAmn, kBmn);
        const int mw = warp == 1 ? 0 : 1;
        int i = 0;  // K blocks of this CTA so far, over all its work
        bool ok = true;
        Work w;
        for (int it = 0; ok && next_work(p, tiles, it, w); ++it) {
            const Tile tl = decode_tile<BN, MODE>(p, w.t, m_blocks, mb_prefix);
            if (!tl.valid) continue;
            group_k_range<MODE>(p, tl, w);
            for (int kb = w.kb0; kb < w.kb1; ++kb, ++i) {
                if ((i & 1) != mw) continue;
                const int stage = i % STAGES, buf = i % kNBuf;
                const uint32_t phase = static_cast<uint32_t>(i / STAGES) & 1u;
                const uint32_t bphase = static_cast<uint32_t>(i / kNBuf) & 1u;
                if (!mbar_wait(tempty + buf, bphase ^ 1u, abort_flag)) { ok = false; break; }
                if (!mbar_wait(full + stage, phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a_addr = smem_u32(sA + stage * kTileABytes);
                    const uint32_t b_addr = smem_u32(sB + stage * C::kTileBBytes);
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
#pragma unroll
                    for (int k = 0; k < kBK / 32; ++k) {
                        const uint64_t ad = kAmn ? sdesc_mnmajor_sw128(a_addr + k * 32 * 128, 128 * kBK)
                                                 : sdesc_kmajor_sw128(a_addr + k * 32);
                        const uint64_t bd = kBmn ? sdesc_mnmajor_sw128(b_addr + k * 32 * 128, 128 * kBK)
                                                 : sdesc_kmajor_sw128(b_addr + k * 32);
                        umma_f8(d_tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
                    }
                    umma_commit(empty + stage);
                    umma_commit(tfull + buf);
                }
                __syncwarp();
            }
        }
        // All MMAs of this warp must have finished before TMEM is released.
        if (lane == 0) {
            umma_commit(done + mw);
            mbar_wait_drain(done + mw, 0);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------------------------ scale producer ----
        // Per K block: lane l copies sa rows m0+4l..m0+4l+3 (16 bytes) and
        // lanes 0..3 the tile's sb values; the copies run asynchronously.  A
        // group of up to kScaleGroup consecutive K blocks of the tile shares
        // one ring slot and one barrier, completed when all of its copies
        // land, so this warp only ever waits for a free slot.  Rows past the
        // data and sb blocks past N are zero-filled, nothing outside the
        // tensors is read.
        int slot = 0;
        uint32_t sphase = 0;
        const int row_limit = p.M;  // rows of sa that exist (dense M, M_total or M_max)
        Work w;
        for (int it = 0; next_work(p, tiles, it, w); ++it) {
            const Tile tl = decode_tile<BN, MODE>(p, w.t, m_blocks, mb_prefix);
            if (!tl.valid) continue;
            group_k_range<MODE>(p, tl, w);
            const float* sa_base = p.sa + (MODE == kMasked ? static_cast<int64_t>(tl.g) * nkb * p.sa_stride : 0);
            const float* sb_g = p.sb + (MODE == kKGrouped ? 0 : static_cast<int64_t>(tl.g) * p.nbn * nkb);
            const int nb = tl.n0 / 128 + (lane & 3);
            const bool nb_ok = nb < p.nbn;
            const int r4 = tl.m0 + lane * 4;
            const int left = row_limit - r4;
            const uint32_t sa_bytes = left >= 4 ? 16u : (left > 0 ? static_cast<uint32_t>(left) * 4u : 0u);
            bool ok = true;
            for (int kg = w.kb0; kg < w.kb1; kg += kScaleGroup) {
                if (!mbar_wait(sempty + slot, sphase ^ 1u, abort_flag)) { ok = false; break; }
                const int n = min(kScaleGroup, w.kb1 - kg);
                for (int j = 0; j < n; ++j) {
                    const int kb = kg + j;
                    const uint32_t dst = smem_u32(sring + (slot * kScaleGroup + j) * kScaleSlotFloats);
                    const float* src = sa_bytes ? sa_base + static_cast<int64_t>(kb) * p.sa_stride + r4 : p.sa;
                    cp_async_16(dst + lane * 16, src, sa_bytes);
                    if (lane < 4)
                        cp_async_4(dst + (kBM + lane) * 4, nb_ok ? sb_g + static_cast<int64_t>(nb) * nkb + kb : p.sb,
                                   nb_ok ? 4u : 0u);
                }
                cp_async_arrive(sfull + slot);
                if (++slot == kScaleGroups) { slot = 0; sphase ^= 1u; }
            }
            if (!ok) break;
        }
        // Let every copy land before the CTA can exit.
        asm volatile("cp.async.wait_all;" ::: "memory");
    }
    } else {
        // ------------------------------------------ promotion + epilogue ----
        if (C::kSplitRegs) regs_inc<C::kRegsHigh>();
        const int ew = warp - kFirstEpiWarp;
        const int half = ew >> 2;                 // which warpgroup's share of the tile's columns
        const int quarter = warp & 3;             // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;        // row inside the tile
        const int col0 = half * C::kColsPerWarp;  // first column inside the tile
        const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        int buf = 0, slot = 0;
        uint32_t bphase = 0, sphase = 0;
        bool ok = true;
        Work w;
        for (int it = 0; ok && next_work(p, tiles, it, w); ++it) {
            const Tile tl = decode_tile<BN, MODE>(p, w.t, m_blocks, mb_prefix);
            if (!tl.valid) continue;
            group_k_range<MODE>(p, tl, w);
            const int g = tl.g;
            // Row validity and the row's output address.
            const int row = tl.m0 + r;
            bool row_ok;
            int64_t d_row;
            if (MODE == kMasked) {
                const int mm = min(max(__ldg(p.masked_m + g), 0), p.M);
                row_ok = row < mm;
                d_row = static_cast<int64_t>(g) * p.M + row;
            } else if (MODE == kContiguous) {
                const int gi = __ldg(p.m_indices + row);
                row_ok = (gi == g);
                if (gi != g && gi != -1) atomicOr(&g_dg_error, 2u);
                d_row = row;
            } else if (MODE == kKGrouped) {
                row_ok = row < p.M;
                d_row = static_cast<int64_t>(g) * p.M + row;
            } else {
                row_ok = row < p.M;
                d_row = row;
            }
            // Which of the scale ring's sb values each 32-column chunk uses.
            int sb_sel[C::kChunks];
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c) sb_sel[c] = (tl.n0 + col0 + c * 32) / 128 - tl.n0 / 128;

            float2 acc[C::kColsPerWarp / 2];
#pragma unroll
            for (int j = 0; j < C::kColsPerWarp / 2; ++j) acc[j] = make_float2(0.f, 0.f);

            for (int kb = w.kb0; kb < w.kb1; ++kb) {
                const int jg = (kb - w.kb0) % kScaleGroup;  // K block inside its scale group
                if (jg == 0 && !mbar_wait(sfull + slot, sphase, abort_flag)) { ok = false; break; }
                const float* sc = sring + (slot * kScaleGroup + jg) * kScaleSlotFloats;
                const float s_a = sc[r];
                float2 s2[C::kChunks];
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c) {
                    const float s = s_a * sc[kBM + sb_sel[c]];
                    s2[c] = make_float2(s, s);
                }
                if (jg == kScaleGroup - 1 || kb == w.kb1 - 1) {
                    // The group's last K block has read its scales: release the slot.
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sempty + slot);
                    if (++slot == kScaleGroups) { slot = 0; sphase ^= 1u; }
                }

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
                        // Last TMEM read of this buffer: hand it back to the MMA warp.
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(tempty + buf);
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

            if (w.slice >= 0) {
                // Split tail tile.  Partial (r, s) for slices s >= 1 lives at
                // ws + ((r*(S-1) + s-1) * 128*BN) floats in the layout
                // [promotion warp][float4 j][lane], so a warp moves 512
                // contiguous bytes per access.  Slice s >= 1 writes its partial
                // and raises its flag; slice 0 waits for every flag, adds the
                // partials in slice order (fixed, so the result is
                // deterministic), resets the flags and stores D.
                constexpr int kF4 = C::kColsPerWarp / 4;
                const int S = p.tail_split;
                const int rt = w.t - p.full_tiles;
                const int nthreads = 32 * C::kEpiWarpsC;
                const bool leader = (warp == kFirstEpiWarp && lane == 0);
                if (w.slice > 0) {
                    float4* dst = reinterpret_cast<float4*>(p.ws + static_cast<int64_t>(rt * (S - 1) + w.slice - 1) * kBM * BN);
#pragma unroll
                    for (int j = 0; j < kF4; ++j)
                        __stcg(dst + (ew * kF4 + j) * 32 + lane,
                               make_float4(acc[2 * j].x, acc[2 * j].y, acc[2 * j + 1].x, acc[2 * j + 1].y));
                    __threadfence();
                    named_barrier_sync(1, nthreads);
                    if (leader) st_release_gpu(p.ws_flags + rt * (S - 1) + w.slice - 1, 1u);
                    continue;  // slice 0 stores the tile
                }
                // slice 0
                bool got = true;
                if (leader) {
                    for (int s2 = 1; s2 < S && got; ++s2)
                        got = wait_flag_gpu(p.ws_flags + rt * (S - 1) + s2 - 1);
                    for (int s2 = 1; s2 < S; ++s2) p.ws_flags[rt * (S - 1) + s2 - 1] = 0u;
                    if (!got) atomicOr(&g_dg_error, 1u);
                }
                named_barrier_sync(1, nthreads);
                for (int s2 = 1; s2 < S; ++s2) {
                    const float4* src = reinterpret_cast<const float4*>(
                        p.ws + static_cast<int64_t>(rt * (S - 1) + s2 - 1) * kBM * BN);
#pragma unroll
                    for (int j = 0; j < kF4; ++j) {
                        const float4 v = __ldcg(src + (ew * kF4 + j) * 32 + lane);
                        acc[2 * j].x += v.x;
                        acc[2 * j].y += v.y;
                        acc[2 * j + 1].x += v.z;
                        acc[2 * j + 1].y += v.w;
                    }
                }
            }

            // Epilogue: bf16 round-to-nearest-even.  When every row of this
            // warp may be written (valid, or outside D where the TMA store
            // clips it), the warp stages 32 rows x 32 columns at a time in
            // shared memory (64-byte swizzle: 16-byte chunk q of row r sits at
            // r*64 + 16*(q ^ ((r >> 1) & 3)), conflict-free for the warp) and
            // one lane issues a TMA store; the copy drains while the warp
            // moves on.  Warps holding rows that must stay untouched (padding
            // rows, rows past masked_m) store their valid rows directly.
            const bool clip_ok = row_ok || MODE == kDense || MODE == kKGrouped || (MODE == kMasked && row >= p.M);
            if (__all_sync(0xffffffffu, clip_ok)) {
                static_assert(SP == 1 || SP == C::kColsPerWarp / 32, "one staging piece, or one per piece");
                if (SP > 1) {
                    if (lane == 0) bulk_wait_read<0>();  // the previous tile's stores have read every piece
                    __syncwarp();
                }
#pragma unroll
                for (int pc = 0; pc < C::kColsPerWarp / 32; ++pc) {
                    uint8_t* piece = sOut + (ew * SP + (SP > 1 ? pc : 0)) * kStageOutBytes;
                    const uint32_t stg = smem_u32(piece);
                    if (SP == 1) {
                        if (lane == 0) bulk_wait_read<0>();  // previous store has read the buffer
                        __syncwarp();
                    }
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
                        if (MODE == kMasked || MODE == kKGrouped)
                            tma_store_3d(&tmD, piece, x, tl.m0 + quarter * 32, g);
                        else
                            tma_store_2d(&tmD, piece, x, tl.m0 + quarter * 32);
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
        // Every TMA store of this warp must have completed before the CTA exits.
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

}  // namespace dg
