// dg_kernel.cuh -- persistent, warp-specialised sm_100a kernel for the FP8
// block-scaled NT GEMM (dense, grouped-contiguous and grouped-masked forms).
//
// Per output tile of 128 x BN:
//   * warp 0 (producer): TMA-loads, for every 128-wide K block kb, the A tile
//     [128 rows x 128 K] and the B tile [BN rows x 128 K] (128-byte swizzle)
//     into a STAGES-deep shared-memory ring.
//   * warp 1 (MMA): issues four tcgen05.mma kind::f8f6f4 (K = 32 each) that
//     write P_kb = A_kb . B_kb^T into a FRESH TMEM buffer (one of NBUF), then
//     commits to the ring's "empty" barrier and the buffer's "full" barrier.
//   * warps 4..11 (promotion + epilogue): pull P_kb out of TMEM with
//     tcgen05.ld, release the buffer, and accumulate
//         acc[m,n] += (sa[m,kb] * sb[n/128,kb]) * P_kb[m,n]
//     in FP32 registers -- the two-level accumulation with promotion interval
//     128 described on the page "Deepseek DeepGEMM 技术原理的深入分析" (section
//     "技术背景与核心原理").  After the last kb they round to bf16 and store
//     the valid rows and columns.
// TMEM buffers let the tensor core run up to NBUF-1 blocks ahead of the
// promotion, and the next tile's MMAs overlap the previous tile's epilogue.
// Tiles are handed out round-robin over a rasterised order (groups of
// `raster` m-blocks, m fastest) so CTAs running together share A and B in L2.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "dg_ptx.cuh"

namespace dg {

enum Mode : int { kDense = 0, kContiguous = 1, kMasked = 2 };

constexpr int kBM = 128;                 // tile rows = tcgen05 M
constexpr int kBK = 128;                 // K per block = scale granularity
constexpr int kThreads = 384;            // 12 warps
constexpr int kFirstEpiWarp = 4;         // warps 4..11: promotion/epilogue
constexpr int kEpiWarps = 8;
constexpr int kTileABytes = kBM * kBK;   // 16 KiB of e4m3
constexpr int kMaxMaskedGroups = 1024;   // masked mode: prefix table in smem

struct Params {
    uint16_t* D;
    const float* sa;
    const float* sb;
    const int32_t* m_indices;  // contiguous mode
    const int32_t* masked_m;   // masked mode
    int sa_stride;
    int M;          // dense: M; contiguous: M_total; masked: M_max
    int N, K, G;
    int nkb;        // K / 128
    int nbn;        // ceil(N / 128): rows of sb per group
    int n_blocks;   // ceil(N / BN)
    int m_blocks;   // dense/contiguous: ceil(M / 128); masked: unused (device prefix)
    int raster;     // m-blocks per raster group
};

template <int BN>
struct Cfg {
    static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN must be 64, 128, 192 or 256");
    static constexpr int kTileBBytes = BN * kBK;
    static constexpr int kNBuf = (BN <= 128) ? 4 : 2;
    static constexpr int kTmemCols = (kNBuf * BN <= 256) ? 256 : 512;
    static constexpr int kColsPerWarp = BN / 2;       // two warpgroups split the columns
    static constexpr int kChunks = kColsPerWarp / 32;  // tcgen05.ld 32x32b.x32 chunks
    static_assert(kNBuf * BN <= kTmemCols, "TMEM buffers overflow the allocation");
};

template <int BN, int STAGES>
constexpr int smem_bytes() {
    // 1 KiB alignment slack + operand ring + barriers / bookkeeping + masked prefix table.
    return 1024 + STAGES * (kTileABytes + Cfg<BN>::kTileBBytes) + 256 + 4 * (kMaxMaskedGroups + 1);
}

struct Tile {
    int g;        // group
    int a_row;    // A row coordinate (dense/contiguous: global row; masked: row inside group)
    int n0;       // first output column
    int m0;       // first output row (dense/contiguous: global; masked: inside group)
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
    raster_tile(t, m_blocks, p.n_blocks, p.raster, mb, nb);
    Tile tl;
    tl.n0 = nb * BN;
    tl.valid = true;
    if (MODE == kDense) {
        tl.g = 0;
        tl.m0 = tl.a_row = mb * kBM;
    } else if (MODE == kContiguous) {
        tl.m0 = tl.a_row = mb * kBM;
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
        tl.m0 = tl.a_row = (mb - mb_prefix[lo]) * kBM;
    }
    return tl;
}

template <int BN, int STAGES, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
fp8_gemm_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tmA,
                const __grid_constant__ CUtensorMap tmB) {
    using C = Cfg<BN>;
    constexpr int kNBuf = C::kNBuf;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = sA + STAGES * kTileABytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * C::kTileBBytes);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + kNBuf;
    uint64_t* done = tempty + kNBuf;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* mb_prefix = const_cast<int*>(reinterpret_cast<volatile int*>(abort_flag + 1));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int b = 0; b < kNBuf; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, kEpiWarps);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    int m_blocks = p.m_blocks;
    if (MODE == kMasked) {
        // Per-group m-block counts from the device-resident masked_m, then an
        // exclusive prefix over groups.  Counts outside [0, M_max] are clamped
        // and flagged.
        for (int g = threadIdx.x; g < p.G; g += kThreads) {
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
    const int tiles = m_blocks * p.n_blocks;
    const int nkb = p.nkb;

    if (warp == 0) {
        // ------------------------------------------------------ producer ----
        const uint64_t pol_a = l2_policy_evict_last();
        const uint64_t pol_b = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        int fills = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            const Tile tl = decode_tile<BN, MODE>(p, t, m_blocks, mb_prefix);
            if (!tl.valid) continue;
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(empty + stage, phase ^ 1u, abort_flag)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(full + stage, kTileABytes + C::kTileBBytes);
                    if (MODE == kMasked)
                        tma_load_3d(sA + stage * kTileABytes, &tmA, full + stage, kb * kBK, tl.a_row, tl.g, pol_a);
                    else
                        tma_load_2d(sA + stage * kTileABytes, &tmA, full + stage, kb * kBK, tl.a_row, pol_a);
                    tma_load_3d(sB + stage * C::kTileBBytes, &tmB, full + stage, kb * kBK, tl.n0, tl.g, pol_b);
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
    } else if (warp == 1) {
        // ----------------------------------------------------------- MMA ----
        constexpr uint32_t idesc = idesc_e4m3_f32(kBM, BN);
        int stage = 0, buf = 0;
        uint32_t phase = 0, bphase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            const Tile tl = decode_tile<BN, MODE>(p, t, m_blocks, mb_prefix);
            if (!tl.valid) continue;
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
                        umma_f8(d_tmem, sdesc_kmajor_sw128(a_addr + k * 32), sdesc_kmajor_sw128(b_addr + k * 32),
                                idesc, k > 0 ? 1u : 0u);
                    umma_commit(empty + stage);
                    umma_commit(tfull + buf);
                }
                __syncwarp();
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                if (++buf == kNBuf) { buf = 0; bphase ^= 1u; }
            }
        }
        // All MMAs of this CTA must have finished before TMEM is released.
        if (lane == 0) {
            umma_commit(done);
            mbar_wait_drain(done, 0);
        }
        __syncwarp();
    } else if (warp >= kFirstEpiWarp) {
        // ------------------------------------------ promotion + epilogue ----
        const int ew = warp - kFirstEpiWarp;
        const int half = ew >> 2;                 // which half of the tile's columns
        const int quarter = warp & 3;             // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;        // row inside the tile
        const int col0 = half * C::kColsPerWarp;  // first column inside the tile
        const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        int buf = 0;
        uint32_t bphase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            const Tile tl = decode_tile<BN, MODE>(p, t, m_blocks, mb_prefix);
            if (!tl.valid) continue;
            const int g = tl.g;
            // Row validity and the row's output / scale addresses.
            const int row = tl.m0 + r;
            bool row_ok;
            int64_t d_row;
            const float* sa_row;
            if (MODE == kMasked) {
                const int mm = min(max(__ldg(p.masked_m + g), 0), p.M);
                row_ok = row < mm;
                d_row = static_cast<int64_t>(g) * p.M + row;
                sa_row = p.sa + static_cast<int64_t>(g) * nkb * p.sa_stride + row;
            } else if (MODE == kContiguous) {
                const int gi = __ldg(p.m_indices + row);
                row_ok = (gi == g);
                if (gi != g && gi != -1) atomicOr(&g_dg_error, 2u);
                d_row = row;
                sa_row = p.sa + row;
            } else {
                row_ok = row < p.M;
                d_row = row;
                sa_row = p.sa + row;
            }
            const float* sb_g = p.sb + static_cast<int64_t>(g) * p.nbn * nkb;
            int nb_idx[C::kChunks];
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
                nb_idx[c] = min((tl.n0 + col0 + c * 32) / 128, p.nbn - 1);

            float acc[C::kColsPerWarp];
#pragma unroll
            for (int j = 0; j < C::kColsPerWarp; ++j) acc[j] = 0.f;

            for (int kb = 0; kb < nkb; ++kb) {
                const float s_a = row_ok ? __ldg(sa_row + static_cast<int64_t>(kb) * p.sa_stride) : 0.f;
                float s[C::kChunks];
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c) s[c] = s_a * __ldg(sb_g + nb_idx[c] * nkb + kb);

                if (!mbar_wait(tfull + buf, bphase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                uint32_t v[C::kChunks][32];
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
                    tmem_ld_32x32b_x32(t_lane + static_cast<uint32_t>(buf * BN + col0 + c * 32), v[c]);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c) reg_fence(v[c]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty + buf);
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c)
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        acc[c * 32 + j] = fmaf(__uint_as_float(v[c][j]), s[c], acc[c * 32 + j]);
                if (++buf == kNBuf) { buf = 0; bphase ^= 1u; }
            }
            if (!ok) break;

            // Epilogue: bf16 round-to-nearest-even, 16-byte stores of the valid
            // part of this row (N % 8 == 0, so 8-column groups are all-or-none).
            if (row_ok) {
                uint16_t* drow = p.D + d_row * p.N;
#pragma unroll
                for (int c = 0; c < C::kChunks; ++c) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int col = tl.n0 + col0 + c * 32 + q * 8;
                        if (col < p.N) {
                            uint4 pk;
                            const float* a8 = acc + c * 32 + q * 8;
                            __nv_bfloat162 h0 = __floats2bfloat162_rn(a8[0], a8[1]);
                            __nv_bfloat162 h1 = __floats2bfloat162_rn(a8[2], a8[3]);
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(a8[4], a8[5]);
                            __nv_bfloat162 h3 = __floats2bfloat162_rn(a8[6], a8[7]);
                            pk.x = *reinterpret_cast<uint32_t*>(&h0);
                            pk.y = *reinterpret_cast<uint32_t*>(&h1);
                            pk.z = *reinterpret_cast<uint32_t*>(&h2);
                            pk.w = *reinterpret_cast<uint32_t*>(&h3);
                            *reinterpret_cast<uint4*>(drow + col) = pk;
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

}  // namespace dg
