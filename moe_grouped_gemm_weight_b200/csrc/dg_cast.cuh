// dg_cast.cuh -- sm_100a FP8 cast kernels (the GEMM's operand preparation).
//
// The pages leave the cast to the caller ("DeepGEMM项目介绍与本地部署指南",
// section "接口": e4m3 inputs, transposed TMA-aligned LHS scales) and name a
// helper to_fp8 that returns the FP8 tensor with its scales (the later-version
// article, section 4.1).  Per tile (1x128 of an activation row, 128x128 of a
// weight matrix), in IEEE single precision:
//
//   amax = max(max |x|, 1e-4)      s = amax / 448      r = 448 / amax
//   q    = e4m3 (round to nearest even, saturating to +-448) of x * r
//
// s is the scale the GEMM reads (sa transposed: sa[kb*sa_stride + m]; sb row
// major [N/128][K/128]); s * q ~ x, and the largest |x| of a tile maps to 448.
// Both kernels are bound by HBM: per element 2 bytes in, 1 byte out.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "dg_ptx.cuh"

namespace dg {

constexpr int kCastThreads = 256;
constexpr int kCastRowsPerCta = 16;  // 1x128 cast: one half-warp per row tile

struct CastParams {
    uint8_t* Q;
    float* s;          // 1x128: sa (transposed, sa_stride); 128x128: sb [N/128][K/128]
    const uint16_t* X;
    int rows, K, nkb;
    int sa_stride;
};

// 8 bf16 (one 16-byte load) -> floats.
__device__ __forceinline__ void bf16x8_to_float(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// 8 floats times r -> 8 e4m3 codes (RNE, saturating), packed little-endian.
__device__ __forceinline__ uint2 e4m3x8(const float (&f)[8], float r) {
    uint32_t p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 y = make_float2(__fmul_rn(f[2 * i], r), __fmul_rn(f[2 * i + 1], r));
        p[i] = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
    }
    return make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
}

__device__ __forceinline__ float amax8(const float (&f)[8]) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(f[i]));
    return a;
}

__device__ __forceinline__ uint4 ld_stream_16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Activations.  Work item = (16 rows, kCastBlocks K blocks): half-warp h of
// the CTA takes row 16*i + h, its lanes 8 consecutive bf16 of each block
// (kCastBlocks 16-byte loads in flight per thread before any is used).  The
// 16 half-warps of a CTA write 16 consecutive scales of each K block.
constexpr int kCastBlocks = 4;

__global__ void __launch_bounds__(kCastThreads)
cast_1x128_kernel(const CastParams p) {
    griddep_wait();
    griddep_launch_dependents();
    const int half = threadIdx.x >> 4;  // 0..15: row inside the item
    const int hl = threadIdx.x & 15;    // lane inside the half-warp
    const int row_groups = (p.rows + kCastRowsPerCta - 1) / kCastRowsPerCta;
    const int kb_groups = (p.nkb + kCastBlocks - 1) / kCastBlocks;
    const int64_t items = static_cast<int64_t>(row_groups) * kb_groups;
    for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
        const int rg = static_cast<int>(it % row_groups);
        const int kb0 = static_cast<int>(it / row_groups) * kCastBlocks;
        const int m = rg * kCastRowsPerCta + half;
        const bool row_ok = m < p.rows;
        const uint16_t* xr = p.X + static_cast<int64_t>(m) * p.K + kb0 * 128 + hl * 8;
        uint4 v[kCastBlocks];
#pragma unroll
        for (int b = 0; b < kCastBlocks; ++b)
            v[b] = (row_ok && kb0 + b < p.nkb) ? ld_stream_16(xr + b * 128) : make_uint4(0, 0, 0, 0);
        uint8_t* qr = p.Q + static_cast<int64_t>(m) * p.K + kb0 * 128 + hl * 8;
#pragma unroll
        for (int b = 0; b < kCastBlocks; ++b) {
            float f[8];
            bf16x8_to_float(v[b], f);
            float a = amax8(f);
#pragma unroll
            for (int off = 8; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));  // half-warp
            a = fmaxf(a, 1e-4f);
            if (row_ok && kb0 + b < p.nkb) {
                *reinterpret_cast<uint2*>(qr + b * 128) = e4m3x8(f, __fdiv_rn(448.f, a));
                if (hl == 0) p.s[static_cast<int64_t>(kb0 + b) * p.sa_stride + m] = __fdiv_rn(a, 448.f);
            }
        }
    }
}

// Weights.  One CTA per 128x128 block (grid x = K block, y = 128-row block):
// thread t holds rows t/16 + 16j (j < 8) at columns 8*(t%16) .. +8, so every
// 16 threads read one 256-byte row segment.
__global__ void __launch_bounds__(kCastThreads)
cast_128x128_kernel(const CastParams p) {
    griddep_wait();
    griddep_launch_dependents();
    __shared__ float warp_max[kCastThreads / 32];
    const int kb = blockIdx.x, nb = blockIdx.y;
    const int r0 = nb * 128 + (threadIdx.x >> 4);
    const int c = kb * 128 + (threadIdx.x & 15) * 8;
    uint4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int r = r0 + 16 * j;
        v[j] = r < p.rows ? ld_stream_16(p.X + static_cast<int64_t>(r) * p.K + c) : make_uint4(0, 0, 0, 0);
    }
    float a = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float f[8];
        bf16x8_to_float(v[j], f);
        a = fmaxf(a, amax8(f));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = a;
    __syncthreads();
    a = warp_max[0];
#pragma unroll
    for (int w = 1; w < kCastThreads / 32; ++w) a = fmaxf(a, warp_max[w]);
    a = fmaxf(a, 1e-4f);
    const float r = __fdiv_rn(448.f, a);
    if (threadIdx.x == 0) p.s[static_cast<int64_t>(nb) * p.nkb + kb] = __fdiv_rn(a, 448.f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int row = r0 + 16 * j;
        if (row < p.rows) {
            float f[8];
            bf16x8_to_float(v[j], f);
            *reinterpret_cast<uint2*>(p.Q + static_cast<int64_t>(row) * p.K + c) = e4m3x8(f, r);
        }
    }
}

}  // namespace dg
