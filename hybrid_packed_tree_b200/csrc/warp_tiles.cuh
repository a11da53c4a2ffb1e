// warp_tiles.cuh -- CUDA-core building blocks of the small-batch kernels: rows of
// 128 fp32 state columns held four per lane, a warp reduce-scatter of per-lane
// partial sums, and 32-column dot products of bf16 or fp32 shared-memory rows.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace stree {
namespace tiles {

constexpr int kCols = 128;                  // state columns (dstate, or d_k)

__device__ __forceinline__ float in_to_f(float v) { return v; }
__device__ __forceinline__ float in_to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename In> __device__ __forceinline__ In f_to_in(float v);
template <> __device__ __forceinline__ float f_to_in<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 f_to_in<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Four consecutive state columns 4 lane .. 4 lane + 3 of row `row` of a [*][128] array.
__device__ __forceinline__ float4 row4(const float *base, int row, int lane)
{
    return *reinterpret_cast<const float4 *>(base + row * kCols + 4 * lane);
}
__device__ __forceinline__ float4 row4(const __nv_bfloat16 *base, int row, int lane)
{
    const uint2 raw = *reinterpret_cast<const uint2 *>(base + row * kCols + 4 * lane);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
    return make_float4(__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi));
}

// C_i . B_j over the 32 state columns 32 s .. 32 s + 31 (four independent sums).
__device__ __forceinline__ float dot32(const float *C, const float *B, int i, int j, int s, int rot)
{
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const int cc = (c + rot) & 7;
        const float4 cv = *reinterpret_cast<const float4 *>(C + i * kCols + 32 * s + 4 * cc);
        const float4 bv = *reinterpret_cast<const float4 *>(B + j * kCols + 32 * s + 4 * cc);
        d[c & 3] = fmaf(cv.x, bv.x, fmaf(cv.y, bv.y, fmaf(cv.z, bv.z, fmaf(cv.w, bv.w, d[c & 3]))));
    }
    return (d[0] + d[1]) + (d[2] + d[3]);
}
__device__ __forceinline__ float dot32(const __nv_bfloat16 *C, const __nv_bfloat16 *B, int i, int j, int s, int rot)
{
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int cc = (c + rot) & 3;
        const uint4 cr = *reinterpret_cast<const uint4 *>(C + i * kCols + 32 * s + 8 * cc);
        const uint4 br = *reinterpret_cast<const uint4 *>(B + j * kCols + 32 * s + 8 * cc);
        const __nv_bfloat162 *c2 = reinterpret_cast<const __nv_bfloat162 *>(&cr);
        const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&br);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float2 cf = __bfloat1622float2(c2[u]), bf = __bfloat1622float2(b2[u]);
            d[c] = fmaf(cf.x, bf.x, fmaf(cf.y, bf.y, d[c]));
        }
    }
    return (d[0] + d[1]) + (d[2] + d[3]);
}

// Chunk rotation of dot32 for a lane whose pair is lane / 4 and quarter lane % 4.
// Rows lie 256 (bf16) or 512 (fp32) bytes apart, so without it the lanes of one
// 16-byte load phase (eight lanes: two pairs, four quarters) would hit the same
// banks; with it those eight lanes read eight different bank groups.
template <typename In>
__device__ __forceinline__ int dot32_rot(int lane)
{
    const int pair = (lane >> 2) & 1, quarter = lane & 3;
    return sizeof(In) == 4 ? 4 * pair + quarter : 2 * pair + (quarter >> 1);
}

__device__ __forceinline__ void named_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float dot4(float4 a, float4 b)
{
    return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, a.x * b.x)));
}

// Butterfly reduce-scatter of 64 per-lane values over the warp: afterwards
// v[0] and v[1] hold the warp-wide sums of entries 2*lane and 2*lane + 1.
// At the stage with xor distance m the lanes with bit m set keep the upper half
// of their current block and the others the lower half; lane bit m thereby
// selects index weight 2m, which makes the surviving index 2*lane + k.
__device__ __forceinline__ void reduce_scatter64(float (&v)[64], int lane)
{
#pragma unroll
    for (int st = 0; st < 5; ++st) {
        const int m = 16 >> st, half = 32 >> st;
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int k = 0; k < half; ++k) {
            const float send = up ? v[k] : v[k + half];
            const float keep = up ? v[k + half] : v[k];
            v[k] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
}


}  // namespace tiles
}  // namespace stree
