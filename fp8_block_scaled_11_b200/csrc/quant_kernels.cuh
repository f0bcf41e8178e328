// quant_kernels.cuh -- dynamic FP8 (e4m3) quantization kernels (memory-bound).
//
// One rule for every group shape: amax = max|x| over the group, s = 448 /
// max(amax, 1e-12) (IEEE fp32 division), q = e4m3(x * s) with round-to-
// nearest-even and saturation (cvt.rn.satfinite), stored scale = 1/s (IEEE).
// Group shapes follow pytorch/ao PR #2592 "add more generic kernel for fp8
// blockwise scaling" (Performance table: (1,128) and (128,128)); reciprocal,
// column-major scales follow pytorch/ao PR #2785 "integrate torch._scaled_mm
// into Float8BlockwiseLinear and add bench script" (Summary).
//
// Design for B200: 16-byte vector loads/stores only, every warp access covers
// whole 32-byte sectors, scale grids written as contiguous runs (the grid is
// column-major, so consecutive rows of one group column are adjacent), and
// persistent grid-stride launches sized from the occupancy calculator.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace fp8bs {

constexpr float kE4M3Max = 448.0f;
constexpr float kAmaxFloor = 1e-12f;

__device__ __forceinline__ float scale_from_amax(float amax)
{
    return __fdiv_rn(kE4M3Max, fmaxf(amax, kAmaxFloor));
}

// 8 consecutive inputs as fp32.  bf16: one 16-byte load; fp32: two.
template <typename T>
struct Vec8;

template <>
struct Vec8<__nv_bfloat16> {
    uint4 raw;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { raw = __ldcs(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ void get(float (&f)[8]) const
    {
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    __device__ __forceinline__ void zero() { raw = make_uint4(0, 0, 0, 0); }
};

template <>
struct Vec8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p)
    {
        a = __ldcs(reinterpret_cast<const float4*>(p));
        b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ void get(float (&f)[8]) const
    {
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
};

__device__ __forceinline__ float absmax8(const float (&f)[8])
{
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
    return m;
}

// 8 values * s -> 8 e4m3 bytes packed little-endian in a uint2.
__device__ __forceinline__ uint2 quant8(const float (&f)[8], float s)
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        w[i] = cvt_e4m3x2(__fmul_rn(f[2 * i], s), __fmul_rn(f[2 * i + 1], s));
    }
    return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// --------------------------------------------------------------------------
// 1x128 groups along the contiguous dimension.
// Work item = 32 rows x one 128-column group, owned by one warp.  A half-warp
// covers one row's group (16 lanes x 8 values); the warp walks 2 rows per step
// in batches of 8 steps (8 x 16 B loads in flight per lane).  Each lane ends
// up holding the scale of row (32*item + lane), so the 32 scales of the item
// (adjacent in the column-major grid) leave in one coalesced 128-byte store.
// --------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) quant_1x128_rows_kernel(
    const T* __restrict__ x, int64_t rows, int64_t cols, int64_t ldx,
    uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sinv, int64_t ld_s)
{
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4;       // which of the two rows of a step
    const int hl = lane & 15;         // position inside the 128-wide group
    const int64_t groups = (cols + 127) >> 7;
    const int64_t rblocks = (rows + 31) >> 5;
    const int64_t items = rblocks * groups;
    const int64_t warp0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);

    for (int64_t it = warp0; it < items; it += nwarps) {
        const int64_t rb = it / groups;
        const int64_t g = it - rb * groups;
        const int64_t c = (g << 7) + (hl << 3);
        const bool col_ok = c < cols;   // cols % 16 == 0: a chunk of 8 is all-in or all-out
        float my_scale = 0.f;
#pragma unroll
        for (int batch = 0; batch < 2; ++batch) {
            Vec8<T> v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int64_t r = (rb << 5) + ((batch * 8 + i) << 1) + half;
                if (col_ok && r < rows) v[i].load(x + r * ldx + c);
                else v[i].zero();
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int step = batch * 8 + i;
                const int64_t r = (rb << 5) + (step << 1) + half;
                float f[8];
                v[i].get(f);
                float amax = absmax8(f);
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                const float s = scale_from_amax(amax);
                if (col_ok && r < rows) {
                    *reinterpret_cast<uint2*>(q + r * ldq + c) = quant8(f, s);
                }
                const float rinv = __frcp_rn(s);
                // lane 2*step + h receives the scale of row 2*step + h
                const float other = __shfl_sync(0xffffffffu, rinv, (lane & 1) << 4);
                if ((lane >> 1) == step) my_scale = other;
            }
        }
        const int64_t r = (rb << 5) + lane;
        if (r < rows) sinv[r + g * ld_s] = my_scale;
    }
}

// --------------------------------------------------------------------------
// 128 x 128 tiles held as 8 x 8 register blocks.
// Thread layout in a 256-thread CTA: warp w = (wr, wc) = (w >> 2, w & 3),
// lane l = (ls, lg) = (l >> 3, l & 7); strip s = 4 wc + ls owns columns
// [8s, 8s+8) of the tile, row group g = 8 wr + lg owns rows [8g, 8g+8).  For a
// fixed row i a warp reads 8 rows x 64 contiguous bytes (bf16); for a fixed
// column j it writes 4 transposed rows x 64 contiguous bytes, and row-major
// output rows go out as 8 rows x 32 contiguous bytes: whole 32-byte sectors.
// --------------------------------------------------------------------------
template <typename T>
struct Block8x8 {
    Vec8<T> row[8];

    __device__ __forceinline__ void load(const T* __restrict__ x, int64_t rows, int64_t cols, int64_t ldx,
                                         int64_t r0, int64_t c0)
    {
        const bool col_ok = c0 < cols;           // cols % 16 == 0: a strip of 8 is all-in or all-out
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (col_ok && r0 + i < rows) row[i].load(x + (r0 + i) * ldx + c0);
            else row[i].zero();
        }
    }

    __device__ __forceinline__ void col_absmax(float (&m)[8]) const
    {
#pragma unroll
        for (int j = 0; j < 8; ++j) m[j] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float f[8];
            row[i].get(f);
#pragma unroll
            for (int j = 0; j < 8; ++j) m[j] = fmaxf(m[j], fabsf(f[j]));
        }
    }

    // Column j quantized with scale s: the 8 bytes of rows 0..7 (row 0 lowest).
    __device__ __forceinline__ uint2 quant_col(int j, float s) const
    {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float f[8];
            row[i].get(f);
            v[i] = __fmul_rn(f[j], s);
        }
        const uint32_t w0 = cvt_e4m3x2(v[0], v[1]) | ((uint32_t)cvt_e4m3x2(v[2], v[3]) << 16);
        const uint32_t w1 = cvt_e4m3x2(v[4], v[5]) | ((uint32_t)cvt_e4m3x2(v[6], v[7]) << 16);
        return make_uint2(w0, w1);
    }
};

__device__ __forceinline__ void block_coords(int& strip, int& group)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    strip = 4 * (w & 3) + (l >> 3);
    group = 8 * (w >> 2) + (l & 7);
}

// --------------------------------------------------------------------------
// 1x128 groups along the ROWS, writing the quantized transpose: the group of
// output row c (input column c) is input rows [128 t, 128 t + 128).
// Per column: max over the thread's 8 rows, over the 8 row groups of the warp
// (lane shuffles), then over the two warps holding the tile's upper and lower
// 64 rows (shared memory).  Output row c of the tile gets its 128 bytes from
// 16 threads, 8 bytes each.
// --------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) quant_1x128_cols_kernel(
    const T* __restrict__ x, int64_t rows, int64_t cols, int64_t ldx,
    uint8_t* __restrict__ qt, int64_t ldq, float* __restrict__ sinv, int64_t ld_s)
{
    __shared__ float s_half[2][128];           // column maxima of the tile's two 64-row halves
    int strip, group;
    block_coords(strip, group);
    const int wr = (threadIdx.x >> 5) >> 2;
    const int64_t tiles_c = (cols + 127) >> 7;
    const int64_t ntiles = ((rows + 127) >> 7) * tiles_c;

    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        const int64_t r0 = (tr << 7) + 8 * group;
        const int64_t c0 = (tc << 7) + 8 * strip;
        Block8x8<T> blk;
        blk.load(x, rows, cols, ldx, r0, c0);
        float m[8];
        blk.col_absmax(m);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int o = 1; o <= 4; o <<= 1) m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], o));
        }
        if ((threadIdx.x & 7) == 0) {
#pragma unroll
            for (int j = 0; j < 8; ++j) s_half[wr][8 * strip + j] = m[j];
        }
        __syncthreads();
        float sc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            sc[j] = scale_from_amax(fmaxf(s_half[0][8 * strip + j], s_half[1][8 * strip + j]));
        if (c0 < cols && r0 < rows) {          // rows % 16 == 0: a group of 8 rows is all-in or all-out
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint2*>(qt + (c0 + j) * ldq + r0) = blk.quant_col(j, sc[j]);
        }
        if (group == 0 && c0 < cols) {
            float* dst = sinv + c0 + tr * ld_s;
            *reinterpret_cast<float4*>(dst) = make_float4(__frcp_rn(sc[0]), __frcp_rn(sc[1]), __frcp_rn(sc[2]), __frcp_rn(sc[3]));
            *reinterpret_cast<float4*>(dst + 4) = make_float4(__frcp_rn(sc[4]), __frcp_rn(sc[5]), __frcp_rn(sc[6]), __frcp_rn(sc[7]));
        }
        __syncthreads();
    }
}

// --------------------------------------------------------------------------
// 128x128 tiles: one CTA per tile, the tile in registers as 8x8 blocks, amax
// over the tile (shuffles + shared memory), then row-major and/or transposed
// bytes straight from registers.
// --------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) quant_128x128_kernel(
    const T* __restrict__ x, int64_t rows, int64_t cols, int64_t ldx,
    uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sinv, int64_t ld_s,
    uint8_t* __restrict__ qt, int64_t ldqt, float* __restrict__ sinvt, int64_t ld_st)
{
    __shared__ float s_warp[8];
    int strip, group;
    block_coords(strip, group);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t tiles_c = (cols + 127) >> 7;
    const int64_t ntiles = ((rows + 127) >> 7) * tiles_c;

    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const int64_t bi = t / tiles_c, bj = t - bi * tiles_c;
        const int64_t r0 = (bi << 7) + 8 * group;
        const int64_t c0 = (bj << 7) + 8 * strip;
        Block8x8<T> blk;
        blk.load(x, rows, cols, ldx, r0, c0);
        float m8[8];
        blk.col_absmax(m8);
        float m = m8[0];
#pragma unroll
        for (int j = 1; j < 8; ++j) m = fmaxf(m, m8[j]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) s_warp[warp] = m;
        __syncthreads();
        float amax = s_warp[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) amax = fmaxf(amax, s_warp[w]);
        const float s = scale_from_amax(amax);
        const bool in = c0 < cols && r0 < rows;    // rows, cols % 16 == 0: blocks are all-in or all-out
        if (q != nullptr && in) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float f[8];
                blk.row[i].get(f);
                *reinterpret_cast<uint2*>(q + (r0 + i) * ldq + c0) = quant8(f, s);
            }
        }
        if (qt != nullptr && in) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint2*>(qt + (c0 + j) * ldqt + r0) = blk.quant_col(j, s);
        }
        if (threadIdx.x == 0) {
            const float rinv = __frcp_rn(s);
            if (q != nullptr) sinv[bi + bj * ld_s] = rinv;
            if (qt != nullptr) sinvt[bj + bi * ld_st] = rinv;
        }
        __syncthreads();
    }
}

// --------------------------------------------------------------------------
// Rowwise: one warp per row, two passes (amax, then quantize; the second pass
// re-reads the row, usually from L2).
// --------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) quant_rowwise_kernel(
    const T* __restrict__ x, int64_t rows, int64_t cols, int64_t ldx,
    uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sinv)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = warp0; r < rows; r += nwarps) {
        const T* xr = x + r * ldx;
        float m = 0.f;
        for (int64_t c = (int64_t)lane << 3; c < cols; c += 256) {
            Vec8<T> v;
            v.load(xr + c);
            float f[8];
            v.get(f);
            m = fmaxf(m, absmax8(f));
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float s = scale_from_amax(m);
        for (int64_t c = (int64_t)lane << 3; c < cols; c += 256) {
            Vec8<T> v;
            v.load(xr + c);
            float f[8];
            v.get(f);
            *reinterpret_cast<uint2*>(q + r * ldq + c) = quant8(f, s);
        }
        if (lane == 0) sinv[r] = __frcp_rn(s);
    }
}

// --------------------------------------------------------------------------
// Per-tensor: pass 1 writes one |x| maximum per CTA into the workspace; pass 2
// reduces those partials (every CTA, identically), then quantizes.
// --------------------------------------------------------------------------
constexpr int kTensorPartials = 1024;

__device__ __forceinline__ float block_max_256(float m, float* s_warp)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_warp[warp] = m;
    __syncthreads();
    float r = s_warp[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) r = fmaxf(r, s_warp[w]);
    __syncthreads();
    return r;
}

template <typename T>
__global__ void __launch_bounds__(256) tensor_amax_kernel(const T* __restrict__ x, int64_t n,
                                                         float* __restrict__ partial)
{
    __shared__ float s_warp[8];
    float m = 0.f;
    for (int64_t i = ((int64_t)blockIdx.x * 256 + threadIdx.x) << 3; i < n; i += (int64_t)gridDim.x * 256 * 8) {
        Vec8<T> v;
        v.load(x + i);
        float f[8];
        v.get(f);
        m = fmaxf(m, absmax8(f));
    }
    m = block_max_256(m, s_warp);
    if (threadIdx.x == 0) partial[blockIdx.x] = m;
}

template <typename T>
__global__ void __launch_bounds__(256) tensor_quant_kernel(const T* __restrict__ x, int64_t n,
                                                          const float* __restrict__ partial, int nparts,
                                                          uint8_t* __restrict__ q, float* __restrict__ sinv)
{
    __shared__ float s_warp[8];
    float m = 0.f;
    for (int i = threadIdx.x; i < nparts; i += 256) m = fmaxf(m, partial[i]);
    const float amax = block_max_256(m, s_warp);
    const float s = scale_from_amax(amax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *sinv = __frcp_rn(s);
    for (int64_t i = ((int64_t)blockIdx.x * 256 + threadIdx.x) << 3; i < n; i += (int64_t)gridDim.x * 256 * 8) {
        Vec8<T> v;
        v.load(x + i);
        float f[8];
        v.get(f);
        *reinterpret_cast<uint2*>(q + i) = quant8(f, s);
    }
}

}  // namespace fp8bs
