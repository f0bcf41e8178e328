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
// 1x128 groups along the ROWS, writing the quantized transpose.
// Tile = 128 rows x 64 columns, staged through shared memory as fp32 (row
// stride 65 words).  Pass 1: 4 threads per column reduce |x| over 128 rows.
// Pass 2: each thread emits 16 consecutive output bytes (16 rows of one
// column) of the transposed row; 64 scales per tile leave contiguously.
// --------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) quant_1x128_cols_kernel(
    const T* __restrict__ x, int64_t rows, int64_t cols, int64_t ldx,
    uint8_t* __restrict__ qt, int64_t ldq, float* __restrict__ sinv, int64_t ld_s)
{
    constexpr int TR = 128, TC = 64, PITCH = TC + 1;
    __shared__ float tile[TR * PITCH];
    __shared__ float s_scale[TC];
    const int tid = threadIdx.x;
    const int64_t tiles_r = (rows + TR - 1) / TR;
    const int64_t tiles_c = (cols + TC - 1) / TC;
    const int64_t ntiles = tiles_r * tiles_c;

    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const int64_t tr = t / tiles_c;
        const int64_t tc = t - tr * tiles_c;
        const int64_t r0 = tr * TR, c0 = tc * TC;
        // load: 128 rows x 8 chunks of 8 values = 1024 chunks, 4 per thread
        {
            Vec8<T> v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int id = tid + 256 * j;
                const int lr = id >> 3, lc = (id & 7) << 3;
                const int64_t r = r0 + lr, c = c0 + lc;
                if (r < rows && c < cols) v[j].load(x + r * ldx + c);
                else v[j].zero();
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int id = tid + 256 * j;
                const int lr = id >> 3, lc = (id & 7) << 3;
                float f[8];
                v[j].get(f);
#pragma unroll
                for (int e = 0; e < 8; ++e) tile[lr * PITCH + lc + e] = f[e];
            }
        }
        __syncthreads();
        // column amax: thread -> column tid/4, rows (tid%4)*32 .. +32
        {
            const int lc = tid >> 2, part = tid & 3;
            float m = 0.f;
#pragma unroll 8
            for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(tile[(part * 32 + i) * PITCH + lc]));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            if (part == 0) s_scale[lc] = scale_from_amax(m);
        }
        __syncthreads();
        // emit: 64 columns x 8 chunks of 16 rows = 512 chunks, 2 per thread
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int id = tid + 256 * j;
            const int lc = id & 63;          // consecutive threads: consecutive columns (bank-friendly)
            const int ch = id >> 6;          // 16-row chunk
            const int64_t c = c0 + lc, r = r0 + ch * 16;
            if (c < cols && r < rows) {      // rows % 16 == 0: chunks are all-in or all-out
                const float s = s_scale[lc];
                uint32_t w[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int rr = ch * 16 + k * 4;
                    const uint32_t lo = cvt_e4m3x2(__fmul_rn(tile[(rr + 0) * PITCH + lc], s),
                                                   __fmul_rn(tile[(rr + 1) * PITCH + lc], s));
                    const uint32_t hi = cvt_e4m3x2(__fmul_rn(tile[(rr + 2) * PITCH + lc], s),
                                                   __fmul_rn(tile[(rr + 3) * PITCH + lc], s));
                    w[k] = lo | (hi << 16);
                }
                *reinterpret_cast<uint4*>(qt + c * ldq + r) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        if (tid < TC) {
            const int64_t c = c0 + tid;
            if (c < cols) sinv[c + tr * ld_s] = __frcp_rn(s_scale[tid]);
        }
        __syncthreads();
    }
}

// --------------------------------------------------------------------------
// 128x128 tiles.  One CTA (256 threads) per tile: the tile (up to 32 KB of
// bf16) is held in registers, 8 chunks of 8 values per thread; block-wide
// amax through warp shuffles + shared memory; quantized bytes stored row-wise
// and, when requested, staged in shared memory and stored transposed.
// --------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) quant_128x128_kernel(
    const T* __restrict__ x, int64_t rows, int64_t cols, int64_t ldx,
    uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sinv, int64_t ld_s,
    uint8_t* __restrict__ qt, int64_t ldqt, float* __restrict__ sinvt, int64_t ld_st)
{
    constexpr int QP = 128 + 16;             // byte pitch of the staged tile
    __shared__ float s_warp[8];
    __shared__ __align__(16) uint8_t s_q[128 * QP];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t tiles_c = (cols + 127) >> 7;
    const int64_t tiles_r = (rows + 127) >> 7;
    const int64_t ntiles = tiles_r * tiles_c;

    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const int64_t bi = t / tiles_c, bj = t - bi * tiles_c;
        const int64_t r0 = bi << 7, c0 = bj << 7;
        // chunk id = tid + 256*j: row id/16, column chunk id%16 -> a warp reads 2 full 128-wide rows
        Vec8<T> v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int id = tid + 256 * j;
            const int64_t r = r0 + (id >> 4), c = c0 + ((id & 15) << 3);
            if (r < rows && c < cols) v[j].load(x + r * ldx + c);
            else v[j].zero();
        }
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float f[8];
            v[j].get(f);
            m = fmaxf(m, absmax8(f));
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) s_warp[warp] = m;
        __syncthreads();
        float amax = s_warp[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) amax = fmaxf(amax, s_warp[w]);
        const float s = scale_from_amax(amax);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int id = tid + 256 * j;
            const int lr = id >> 4, lc = (id & 15) << 3;
            const int64_t r = r0 + lr, c = c0 + lc;
            float f[8];
            v[j].get(f);
            const uint2 b = quant8(f, s);
            if (q != nullptr && r < rows && c < cols) *reinterpret_cast<uint2*>(q + r * ldq + c) = b;
            if (qt != nullptr) *reinterpret_cast<uint2*>(s_q + lr * QP + lc) = b;
        }
        if (tid == 0) {
            const float rinv = __frcp_rn(s);
            if (q != nullptr) sinv[bi + bj * ld_s] = rinv;
            if (qt != nullptr) sinvt[bj + bi * ld_st] = rinv;
        }
        if (qt != nullptr) {
            __syncthreads();
            // transposed: output row (c0+lc) gets bytes r0..r0+127; 128 cols x 8 chunks of 16 = 1024, 4 per thread
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int id = tid + 256 * j;
                const int lc = id & 127, ch = id >> 7;
                const int64_t c = c0 + lc, r = r0 + ch * 16;
                if (c < cols && r < rows) {
                    uint32_t w[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int rr = ch * 16 + k * 4;
                        w[k] = (uint32_t)s_q[(rr + 0) * QP + lc] | ((uint32_t)s_q[(rr + 1) * QP + lc] << 8) |
                               ((uint32_t)s_q[(rr + 2) * QP + lc] << 16) | ((uint32_t)s_q[(rr + 3) * QP + lc] << 24);
                    }
                    *reinterpret_cast<uint4*>(qt + c * ldqt + r) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
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
