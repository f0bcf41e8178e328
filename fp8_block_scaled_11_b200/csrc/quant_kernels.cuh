// quant_kernels.cuh -- dynamic FP8 (e4m3) quantization kernels (memory-bound).
//
// One rule for every group shape: amax = max|x| over the group, s = 448 /
// max(amax, 1e-12) (IEEE fp32 division), q = e4m3(x * s) with round-to-
// nearest-even and saturation (cvt.rn.satfinite), stored scale = 1/s (IEEE).
// The group kernels also have a POW2 instantiation that rounds s down to a
// power of two first (scale_rule), for the GEMM's power-of-two recipes.
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

// The power-of-two rule (POW2): the largest power of two not above the fp32
// scale, so that the reciprocal is exactly representable as a UE8M0 scale
// factor (8-bit biased exponent, the scale type of the tensor cores' block-
// scaled MMA).  s is positive and normal (amax is floored at 1e-12 and
// finite), so clearing its mantissa bits gives that power of two.
template <bool POW2>
__device__ __forceinline__ float scale_rule(float amax)
{
    const float s = scale_from_amax(amax);
    return POW2 ? __uint_as_float(__float_as_uint(s) & 0x7F800000u) : s;
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
// in two batches of 8 steps (8 loads of 16 B in flight per lane).  A batch's
// 16 row maxima are gathered so that lane L holds the amax of row L, each lane
// computes one scale (one IEEE divide per row, not per lane) and the scales
// are broadcast back by shuffles.  A batch's 16 reciprocal scales (adjacent in
// the column-major grid) leave in one coalesced 64-byte store.
// --------------------------------------------------------------------------
template <typename T, bool POW2 = false>
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
        // two batches of 8 steps (16 rows each): 8 loads of 16 B in flight per lane
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            Vec8<T> v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int64_t r = (rb << 5) + (b << 4) + (i << 1) + half;
                if (col_ok && r < rows) v[i].load(x + r * ldx + c);
                else v[i].zero();
            }
            float my_amax = 0.f;        // lanes 0..15: amax of row (32 rb + 16 b + lane)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float f[8];
                v[i].get(f);
                float amax = absmax8(f);
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                // lane 2i + h receives the amax of row 2i + h of the batch (held by half-warp h)
                const float other = __shfl_sync(0xffffffffu, amax, (lane & 1) << 4);
                if ((lane >> 1) == i) my_amax = other;
            }
            const float my_s = scale_rule<POW2>(my_amax);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int64_t r = (rb << 5) + (b << 4) + (i << 1) + half;
                const float s = __shfl_sync(0xffffffffu, my_s, 2 * i + half);
                float f[8];
                v[i].get(f);
                if (col_ok && r < rows) *reinterpret_cast<uint2*>(q + r * ldq + c) = quant8(f, s);
            }
            const int64_t r = (rb << 5) + (b << 4) + lane;
            if (lane < 16 && r < rows) sinv[r + g * ld_s] = __frcp_rn(my_s);
        }
    }
}

// --------------------------------------------------------------------------
// 128 x 128 tiles through a TMA ring in shared memory.
//
// One elected thread keeps kQStages tiles (the CTA's next ones in grid-stride
// order) in flight with 2-D bulk tensor loads into a ring of shared-memory
// stages, one mbarrier per stage; all 256 threads then read the current tile
// from shared memory as 8 x 8 blocks: warp w = (wr, wc) = (w >> 1, w & 1),
// lane l = (lg, ls) = (l >> 3, l & 7); strip s = 8 wc + ls owns tile columns
// [8s, 8s+8), row group g = 4 wr + lg owns rows [8g, 8g+8).  Each 8-lane
// phase of a 16-byte shared load reads 128 contiguous bytes (no bank
// conflicts); for a fixed column j a warp writes 8 transposed rows x 32
// contiguous bytes, and for a fixed row i 4 rows x 64 contiguous bytes.
// The stage is refilled as soon as every thread holds its block in registers
// (the amax reduction's barrier), so the next loads overlap the compute.
// --------------------------------------------------------------------------
constexpr int kQStages = 3;
constexpr uint64_t kQWaitLimitNs = 2000000000ull;

template <typename T>
struct QTile {
    static constexpr uint32_t row_bytes = 128 * sizeof(T);
    static constexpr uint32_t bytes = 128 * row_bytes;                  // 32 KB (bf16) / 64 KB (fp32)
    static constexpr uint32_t bar_off = kQStages * bytes;
    static constexpr uint32_t smem = bar_off + 8 * kQStages + 1024;     // + alignment slack
};

// 8 consecutive values of row r, columns [8s, 8s+8), from a staged tile.
template <typename T>
__device__ __forceinline__ void lds_vec8(const uint8_t* tile, int r, int s, Vec8<T>& v);

// 16 bytes from shared memory as an explicit shared-space load (the tile
// pointer reaches the callers through a lambda, where a plain dereference may
// compile to a generic load).
__device__ __forceinline__ uint4 lds_u4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

template <>
__device__ __forceinline__ void lds_vec8<__nv_bfloat16>(const uint8_t* tile, int r, int s, Vec8<__nv_bfloat16>& v)
{
    v.raw = lds_u4(smem_u32(tile) + r * QTile<__nv_bfloat16>::row_bytes + s * 16);
}

template <>
__device__ __forceinline__ void lds_vec8<float>(const uint8_t* tile, int r, int s, Vec8<float>& v)
{
    const uint32_t a = smem_u32(tile) + r * QTile<float>::row_bytes + s * 32;
    const uint4 x = lds_u4(a), y = lds_u4(a + 16);
    v.a = make_float4(__uint_as_float(x.x), __uint_as_float(x.y), __uint_as_float(x.z), __uint_as_float(x.w));
    v.b = make_float4(__uint_as_float(y.x), __uint_as_float(y.y), __uint_as_float(y.z), __uint_as_float(y.w));
}

template <typename T>
struct Block8x8 {
    Vec8<T> row[8];

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

// The shared pipeline of both tile kernels: grid-stride tiles, a kQStages
// ring of TMA loads, and a callback per tile that receives the staged tile.
// `process(tile_smem, tile_index, release)` must call release() once its
// block is in registers (after a __syncthreads); release() refills the stage.
template <typename T, typename Process>
__device__ __forceinline__ void tile_pipeline(const CUtensorMap* map, int64_t ntiles, int64_t tiles_c, int* err,
                                              Process&& process)
{
    extern __shared__ uint8_t qsmem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsmem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    auto full = [&](int st) { return sbase + QTile<T>::bar_off + 8u * st; };
    __shared__ int s_abort;
    __shared__ int s_fills[kQStages];                 // loads issued per stage (thread 0 only)
    if (threadIdx.x == 0) {
        for (int st = 0; st < kQStages; ++st) {
            mbar_init(full(st), 1);
            s_fills[st] = 0;
        }
        s_abort = 0;
        fence_barrier_init();
        prefetch_tensormap(map);
    }
    __syncthreads();
    auto issue = [&](int64_t t, int st) {
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        ++s_fills[st];
        mbar_arrive_expect_tx(full(st), QTile<T>::bytes);
        tma_load_2d(sbase + st * QTile<T>::bytes, map, full(st), (int32_t)(tc * 128), (int32_t)(tr * 128));
    };
    // prologue: the first kQStages tiles of this CTA
    if (threadIdx.x == 0) {
        for (int st = 0; st < kQStages; ++st) {
            const int64_t t = blockIdx.x + (int64_t)st * gridDim.x;
            if (t < ntiles) issue(t, st);
        }
    }
    int st = 0;
    uint32_t phase = 0;
    int64_t k = 0;                                    // this CTA's tile counter
    for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++k) {
        bool ok = mbar_wait_bounded(full(st), phase, &s_abort, kQWaitLimitNs);
        if (!__syncthreads_and(ok)) {
            if (threadIdx.x == 0) { s_abort = 1; atomicOr(err, 1); }
            break;
        }
        const int this_st = st;
        auto release = [&]() {
            const int64_t tn = t + (int64_t)kQStages * gridDim.x;
            if (threadIdx.x == 0 && tn < ntiles) issue(tn, this_st);
        };
        process(sm + this_st * QTile<T>::bytes, t, release);
        if (++st == kQStages) { st = 0; phase ^= 1u; }
    }
    // every issued load has landed before the CTA exits (immediate unless a
    // wait gave up with loads still in flight)
    if (threadIdx.x == 0) {
        for (int j = 0; j < kQStages; ++j)
            if (s_fills[j] > 0) mbar_wait_bounded(full(j), (uint32_t)((s_fills[j] - 1) & 1), nullptr, kQWaitLimitNs / 2);
    }
    __syncthreads();
}

__device__ __forceinline__ void qblock_coords(int& strip, int& group, int& wr, int& wc)
{
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    wr = w >> 1;
    wc = w & 1;
    strip = 8 * wc + (l & 7);
    group = 4 * wr + (l >> 3);
}

// 1x128 groups along the ROWS, writing the quantized transpose: the group of
// output row c (input column c) is input rows [128 t, 128 t + 128).  Column
// maxima: the thread's 8 rows, the warp's 4 row groups (shuffles), the 4
// warps holding the tile's 32-row quarters (shared memory).
template <typename T, bool POW2 = false>
__global__ void __launch_bounds__(256) quant_1x128_cols_kernel(
    const __grid_constant__ CUtensorMap map, int64_t rows, int64_t cols,
    uint8_t* __restrict__ qt, int64_t ldq, float* __restrict__ sinv, int64_t ld_s, int* err)
{
    __shared__ float s_part[4][128];
    __shared__ __align__(16) float s_scale[128];
    int strip, group, wr, wc;
    qblock_coords(strip, group, wr, wc);
    const int64_t tiles_c = (cols + 127) >> 7;
    const int64_t ntiles = ((rows + 127) >> 7) * tiles_c;
    tile_pipeline<T>(&map, ntiles, tiles_c, err, [&](const uint8_t* tile, int64_t t, auto&& release) {
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        Block8x8<T> blk;
#pragma unroll
        for (int i = 0; i < 8; ++i) lds_vec8<T>(tile, 8 * group + i, strip, blk.row[i]);
        float m[8];
        blk.col_absmax(m);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], 8));
            m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], 16));
        }
        if ((threadIdx.x & 31) < 8) {
#pragma unroll
            for (int j = 0; j < 8; ++j) s_part[wr][8 * strip + j] = m[j];
        }
        __syncthreads();
        release();
        // one scale per output row (tile column): threads 0..127
        if (threadIdx.x < 128) {
            const int c = threadIdx.x;
            const float sc = scale_rule<POW2>(fmaxf(fmaxf(s_part[0][c], s_part[1][c]), fmaxf(s_part[2][c], s_part[3][c])));
            s_scale[c] = sc;
            const int64_t cg = (tc << 7) + c;
            if (cg < cols) sinv[cg + tr * ld_s] = __frcp_rn(sc);
        }
        __syncthreads();
        const float4 sa = *reinterpret_cast<const float4*>(&s_scale[8 * strip]);
        const float4 sb = *reinterpret_cast<const float4*>(&s_scale[8 * strip + 4]);
        const float sc[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
        const int64_t r0 = (tr << 7) + 8 * group;
        const int64_t c0 = (tc << 7) + 8 * strip;
        if (c0 < cols && r0 < rows) {          // rows, cols % 16 == 0: 8-blocks are all-in or all-out
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint2*>(qt + (c0 + j) * ldq + r0) = blk.quant_col(j, sc[j]);
        }
        __syncthreads();                       // s_part / s_scale are rewritten by the next tile
    });
}

// 1x128 groups along the contiguous dimension, through the tile pipeline: a
// 128 x 128 tile holds 128 whole row groups; row maxima over the thread's 8
// columns, the warp's 8 strips (shuffles) and the tile's two 64-column halves
// (shared memory).  Byte-identical to quant_1x128_rows_kernel; used when the
// row count is a multiple of 16.
template <typename T, bool POW2 = false>
__global__ void __launch_bounds__(256) quant_1x128_rowtile_kernel(
    const __grid_constant__ CUtensorMap map, int64_t rows, int64_t cols,
    uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sinv, int64_t ld_s, int* err)
{
    __shared__ float s_rpart[2][128];                 // row maxima per 64-column half
    __shared__ float s_rscale[128];
    int strip, group, wr, wc;
    qblock_coords(strip, group, wr, wc);
    const int lane = threadIdx.x & 31;
    const int64_t tiles_c = (cols + 127) >> 7;
    const int64_t ntiles = ((rows + 127) >> 7) * tiles_c;
    tile_pipeline<T>(&map, ntiles, tiles_c, err, [&](const uint8_t* tile, int64_t t, auto&& release) {
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        Block8x8<T> blk;
#pragma unroll
        for (int i = 0; i < 8; ++i) lds_vec8<T>(tile, 8 * group + i, strip, blk.row[i]);
        float rm[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float f[8];
            blk.row[i].get(f);
            rm[i] = absmax8(f);
            rm[i] = fmaxf(rm[i], __shfl_xor_sync(0xffffffffu, rm[i], 1));
            rm[i] = fmaxf(rm[i], __shfl_xor_sync(0xffffffffu, rm[i], 2));
            rm[i] = fmaxf(rm[i], __shfl_xor_sync(0xffffffffu, rm[i], 4));
        }
        if ((lane & 7) == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i) s_rpart[wc][8 * group + i] = rm[i];
        }
        __syncthreads();
        release();
        if (threadIdx.x < 128) {
            const int r = threadIdx.x;
            const float sr = scale_rule<POW2>(fmaxf(s_rpart[0][r], s_rpart[1][r]));
            s_rscale[r] = sr;
            const int64_t rg = (tr << 7) + r;
            if (rg < rows) sinv[rg + tc * ld_s] = __frcp_rn(sr);
        }
        __syncthreads();
        const int64_t r0 = (tr << 7) + 8 * group;
        const int64_t c0 = (tc << 7) + 8 * strip;
        if (c0 < cols && r0 < rows) {          // rows, cols % 16 == 0: 8-blocks are all-in or all-out
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float f[8];
                blk.row[i].get(f);
                *reinterpret_cast<uint2*>(q + (r0 + i) * ldq + c0) = quant8(f, s_rscale[8 * group + i]);
            }
        }
        __syncthreads();                       // the shared arrays are rewritten by the next tile
    });
}

// Both 1x128 directions from one read of the input.  A 128 x 128 tile holds
// 128 whole row groups (1x128 along the columns) and 128 whole column groups
// (1x128 along the rows), so one pass over the tile gives both sets of
// maxima: column maxima as in quant_1x128_cols_kernel, row maxima over the
// thread's 8 columns, the warp's 8 strips (shuffles) and the tile's two
// 64-column halves (shared memory).  Outputs are byte-identical to the
// row-direction and transposed column-direction launches.
template <typename T, bool POW2 = false>
__global__ void __launch_bounds__(256) quant_1x128_dual_kernel(
    const __grid_constant__ CUtensorMap map, int64_t rows, int64_t cols,
    uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sinv, int64_t ld_s,
    uint8_t* __restrict__ qt, int64_t ldqt, float* __restrict__ sinvt, int64_t ld_st, int* err)
{
    __shared__ float s_cpart[4][128];                 // column maxima per 32-row quarter
    __shared__ float s_rpart[2][128];                 // row maxima per 64-column half
    __shared__ __align__(16) float s_cscale[128];
    __shared__ float s_rscale[128];
    int strip, group, wr, wc;
    qblock_coords(strip, group, wr, wc);
    const int lane = threadIdx.x & 31;
    const int64_t tiles_c = (cols + 127) >> 7;
    const int64_t ntiles = ((rows + 127) >> 7) * tiles_c;
    tile_pipeline<T>(&map, ntiles, tiles_c, err, [&](const uint8_t* tile, int64_t t, auto&& release) {
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        Block8x8<T> blk;
#pragma unroll
        for (int i = 0; i < 8; ++i) lds_vec8<T>(tile, 8 * group + i, strip, blk.row[i]);
        float cm[8], rm[8];
        blk.col_absmax(cm);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float f[8];
            blk.row[i].get(f);
            rm[i] = absmax8(f);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            cm[j] = fmaxf(cm[j], __shfl_xor_sync(0xffffffffu, cm[j], 8));
            cm[j] = fmaxf(cm[j], __shfl_xor_sync(0xffffffffu, cm[j], 16));
            rm[j] = fmaxf(rm[j], __shfl_xor_sync(0xffffffffu, rm[j], 1));
            rm[j] = fmaxf(rm[j], __shfl_xor_sync(0xffffffffu, rm[j], 2));
            rm[j] = fmaxf(rm[j], __shfl_xor_sync(0xffffffffu, rm[j], 4));
        }
        if (lane < 8) {
#pragma unroll
            for (int j = 0; j < 8; ++j) s_cpart[wr][8 * strip + j] = cm[j];
        }
        if ((lane & 7) == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i) s_rpart[wc][8 * group + i] = rm[i];
        }
        __syncthreads();
        release();
        // threads 0..127: one scale per tile column; 128..255: one per tile row
        if (threadIdx.x < 128) {
            const int c = threadIdx.x;
            const float sc = scale_rule<POW2>(fmaxf(fmaxf(s_cpart[0][c], s_cpart[1][c]), fmaxf(s_cpart[2][c], s_cpart[3][c])));
            s_cscale[c] = sc;
            const int64_t cg = (tc << 7) + c;
            if (cg < cols) sinvt[cg + tr * ld_st] = __frcp_rn(sc);
        } else {
            const int r = threadIdx.x - 128;
            const float sr = scale_rule<POW2>(fmaxf(s_rpart[0][r], s_rpart[1][r]));
            s_rscale[r] = sr;
            const int64_t rg = (tr << 7) + r;
            if (rg < rows) sinv[rg + tc * ld_s] = __frcp_rn(sr);
        }
        __syncthreads();
        const int64_t r0 = (tr << 7) + 8 * group;
        const int64_t c0 = (tc << 7) + 8 * strip;
        if (c0 < cols && r0 < rows) {          // rows, cols % 16 == 0: 8-blocks are all-in or all-out
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float f[8];
                blk.row[i].get(f);
                *reinterpret_cast<uint2*>(q + (r0 + i) * ldq + c0) = quant8(f, s_rscale[8 * group + i]);
            }
            const float4 sa = *reinterpret_cast<const float4*>(&s_cscale[8 * strip]);
            const float4 sb = *reinterpret_cast<const float4*>(&s_cscale[8 * strip + 4]);
            const float sc[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint2*>(qt + (c0 + j) * ldqt + r0) = blk.quant_col(j, sc[j]);
        }
        __syncthreads();                       // the shared arrays are rewritten by the next tile
    });
}

// 128x128 tiles: amax over the tile (shuffles + shared memory), then
// row-major and/or transposed bytes straight from registers.
template <typename T, bool POW2 = false>
__global__ void __launch_bounds__(256) quant_128x128_kernel(
    const __grid_constant__ CUtensorMap map, int64_t rows, int64_t cols,
    uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ sinv, int64_t ld_s,
    uint8_t* __restrict__ qt, int64_t ldqt, float* __restrict__ sinvt, int64_t ld_st, int* err)
{
    __shared__ float s_warp[8];
    int strip, group, wr, wc;
    qblock_coords(strip, group, wr, wc);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t tiles_c = (cols + 127) >> 7;
    const int64_t ntiles = ((rows + 127) >> 7) * tiles_c;
    tile_pipeline<T>(&map, ntiles, tiles_c, err, [&](const uint8_t* tile, int64_t t, auto&& release) {
        const int64_t bi = t / tiles_c, bj = t - bi * tiles_c;
        Block8x8<T> blk;
#pragma unroll
        for (int i = 0; i < 8; ++i) lds_vec8<T>(tile, 8 * group + i, strip, blk.row[i]);
        float m8[8];
        blk.col_absmax(m8);
        float m = m8[0];
#pragma unroll
        for (int j = 1; j < 8; ++j) m = fmaxf(m, m8[j]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) s_warp[warp] = m;
        __syncthreads();
        release();
        float amax = s_warp[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) amax = fmaxf(amax, s_warp[w]);
        const float s = scale_rule<POW2>(amax);
        const int64_t r0 = (bi << 7) + 8 * group;
        const int64_t c0 = (bj << 7) + 8 * strip;
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
        __syncthreads();                       // s_warp is rewritten by the next tile
    });
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
