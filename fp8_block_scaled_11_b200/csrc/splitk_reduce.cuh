// splitk_reduce.cuh -- the split-K reduction of the scaled GEMM.
//
// D[m,n] = sum over splits s = 0, 1, ..., splits-1 (in that order) of
// ws[s][m][n], rounded once to the output type (bf16 RNE or fp32).  The fixed
// order makes the result independent of the launch geometry.
//
// Memory-bound (the partials were just written by the GEMM and are normally
// still in L2): each thread owns one 4-column chunk of a row and issues the
// loads of up to sixteen splits before adding them in split order, so that
// sixteen 16-byte loads per thread are in flight instead of one.
//
// Launched as a programmatic dependent of the GEMM (its CTAs may start while
// the GEMM's last tiles run): griddepcontrol.wait holds every thread until the
// GEMM grid has completed and its partial sums are visible (without that
// launch attribute the wait returns at once).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace fp8bs {

constexpr int kReduceThreads = 128;
constexpr int kReduceBatch = 16;         // split loads in flight per thread

__global__ void __launch_bounds__(kReduceThreads) splitk_reduce_kernel(const float* __restrict__ ws, int splits,
                                                                       int64_t M, int64_t N, int64_t ldw,
                                                                       void* __restrict__ D, int64_t ldd, int out_f32,
                                                                       int vec_out)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t nq = (N + 3) >> 2;          // 4-column chunks per row
    const int64_t total = M * nq;
    const int64_t plane = M * ldw;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = i / nq;
        const int64_t n = (i - m * nq) << 2;
        const float* src = ws + m * ldw + n;
        float4 s = __ldcg(reinterpret_cast<const float4*>(src));
        int k = 1;
        for (; k + kReduceBatch <= splits; k += kReduceBatch) {
            float4 v[kReduceBatch];
#pragma unroll
            for (int j = 0; j < kReduceBatch; ++j) v[j] = __ldcg(reinterpret_cast<const float4*>(src + (k + j) * plane));
#pragma unroll
            for (int j = 0; j < kReduceBatch; ++j) {
                s.x += v[j].x; s.y += v[j].y; s.z += v[j].z; s.w += v[j].w;
            }
        }
        for (; k < splits; ++k) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(src + k * plane));
            s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
        }
        const float v[4] = {s.x, s.y, s.z, s.w};
        const int valid = (int)((N - n) < 4 ? (N - n) : 4);
        if (out_f32) {
            float* d = reinterpret_cast<float*>(D) + m * ldd + n;
            if (vec_out && valid == 4) *reinterpret_cast<float4*>(d) = s;
            else for (int t = 0; t < valid; ++t) d[t] = v[t];
        } else {
            __nv_bfloat16* d = reinterpret_cast<__nv_bfloat16*>(D) + m * ldd + n;
            const uint32_t lo = cvt_bf16x2(s.x, s.y), hi = cvt_bf16x2(s.z, s.w);
            if (vec_out && valid == 4) {
                *reinterpret_cast<uint2*>(d) = make_uint2(lo, hi);
            } else {
                const uint32_t ww[2] = {lo, hi};
                uint16_t* d16 = reinterpret_cast<uint16_t*>(d);
                for (int t = 0; t < valid; ++t) d16[t] = (uint16_t)((ww[t >> 1] >> ((t & 1) * 16)) & 0xFFFFu);
            }
        }
    }
}

}  // namespace fp8bs
