// gemm_bs_kernel.cuh -- the block recipes of the scaled GEMM with power-of-two
// scales, applied by the tensor cores (block-scaled MMA).
//
// Computes the same D[m,n] = sum_kb rA(m,kb) * rB(n,kb) * P_kb[m,n] as
// gemm_kernel.cuh for the (1x128, 128x128) and (1x128, 1x128) recipes of
// pytorch/ao PR #4209 "[codex] add repro for blockwise _scaled_mm
// investigation" (Findings So Far), when every scale is an exact power of two.
// tcgen05.mma kind::mxf8f6f4.block_scale multiplies the products of each
// 32-wide K step by its row's and column's UE8M0 scale factors (a 128-wide
// K block is four such steps with the same factor) and accumulates every K
// block of a unit in one fp32 TMEM accumulator: no promotion warps and no
// per-K-block hand-off.  This is the fast-accumulation variant of
// pytorch/pytorch issue #159940 (Describe the bug: USE_FAST_ACCUM) in its B200
// form: the work the flag skips on the earlier part (software promotion) is
// skipped here too, at the price of scales restricted to powers of two.
//
// One persistent CTA per SM computes 128 x 256 output tiles (units: tiles, or
// tile x K-split with split-K), 12 warps:
//   warp 0      TMA producer: per K-block a 128x128 tile of A and a 256x128
//               tile of B^T (128-byte swizzle) into a 4-stage ring.
//   warp 1      TMEM allocation; lane 0, per group of four K-blocks, copies
//               the group's scale factors from shared memory into a stage of
//               the TMEM scale-factor ring (columns 256..) with three
//               tcgen05.cp 32x128b.warpx4 (every lane quarter gets its copy,
//               as the MMA reads it), then issues four 128x256x32 block-scaled
//               MMAs per K-block into the accumulator (TMEM columns 0..255).
//   warp 2      scale producer: per group of four K-blocks one TMA load of the
//               A scale grid's 128 x 4 block and one of B's (256 x 4, or the
//               aligned 4 x 4 group of 128-column blocks) into a shared-memory
//               scale ring, running up to four groups ahead.
//   warp 3      scale-factor converter: per group it reads the fp32 scales,
//               takes each one's exponent byte and writes the bytes in the
//               TMEM layout (one 16-byte row per lane) into a staging ring.
//   warps 4-11  epilogue: load the finished accumulator into registers
//               (128 columns per thread), release it to the next unit's MMAs,
//               then convert and store.
// The scale-factor work stays on the first warpgroup: a first form with four
// writer warps (one per lane quarter, each tcgen05.st-ing its quarter's copy),
// which share every SM sub-partition with the MMA and TMA threads, measured
// 628-636 us against 619 us on the Llama4 forward GEMM.
// Scale-factor layout in TMEM (M = 128, N = 256, one CTA, one factor per 32
// K): the factor of row r (of A, or of B^T) sits in lane 32*q + r % 32 for
// each sub-partition q, in 32-bit column r / 32 of the operand's part of the
// stage; the byte of that word is the scale-factor id the MMA names.  A stage
// holds four K-blocks: byte b of every word belongs to the stage's K-block b,
// and all four MMAs of that K-block name id b.
//
// Every mbarrier wait is bounded (kWaitLimitNs); a wait that runs out sets the
// library error flag (bit 0) and the CTA abort flag, and every role leaves as
// in gemm_kernel.cuh.  A scale that is not a positive normal power of two sets
// bit 1 of the error flag.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "ptx_bs.cuh"
#include "gemm_kernel.cuh"

namespace fp8bs {

constexpr int kBsStages = 4;                    // A/B shared-memory ring
constexpr int kSfStages = 4;                    // TMEM scale-factor ring
constexpr int kSfKb = 4;                        // K-blocks per scale-factor stage (bytes per word)
constexpr uint32_t kSfCols = 16;                // TMEM columns per stage
constexpr uint32_t kSfColA = 0;                 // A's 4 words (128 rows / 32) within a stage
constexpr uint32_t kSfColB = 8;                 // B's 8 words (256 columns / 32)
constexpr uint32_t kSfCol0 = kBN;               // the ring follows the accumulator
constexpr int kBsEpiWarps = 8;
constexpr int kBsThreads = 32 * (4 + kBsEpiWarps);
static_assert(kSfCol0 + kSfStages * kSfCols <= kTmemCols, "scale-factor ring exceeds TMEM");

// one scale-ring stage: A's scales [b][128 rows], then B's [b][256 columns]
// (or [b][4 blocks]), b = the stage's four K-blocks
constexpr uint32_t kScStageBytes = (kBM + kBN) * kSfKb * 4;
// one staging stage of scale-factor bytes, each part 32 rows of 16 bytes (the
// source of one tcgen05.cp 32x128b): A, then B's columns 0..127, then 128..255
constexpr uint32_t kSfPartBytes = 32 * 16;
constexpr uint32_t kSfStageBytes = 3 * kSfPartBytes;

struct BsSmem {
    static constexpr uint32_t a_off = 0;
    static constexpr uint32_t b_off = a_off + kBsStages * kATileBytes;
    static constexpr uint32_t sc_off = b_off + kBsStages * kBTileBytes;
    static constexpr uint32_t sf_off = sc_off + kSfStages * kScStageBytes;
    static constexpr uint32_t bar_off = sf_off + kSfStages * kSfStageBytes;
    // ab_full[S], ab_empty[S], sf_full[SS], sf_empty[SS], sc_full[SS], sc_empty[SS], tm_full, tm_empty, drain
    static constexpr uint32_t n_bars = 2 * kBsStages + 4 * kSfStages + 3;
    static constexpr uint32_t misc_off = bar_off + n_bars * 8;
    static constexpr uint32_t total = misc_off + 16;
    static constexpr uint32_t alloc = total + 1024;     // slack to align the base to 1024 B
};
static_assert(BsSmem::alloc <= 232448, "shared memory per CTA");

// The UE8M0 byte of a power-of-two scale r = 2^(e-127): its fp32 biased
// exponent.  Anything else (a mantissa bit, the sign, zero or subnormal,
// inf or NaN) is recorded in `bad`.
__device__ __forceinline__ uint32_t ue8m0_of(float r, uint32_t& bad)
{
    const uint32_t bits = __float_as_uint(r);
    const uint32_t e = bits >> 23;                  // includes the sign bit
    bad |= (bits & 0x7FFFFFu) | (uint32_t)(e - 1u >= 254u);
    return e & 0xFFu;
}

template <int MODE>
__global__ void __launch_bounds__(kBsThreads, 1)
gemm_fp8_bs_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                   const GemmParams p)
{
    static_assert(MODE == kModeBlock128 || MODE == kModeBlock1x128, "block recipes only");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bars = sbase + BsSmem::bar_off;
    auto ab_full = [&](int s) { return bars + 8u * s; };
    auto ab_empty = [&](int s) { return bars + 8u * (kBsStages + s); };
    auto sf_full = [&](int s) { return bars + 8u * (2 * kBsStages + s); };
    auto sf_empty = [&](int s) { return bars + 8u * (2 * kBsStages + kSfStages + s); };
    auto sc_full = [&](int s) { return bars + 8u * (2 * kBsStages + 2 * kSfStages + s); };
    auto sc_empty = [&](int s) { return bars + 8u * (2 * kBsStages + 3 * kSfStages + s); };
    const uint32_t tm_full = bars + 8u * (2 * kBsStages + 4 * kSfStages);
    const uint32_t tm_empty = tm_full + 8u;
    const uint32_t drain_bar = tm_full + 16u;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + BsSmem::misc_off);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + BsSmem::misc_off + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kBsStages; ++s) {
            mbar_init(ab_full(s), 1);
            mbar_init(ab_empty(s), 1);
        }
        for (int s = 0; s < kSfStages; ++s) {
            mbar_init(sf_full(s), 1);
            mbar_init(sf_empty(s), 1);
            mbar_init(sc_full(s), 1);
            mbar_init(sc_empty(s), 1);
        }
        mbar_init(tm_full, 1);
        mbar_init(tm_empty, kBsEpiWarps);
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
    }
    if (warp == 2 && lane == 0) {
        prefetch_tensormap(&tmSA);
        prefetch_tensormap(&tmSB);
    }
    if (warp == 1) {
        tmem_alloc(sbase + BsSmem::misc_off, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicOr(p.err, 1);
    };

    if (warp < 4) {
        if (warp == 0) {
            // ------------------------------------------------------------ producer
            if (lane == 0) {
                int stage = 0;
                uint32_t phase = 0;
                bool ok = true;
                uint32_t filled = 0, fill_par = 0;      // per stage: ever filled, parity of its latest fill
                for (int64_t u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
                    int tm, tn, kb0, kb1, split;
                    decode_unit(p, u, tm, tn, kb0, kb1, split);
                    const int m0 = tm * kBM, n0 = tn * kBN;
                    for (int kb = kb0; kb < kb1; ++kb) {
                        if (!mbar_wait_bounded(ab_empty(stage), phase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
                        mbar_arrive_expect_tx(ab_full(stage), kATileBytes + kBTileBytes);
                        tma_load_2d(sbase + BsSmem::a_off + stage * kATileBytes, &tmA, ab_full(stage), kb * kBK, m0);
                        tma_load_2d(sbase + BsSmem::b_off + stage * kBTileBytes, &tmB, ab_full(stage), kb * kBK, n0);
                        filled |= 1u << stage;
                        fill_par = (fill_par & ~(1u << stage)) | (phase << stage);
                        if (++stage == kBsStages) { stage = 0; phase ^= 1u; }
                    }
                }
                if (!ok) give_up();
                for (int s = 0; s < kBsStages; ++s)
                    if (filled >> s & 1u) mbar_wait_bounded(ab_full(s), fill_par >> s & 1u, nullptr, kDrainLimitNs);
            }
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                int stage = 0, ss = 0;
                uint32_t phase = 0, sphase = 0, tphase = 0;
                bool ok = true, issued = false;
                for (int64_t u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
                    int tm, tn, kb0, kb1, split;
                    decode_unit(p, u, tm, tn, kb0, kb1, split);
                    // the first stage is normally ready before the accumulator is released
                    if (!mbar_wait_bounded(ab_full(stage), phase, abort_flag, kWaitLimitNs)) { ok = false; break; }
                    if (!mbar_wait_bounded(tm_empty, tphase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
                    for (int kb = kb0; kb < kb1; ++kb) {
                        const uint32_t j = (uint32_t)(kb - kb0) & (kSfKb - 1);
                        if (kb != kb0 && !mbar_wait_bounded(ab_full(stage), phase, abort_flag, kWaitLimitNs)) { ok = false; break; }
                        if (j == 0 && !mbar_wait_bounded(sf_full(ss), sphase, abort_flag, kWaitLimitNs)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t sf = tmem_base + kSfCol0 + (uint32_t)ss * kSfCols;
                        if (j == 0) {
                            // the stage's factors: A's 4 words, B's 8 words (two copies of 4)
                            const uint32_t src = sbase + BsSmem::sf_off + (uint32_t)ss * kSfStageBytes;
                            tmem_cp_32x128b_x4(sf + kSfColA, smem_desc_cp_rows16(src));
                            tmem_cp_32x128b_x4(sf + kSfColB, smem_desc_cp_rows16(src + kSfPartBytes));
                            tmem_cp_32x128b_x4(sf + kSfColB + 4, smem_desc_cp_rows16(src + 2 * kSfPartBytes));
                        }
                        const uint32_t sfa = (sf + kSfColA) | (j << 30);
                        const uint32_t sfb = (sf + kSfColB) | (j << 30);
                        const uint32_t idesc = idesc_e4m3_bs(kBM, kBN, j);
                        const uint32_t a_addr = sbase + BsSmem::a_off + stage * kATileBytes;
                        const uint32_t b_addr = sbase + BsSmem::b_off + stage * kBTileBytes;
#pragma unroll
                        for (int k = 0; k < kBK / 32; ++k) {
                            umma_f8_bs(tmem_base, smem_desc_k_sw128(a_addr + k * 32), smem_desc_k_sw128(b_addr + k * 32),
                                       idesc, sfa, sfb, (kb > kb0 || k > 0) ? 1u : 0u);
                        }
                        issued = true;
                        if (kb + 1 == kb1) umma_commit(tm_full);
                        umma_commit(ab_empty(stage));
                        if (j == kSfKb - 1 || kb + 1 == kb1) {
                            umma_commit(sf_empty(ss));
                            if (++ss == kSfStages) { ss = 0; sphase ^= 1u; }
                        }
                        if (++stage == kBsStages) { stage = 0; phase ^= 1u; }
                    }
                    tphase ^= 1u;
                }
                if (!ok) give_up();
                if (issued) {
                    umma_commit(drain_bar);
                    mbar_wait_bounded(drain_bar, 0, nullptr, kDrainLimitNs);
                }
            }
        } else if (warp == 2) {
            // ------------------------------------------------------------ scale producer
            if (lane == 0) {
                constexpr uint32_t kTx = kBM * kSfKb * 4 + (MODE == kModeBlock128 ? 4 : kBN) * kSfKb * 4;
                int ss = 0;
                uint32_t sphase = 0;
                bool ok = true;
                uint32_t filled = 0, fill_par = 0;
                for (int64_t u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
                    int tm, tn, kb0, kb1, split;
                    decode_unit(p, u, tm, tn, kb0, kb1, split);
                    for (int kbase = kb0; kbase < kb1; kbase += kSfKb) {
                        if (!mbar_wait_bounded(sc_empty(ss), sphase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
                        const uint32_t dst = sbase + BsSmem::sc_off + (uint32_t)ss * kScStageBytes;
                        mbar_arrive_expect_tx(sc_full(ss), kTx);
                        tma_load_2d(dst, &tmSA, sc_full(ss), tm * kBM, kbase);
                        // B: 256 columns, or the 16-byte-aligned group of four 128-column blocks
                        tma_load_2d(dst + kBM * kSfKb * 4, &tmSB, sc_full(ss),
                                    MODE == kModeBlock128 ? ((tn * kBN) >> 7) & ~3 : tn * kBN, kbase);
                        filled |= 1u << ss;
                        fill_par = (fill_par & ~(1u << ss)) | (sphase << ss);
                        if (++ss == kSfStages) { ss = 0; sphase ^= 1u; }
                    }
                }
                if (!ok) give_up();
                for (int s = 0; s < kSfStages; ++s)
                    if (filled >> s & 1u) mbar_wait_bounded(sc_full(s), fill_par >> s & 1u, nullptr, kDrainLimitNs);
            }
        } else {
            // ------------------------------------------------------------ scale-factor converter
            int ss = 0;
            uint32_t sphase = 0;
            bool ok = true;
            uint32_t bad = 0;
            for (int64_t u = blockIdx.x; u < p.num_units; u += gridDim.x) {
                int tm, tn, kb0, kb1, split;
                decode_unit(p, u, tm, tn, kb0, kb1, split);
                const int m0 = tm * kBM, n0 = tn * kBN;
                for (int kbase = kb0; kbase < kb1; kbase += kSfKb) {
                    // every lane waits; a wait that gives up raises the abort
                    // flag, the outcome is voted per unit
                    if (!mbar_wait_bounded(sc_full(ss), sphase, abort_flag, kWaitLimitNs)) ok = false;
                    const float* sc = reinterpret_cast<const float*>(smem + BsSmem::sc_off + (uint32_t)ss * kScStageBytes);
                    const float* scb = sc + kBM * kSfKb;
                    // lane l's 16-byte row of each part: word j = rows (columns) 32j + l,
                    // byte b = K-block kbase + b
                    uint32_t wa[4], wb[8];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int m = m0 + 32 * j + lane;
                        uint32_t word = 0;
#pragma unroll
                        for (int b = 0; b < kSfKb; ++b) {
                            uint32_t e = 127u;                       // 1.0 where no row or K-block is
                            if (m < p.M && kbase + b < kb1) e = ue8m0_of(sc[b * kBM + 32 * j + lane], bad);
                            word |= e << (8 * b);
                        }
                        wa[j] = word;
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        int idx, col;                                 // global index, index within the ring stage
                        if (MODE == kModeBlock128) {
                            idx = (n0 >> 7) + (j >> 2);               // the 128-column block of columns n0+32j ..
                            col = (idx & 3);
                        } else {
                            idx = n0 + 32 * j + lane;
                            col = 32 * j + lane;
                        }
                        const bool valid = MODE == kModeBlock128 ? idx * 128 < p.N : idx < p.N;
                        constexpr int kBW = MODE == kModeBlock128 ? 4 : kBN;   // B entries per K-block in the stage
                        uint32_t word = 0;
#pragma unroll
                        for (int b = 0; b < kSfKb; ++b) {
                            uint32_t e = 127u;
                            if (valid && kbase + b < kb1) e = ue8m0_of(scb[b * kBW + col], bad);
                            word |= e << (8 * b);
                        }
                        wb[j] = word;
                    }
                    // the fp32 stage is read: back to the scale producer
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sc_empty(ss));
                    // the staging stage is free once the MMA thread's copies from it
                    // (and the MMAs reading the TMEM stage they fill) have completed
                    if (!mbar_wait_bounded(sf_empty(ss), sphase ^ 1u, abort_flag, kWaitLimitNs)) ok = false;
                    const uint32_t dst = sbase + BsSmem::sf_off + (uint32_t)ss * kSfStageBytes + (uint32_t)lane * 16u;
                    sts128(dst, wa[0], wa[1], wa[2], wa[3]);
                    sts128(dst + kSfPartBytes, wb[0], wb[1], wb[2], wb[3]);
                    sts128(dst + 2 * kSfPartBytes, wb[4], wb[5], wb[6], wb[7]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sf_full(ss));
                    if (++ss == kSfStages) { ss = 0; sphase ^= 1u; }
                }
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
            }
            if (!ok && lane == 0) give_up();
            if (__any_sync(0xffffffffu, bad != 0) && lane == 0) atomicOr(p.err, 2);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int e = warp - 4;                  // 0 .. 7
        const int lq = warp & 3;                 // TMEM lane quarter this warp may access
        const int col0 = (e >> 2) * 128;         // this warp's 128 columns of the tile
        const uint32_t taddr = tmem_base + ((uint32_t)(lq * 32) << 16) + (uint32_t)col0;
        uint32_t tphase = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < p.num_units; u += gridDim.x) {
            int tm, tn, kb0, kb1, split;
            decode_unit(p, u, tm, tn, kb0, kb1, split);
            if (!mbar_wait_bounded(tm_full, tphase, abort_flag, kWaitLimitNs)) ok = false;
            tc_fence_after();
            uint32_t r0[32], r1[32], r2[32], r3[32];
            tmem_ld_32x32b_x32(taddr, r0);
            tmem_ld_32x32b_x32(taddr + 32, r1);
            tmem_ld_32x32b_x32(taddr + 64, r2);
            tmem_ld_32x32b_x32(taddr + 96, r3);
            tmem_ld_wait();
            reg_after_wait32(r0);
            reg_after_wait32(r1);
            reg_after_wait32(r2);
            reg_after_wait32(r3);
            // the warp-collective wait above leaves all lanes' loads complete:
            // the accumulator goes back to the MMA warp before the stores
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tm_empty);
            tphase ^= 1u;
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;

            const int64_t m = (int64_t)tm * kBM + lq * 32 + lane;
            const int n_base = tn * kBN + col0;
            auto val = [&](int c) -> float {
                const uint32_t* rr = c < 32 ? r0 : c < 64 ? r1 : c < 96 ? r2 : r3;
                return __uint_as_float(rr[c & 31]);
            };
            if (m < p.M) {
                if (p.splits > 1 || p.out_f32) {
                    float* dst = p.splits > 1 ? p.ws + ((int64_t)split * p.M + m) * p.ldw
                                              : reinterpret_cast<float*>(p.D) + m * p.ldd;
                    const bool vec = p.splits > 1 || p.vec_out;   // the partials' pitch is a multiple of 4
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int n = n_base + 4 * j;
                        const float4 v = make_float4(val(4 * j), val(4 * j + 1), val(4 * j + 2), val(4 * j + 3));
                        if (vec && n + 4 <= p.N) {
                            *reinterpret_cast<float4*>(dst + n) = v;
                        } else if (n < p.N) {
                            const float vv[4] = {v.x, v.y, v.z, v.w};
                            for (int t = 0; t < min(4, p.N - n); ++t) dst[n + t] = vv[t];
                        }
                    }
                } else {
                    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.D) + m * p.ldd;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = n_base + 8 * j;
                        const uint4 w = make_uint4(cvt_bf16x2(val(8 * j), val(8 * j + 1)),
                                                   cvt_bf16x2(val(8 * j + 2), val(8 * j + 3)),
                                                   cvt_bf16x2(val(8 * j + 4), val(8 * j + 5)),
                                                   cvt_bf16x2(val(8 * j + 6), val(8 * j + 7)));
                        if (p.vec_out && n + 8 <= p.N) {
                            *reinterpret_cast<uint4*>(dst + n) = w;
                        } else if (n < p.N) {
                            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                            uint16_t* d16 = reinterpret_cast<uint16_t*>(dst);
                            for (int t = 0; t < min(8, p.N - n); ++t)
                                d16[n + t] = (uint16_t)((ww[t >> 1] >> ((t & 1) * 16)) & 0xFFFFu);
                        }
                    }
                }
            }
        }
        if (!ok && lane == 0) give_up();
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace fp8bs
