// gemm_kernel.cuh -- FP8 (e4m3) scaled GEMM on the sm_100a tensor cores.
//
// Computes  D[m,n] = sum_kb rA(m,kb) * rB(n,kb) * P_kb[m,n],
//           P_kb[m,n] = sum_{k in K-block kb} qA[m,k] * qB[n,k]
// i.e. the dequantized matmul that pytorch/ao PR #4209 "[codex] add repro for
// blockwise _scaled_mm investigation" (What Changed) uses as ground truth, for
// the (1x128, 128x128) and (1x128, 1x128) recipes of that page and the
// per-tensor / rowwise recipes of ROCm/aiter issue #1765 and pytorch/pytorch
// issue #159940.
//
// One persistent CTA per SM computes 128 x 256 output tiles:
//   warp 0      TMA producer: per K-block one 128x128 tile of A and one
//               256x128 tile of B^T (bytes, 128-byte swizzle) into a 4-stage
//               shared-memory ring; for the rowwise and 1x128 x 1x128 recipes
//               also the K-block's scale vectors into a separate ring (the
//               1x128 x 128x128 promotion warps read their two scalars per
//               K-block from L2 themselves).
//   warp 1      TMEM allocation; lane 0 issues four tcgen05.mma (128x256x32,
//               e4m3 x e4m3 -> fp32) per K-block into one of two 256-column
//               TMEM accumulators and commits the accumulator and the smem
//               stage when the MMAs complete.
//   warps 2..   promotion / epilogue (8 warps, or 16 for the 1x128 x 1x128
//               recipe whose per-column scales double the per-element work;
//               with both block recipes the promotion warps start at warp 4,
//               after a first warpgroup whose two idle warps let it hand its
//               registers over to them):
//               per accumulation group (one K-block for the block recipes; the
//               whole K range for tensor/rowwise) they tcgen05.ld the partial
//               sums, multiply by the scale product and add into fp32 registers
//               (packed f32x2 FMA), then release the TMEM buffer so the MMA of
//               group g+2 can start.  At the end of a tile the registers are
//               converted and stored.
// The per-K-block promotion keeps every partial sum in fp32 with the exact
// scale product of its block, which is what makes any number of K blocks
// (1000, 1001, 1002, ...) safe: scale indexing is kb*ld + i with no padding
// or parity assumption.
//
// Every mbarrier wait is bounded (kWaitLimitNs).  A wait that runs out sets
// the library error flag and a CTA-wide abort flag; all roles then leave their
// loops, the producer waits (bounded) for its TMA copies in flight, the MMA
// thread waits (bounded) for its MMAs in flight, and TMEM is freed before exit.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "quant_kernels.cuh"

namespace fp8bs {

constexpr int kBM = 128;                        // tile rows (TMEM lanes)
constexpr int kBN = 256;                        // tile columns (TMEM columns per accumulator)
constexpr int kBK = 128;                        // K-block = scale block = one 128-byte swizzle row
constexpr uint32_t kTmemCols = 512;             // all of TMEM
constexpr int kTmemBufs = kTmemCols / kBN;      // two accumulators in flight
constexpr int kStages = 4;                      // A/B smem ring depth
constexpr int kScaleStages = kStages + kTmemBufs + 2;   // scale ring depth (> kStages + kTmemBufs)
constexpr uint64_t kWaitLimitNs = 4000000000ull;   // pipeline waits
constexpr uint64_t kDrainLimitNs = 1000000000ull;  // exit-time waits for work in flight

constexpr uint32_t kATileBytes = kBM * kBK;             // 16 KB
constexpr uint32_t kBTileBytes = kBN * kBK;             // 32 KB
constexpr uint32_t kScaleEntryBytes = (kBM + kBN) * 4;  // sa[128] then sb[256]

struct SmemLayout {
    static constexpr uint32_t a_off = 0;
    static constexpr uint32_t b_off = a_off + kStages * kATileBytes;
    static constexpr uint32_t sc_off = b_off + kStages * kBTileBytes;
    static constexpr uint32_t bar_off = sc_off + kScaleStages * kScaleEntryBytes;
    // ab_full[S], ab_empty[S], sc_full[SS], sc_empty[SS], tm_full[2], tm_empty[2], drain
    static constexpr uint32_t n_bars = 2 * kStages + 2 * kScaleStages + 2 * kTmemBufs + 1;
    static constexpr uint32_t misc_off = bar_off + n_bars * 8;
    static constexpr uint32_t total = misc_off + 16;
    static constexpr uint32_t alloc = total + 1024;     // slack to align the base to 1024 B
};

enum GemmMode : int { kModeTensor = 0, kModeRowwise = 1, kModeBlock128 = 2, kModeBlock1x128 = 3 };

// Warp roles per recipe.  Warp 0 issues the TMA loads, warp 1 the MMAs, the
// rest promote and store.  With `reg_split` the first warpgroup (producer, MMA
// issuer and two idle warps) hands registers over to the promotion warps
// (setmaxnreg), which then run their loop without spills; the hand-over is
// sized for exactly `launch_regs` registers per thread at launch, which the
// host checks before the first launch.  Measured on B200: the 1x128 x 128x128
// recipe is fastest with 8 promotion warps at 232 registers that issue four
// 16-column TMEM loads per wait (the per-warp promotion time follows the
// number of load round trips, not the bytes), the 1x128 x 1x128 recipe with
// 16 promotion warps keeping two chunks in flight, at 104 registers after the
// hand-over (96 at launch, where the loop spilled: 6% slower).
template <int MODE>
struct EpiCfg {
    static constexpr int warps = MODE == kModeBlock1x128 ? 16 : 8;
    static constexpr bool reg_split = MODE == kModeBlock1x128 || MODE == kModeBlock128;
    static constexpr bool quad_loads = MODE == kModeBlock128;   // four TMEM loads per wait; else two in flight
    static constexpr int ctrl_warps = reg_split ? 4 : 2;
    static constexpr int threads = 32 * (ctrl_warps + warps);
    static constexpr int cols = kBN * 4 / warps;        // accumulator columns per thread
    static constexpr int chunks = cols / 16;            // 16-column TMEM loads per group
    // registers per thread at launch: the per-sub-partition limit of
    // __launch_bounds__(threads, 1) (16384 registers shared by the
    // ceil(warps / 4) warps of each SM sub-partition, in steps of 8); after
    // the hand-over the first warpgroup keeps ctrl_regs, the promotion warps
    // take the rest (at most 232)
    static constexpr int launch_regs = (16384 / (32 * ((ctrl_warps + warps + 3) / 4))) / 8 * 8;
    static constexpr int ctrl_regs = 40;
    static constexpr int epi_regs_raw = (threads * launch_regs - 128 * ctrl_regs) / (32 * warps) / 8 * 8;
    static constexpr int epi_regs = epi_regs_raw > 232 ? 232 : epi_regs_raw;
    static_assert(!reg_split || (ctrl_warps == 4 && warps % 4 == 0 &&
                                 128 * ctrl_regs + 32 * warps * epi_regs <= threads * launch_regs),
                  "register hand-over exceeds the launch allocation");
    static_assert(!quad_loads || chunks % 4 == 0, "four TMEM loads per wait");
};

struct GemmParams {
    int32_t M, N, K;
    int32_t Kb;                 // number of K blocks
    int32_t tiles_m, tiles_n;
    int32_t splits;             // K splits per tile (1 = no split-K)
    int32_t group_m;            // rasterization band height in tiles
    int64_t num_units;          // tiles_m * tiles_n * splits
    void* D;                    // output (bf16 or fp32) when splits == 1
    int64_t ldd;
    int32_t out_f32;
    int32_t vec_out;            // 1: D and ldd allow 16-byte row-chunk stores
    float* ws;                  // split-K partials [splits][M][ldw] fp32
    int64_t ldw;
    const float* sa;            // scale pointers read directly (tensor mode, 1x128 x 128x128 mode)
    const float* sb;
    int64_t ld_sa, ld_sb;       // their leading dimensions (block modes)
    int* err;                   // library error flag
};

// The fused-quantization instantiation's parameters: the bf16 output's 1x128
// groups along N as e4m3 bytes and reciprocal scales.  (A separate type, so
// that the other instantiations keep their parameter block as it is.)
struct GemmParamsQ : GemmParams {
    uint8_t* qout;
    int64_t ldq_out;
    float* sout;
    int64_t lds_out;
};

// The grouped instantiation's parameters (a grouped / MoE GEMM: G independent
// GEMMs D_g = scaled(A_g . B_g^T) in one persistent launch).  The groups' rows
// of A, D and of A's scale grid are packed one after another (group g starts
// at row row_start[g]); group g's B^T is rows g*N .. g*N + N - 1 of a stacked
// G*N x K matrix, its 128x128 scale grid starts sb_stride floats after group
// g-1's.  Tiles of group g are units tile_start[g] .. tile_start[g+1] - 1.
constexpr int kMaxGroups = 64;
struct GemmParamsG : GemmParams {
    int32_t groups;
    int32_t row_start[kMaxGroups + 1];
    int32_t tile_start[kMaxGroups + 1];
    int64_t sb_stride;
};

__device__ __forceinline__ void decode_unit(const GemmParams& p, int64_t u, int& tm, int& tn, int& kb0, int& kb1,
                                            int& split)
{
    const int64_t tile = u / p.splits;
    split = (int)(u - tile * p.splits);
    // grouped rasterization: bands of group_m tile-rows, column-major inside a band
    const int64_t band_tiles = (int64_t)p.group_m * p.tiles_n;
    const int64_t band = tile / band_tiles;
    const int64_t in_band = tile - band * band_tiles;
    const int band_m0 = (int)(band * p.group_m);
    const int band_h = min(p.group_m, p.tiles_m - band_m0);
    tm = band_m0 + (int)(in_band % band_h);
    tn = (int)(in_band / band_h);
    kb0 = (int)(((int64_t)p.Kb * split) / p.splits);
    kb1 = (int)(((int64_t)p.Kb * (split + 1)) / p.splits);
}

// Group of unit u of a grouped launch, its tile within the group (the same
// banded rasterization as decode_unit, over the group's tile rows), its first
// row, one past its last row, and the first row of its B^T in the stack.
__device__ __forceinline__ void decode_group_unit(const GemmParamsG& p, int64_t u, int& g, int& tm, int& tn,
                                                  int& row0, int& row_end, int& brow0)
{
    int lo = 0, hi = p.groups - 1;
    while (lo < hi) {                  // last group whose first tile is <= u
        const int mid = (lo + hi + 1) >> 1;
        if (p.tile_start[mid] <= u) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const int64_t local = u - p.tile_start[g];
    row0 = p.row_start[g];
    row_end = p.row_start[g + 1];
    const int tiles_m = (row_end - row0 + kBM - 1) / kBM;
    const int64_t band_tiles = (int64_t)p.group_m * p.tiles_n;
    const int64_t band = local / band_tiles;
    const int64_t in_band = local - band * band_tiles;
    const int band_m0 = (int)(band * p.group_m);
    const int band_h = min(p.group_m, tiles_m - band_m0);
    tm = band_m0 + (int)(in_band % band_h);
    tn = (int)(in_band / band_h);
    brow0 = g * p.N;
}

// QOUT: the epilogue also quantizes the bf16 output, 1x128 along N (each
// promotion thread holds one row's 128 consecutive columns: one whole group),
// byte-identical to quantizing the stored bf16 output afterwards.
// GROUPED: a grouped launch (GemmParamsG); 1x128 x 128x128 recipe, no split-K.
// The tile's rows past its group's last row are multiplied with the next
// group's rows of A (or TMA's zero fill) and never stored.
// BMN: B given MN-major (stored K x N, N contiguous): each K-block's B tile is
// two 128 x 128-byte boxes (K rows x N bytes, 128-byte swizzle), N-halves 16 KB
// apart, read by the MMA through the MN-major descriptor; the 1x128 x 128x128
// scale grid is then B's in storage order, rB(n, kb) = sb[kb + (n/128) ld_sb].
template <int MODE, bool QOUT = false, bool GROUPED = false, bool BMN = false>
__global__ void __launch_bounds__(EpiCfg<MODE>::threads, 1)
gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                const std::conditional_t<QOUT, GemmParamsQ, std::conditional_t<GROUPED, GemmParamsG, GemmParams>> p)
{
    static_assert(!GROUPED || (MODE == kModeBlock128 && !QOUT), "grouped launches: 1x128 x 128x128, plain output");
    static_assert(!BMN || (!GROUPED && !QOUT && MODE != kModeBlock1x128), "MN-major B: plain launches, not 1x128 x 1x128");
    using E = EpiCfg<MODE>;
    static_assert(!QOUT || E::cols == 128, "fused output quantization needs one 1x128 group per thread");
    constexpr int kEpiWarps = E::warps;
    constexpr int kColsPerThread = E::cols;
    constexpr int kChunks = E::chunks;
    constexpr bool kPromote = (MODE == kModeBlock128 || MODE == kModeBlock1x128);
    // The 1x128 x 128x128 recipe needs two scalars per thread and K-block:
    // they are read straight from global memory (L2), prefetched two K-blocks
    // ahead.  Per-column scales (rowwise, 1x128 x 1x128) go through a
    // shared-memory ring filled by TMA.
    constexpr bool kScaleRing = (MODE == kModeRowwise || MODE == kModeBlock1x128);
    constexpr bool kColScales = (MODE == kModeBlock1x128 || MODE == kModeRowwise);
    constexpr uint32_t kScaleTx = kBM * 4 + (kColScales ? kBN * 4 : 16);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bars = sbase + SmemLayout::bar_off;
    auto ab_full = [&](int s) { return bars + 8u * s; };
    auto ab_empty = [&](int s) { return bars + 8u * (kStages + s); };
    auto sc_full = [&](int s) { return bars + 8u * (2 * kStages + s); };
    auto sc_empty = [&](int s) { return bars + 8u * (2 * kStages + kScaleStages + s); };
    auto tm_full = [&](int b) { return bars + 8u * (2 * kStages + 2 * kScaleStages + b); };
    auto tm_empty = [&](int b) { return bars + 8u * (2 * kStages + 2 * kScaleStages + kTmemBufs + b); };
    const uint32_t drain_bar = bars + 8u * (2 * kStages + 2 * kScaleStages + 2 * kTmemBufs);
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + SmemLayout::misc_off);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SmemLayout::misc_off + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(ab_full(s), 1);
            mbar_init(ab_empty(s), 1);
        }
        for (int s = 0; s < kScaleStages; ++s) {
            mbar_init(sc_full(s), 1);
            mbar_init(sc_empty(s), kEpiWarps);
        }
        for (int b = 0; b < kTmemBufs; ++b) {
            mbar_init(tm_full(b), 1);
            mbar_init(tm_empty(b), kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        if (kScaleRing) {
            prefetch_tensormap(&tmSA);
            prefetch_tensormap(&tmSB);
        }
    }
    if (warp == 1) {
        tmem_alloc(sbase + SmemLayout::misc_off, kTmemCols);
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

    if (warp < E::ctrl_warps) {
        // the first warpgroup's roles (its hand-over is warpgroup-uniform)
        if constexpr (E::reg_split) setmaxnreg_dec<E::ctrl_regs>();
        if (warp == 0) {
            // ------------------------------------------------------------ producer
            if (lane == 0) {
                int stage = 0;
                uint32_t phase = 0;
                int ss = 0;
                uint32_t sphase = 0;
                bool ok = true;
                // per stage: was it ever filled, and the parity of its latest fill
                uint32_t filled = 0, fill_par = 0, sfilled = 0, sfill_par = 0;
                auto issue_scales = [&](int m0, int n0, int kb) -> bool {
                    if (!mbar_wait_bounded(sc_empty(ss), sphase ^ 1u, abort_flag, kWaitLimitNs)) return false;
                    const uint32_t dst = sbase + SmemLayout::sc_off + ss * kScaleEntryBytes;
                    mbar_arrive_expect_tx(sc_full(ss), kScaleTx);
                    tma_load_2d(dst, &tmSA, sc_full(ss), m0, kb);
                    if (kColScales) {
                        tma_load_2d(dst + kBM * 4, &tmSB, sc_full(ss), n0, kb);
                    } else {
                        tma_load_2d(dst + kBM * 4, &tmSB, sc_full(ss), (n0 / 128) & ~3, kb);
                    }
                    sfilled |= 1u << ss;
                    sfill_par = (sfill_par & ~(1u << ss)) | (sphase << ss);
                    if (++ss == kScaleStages) { ss = 0; sphase ^= 1u; }
                    return true;
                };
                for (int64_t u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
                    int tm, tn, kb0, kb1, split;
                    decode_unit(p, u, tm, tn, kb0, kb1, split);
                    int m0 = tm * kBM, n0 = tn * kBN;
                    if constexpr (GROUPED) {
                        int g, row0, row_end, brow0;
                        decode_group_unit(p, u, g, tm, tn, row0, row_end, brow0);
                        m0 = row0 + tm * kBM;
                        n0 = brow0 + tn * kBN;
                        kb0 = 0;
                        kb1 = p.Kb;
                    }
                    if (MODE == kModeRowwise) ok = issue_scales(m0, n0, 0);
                    for (int kb = kb0; kb < kb1 && ok; ++kb) {
                        if (!mbar_wait_bounded(ab_empty(stage), phase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
                        mbar_arrive_expect_tx(ab_full(stage), kATileBytes + kBTileBytes);
                        tma_load_2d(sbase + SmemLayout::a_off + stage * kATileBytes, &tmA, ab_full(stage), kb * kBK, m0);
                        if constexpr (BMN) {
                            const uint32_t bdst = sbase + SmemLayout::b_off + stage * kBTileBytes;
                            tma_load_2d(bdst, &tmB, ab_full(stage), n0, kb * kBK);
                            tma_load_2d(bdst + kBTileBytes / 2, &tmB, ab_full(stage), n0 + kBN / 2, kb * kBK);
                        } else {
                            tma_load_2d(sbase + SmemLayout::b_off + stage * kBTileBytes, &tmB, ab_full(stage), kb * kBK, n0);
                        }
                        filled |= 1u << stage;
                        fill_par = (fill_par & ~(1u << stage)) | (phase << stage);
                        if (++stage == kStages) { stage = 0; phase ^= 1u; }
                        if (kPromote && kScaleRing) ok = issue_scales(m0, n0, kb);
                    }
                }
                if (!ok) give_up();
                // drain: every issued TMA copy must have landed before the CTA exits
                for (int s = 0; s < kStages; ++s)
                    if (filled >> s & 1u) mbar_wait_bounded(ab_full(s), fill_par >> s & 1u, nullptr, kDrainLimitNs);
                for (int s = 0; s < kScaleStages; ++s)
                    if (sfilled >> s & 1u) mbar_wait_bounded(sc_full(s), sfill_par >> s & 1u, nullptr, kDrainLimitNs);
            }
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idesc = BMN ? idesc_e4m3_f32_major(kBM, kBN, 1) : idesc_e4m3_f32(kBM, kBN);
                int stage = 0;
                uint32_t phase = 0;
                int tb = 0;
                uint32_t tphase = 0;
                bool ok = true, issued = false;
                for (int64_t u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
                    int tm, tn, kb0, kb1, split;
                    decode_unit(p, u, tm, tn, kb0, kb1, split);
                    const int ngroups = kPromote ? (kb1 - kb0) : 1;
                    int kb = kb0;
                    for (int g = 0; g < ngroups && ok; ++g) {
                        const int kb_end = kPromote ? kb + 1 : kb1;
                        // The smem stage of the group's first K-block is normally
                        // ready long before the TMEM buffer is free: wait for it
                        // first, so that only the TMEM hand-off is on the critical path.
                        if (!mbar_wait_bounded(ab_full(stage), phase, abort_flag, kWaitLimitNs)) { ok = false; break; }
                        if (!mbar_wait_bounded(tm_empty(tb), tphase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t d_tmem = tmem_base + (uint32_t)(tb * kBN);
                        const int kb_first = kb;         // its stage was waited for above
                        for (; kb < kb_end; ++kb) {
                            if (kb != kb_first) {
                                if (!mbar_wait_bounded(ab_full(stage), phase, abort_flag, kWaitLimitNs)) { ok = false; break; }
                                tc_fence_after();
                            }
                            const uint32_t a_addr = sbase + SmemLayout::a_off + stage * kATileBytes;
                            const uint32_t b_addr = sbase + SmemLayout::b_off + stage * kBTileBytes;
    #pragma unroll
                            for (int k = 0; k < kBK / 32; ++k) {
                                const uint64_t adesc = smem_desc_k_sw128(a_addr + k * 32);
                                // MN-major: a 32-deep K step is 4 groups of 8 K-rows (4 KB)
                                const uint64_t bdesc = BMN ? smem_desc_mn_sw128(b_addr + k * 4096, kBTileBytes / 2)
                                                           : smem_desc_k_sw128(b_addr + k * 32);
                                const uint32_t acc = (kPromote ? (k > 0) : (kb > kb0 || k > 0)) ? 1u : 0u;
                                umma_f8(d_tmem, adesc, bdesc, idesc, acc);
                            }
                            issued = true;
                            // the accumulator hand-off is on the critical path: signal it first
                            if (kb + 1 == kb_end) umma_commit(tm_full(tb));
                            umma_commit(ab_empty(stage));
                            if (++stage == kStages) { stage = 0; phase ^= 1u; }
                        }
                        if (!ok) break;
                        if (++tb == kTmemBufs) { tb = 0; tphase ^= 1u; }
                    }
                }
                if (!ok) give_up();
                if (issued) {
                    // all MMAs of this thread complete before TMEM can be freed
                    umma_commit(drain_bar);
                    mbar_wait_bounded(drain_bar, 0, nullptr, kDrainLimitNs);
                }
            }
        }
    } else {
        if constexpr (E::reg_split) setmaxnreg_inc<E::epi_regs>();
        // ------------------------------------------------------------ promotion / epilogue
        const int e = warp - E::ctrl_warps;     // 0 .. kEpiWarps-1
        const int lq = warp & 3;                // TMEM lane quarter this warp may access
        const int col0 = (e >> 2) * kColsPerThread;   // this warp's columns within the tile
        const int row_in_tile = lq * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(lq * 32) << 16;
        int tb = 0;
        uint32_t tphase = 0;
        int ss = 0;
        uint32_t sphase = 0;
        bool ok = true;
        float tensor_scale = 1.0f;
        if (MODE == kModeTensor) tensor_scale = __ldg(p.sa) * __ldg(p.sb);

        for (int64_t u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
            int tm, tn, kb0, kb1, split;
            decode_unit(p, u, tm, tn, kb0, kb1, split);
            const int ngroups = kPromote ? (kb1 - kb0) : 1;
            float2 acc[kColsPerThread / 2];
#pragma unroll
            for (int i = 0; i < kColsPerThread / 2; ++i) acc[i] = make_float2(0.f, 0.f);

            // 1x128 x 128x128: this thread's row scale and its columns' block
            // scale, for K-blocks kb0, kb0+1 (loaded now) and kb0+2.. (loaded
            // two groups ahead, from L2)
            int64_t m_glob = (int64_t)tm * kBM + row_in_tile;
            int64_t m_end = p.M;                        // rows at or past this are never stored
            const float* sb_g = p.sb;
            if constexpr (GROUPED) {
                int g, row0, row_end, brow0;
                decode_group_unit(p, u, g, tm, tn, row0, row_end, brow0);
                m_glob = row0 + (int64_t)tm * kBM + row_in_tile;
                m_end = row_end;
                sb_g = p.sb + (int64_t)g * p.sb_stride;
                kb0 = 0;
                kb1 = p.Kb;
            }
            const bool row_ok = m_glob < m_end;
            const int nb_glob = (tn * kBN + col0) / 128;
            const bool nb_ok = nb_glob * 128 < p.N;     // columns past N are never stored
            // raw values only: the product is formed when the group is promoted,
            // so the loads stay in flight for two groups
            auto load_scales = [&](int kb, float& a, float& b) {
                if (MODE != kModeBlock128 || kb >= kb1 || !row_ok || !nb_ok) { a = b = 0.f; return; }
                a = __ldg(p.sa + m_glob + (int64_t)kb * p.ld_sa);
                b = BMN ? __ldg(sb_g + kb + (int64_t)nb_glob * p.ld_sb) : __ldg(sb_g + nb_glob + (int64_t)kb * p.ld_sb);
            };
            float pa0, pb0, pa1, pb1;
            load_scales(kb0, pa0, pb0);
            load_scales(kb0 + 1, pa1, pb1);

            for (int g = 0; g < ngroups; ++g) {
                // Every lane waits.  A wait that gives up raises the abort flag
                // and the warp carries on (no warp vote per K-block); the
                // outcome is voted once per tile, below.
                uint32_t sc_addr = 0;
                float rowf = tensor_scale;
                if (MODE == kModeBlock128) {
                    rowf = pa0 * pb0;
                    pa0 = pa1;
                    pb0 = pb1;
                    load_scales(kb0 + g + 2, pa1, pb1);
                }
                if (kScaleRing) {
                    if (!mbar_wait_bounded(sc_full(ss), sphase, abort_flag, kWaitLimitNs)) { ok = false; give_up(); }
                    const float* sc = reinterpret_cast<const float*>(smem + SmemLayout::sc_off + ss * kScaleEntryBytes);
                    sc_addr = sbase + SmemLayout::sc_off + ss * kScaleEntryBytes;
                    rowf = sc[row_in_tile];
                }
                if (!mbar_wait_bounded(tm_full(tb), tphase, abort_flag, kWaitLimitNs)) { ok = false; give_up(); }
                tc_fence_after();
                const float2 rowf2 = make_float2(rowf, rowf);
                const uint32_t tcol = tmem_base + lane_addr + (uint32_t)(tb * kBN + col0);
                auto promote = [&](int c, const uint32_t (&r)[16]) {
                    if (kColScales) {
                        const uint32_t sb_addr = sc_addr + (uint32_t)((kBM + col0 + c * 16) * 4);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float4 b4 = lds128(sb_addr + 16 * j);
                            const float2 f0 = fmul2(rowf2, make_float2(b4.x, b4.y));
                            const float2 f1 = fmul2(rowf2, make_float2(b4.z, b4.w));
                            acc[c * 8 + 2 * j] = ffma2(make_float2(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1])), f0, acc[c * 8 + 2 * j]);
                            acc[c * 8 + 2 * j + 1] = ffma2(make_float2(__uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])), f1, acc[c * 8 + 2 * j + 1]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            acc[c * 8 + j] = ffma2(make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])), rowf2, acc[c * 8 + j]);
                    }
                };
                if constexpr (E::quad_loads) {
                    // four 16-column loads per wait (64 registers in flight)
#pragma unroll
                    for (int h = 0; h < kChunks / 4; ++h) {
                        uint32_t r0[16], r1[16], r2[16], r3[16];
                        tmem_ld_32x32b_x16(tcol + (4 * h + 0) * 16, r0);
                        tmem_ld_32x32b_x16(tcol + (4 * h + 1) * 16, r1);
                        tmem_ld_32x32b_x16(tcol + (4 * h + 2) * 16, r2);
                        tmem_ld_32x32b_x16(tcol + (4 * h + 3) * 16, r3);
                        tmem_ld_wait(r0);
                        reg_after_wait(r1);
                        reg_after_wait(r2);
                        reg_after_wait(r3);
                        promote(4 * h + 0, r0);
                        promote(4 * h + 1, r1);
                        promote(4 * h + 2, r2);
                        promote(4 * h + 3, r3);
                    }
                } else {
                    // two 16-column loads in flight: chunk c+1 loads while c is promoted
                    uint32_t rbuf[2][16];
                    tmem_ld_32x32b_x16(tcol, rbuf[0]);
                    tmem_ld_wait(rbuf[0]);
#pragma unroll
                    for (int c = 0; c < kChunks; ++c) {
                        if (c + 1 < kChunks) tmem_ld_32x32b_x16(tcol + (c + 1) * 16, rbuf[(c + 1) & 1]);
                        promote(c, rbuf[c & 1]);
                        if (c + 1 < kChunks) tmem_ld_wait(rbuf[(c + 1) & 1]);
                    }
                }
                // the warp-collective tcgen05.wait::ld above leaves all lanes'
                // loads complete: lane 0 may release the buffer
                tc_fence_before();
                if (lane == 0) {
                    mbar_arrive(tm_empty(tb));
                    if (kScaleRing) mbar_arrive(sc_empty(ss));
                }
                if (++tb == kTmemBufs) { tb = 0; tphase ^= 1u; }
                if (kScaleRing) {
                    if (++ss == kScaleStages) { ss = 0; sphase ^= 1u; }
                }
            }
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;

            // ---- store the tile: row m, this thread's kColsPerThread columns
            const int64_t m = m_glob;
            const int n_base = tn * kBN + col0;
            if constexpr (QOUT) {
                const int valid = p.N - n_base;            // columns of this group below N
                if (m < p.M && valid > 0) {
                    // 1. round to bf16 (the output's values) and store them if wanted
                    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.D) + m * p.ldd;
#pragma unroll
                    for (int j = 0; j < kColsPerThread / 8; ++j) {
                        const int n = n_base + 8 * j;
                        const uint32_t ww[4] = {cvt_bf16x2(acc[4 * j].x, acc[4 * j].y),
                                                cvt_bf16x2(acc[4 * j + 1].x, acc[4 * j + 1].y),
                                                cvt_bf16x2(acc[4 * j + 2].x, acc[4 * j + 2].y),
                                                cvt_bf16x2(acc[4 * j + 3].x, acc[4 * j + 3].y)};
                        if (p.D != nullptr) {
                            if (p.vec_out && n + 8 <= p.N) {
                                *reinterpret_cast<uint4*>(dst + n) = make_uint4(ww[0], ww[1], ww[2], ww[3]);
                            } else if (n < p.N) {
                                uint16_t* d16 = reinterpret_cast<uint16_t*>(dst);
                                for (int t = 0; t < min(8, p.N - n); ++t)
                                    d16[n + t] = (uint16_t)((ww[t >> 1] >> ((t & 1) * 16)) & 0xFFFFu);
                            }
                        }
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            acc[4 * j + t] = make_float2(__uint_as_float(ww[t] << 16), __uint_as_float(ww[t] & 0xFFFF0000u));
                    }
                    // 2. the group's amax over its valid columns, scale, bytes
                    float amax = 0.f;
#pragma unroll
                    for (int j = 0; j < kColsPerThread / 2; ++j) {
                        if (2 * j < valid) amax = fmaxf(amax, fabsf(acc[j].x));
                        if (2 * j + 1 < valid) amax = fmaxf(amax, fabsf(acc[j].y));
                    }
                    const float sc = scale_from_amax(amax);
                    uint8_t* qrow = p.qout + m * p.ldq_out + n_base;
#pragma unroll
                    for (int j = 0; j < kColsPerThread / 16; ++j) {
                        float f0[8], f1[8];
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            f0[2 * t] = acc[8 * j + t].x;
                            f0[2 * t + 1] = acc[8 * j + t].y;
                            f1[2 * t] = acc[8 * j + 4 + t].x;
                            f1[2 * t + 1] = acc[8 * j + 4 + t].y;
                        }
                        const uint2 lo = quant8(f0, sc), hi = quant8(f1, sc);
                        if (16 * j + 16 <= valid) {
                            *reinterpret_cast<uint4*>(qrow + 16 * j) = make_uint4(lo.x, lo.y, hi.x, hi.y);
                        } else if (16 * j < valid) {
                            const uint32_t bw[4] = {lo.x, lo.y, hi.x, hi.y};
                            for (int t = 0; t < valid - 16 * j; ++t)
                                qrow[16 * j + t] = (uint8_t)((bw[t >> 2] >> ((t & 3) * 8)) & 0xFFu);
                        }
                    }
                    p.sout[m + (int64_t)(n_base / 128) * p.lds_out] = __frcp_rn(sc);
                }
                continue;
            }
            if (m < m_end) {
                if (p.splits > 1) {
                    float* dst = p.ws + ((int64_t)split * p.M + m) * p.ldw;
#pragma unroll
                    for (int j = 0; j < kColsPerThread / 4; ++j) {
                        const int n = n_base + 4 * j;
                        if (n + 4 <= p.N) {
                            *reinterpret_cast<float4*>(dst + n) = make_float4(acc[2 * j].x, acc[2 * j].y, acc[2 * j + 1].x, acc[2 * j + 1].y);
                        } else if (n < p.N) {
                            const float v[4] = {acc[2 * j].x, acc[2 * j].y, acc[2 * j + 1].x, acc[2 * j + 1].y};
                            for (int t = 0; t < p.N - n; ++t) dst[n + t] = v[t];
                        }
                    }
                } else if (p.out_f32) {
                    float* dst = reinterpret_cast<float*>(p.D) + m * p.ldd;
#pragma unroll
                    for (int j = 0; j < kColsPerThread / 4; ++j) {
                        const int n = n_base + 4 * j;
                        if (p.vec_out && n + 4 <= p.N) {
                            *reinterpret_cast<float4*>(dst + n) = make_float4(acc[2 * j].x, acc[2 * j].y, acc[2 * j + 1].x, acc[2 * j + 1].y);
                        } else if (n < p.N) {
                            const float v[4] = {acc[2 * j].x, acc[2 * j].y, acc[2 * j + 1].x, acc[2 * j + 1].y};
                            for (int t = 0; t < min(4, p.N - n); ++t) dst[n + t] = v[t];
                        }
                    }
                } else {
                    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.D) + m * p.ldd;
#pragma unroll
                    for (int j = 0; j < kColsPerThread / 8; ++j) {
                        const int n = n_base + 8 * j;
                        const uint4 w = make_uint4(cvt_bf16x2(acc[4 * j].x, acc[4 * j].y),
                                                   cvt_bf16x2(acc[4 * j + 1].x, acc[4 * j + 1].y),
                                                   cvt_bf16x2(acc[4 * j + 2].x, acc[4 * j + 2].y),
                                                   cvt_bf16x2(acc[4 * j + 3].x, acc[4 * j + 3].y));
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
        if (!ok) give_up();
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace fp8bs
