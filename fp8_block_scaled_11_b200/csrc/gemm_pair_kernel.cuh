// gemm_pair_kernel.cuh -- FP8 (e4m3) scaled GEMM on CTA pairs (sm_100a,
// tcgen05 cta_group::2).
//
// Computes the same result as gemm_kernel.cuh,
//   D[m,n] = sum_kb rA(m,kb) * rB(n,kb) * P_kb[m,n],
//   P_kb[m,n] = sum_{k in K-block kb} qA[m,k] * qB[n,k],
// the dequantized matmul of pytorch/ao PR #4209 "[codex] add repro for
// blockwise _scaled_mm investigation" (What Changed), for the per-tensor,
// rowwise, (1x128, 128x128) and (1x128, 1x128) recipes.
//
// Why pairs.  In the block recipes every K-block's partial sums leave the
// tensor core through TMEM and are promoted in fp32 registers; the MMA of a
// later K-block can only reuse a TMEM accumulator once the promotion warps
// have drained it.  TMEM holds 512 fp32 columns per lane.  A CTA pair computes
// a 256 x 128 output tile with one cta_group::2 MMA stream: each CTA holds 128
// rows of A, 64 rows of B and its own 128 x 128 slice of the accumulator, so
// four 128-column accumulators fit (the MMA runs up to three K-blocks ahead of
// the promotion), while the operand bytes per flop stay those of a 128 x 256
// single-CTA tile.
//
// Why steps of two K-blocks, two producers and two MMA issuers.  Measured on
// B200: one thread that issues TMA loads into a ring and one that consumes it
// complete a stage about every 450 cycles plus ~90 per TMA instruction,
// however deep the ring; and one thread issuing 256x128x32 pair MMAs (64 tensor
// cycles each) falls behind the tensor core as soon as it also waits on
// barriers.  So a pipeline stage carries two K-blocks (48 KB per CTA), and the
// stages alternate between two producer threads and two MMA-issuing threads:
// each thread handles one stage per four K-blocks (1024 tensor cycles).
//
// Roles, per CTA of the cluster of two (rank 0 = leader):
//   warps 0, 3  TMA producers for the even / odd steps.  Per step: this CTA's
//               two 128 x 128 tiles of A and its two 64 x 128 halves of the B
//               tile (K-major, 128-byte swizzle; or MN-major: 256 K-rows x 64
//               columns, 64-byte swizzle) into a 4-stage ring.  Both CTAs'
//               loads complete on the leader's stage barrier, which the leader
//               arms with both CTAs' bytes.  Rowwise / 1x128 x 1x128 recipes:
//               also the scale vectors of this CTA's rows and of the tile's 128
//               columns into a local ring.
//   warp 1      TMEM allocation (both CTAs, 512 columns).
//   warps 1, 2  in the leader, lane 0 issues the pair MMAs of the even / odd
//               steps: four 256x128x32 MMAs per K-block into one of the four
//               accumulators, commits (multicast to both CTAs) each
//               accumulator and then the smem stage.
//   warps 4-11  promotion / epilogue: warp w reads TMEM lanes 32*(w%4) .. +31
//               (its rows) and 64 of the 128 columns (measured faster than 16
//               warps of 32 columns); per accumulation group
//               (a K-block for the block recipes, one issuer's share of the K
//               range for the tensor / rowwise recipes) it loads the partial
//               sums, multiplies by the scale product and adds into fp32
//               registers (packed f32x2 FMA), then releases the accumulator on
//               the leader's barrier.
// Every wait is bounded (kWaitLimitNs) exactly as in gemm_kernel.cuh: a wait
// that runs out raises the library error flag and both CTAs' abort flags, all
// roles leave their loops, MMAs and loads in flight are drained (bounded), and
// TMEM is freed by both CTAs after a cluster barrier.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "gemm_kernel.cuh"

namespace fp8bs {

constexpr int kPairM = 256;                    // output rows per pair tile
constexpr int kCtaM = 128;                     // of which each CTA computes
constexpr int kPairN = 128;                    // output columns per pair tile
constexpr int kCtaN = kPairN / 2;              // B columns held by each CTA
constexpr int kPairBufs = 4;                   // TMEM accumulators
constexpr uint32_t kPairBufCols = kTmemCols / kPairBufs;   // 128 columns each
constexpr int kStepKb = 2;                     // K-blocks per pipeline step (stage)
constexpr int kPairStages = 4;                 // A/B ring depth (steps)
constexpr int kPairScaleStages = 8;            // scale ring depth (steps, or tiles for rowwise)
constexpr uint32_t kPairATile = kCtaM * kBK;   // 16 KB per K-block
constexpr uint32_t kPairBTile = kCtaN * kBK;   // 8 KB per K-block
constexpr uint32_t kPairAStage = kStepKb * kPairATile;
constexpr uint32_t kPairBStage = kStepKb * kPairBTile;
constexpr uint32_t kPairStageTx = 2 * (kPairAStage + kPairBStage);   // both CTAs' bytes per stage
constexpr uint32_t kPairScaleKb = (kCtaM + kPairN) * 4;             // sa[128] then sb[128], per K-block
constexpr uint32_t kPairScaleEntry = kStepKb * kPairScaleKb;
constexpr int kPairEpiWarps = 8;
constexpr int kPairCtrlWarps = 4;
constexpr int kPairThreads = 32 * (kPairCtrlWarps + kPairEpiWarps);
constexpr int kPairCols = kPairN * 4 / kPairEpiWarps;     // accumulator columns per thread (64)
constexpr uint64_t kPairAbortGraceNs = 100000ull;          // abort path: time for stray loads to land

static_assert(kPairCols % 32 == 0, "pairs of 16-column TMEM loads per wait");
static_assert(kPairStages % 2 == 0 && kPairScaleStages % 2 == 0 && kPairBufs == 4,
              "stages, scale entries and accumulator pairs alternate with the step parity");

struct PairSmem {
    static constexpr uint32_t a_off = 0;
    static constexpr uint32_t b_off = a_off + kPairStages * kPairAStage;
    static constexpr uint32_t sc_off = b_off + kPairStages * kPairBStage;
    static constexpr uint32_t bar_off = sc_off + kPairScaleStages * kPairScaleEntry;
    // ab_full[S], ab_empty[S], sc_full[SS], sc_empty[SS], tm_full[4], tm_empty[4], drain
    static constexpr uint32_t n_bars = 2 * kPairStages + 2 * kPairScaleStages + 2 * kPairBufs + 1;
    static constexpr uint32_t misc_off = bar_off + n_bars * 8;    // tmem slot, abort flag
    static constexpr uint32_t total = misc_off + 16;
    static constexpr uint32_t alloc = total + 1024;               // slack to align the base to 1024 B
};
static_assert(PairSmem::b_off % 1024 == 0 && PairSmem::sc_off % 1024 == 0, "swizzled tiles 1024-byte aligned");
static_assert(PairSmem::alloc <= 232448, "shared memory per CTA");

// BMN: B is given MN-major (stored K x N, row-major) instead of as B^T (N x K).
template <int MODE, bool BMN>
__global__ void __launch_bounds__(kPairThreads, 1)
gemm_fp8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                     const GemmParams p)
{
    constexpr bool kPromote = (MODE == kModeBlock128 || MODE == kModeBlock1x128);
    // scales travel through a shared-memory ring loaded by TMA (only the
    // per-tensor recipe reads its two scalars directly): per K-block the
    // 128 row scales of this CTA and either the tile's 128 column scales
    // (1x128 x 1x128; rowwise once per tile) or the tile's one 128x128-block
    // scale, fetched as the aligned 16-byte group that holds it
    constexpr bool kScaleRing = MODE != kModeTensor;
    constexpr bool kColScales = (MODE == kModeRowwise || MODE == kModeBlock1x128);
    constexpr uint32_t kScaleTx = MODE == kModeBlock1x128 ? kPairScaleEntry
                                : MODE == kModeBlock128 ? kStepKb * (kCtaM * 4 + 16) : kPairScaleKb;
    constexpr int kChunks = kPairCols / 16;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bars = sbase + PairSmem::bar_off;
    auto ab_full = [&](int s) { return bars + 8u * s; };
    auto ab_empty = [&](int s) { return bars + 8u * (kPairStages + s); };
    auto sc_full = [&](int s) { return bars + 8u * (2 * kPairStages + s); };
    auto sc_empty = [&](int s) { return bars + 8u * (2 * kPairStages + kPairScaleStages + s); };
    auto tm_full = [&](int b) { return bars + 8u * (2 * kPairStages + 2 * kPairScaleStages + b); };
    auto tm_empty = [&](int b) { return bars + 8u * (2 * kPairStages + 2 * kPairScaleStages + kPairBufs + b); };
    const uint32_t drain_bar = bars + 8u * (2 * kPairStages + 2 * kPairScaleStages + 2 * kPairBufs);
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + PairSmem::misc_off);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PairSmem::misc_off + 4);
    const uint32_t abort_addr = sbase + PairSmem::misc_off + 4;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int64_t cluster_id = blockIdx.x >> 1;
    const int64_t num_clusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            mbar_init(ab_full(s), 1);
            mbar_init(ab_empty(s), 1);
        }
        for (int s = 0; s < kPairScaleStages; ++s) {
            mbar_init(sc_full(s), 1);
            mbar_init(sc_empty(s), kPairEpiWarps);
        }
        for (int b = 0; b < kPairBufs; ++b) {
            mbar_init(tm_full(b), 1);
            mbar_init(tm_empty(b), 2 * kPairEpiWarps);    // both CTAs' promotion warps
        }
        mbar_init(drain_bar, 2);    // one commit from each MMA issuer
        *abort_flag = 0;
        fence_barrier_init();
    }
    if ((warp == 0 || warp == 3) && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        if (kScaleRing) {
            prefetch_tensormap(&tmSA);
            prefetch_tensormap(&tmSB);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(sbase + PairSmem::misc_off, kTmemCols);
        tmem_relinquish_pair();
    }
    // barriers of both CTAs initialised (remote arrivals and the peer's loads
    // may target them from here on) and TMEM allocated in both
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // a split-K reduction launched after this kernel may start its (waiting)
    // CTAs now: it reads nothing before this grid has completed
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // A wait that gives up stops this CTA's roles and the peer's.
    auto give_up = [&]() {
        *abort_flag = 1;
        st_shared_cluster_u32(mapa_shared(abort_addr, rank ^ 1u), 1u);
        atomicOr(p.err, 1);
    };

    if (warp == 0 || warp == 3) {
        // ---------------------------------------------------------------- producers (even / odd steps)
        if (lane == 0) {
            const int t = warp == 0 ? 0 : 1;
            bool ok = true;
            // per stage / scale entry: was it ever filled by this thread, and
            // the parity of its latest fill
            uint32_t armed = 0, arm_par = 0, sfilled = 0, sfill_par = 0;
            int64_t st = 0;     // step sequence number (all units of this cluster)
            int64_t sq = 0;     // unit sequence number
            auto issue_scales = [&](int64_t idx, int m0c, int n0, int kb, int nkb_entry) -> bool {
                const int e = (int)(idx % kPairScaleStages);
                const uint32_t ph = (uint32_t)((idx / kPairScaleStages) & 1);
                if (!mbar_wait_bounded(sc_empty(e), ph ^ 1u, abort_flag, kWaitLimitNs)) return false;
                const uint32_t dst = sbase + PairSmem::sc_off + e * kPairScaleEntry;
                mbar_arrive_expect_tx(sc_full(e), kScaleTx);
                for (int i = 0; i < nkb_entry; ++i) {
                    tma_load_2d(dst + i * kPairScaleKb, &tmSA, sc_full(e), m0c, kb + i);
                    if (MODE != kModeBlock128)
                        tma_load_2d(dst + i * kPairScaleKb + kCtaM * 4, &tmSB, sc_full(e), n0, kb + i);
                    else if (BMN)   // grid (K-block, N-block): the group of 4 K-blocks holding kb + i
                        tma_load_2d(dst + i * kPairScaleKb + kCtaM * 4, &tmSB, sc_full(e), (kb + i) & ~3, n0 / kPairN);
                    else            // grid (N-block, K-block): the group of 4 N-blocks holding this tile's
                        tma_load_2d(dst + i * kPairScaleKb + kCtaM * 4, &tmSB, sc_full(e), (n0 / kPairN) & ~3, kb + i);
                }
                sfilled |= 1u << e;
                sfill_par = (sfill_par & ~(1u << e)) | (ph << e);
                return true;
            };
            for (int64_t u = cluster_id; u < p.num_units && ok; u += num_clusters, ++sq) {
                int tm, tn, kb0, kb1, split;
                decode_unit(p, u, tm, tn, kb0, kb1, split);
                const int nsteps = (kb1 - kb0 + kStepKb - 1) / kStepKb;
                const int m0c = tm * kPairM + (int)rank * kCtaM;     // this CTA's A rows
                const int n0 = tn * kPairN;
                const int nb = n0 + (int)rank * kCtaN;               // this CTA's B columns
                // rowwise: one scale entry per tile, loaded by the producer of its first step
                if (MODE == kModeRowwise && (int)(st & 1) == t) ok = issue_scales(sq, m0c, n0, 0, 1);
                for (int i = 0; i < nsteps && ok; ++i, ++st) {
                    if ((int)(st & 1) != t) continue;
                    const int stage = (int)(st % kPairStages);
                    const uint32_t phase = (uint32_t)((st / kPairStages) & 1);
                    if (!mbar_wait_bounded(ab_empty(stage), phase ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
                    if (leader) {
                        mbar_arrive_expect_tx(ab_full(stage), kPairStageTx);
                        armed |= 1u << stage;
                        arm_par = (arm_par & ~(1u << stage)) | (phase << stage);
                    }
                    // both K-blocks are always loaded (the bytes the leader
                    // expects); a second K-block past the unit's range is not
                    // multiplied, one past K reads TMA's zero fill
                    const int kb = kb0 + kStepKb * i;
                    const uint32_t full_leader = mapa_shared(ab_full(stage), 0);
                    const uint32_t a_dst = sbase + PairSmem::a_off + stage * kPairAStage;
                    const uint32_t b_dst = sbase + PairSmem::b_off + stage * kPairBStage;
#pragma unroll
                    for (int h = 0; h < kStepKb; ++h)
                        tma_load_2d_pair(a_dst + h * kPairATile, &tmA, full_leader, (kb + h) * kBK, m0c);
                    if (BMN) {
                        // K-rows kb*128 .. +255 of this CTA's 64 columns: both K-blocks
                        tma_load_2d_pair(b_dst, &tmB, full_leader, nb, kb * kBK);
                    } else {
#pragma unroll
                        for (int h = 0; h < kStepKb; ++h)
                            tma_load_2d_pair(b_dst + h * kPairBTile, &tmB, full_leader, (kb + h) * kBK, nb);
                    }
                    if (kPromote && !issue_scales(st, m0c, n0, kb, kStepKb)) { ok = false; break; }
                }
            }
            if (!ok) give_up();
            // drain: the loads this CTA issued must land before the CTA exits.
            // The leader's stage barriers count both CTAs' bytes; in a normal
            // run every armed phase was consumed by the MMA.  After an abort a
            // peer load may target a phase the leader never armed, so both
            // CTAs also give stray loads a fixed grace period.
            for (int s = 0; s < kPairStages; ++s)
                if (armed >> s & 1u) mbar_wait_bounded(ab_full(s), arm_par >> s & 1u, nullptr, kDrainLimitNs);
            for (int s = 0; s < kPairScaleStages; ++s)
                if (sfilled >> s & 1u) mbar_wait_bounded(sc_full(s), sfill_par >> s & 1u, nullptr, kDrainLimitNs);
            if (*abort_flag) {
                const uint64_t t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < kPairAbortGraceNs) {
                }
            }
        }
    } else if (warp == 1 || warp == 2) {
        // ---------------------------------------------------------------- MMA issuers (leader; even / odd steps)
        //  - block recipes: K-block slot h of step st goes to accumulator
        //    2*(st % 2) + h, committed per K-block (a slot past the unit's
        //    range is committed without MMAs so that every accumulator's
        //    phases advance in step);
        //  - tensor / rowwise: the issuer of parity t accumulates its steps of
        //    the tile into accumulator 2*(sq % 2) + t (sq = the tile's sequence
        //    number), committed once per tile; the epilogue adds the pair.
        if (leader && lane == 0) {
            constexpr uint32_t idesc = idesc_e4m3_f32_major(kPairM, kPairN, BMN ? 1u : 0u);
            const int t = warp - 1;
            int64_t st = 0, sq = 0;
            bool ok = true;
            // the four MMAs of slot h of stage `stage` into accumulator `tb`
            auto issue_kblock = [&](int stage, int h, int tb, bool first) {
                const uint32_t a_addr = sbase + PairSmem::a_off + stage * kPairAStage + h * kPairATile;
                const uint32_t b_addr = sbase + PairSmem::b_off + stage * kPairBStage + h * kPairBTile;
                const uint32_t d_tmem = tmem_base + (uint32_t)tb * kPairBufCols;
#pragma unroll
                for (int k = 0; k < kBK / 32; ++k) {
                    const uint64_t adesc = smem_desc_k_sw128(a_addr + k * 32);
                    // K-major: the k-th 32-byte slice of each 128-byte row;
                    // MN-major: K-rows 32k .. 32k+31 (four 512-byte groups)
                    const uint64_t bdesc = BMN ? smem_desc_mn_sw64(b_addr + k * 2048)
                                               : smem_desc_k_sw128(b_addr + k * 32);
                    umma_f8_pair(d_tmem, adesc, bdesc, idesc, (first && k == 0) ? 0u : 1u);
                }
            };
            for (int64_t u = cluster_id; u < p.num_units && ok; u += num_clusters, ++sq) {
                int tm, tn, kb0, kb1, split;
                decode_unit(p, u, tm, tn, kb0, kb1, split);
                const int nsteps = (kb1 - kb0 + kStepKb - 1) / kStepKb;
                const int tbt = (int)(2 * (sq & 1) + t);              // tensor / rowwise accumulator
                const uint32_t tphase_t = (uint32_t)((sq >> 1) & 1);
                bool first = true;
                for (int i = 0; i < nsteps && ok; ++i, ++st) {
                    if ((int)(st & 1) != t) continue;
                    const int stage = (int)(st % kPairStages);
                    if (!mbar_wait_bounded(ab_full(stage), (uint32_t)((st / kPairStages) & 1), abort_flag, kWaitLimitNs)) { ok = false; break; }
                    tc_fence_after();
                    const int kb = kb0 + kStepKb * i;
#pragma unroll
                    for (int h = 0; h < kStepKb; ++h) {
                        const bool valid = kb + h < kb1;
                        if (kPromote) {
                            const int tb = (int)(2 * (st & 1) + h);
                            if (!mbar_wait_bounded(tm_empty(tb), (uint32_t)(((st >> 1) & 1) ^ 1), abort_flag, kWaitLimitNs)) { ok = false; break; }
                            tc_fence_after();
                            if (valid) issue_kblock(stage, h, tb, true);
                            umma_commit_pair_mc(tm_full(tb), 0x3);
                        } else if (valid) {
                            if (first) {
                                if (!mbar_wait_bounded(tm_empty(tbt), tphase_t ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
                                tc_fence_after();
                            }
                            issue_kblock(stage, h, tbt, first);
                            first = false;
                        }
                    }
                    if (!ok) break;
                    umma_commit_pair_mc(ab_empty(stage), 0x3);
                }
                if (!ok) break;
                if (!kPromote) {
                    // a tile whose steps all went to the other issuer leaves
                    // this accumulator unwritten; the epilogue then does not
                    // read it, but its barrier phases still advance
                    if (first && !mbar_wait_bounded(tm_empty(tbt), tphase_t ^ 1u, abort_flag, kWaitLimitNs)) { ok = false; break; }
                    umma_commit_pair_mc(tm_full(tbt), 0x3);
                }
            }
            if (!ok) give_up();
            // every MMA of both issuers has completed (both CTAs' TMEM written,
            // both CTAs' shared memory read) before the cluster may tear down
            umma_commit_pair_mc(drain_bar, 0x1);
            if (t == 0) mbar_wait_bounded(drain_bar, 0, nullptr, kDrainLimitNs);
        }
    } else if (warp >= kPairCtrlWarps) {
        // ---------------------------------------------------------------- promotion / epilogue
        const int e = warp - kPairCtrlWarps;        // 0 .. 7
        const int lq = warp & 3;                    // TMEM lane quarter this warp may access
        const int col0 = (e >> 2) * kPairCols;      // this warp's columns within the tile
        const int row_in_tile = lq * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(lq * 32) << 16;
        int64_t st = 0, sq = 0;
        bool ok = true;
        float tensor_scale = 1.0f;
        if (MODE == kModeTensor) tensor_scale = __ldg(p.sa) * __ldg(p.sb);

        for (int64_t u = cluster_id; u < p.num_units && ok; u += num_clusters, ++sq) {
            int tm, tn, kb0, kb1, split;
            decode_unit(p, u, tm, tn, kb0, kb1, split);
            const int nsteps = (kb1 - kb0 + kStepKb - 1) / kStepKb;
            const int64_t st_first = st;
            float2 acc[kPairCols / 2];
#pragma unroll
            for (int i = 0; i < kPairCols / 2; ++i) acc[i] = make_float2(0.f, 0.f);

            const int64_t m_glob = (int64_t)tm * kPairM + (int64_t)rank * kCtaM + row_in_tile;

            // the warp-collective wait::ld of the promotion leaves all lanes'
            // loads complete: lane 0 releases the accumulator on the leader's barrier
            auto release = [&](int tb) {
                tc_fence_before();
                if (lane == 0) {
                    if (leader) mbar_arrive(tm_empty(tb));
                    else mbar_arrive_remote(mapa_shared(tm_empty(tb), 0));
                }
            };
            // accumulate the partial sums of accumulator tb (TMEM phase tph),
            // scaled by rowf (and per column by the scale entry at sc_addr)
            auto promote_buffer = [&](int tb, uint32_t tph, bool read, float rowf, uint32_t sc_addr) {
                if (!mbar_wait_bounded(tm_full(tb), tph, abort_flag, kWaitLimitNs)) { ok = false; give_up(); }
                tc_fence_after();
                if (read) {
                    const float2 rowf2 = make_float2(rowf, rowf);
                    const uint32_t tcol = tmem_base + lane_addr + (uint32_t)tb * kPairBufCols + (uint32_t)col0;
                    auto promote = [&](int c, const uint32_t (&r)[16]) {
                        if (kColScales) {
                            const uint32_t sb_addr = sc_addr + (uint32_t)((kCtaM + col0 + c * 16) * 4);
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj) {
                                const float4 b4 = lds128(sb_addr + 16 * jj);
                                const float2 f0 = fmul2(rowf2, make_float2(b4.x, b4.y));
                                const float2 f1 = fmul2(rowf2, make_float2(b4.z, b4.w));
                                acc[c * 8 + 2 * jj] = ffma2(make_float2(__uint_as_float(r[4 * jj]), __uint_as_float(r[4 * jj + 1])), f0, acc[c * 8 + 2 * jj]);
                                acc[c * 8 + 2 * jj + 1] = ffma2(make_float2(__uint_as_float(r[4 * jj + 2]), __uint_as_float(r[4 * jj + 3])), f1, acc[c * 8 + 2 * jj + 1]);
                            }
                        } else {
#pragma unroll
                            for (int jj = 0; jj < 8; ++jj)
                                acc[c * 8 + jj] = ffma2(make_float2(__uint_as_float(r[2 * jj]), __uint_as_float(r[2 * jj + 1])), rowf2, acc[c * 8 + jj]);
                        }
                    };
#pragma unroll
                    for (int h = 0; h < kChunks / 2; ++h) {
                        uint32_t r0[16], r1[16];
                        tmem_ld_32x32b_x16(tcol + (2 * h + 0) * 16, r0);
                        tmem_ld_32x32b_x16(tcol + (2 * h + 1) * 16, r1);
                        tmem_ld_wait(r0);
                        reg_after_wait(r1);
                        promote(2 * h + 0, r0);
                        promote(2 * h + 1, r1);
                    }
                }
                release(tb);
            };

            if (kPromote) {
                for (int i = 0; i < nsteps; ++i, ++st) {
                    const int e_sc = (int)(st % kPairScaleStages);
                    if (!mbar_wait_bounded(sc_full(e_sc), (uint32_t)((st / kPairScaleStages) & 1), abort_flag, kWaitLimitNs)) { ok = false; give_up(); }
                    const uint32_t sc_base = sbase + PairSmem::sc_off + e_sc * kPairScaleEntry;
#pragma unroll
                    for (int h = 0; h < kStepKb; ++h) {
                        const int kb = kb0 + kStepKb * i + h;
                        const bool valid = kb < kb1;
                        const uint32_t sc_addr = sc_base + h * kPairScaleKb;
                        const float* sc = reinterpret_cast<const float*>(smem + (sc_addr - sbase));
                        float rowf = sc[row_in_tile];
                        if (MODE == kModeBlock128) rowf *= sc[kCtaM + (BMN ? (kb & 3) : (tn & 3))];
                        promote_buffer((int)(2 * (st & 1) + h), (uint32_t)((st >> 1) & 1), valid, rowf, sc_addr);
                    }
                    if (lane == 0) mbar_arrive(sc_empty(e_sc));
                }
            } else {
                // the two issuers' accumulators of this tile; the one of parity
                // q holds data when one of the tile's steps had parity q
                float rowf = tensor_scale;
                uint32_t sc_addr = 0;
                int e_sc = 0;
                if (MODE == kModeRowwise) {
                    e_sc = (int)(sq % kPairScaleStages);
                    if (!mbar_wait_bounded(sc_full(e_sc), (uint32_t)((sq / kPairScaleStages) & 1), abort_flag, kWaitLimitNs)) { ok = false; give_up(); }
                    sc_addr = sbase + PairSmem::sc_off + e_sc * kPairScaleEntry;
                    rowf = reinterpret_cast<const float*>(smem + (sc_addr - sbase))[row_in_tile];
                }
                for (int q = 0; q < 2; ++q) {
                    const bool has = nsteps >= 2 || (int)(st_first & 1) == q;
                    promote_buffer((int)(2 * (sq & 1) + q), (uint32_t)((sq >> 1) & 1), has, rowf, sc_addr);
                }
                if (MODE == kModeRowwise && lane == 0) mbar_arrive(sc_empty(e_sc));
                st += nsteps;
            }
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;

            // ---- store the tile: row m, this thread's kPairCols columns
            const int64_t m = m_glob;
            const int n_base = tn * kPairN + col0;
            if (m < p.M) {
                if (p.splits > 1) {
                    float* dst = p.ws + ((int64_t)split * p.M + m) * p.ldw;
#pragma unroll
                    for (int j = 0; j < kPairCols / 4; ++j) {
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
                    for (int j = 0; j < kPairCols / 4; ++j) {
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
                    for (int j = 0; j < kPairCols / 8; ++j) {
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

    // Teardown: the leader's MMAs have completed (its MMA thread waited on the
    // drain barrier) before either CTA passes this barrier, so both CTAs' TMEM
    // and shared memory are no longer in use by the pair.
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

}  // namespace fp8bs
