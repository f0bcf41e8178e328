// fp8bs_lib.cu -- the C ABI declared in include/fp8bs.h: argument validation,
// TMA tensor-map encoding, launch configuration, and the device error flag.
// The kernels are in quant_kernels.cuh and gemm_kernel.cuh (one translation
// unit, so the error flag is a plain __device__ variable).  The GEMM runs on
// single CTAs (gemm_kernel.cuh) or CTA pairs (gemm_pair_kernel.cuh), the
// power-of-two block recipes on the block-scaled MMA kernel (gemm_bs_kernel.cuh).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fp8bs.h"
#include "quant_kernels.cuh"
#include "gemm_kernel.cuh"
#include "gemm_pair_kernel.cuh"
#include "gemm_bs_kernel.cuh"
#include "splitk_reduce.cuh"

using namespace fp8bs;

namespace {

__device__ int g_device_error;

constexpr int kMaxDevices = 64;

// Per-device state, filled on first use.  Calls may come from several host
// threads: the flags are atomics (release on set, acquire on test) and every
// first-time set-up runs under g_mutex.
struct DeviceInfo {
    std::atomic<bool> ready{false};
    bool sm100 = false;
    int num_sms = 0;
    int* err_ptr = nullptr;
    std::atomic<bool> gemm_attr_set[20]{};   // per instantiation: plain, fused output quantization, grouped,
                                             // block-scaled, MN-major B
    std::atomic<int> quant_blocks[12]{};     // resident CTAs per SM, per quant kernel kind
    std::atomic<bool> tile_attr_set[16]{};   // per tile kernel kind (+8: power-of-two scale rule)
    std::atomic<int> tile_blocks[16]{};
    std::atomic<int> pair_clusters[8]{};     // co-resident CTA pairs, per pair-kernel instantiation
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_mutex;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

fp8bs_status get_device(DeviceInfo** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8BS_ERR_CUDA;
    DeviceInfo& d = g_dev[dev];
    if (!d.ready.load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!d.ready.load(std::memory_order_relaxed)) {
            int major = 0;
            if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return FP8BS_ERR_CUDA;
            d.sm100 = (major == 10);
            if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return FP8BS_ERR_CUDA;
            if (d.sm100) {
                void* p = nullptr;
                if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return FP8BS_ERR_CUDA;
                d.err_ptr = static_cast<int*>(p);
            }
            if (g_encode == nullptr) {
                void* fn = nullptr;
                cudaDriverEntryPointQueryResult q;
                if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                    q != cudaDriverEntryPointSuccess || fn == nullptr)
                    return FP8BS_ERR_CUDA;
                g_encode = reinterpret_cast<EncodeTiledFn>(fn);
            }
            d.ready.store(true, std::memory_order_release);
        }
    }
    if (!d.sm100) return FP8BS_ERR_NO_SM100;
    *out = &d;
    return FP8BS_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t dtype_size(fp8bs_dtype t) { return t == FP8BS_F32 ? 4 : 2; }
inline bool valid_dtype(fp8bs_dtype t) { return t == FP8BS_BF16 || t == FP8BS_F32; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

fp8bs_status launch_status()
{
    return cudaGetLastError() == cudaSuccess ? FP8BS_OK : FP8BS_ERR_CUDA;
}

// Persistent grid: resident CTAs per SM (occupancy calculator) x SMs, capped by the work.
template <typename Kernel>
int persistent_grid(DeviceInfo* d, int kind, Kernel k, int64_t work_ctas)
{
    int nb = d->quant_blocks[kind].load(std::memory_order_acquire);
    if (nb == 0) {
        // racing first calls compute the same value
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k, 256, 0) != cudaSuccess || nb < 1) nb = 1;
        d->quant_blocks[kind].store(nb, std::memory_order_release);
    }
    const int64_t cap = (int64_t)nb * d->num_sms;
    return (int)std::max<int64_t>(1, std::min<int64_t>(cap, work_ctas));
}

// Persistent launch of a TMA-pipelined tile kernel: resident CTAs per SM (for
// its dynamic shared memory) x SMs, capped by the number of tiles.
template <typename Kernel, typename... Args>
fp8bs_status launch_tile_kernel(DeviceInfo* d, int kind, Kernel k, uint32_t smem, int64_t tiles, cudaStream_t stream,
                                Args... args)
{
    if (!d->tile_attr_set[kind].load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!d->tile_attr_set[kind].load(std::memory_order_relaxed)) {
            if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
                return FP8BS_ERR_CUDA;
            int nb = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k, 256, smem) != cudaSuccess || nb < 1) nb = 1;
            d->tile_blocks[kind].store(nb, std::memory_order_relaxed);
            d->tile_attr_set[kind].store(true, std::memory_order_release);
        }
    }
    const int64_t per_sm = d->tile_blocks[kind].load(std::memory_order_relaxed);
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(tiles, per_sm * d->num_sms));
    k<<<grid, 256, smem, stream>>>(args...);
    return launch_status();
}

// 2-D tensor map over a row-major matrix: inner dim `inner` elements, `outer`
// rows, row pitch `pitch_bytes`, box {box_inner, box_outer}.
fp8bs_status make_map(CUtensorMap* m, CUtensorMapDataType dt, size_t esize, const void* base, uint64_t inner,
                      uint64_t outer, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
                      CUtensorMapSwizzle swz)
{
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {pitch_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    (void)esize;
    CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FP8BS_OK : FP8BS_ERR_CUDA;
}

struct SplitPlan {
    int tiles_m, tiles_n, splits;
    int64_t ldw;
    size_t ws_bytes;
};

SplitPlan plan_gemm(int64_t M, int64_t N, int64_t K, int num_sms)
{
    SplitPlan s;
    s.tiles_m = (int)cdiv(M, kBM);
    s.tiles_n = (int)cdiv(N, kBN);
    const int64_t tiles = (int64_t)s.tiles_m * s.tiles_n;
    const int64_t Kb = cdiv(K, kBK);
    int splits = 1;
    if (tiles * 2 <= num_sms) {
        // fill the SMs, but keep >= 8 K-blocks per split: with fewer, the
        // pipeline fill and the reduction's extra launch outweigh the split
        splits = (int)std::min<int64_t>(num_sms / tiles, std::max<int64_t>(1, Kb / 8));
        splits = std::max(1, std::min(splits, 64));
    }
    s.splits = splits;
    s.ldw = (N + 3) & ~int64_t(3);
    s.ws_bytes = splits > 1 ? (size_t)splits * (size_t)M * (size_t)s.ldw * sizeof(float) : 0;
    return s;
}

// Pair kernel: 256 x 128 output tiles; split-K when the tiles cannot keep half
// the CTA pairs busy (same rule as plan_gemm, over pairs instead of SMs).
SplitPlan plan_pair(int64_t M, int64_t N, int64_t K, int num_sms)
{
    SplitPlan s;
    s.tiles_m = (int)cdiv(M, kPairM);
    s.tiles_n = (int)cdiv(N, kPairN);
    const int64_t tiles = (int64_t)s.tiles_m * s.tiles_n;
    const int64_t Kb = cdiv(K, kBK);
    const int pairs = std::max(1, num_sms / 2);
    int splits = 1;
    if (tiles * 2 <= pairs) {
        splits = (int)std::min<int64_t>(pairs / tiles, std::max<int64_t>(1, Kb / 8));
        splits = std::max(1, std::min(splits, 64));
    }
    s.splits = splits;
    s.ldw = (N + 3) & ~int64_t(3);
    s.ws_bytes = splits > 1 ? (size_t)splits * (size_t)M * (size_t)s.ldw * sizeof(float) : 0;
    return s;
}

// Which GEMM kernel a call runs: the CTA-pair kernel for outputs too small to
// fill the GPU without splitting K (fewer, wider splits: the long-K case), the
// single-CTA kernel otherwise (faster on large outputs, where its two 256-column
// accumulators are fed by a single TMA ring; K-major or MN-major B) and for the
// fused output quantization.
bool use_pair(int64_t M, int64_t N, int64_t K, bool b_mn, bool quant_out, int num_sms)
{
    (void)b_mn;
    if (quant_out) return false;
    return plan_pair(M, N, K, num_sms).splits > 1;
}

int num_sms_current()
{
    DeviceInfo* d = nullptr;
    if (get_device(&d) != FP8BS_OK) return 148;
    return d->num_sms;
}

template <int MODE, bool QOUT = false, bool GROUPED = false, bool BMN = false>
fp8bs_status launch_gemm(DeviceInfo* d, const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tSA,
                         const CUtensorMap& tSB,
                         const std::conditional_t<QOUT, GemmParamsQ, std::conditional_t<GROUPED, GemmParamsG, GemmParams>>& p,
                         cudaStream_t stream)
{
    auto k = gemm_fp8_kernel<MODE, QOUT, GROUPED, BMN>;
    constexpr int slot = BMN ? 14 + MODE : MODE + (QOUT ? 4 : 0) + (GROUPED ? 8 : 0);
    if (!d->gemm_attr_set[slot].load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!d->gemm_attr_set[slot].load(std::memory_order_relaxed)) {
            if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SmemLayout::alloc) !=
                cudaSuccess)
                return FP8BS_ERR_CUDA;
            if (EpiCfg<MODE>::reg_split) {
                // the warpgroups' register hand-over is sized for this exact
                // allocation at launch; with fewer registers the promotion warps'
                // increase could never be granted, so refuse to launch instead
                cudaFuncAttributes fa;
                if (cudaFuncGetAttributes(&fa, k) != cudaSuccess) return FP8BS_ERR_CUDA;
                if (fa.numRegs != EpiCfg<MODE>::launch_regs) return FP8BS_ERR_UNSUPPORTED;
            }
            d->gemm_attr_set[slot].store(true, std::memory_order_release);
        }
    }
    const int grid = (int)std::min<int64_t>(p.num_units, d->num_sms);
    k<<<grid, EpiCfg<MODE>::threads, SmemLayout::alloc, stream>>>(tA, tB, tSA, tSB, p);
    return launch_status();
}

// Launch of the pair kernel: clusters of two CTAs, one pair per two SMs (as
// many as can be co-resident), persistent over the units.
template <int MODE, bool BMN>
fp8bs_status launch_pair(DeviceInfo* d, const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tSA,
                         const CUtensorMap& tSB, const GemmParams& p, cudaStream_t stream)
{
    auto k = gemm_fp8_pair_kernel<MODE, BMN>;
    constexpr int slot = MODE + (BMN ? 4 : 0);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = PairSmem::alloc;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nc = d->pair_clusters[slot].load(std::memory_order_acquire);
    if (nc == 0) {
        std::lock_guard<std::mutex> lock(g_mutex);
        nc = d->pair_clusters[slot].load(std::memory_order_relaxed);
        if (nc == 0) {
            if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PairSmem::alloc) !=
                cudaSuccess)
                return FP8BS_ERR_CUDA;
            cfg.gridDim = dim3(2 * std::max(1, d->num_sms / 2), 1, 1);
            if (cudaOccupancyMaxActiveClusters(&nc, k, &cfg) != cudaSuccess) return FP8BS_ERR_CUDA;
            if (nc < 1) return FP8BS_ERR_UNSUPPORTED;
            d->pair_clusters[slot].store(nc, std::memory_order_release);
        }
    }
    const int64_t clusters = std::min<int64_t>(p.num_units, nc);
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
    if (cudaLaunchKernelEx(&cfg, k, tA, tB, tSA, tSB, p) != cudaSuccess) return FP8BS_ERR_CUDA;
    return launch_status();
}

// Launch of the block-scaled MMA kernel (power-of-two recipes): one persistent
// CTA per SM.
template <int MODE>
fp8bs_status launch_bs(DeviceInfo* d, const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tSA,
                       const CUtensorMap& tSB, const GemmParams& p, cudaStream_t stream)
{
    auto k = gemm_fp8_bs_kernel<MODE>;
    const int slot = 12 + (MODE == kModeBlock1x128 ? 1 : 0);
    if (!d->gemm_attr_set[slot].load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!d->gemm_attr_set[slot].load(std::memory_order_relaxed)) {
            if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BsSmem::alloc) !=
                cudaSuccess)
                return FP8BS_ERR_CUDA;
            d->gemm_attr_set[slot].store(true, std::memory_order_release);
        }
    }
    const int grid = (int)std::min<int64_t>(p.num_units, d->num_sms);
    k<<<grid, kBsThreads, BsSmem::alloc, stream>>>(tA, tB, tSA, tSB, p);
    return launch_status();
}

// ---------------------------------------------------------------- quantization
// The group-quantization entry points, over the scale rule (POW2: the
// power-of-two rule; the kernels are otherwise the same instantiations).

template <bool POW2>
fp8bs_status quant_1x128_impl(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx, uint8_t* q,
                             int64_t ldq, float* scale_inv, int64_t ld_scale, int transpose_out, cudaStream_t stream)
{
    if (!valid_dtype(xt)) return FP8BS_ERR_UNSUPPORTED;
    if (x == nullptr || q == nullptr || scale_inv == nullptr || rows < 1 || cols < 1) return FP8BS_ERR_INVALID_ARG;
    if (transpose_out != 0 && transpose_out != 1) return FP8BS_ERR_INVALID_ARG;
    if (ldx < cols) return FP8BS_ERR_INVALID_ARG;
    const int64_t out_rows = transpose_out ? cols : rows;
    const int64_t out_cols = transpose_out ? rows : cols;
    if (ldq < out_cols || ld_scale < out_rows) return FP8BS_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(q) || !aligned16(scale_inv)) return FP8BS_ERR_ALIGNMENT;
    if ((ldx * (int64_t)dtype_size(xt)) % 16 || ldq % 16 || ld_scale % 4 || cols % 16) return FP8BS_ERR_ALIGNMENT;
    if (transpose_out && rows % 16) return FP8BS_ERR_ALIGNMENT;
    DeviceInfo* d = nullptr;
    fp8bs_status st = get_device(&d);
    if (st != FP8BS_OK) return st;

    if (!transpose_out && rows % 16 == 0) {
        // whole 16-row blocks: the TMA tile pipeline (higher HBM throughput)
        const int64_t ctas = cdiv(rows, 128) * cdiv(cols, 128);
        CUtensorMap map;
        if (xt == FP8BS_BF16) {
            if ((st = make_map(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, cols, rows, ldx * 2, 128, 128,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK)
                return st;
            st = launch_tile_kernel(d, 6 + (POW2 ? 8 : 0), quant_1x128_rowtile_kernel<__nv_bfloat16, POW2>, QTile<__nv_bfloat16>::smem, ctas,
                                    stream, map, rows, cols, q, ldq, scale_inv, ld_scale, d->err_ptr);
        } else {
            if ((st = make_map(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, x, cols, rows, ldx * 4, 128, 128,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK)
                return st;
            st = launch_tile_kernel(d, 7 + (POW2 ? 8 : 0), quant_1x128_rowtile_kernel<float, POW2>, QTile<float>::smem, ctas, stream, map,
                                    rows, cols, q, ldq, scale_inv, ld_scale, d->err_ptr);
        }
        if (st != FP8BS_OK) return st;
    } else if (!transpose_out) {
        const int64_t items = cdiv(rows, 32) * cdiv(cols, 128);
        const int64_t ctas = cdiv(items, 8);
        if (xt == FP8BS_BF16) {
            auto k = quant_1x128_rows_kernel<__nv_bfloat16, POW2>;
            int g = persistent_grid(d, 0 + (POW2 ? 10 : 0), k, ctas);
            k<<<g, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), rows, cols, ldx, q, ldq, scale_inv, ld_scale);
        } else {
            auto k = quant_1x128_rows_kernel<float, POW2>;
            int g = persistent_grid(d, 1 + (POW2 ? 10 : 0), k, ctas);
            k<<<g, 256, 0, stream>>>(static_cast<const float*>(x), rows, cols, ldx, q, ldq, scale_inv, ld_scale);
        }
    } else {
        const int64_t ctas = cdiv(rows, 128) * cdiv(cols, 128);
        CUtensorMap map;
        if (xt == FP8BS_BF16) {
            if ((st = make_map(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, cols, rows, ldx * 2, 128, 128,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK)
                return st;
            st = launch_tile_kernel(d, 0 + (POW2 ? 8 : 0), quant_1x128_cols_kernel<__nv_bfloat16, POW2>, QTile<__nv_bfloat16>::smem, ctas,
                                    stream, map, rows, cols, q, ldq, scale_inv, ld_scale, d->err_ptr);
        } else {
            if ((st = make_map(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, x, cols, rows, ldx * 4, 128, 128,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK)
                return st;
            st = launch_tile_kernel(d, 1 + (POW2 ? 8 : 0), quant_1x128_cols_kernel<float, POW2>, QTile<float>::smem, ctas, stream, map, rows,
                                    cols, q, ldq, scale_inv, ld_scale, d->err_ptr);
        }
        if (st != FP8BS_OK) return st;
    }
    return launch_status();
}

template <bool POW2>
fp8bs_status quant_1x128_dual_impl(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx,
                                  uint8_t* q, int64_t ldq, float* scale_inv, int64_t ld_scale, uint8_t* q_t,
                                  int64_t ldq_t, float* scale_inv_t, int64_t ld_scale_t, cudaStream_t stream)
{
    if (!valid_dtype(xt)) return FP8BS_ERR_UNSUPPORTED;
    if (x == nullptr || q == nullptr || scale_inv == nullptr || q_t == nullptr || scale_inv_t == nullptr ||
        rows < 1 || cols < 1)
        return FP8BS_ERR_INVALID_ARG;
    if (ldx < cols || ldq < cols || ld_scale < rows || ldq_t < rows || ld_scale_t < cols) return FP8BS_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(q) || !aligned16(scale_inv) || !aligned16(q_t) || !aligned16(scale_inv_t))
        return FP8BS_ERR_ALIGNMENT;
    if ((ldx * (int64_t)dtype_size(xt)) % 16 || ldq % 16 || ldq_t % 16 || ld_scale % 4 || ld_scale_t % 4 ||
        rows % 16 || cols % 16)
        return FP8BS_ERR_ALIGNMENT;
    DeviceInfo* d = nullptr;
    fp8bs_status st = get_device(&d);
    if (st != FP8BS_OK) return st;
    const int64_t ctas = cdiv(rows, 128) * cdiv(cols, 128);
    CUtensorMap map;
    if (xt == FP8BS_BF16) {
        if ((st = make_map(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, cols, rows, ldx * 2, 128, 128,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK)
            return st;
        st = launch_tile_kernel(d, 4 + (POW2 ? 8 : 0), quant_1x128_dual_kernel<__nv_bfloat16, POW2>, QTile<__nv_bfloat16>::smem, ctas, stream,
                                map, rows, cols, q, ldq, scale_inv, ld_scale, q_t, ldq_t, scale_inv_t, ld_scale_t,
                                d->err_ptr);
    } else {
        if ((st = make_map(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, x, cols, rows, ldx * 4, 128, 128,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK)
            return st;
        st = launch_tile_kernel(d, 5 + (POW2 ? 8 : 0), quant_1x128_dual_kernel<float, POW2>, QTile<float>::smem, ctas, stream, map, rows,
                                cols, q, ldq, scale_inv, ld_scale, q_t, ldq_t, scale_inv_t, ld_scale_t, d->err_ptr);
    }
    return st;
}

template <bool POW2>
fp8bs_status quant_128x128_impl(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx, uint8_t* q,
                               int64_t ldq, float* scale_inv, int64_t ld_scale, uint8_t* q_t, int64_t ldq_t,
                               float* scale_inv_t, int64_t ld_scale_t, cudaStream_t stream)
{
    if (!valid_dtype(xt)) return FP8BS_ERR_UNSUPPORTED;
    if (x == nullptr || rows < 1 || cols < 1 || (q == nullptr && q_t == nullptr)) return FP8BS_ERR_INVALID_ARG;
    if (ldx < cols) return FP8BS_ERR_INVALID_ARG;
    const int64_t rb = cdiv(rows, 128), cb = cdiv(cols, 128);
    if (q != nullptr) {
        if (scale_inv == nullptr || ldq < cols || ld_scale < rb) return FP8BS_ERR_INVALID_ARG;
        if (!aligned16(q) || !aligned16(scale_inv) || ldq % 16 || ld_scale % 4) return FP8BS_ERR_ALIGNMENT;
    }
    if (q_t != nullptr) {
        if (scale_inv_t == nullptr || ldq_t < rows || ld_scale_t < cb) return FP8BS_ERR_INVALID_ARG;
        if (!aligned16(q_t) || !aligned16(scale_inv_t) || ldq_t % 16 || ld_scale_t % 4) return FP8BS_ERR_ALIGNMENT;
    }
    if (!aligned16(x) || (ldx * (int64_t)dtype_size(xt)) % 16 || rows % 16 || cols % 16) return FP8BS_ERR_ALIGNMENT;
    DeviceInfo* d = nullptr;
    fp8bs_status st = get_device(&d);
    if (st != FP8BS_OK) return st;
    const int64_t ctas = rb * cb;
    CUtensorMap map;
    if (xt == FP8BS_BF16) {
        if ((st = make_map(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, cols, rows, ldx * 2, 128, 128,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK)
            return st;
        st = launch_tile_kernel(d, 2 + (POW2 ? 8 : 0), quant_128x128_kernel<__nv_bfloat16, POW2>, QTile<__nv_bfloat16>::smem, ctas, stream,
                                map, rows, cols, q, ldq, scale_inv, ld_scale, q_t, ldq_t, scale_inv_t, ld_scale_t,
                                d->err_ptr);
    } else {
        if ((st = make_map(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, x, cols, rows, ldx * 4, 128, 128,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK)
            return st;
        st = launch_tile_kernel(d, 3 + (POW2 ? 8 : 0), quant_128x128_kernel<float, POW2>, QTile<float>::smem, ctas, stream, map, rows, cols,
                                q, ldq, scale_inv, ld_scale, q_t, ldq_t, scale_inv_t, ld_scale_t, d->err_ptr);
    }
    return st;
}

}  // namespace

extern "C" {

const char* fp8bs_status_string(fp8bs_status s)
{
    switch (s) {
    case FP8BS_OK: return "FP8BS_OK";
    case FP8BS_ERR_INVALID_ARG: return "FP8BS_ERR_INVALID_ARG";
    case FP8BS_ERR_UNSUPPORTED: return "FP8BS_ERR_UNSUPPORTED";
    case FP8BS_ERR_ALIGNMENT: return "FP8BS_ERR_ALIGNMENT";
    case FP8BS_ERR_WORKSPACE: return "FP8BS_ERR_WORKSPACE";
    case FP8BS_ERR_CUDA: return "FP8BS_ERR_CUDA";
    case FP8BS_ERR_TIMEOUT: return "FP8BS_ERR_TIMEOUT";
    case FP8BS_ERR_NO_SM100: return "FP8BS_ERR_NO_SM100";
    case FP8BS_ERR_SCALE: return "FP8BS_ERR_SCALE";
    }
    return "FP8BS_UNKNOWN_STATUS";
}

fp8bs_status fp8bs_check_device_error(cudaStream_t stream)
{
    DeviceInfo* d = nullptr;
    fp8bs_status st = get_device(&d);
    if (st != FP8BS_OK) return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return FP8BS_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return FP8BS_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return FP8BS_ERR_CUDA;
        // bit 0: a bounded wait ran out; bit 1: a power-of-two recipe met another scale
        return (v & 1) || !(v & 2) ? FP8BS_ERR_TIMEOUT : FP8BS_ERR_SCALE;
    }
    return FP8BS_OK;
}

// ---------------------------------------------------------------- quantization

fp8bs_status fp8_quant_1x128(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx, uint8_t* q,
                             int64_t ldq, float* scale_inv, int64_t ld_scale, int transpose_out, cudaStream_t stream)
{
    return quant_1x128_impl<false>(x, xt, rows, cols, ldx, q, ldq, scale_inv, ld_scale, transpose_out, stream);
}

fp8bs_status fp8_quant_1x128_ex(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx, uint8_t* q,
                                int64_t ldq, float* scale_inv, int64_t ld_scale, int transpose_out,
                                fp8bs_scale_rule rule, cudaStream_t stream)
{
    switch (rule) {
    case FP8BS_SCALE_RULE_FP32:
        return quant_1x128_impl<false>(x, xt, rows, cols, ldx, q, ldq, scale_inv, ld_scale, transpose_out, stream);
    case FP8BS_SCALE_RULE_POW2:
        return quant_1x128_impl<true>(x, xt, rows, cols, ldx, q, ldq, scale_inv, ld_scale, transpose_out, stream);
    }
    return FP8BS_ERR_UNSUPPORTED;
}

fp8bs_status fp8_quant_1x128_dual(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx,
                                  uint8_t* q, int64_t ldq, float* scale_inv, int64_t ld_scale, uint8_t* q_t,
                                  int64_t ldq_t, float* scale_inv_t, int64_t ld_scale_t, cudaStream_t stream)
{
    return quant_1x128_dual_impl<false>(x, xt, rows, cols, ldx, q, ldq, scale_inv, ld_scale, q_t, ldq_t,
                                        scale_inv_t, ld_scale_t, stream);
}

fp8bs_status fp8_quant_1x128_dual_ex(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx,
                                     uint8_t* q, int64_t ldq, float* scale_inv, int64_t ld_scale, uint8_t* q_t,
                                     int64_t ldq_t, float* scale_inv_t, int64_t ld_scale_t, fp8bs_scale_rule rule,
                                     cudaStream_t stream)
{
    switch (rule) {
    case FP8BS_SCALE_RULE_FP32:
        return quant_1x128_dual_impl<false>(x, xt, rows, cols, ldx, q, ldq, scale_inv, ld_scale, q_t, ldq_t,
                                            scale_inv_t, ld_scale_t, stream);
    case FP8BS_SCALE_RULE_POW2:
        return quant_1x128_dual_impl<true>(x, xt, rows, cols, ldx, q, ldq, scale_inv, ld_scale, q_t, ldq_t,
                                           scale_inv_t, ld_scale_t, stream);
    }
    return FP8BS_ERR_UNSUPPORTED;
}

fp8bs_status fp8_quant_128x128(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx, uint8_t* q,
                               int64_t ldq, float* scale_inv, int64_t ld_scale, uint8_t* q_t, int64_t ldq_t,
                               float* scale_inv_t, int64_t ld_scale_t, cudaStream_t stream)
{
    return quant_128x128_impl<false>(x, xt, rows, cols, ldx, q, ldq, scale_inv, ld_scale, q_t, ldq_t, scale_inv_t,
                                     ld_scale_t, stream);
}

fp8bs_status fp8_quant_128x128_ex(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx,
                                  uint8_t* q, int64_t ldq, float* scale_inv, int64_t ld_scale, uint8_t* q_t,
                                  int64_t ldq_t, float* scale_inv_t, int64_t ld_scale_t, fp8bs_scale_rule rule,
                                  cudaStream_t stream)
{
    switch (rule) {
    case FP8BS_SCALE_RULE_FP32:
        return quant_128x128_impl<false>(x, xt, rows, cols, ldx, q, ldq, scale_inv, ld_scale, q_t, ldq_t,
                                         scale_inv_t, ld_scale_t, stream);
    case FP8BS_SCALE_RULE_POW2:
        return quant_128x128_impl<true>(x, xt, rows, cols, ldx, q, ldq, scale_inv, ld_scale, q_t, ldq_t,
                                        scale_inv_t, ld_scale_t, stream);
    }
    return FP8BS_ERR_UNSUPPORTED;
}

size_t fp8_quant_tensor_workspace_size(int64_t n)
{
    (void)n;
    return (size_t)kTensorPartials * sizeof(float);
}

fp8bs_status fp8_quant_tensor(const void* x, fp8bs_dtype xt, int64_t n, uint8_t* q, float* scale_inv,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    if (!valid_dtype(xt)) return FP8BS_ERR_UNSUPPORTED;
    if (x == nullptr || q == nullptr || scale_inv == nullptr || n < 1) return FP8BS_ERR_INVALID_ARG;
    if (workspace == nullptr || workspace_bytes < fp8_quant_tensor_workspace_size(n)) return FP8BS_ERR_WORKSPACE;
    if (!aligned16(x) || !aligned16(q) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(scale_inv) & 3) ||
        n % 16)
        return FP8BS_ERR_ALIGNMENT;
    DeviceInfo* d = nullptr;
    fp8bs_status st = get_device(&d);
    if (st != FP8BS_OK) return st;
    const int64_t chunks = n / 8;
    const int parts = (int)std::max<int64_t>(1, std::min<int64_t>(kTensorPartials, cdiv(chunks, 256 * 4)));
    float* partial = static_cast<float*>(workspace);
    if (xt == FP8BS_BF16) {
        tensor_amax_kernel<__nv_bfloat16><<<parts, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), n, partial);
        auto k = tensor_quant_kernel<__nv_bfloat16>;
        int g = persistent_grid(d, 6, k, cdiv(chunks, 256));
        k<<<g, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), n, partial, parts, q, scale_inv);
    } else {
        tensor_amax_kernel<float><<<parts, 256, 0, stream>>>(static_cast<const float*>(x), n, partial);
        auto k = tensor_quant_kernel<float>;
        int g = persistent_grid(d, 7, k, cdiv(chunks, 256));
        k<<<g, 256, 0, stream>>>(static_cast<const float*>(x), n, partial, parts, q, scale_inv);
    }
    return launch_status();
}

fp8bs_status fp8_quant_rowwise(const void* x, fp8bs_dtype xt, int64_t rows, int64_t cols, int64_t ldx, uint8_t* q,
                               int64_t ldq, float* scale_inv, cudaStream_t stream)
{
    if (!valid_dtype(xt)) return FP8BS_ERR_UNSUPPORTED;
    if (x == nullptr || q == nullptr || scale_inv == nullptr || rows < 1 || cols < 1) return FP8BS_ERR_INVALID_ARG;
    if (ldx < cols || ldq < cols) return FP8BS_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scale_inv) & 3) ||
        (ldx * (int64_t)dtype_size(xt)) % 16 || ldq % 16 || cols % 16)
        return FP8BS_ERR_ALIGNMENT;
    DeviceInfo* d = nullptr;
    fp8bs_status st = get_device(&d);
    if (st != FP8BS_OK) return st;
    const int64_t ctas = cdiv(rows, 8);
    if (xt == FP8BS_BF16) {
        auto k = quant_rowwise_kernel<__nv_bfloat16>;
        int g = persistent_grid(d, 8, k, ctas);
        k<<<g, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), rows, cols, ldx, q, ldq, scale_inv);
    } else {
        auto k = quant_rowwise_kernel<float>;
        int g = persistent_grid(d, 9, k, ctas);
        k<<<g, 256, 0, stream>>>(static_cast<const float*>(x), rows, cols, ldx, q, ldq, scale_inv);
    }
    return launch_status();
}

// ---------------------------------------------------------------- GEMM

size_t fp8_scaled_gemm_workspace_size(int64_t M, int64_t N, int64_t K, fp8bs_scale_mode mode)
{
    if (M < 1 || N < 1 || K < 1) return 0;
    const int sms = num_sms_current();
    // the power-of-two recipes run on single CTAs only
    if (mode == FP8BS_SCALE_BLOCK_1x128_128x128_POW2 || mode == FP8BS_SCALE_BLOCK_1x128_1x128_POW2)
        return plan_gemm(M, N, K, sms).ws_bytes;
    // the larger of the two kernels' needs: fp8_scaled_gemm_ex with an
    // MN-major B always runs the pair kernel
    return std::max(plan_pair(M, N, K, sms).ws_bytes,
                    use_pair(M, N, K, false, false, sms) ? size_t(0) : plan_gemm(M, N, K, sms).ws_bytes);
}

}  // extern "C"

namespace {

// Output quantization requested by fp8_scaled_gemm_quant (q == nullptr: none).
struct QuantOut {
    uint8_t* q = nullptr;
    int64_t ldq = 0;
    float* s = nullptr;
    int64_t lds = 0;
};

fp8bs_status scaled_gemm(int64_t M, int64_t N, int64_t K, const uint8_t* A, int64_t lda, const uint8_t* B,
                         int64_t ldb, bool b_mn, const float* scale_a, int64_t ld_sa, const float* scale_b,
                         int64_t ld_sb, fp8bs_scale_mode mode, fp8bs_scale_layout layout, void* D, int64_t ldd,
                         fp8bs_dtype out_dtype, void* workspace, size_t workspace_bytes, const QuantOut& qo,
                         cudaStream_t stream)
{
    const bool quant_out = qo.q != nullptr;
    if (mode < FP8BS_SCALE_TENSOR || mode > FP8BS_SCALE_BLOCK_1x128_1x128_POW2) return FP8BS_ERR_UNSUPPORTED;
    // the power-of-two recipes: the block recipes' scale grids, block-scaled MMA
    const bool pow2 = mode == FP8BS_SCALE_BLOCK_1x128_128x128_POW2 || mode == FP8BS_SCALE_BLOCK_1x128_1x128_POW2;
    if (pow2 && (quant_out || b_mn)) return FP8BS_ERR_UNSUPPORTED;
    const bool grid128 = mode == FP8BS_SCALE_BLOCK_1x128_128x128 || mode == FP8BS_SCALE_BLOCK_1x128_128x128_POW2;
    if (layout != FP8BS_SCALE_COL_MAJOR || !valid_dtype(out_dtype)) return FP8BS_ERR_UNSUPPORTED;
    if (quant_out && (mode == FP8BS_SCALE_BLOCK_1x128_1x128 || out_dtype != FP8BS_BF16)) return FP8BS_ERR_UNSUPPORTED;
    if (b_mn && (quant_out || mode == FP8BS_SCALE_BLOCK_1x128_1x128)) return FP8BS_ERR_UNSUPPORTED;
    if (A == nullptr || B == nullptr || scale_a == nullptr || scale_b == nullptr) return FP8BS_ERR_INVALID_ARG;
    if (D == nullptr && !quant_out) return FP8BS_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < 16) return FP8BS_ERR_INVALID_ARG;
    if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return FP8BS_ERR_INVALID_ARG;
    if (lda < K || ldb < (b_mn ? N : K) || (D != nullptr && ldd < N)) return FP8BS_ERR_INVALID_ARG;
    if (quant_out) {
        if (qo.s == nullptr || qo.ldq < N || qo.lds < M) return FP8BS_ERR_INVALID_ARG;
        if (!aligned16(qo.q) || !aligned16(qo.s) || qo.ldq % 16 || qo.lds % 4) return FP8BS_ERR_ALIGNMENT;
    }
    const int64_t Kb = cdiv(K, kBK), Nb = cdiv(N, 128);
    const bool block = (mode == FP8BS_SCALE_BLOCK_1x128_128x128 || mode == FP8BS_SCALE_BLOCK_1x128_1x128 || pow2);
    if (block) {
        if (ld_sa < M) return FP8BS_ERR_INVALID_ARG;
        if (grid128 && ld_sb < (b_mn ? Kb : Nb)) return FP8BS_ERR_INVALID_ARG;
        if (!grid128 && ld_sb < N) return FP8BS_ERR_INVALID_ARG;
        if (ld_sa % 4 || ld_sb % 4) return FP8BS_ERR_ALIGNMENT;
    }
    if (K % 16 || lda % 16 || ldb % 16) return FP8BS_ERR_ALIGNMENT;
    if (!aligned16(A) || !aligned16(B) || !aligned16(scale_a) || !aligned16(scale_b)) return FP8BS_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(D) % dtype_size(out_dtype)) return FP8BS_ERR_ALIGNMENT;
    const int vec_out = D != nullptr && aligned16(D) && (ldd * (int64_t)dtype_size(out_dtype)) % 16 == 0;
    DeviceInfo* d = nullptr;
    fp8bs_status st = get_device(&d);
    if (st != FP8BS_OK) return st;

    // single-CTA tiles (128 x 256) or CTA pairs (256 x 128)
    const bool pair = !pow2 && use_pair(M, N, K, b_mn, quant_out, d->num_sms);
    SplitPlan plan = pair ? plan_pair(M, N, K, d->num_sms) : plan_gemm(M, N, K, d->num_sms);
    if (quant_out) plan.splits = 1;              // the epilogue quantizes whole tiles
    if (plan.splits > 1) {
        if (workspace == nullptr && workspace_bytes == 0) {
            plan.splits = 1;                     // split-K disabled by the caller
        } else if (workspace == nullptr || workspace_bytes < plan.ws_bytes) {
            return FP8BS_ERR_WORKSPACE;
        } else if (!aligned16(workspace)) {
            return FP8BS_ERR_ALIGNMENT;
        }
    }

    // operand maps: A rows x 128-byte K slices; B^T likewise (K-major), or B
    // as the 256 K-rows of a pair-kernel step x 64-byte column slices (MN-major)
    const uint32_t a_rows = pair ? kCtaM : kBM;
    const uint32_t bt_rows = pair ? kCtaN : kBN;
    CUtensorMap tA, tB, tSA, tSB;
    std::memset(&tSA, 0, sizeof tSA);
    std::memset(&tSB, 0, sizeof tSB);
    if ((st = make_map(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, K, M, lda, kBK, a_rows, CU_TENSOR_MAP_SWIZZLE_128B)) != FP8BS_OK)
        return st;
    if (b_mn && pair) {
        if ((st = make_map(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, N, K, ldb, kCtaN, kStepKb * kBK, CU_TENSOR_MAP_SWIZZLE_64B)) != FP8BS_OK)
            return st;
    } else if (b_mn) {
        // single-CTA kernel: K-rows x 128 N-bytes boxes, two per 256-column tile
        if ((st = make_map(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, N, K, ldb, kBN / 2, kBK, CU_TENSOR_MAP_SWIZZLE_128B)) != FP8BS_OK)
            return st;
    } else if ((st = make_map(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, K, N, ldb, kBK, bt_rows, CU_TENSOR_MAP_SWIZZLE_128B)) != FP8BS_OK) {
        return st;
    }
    const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const uint32_t sa_box = pair ? 128 : kBM;
    const uint32_t sb_box = pair ? 128 : kBN;
    switch (mode) {
    case FP8BS_SCALE_TENSOR:
        break;
    case FP8BS_SCALE_ROWWISE:
        if ((st = make_map(&tSA, f32, 4, scale_a, M, 1, (M * 4 + 15) & ~int64_t(15), sa_box, 1, CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK) return st;
        if ((st = make_map(&tSB, f32, 4, scale_b, N, 1, (N * 4 + 15) & ~int64_t(15), sb_box, 1, CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK) return st;
        break;
    case FP8BS_SCALE_BLOCK_1x128_128x128:
        // single-CTA kernel: the promotion warps read both scales directly;
        // pair kernel: row scales as for 1x128 x 1x128, the B grid in 16-byte
        // groups of four blocks ((N-block, K-block), or (K-block, N-block) for MN-major B)
        if (pair) {
            if ((st = make_map(&tSA, f32, 4, scale_a, M, Kb, ld_sa * 4, sa_box, 1, CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK) return st;
            if (b_mn) {
                if ((st = make_map(&tSB, f32, 4, scale_b, Kb, Nb, ld_sb * 4, 4, 1, CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK) return st;
            } else if ((st = make_map(&tSB, f32, 4, scale_b, Nb, Kb, ld_sb * 4, 4, 1, CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK) {
                return st;
            }
        }
        break;
    case FP8BS_SCALE_BLOCK_1x128_1x128:
        if ((st = make_map(&tSA, f32, 4, scale_a, M, Kb, ld_sa * 4, sa_box, 1, CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK) return st;
        if ((st = make_map(&tSB, f32, 4, scale_b, N, Kb, ld_sb * 4, sb_box, 1, CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK) return st;
        break;
    case FP8BS_SCALE_BLOCK_1x128_128x128_POW2:
    case FP8BS_SCALE_BLOCK_1x128_1x128_POW2:
        // block-scaled kernel: four K-blocks of each grid per load (rows x 4,
        // or the aligned group of four 128-column blocks of B x 4)
        if ((st = make_map(&tSA, f32, 4, scale_a, M, Kb, ld_sa * 4, kBM, kSfKb, CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK) return st;
        if (grid128) {
            if ((st = make_map(&tSB, f32, 4, scale_b, Nb, Kb, ld_sb * 4, 4, kSfKb, CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK) return st;
        } else if ((st = make_map(&tSB, f32, 4, scale_b, N, Kb, ld_sb * 4, kBN, kSfKb, CU_TENSOR_MAP_SWIZZLE_NONE)) != FP8BS_OK) {
            return st;
        }
        break;
    }

    GemmParamsQ p;
    p.M = (int32_t)M;
    p.N = (int32_t)N;
    p.K = (int32_t)K;
    p.Kb = (int32_t)Kb;
    p.tiles_m = plan.tiles_m;
    p.tiles_n = plan.tiles_n;
    p.splits = plan.splits;
    p.group_m = pair ? 8 : 16;
    p.num_units = (int64_t)plan.tiles_m * plan.tiles_n * plan.splits;
    p.D = D;
    p.ldd = ldd;
    p.out_f32 = out_dtype == FP8BS_F32;
    p.vec_out = vec_out;
    p.ws = static_cast<float*>(workspace);
    p.ldw = plan.ldw;
    p.sa = scale_a;
    p.sb = scale_b;
    p.ld_sa = ld_sa;
    p.ld_sb = ld_sb;
    p.err = d->err_ptr;
    p.qout = qo.q;
    p.ldq_out = qo.ldq;
    p.sout = qo.s;
    p.lds_out = qo.lds;

    if (quant_out) {
        switch (mode) {
        case FP8BS_SCALE_TENSOR: return launch_gemm<kModeTensor, true>(d, tA, tB, tSA, tSB, p, stream);
        case FP8BS_SCALE_ROWWISE: return launch_gemm<kModeRowwise, true>(d, tA, tB, tSA, tSB, p, stream);
        default: return launch_gemm<kModeBlock128, true>(d, tA, tB, tSA, tSB, p, stream);
        }
    }
    const GemmParams& pb = p;                    // the plain kernels take the base block
    if (pow2) {
        st = mode == FP8BS_SCALE_BLOCK_1x128_128x128_POW2 ? launch_bs<kModeBlock128>(d, tA, tB, tSA, tSB, pb, stream)
                                                          : launch_bs<kModeBlock1x128>(d, tA, tB, tSA, tSB, pb, stream);
    } else if (!pair && b_mn) {
        switch (mode) {
        case FP8BS_SCALE_TENSOR: st = launch_gemm<kModeTensor, false, false, true>(d, tA, tB, tSA, tSB, pb, stream); break;
        case FP8BS_SCALE_ROWWISE: st = launch_gemm<kModeRowwise, false, false, true>(d, tA, tB, tSA, tSB, pb, stream); break;
        default: st = launch_gemm<kModeBlock128, false, false, true>(d, tA, tB, tSA, tSB, pb, stream); break;
        }
    } else if (!pair) {
        switch (mode) {
        case FP8BS_SCALE_TENSOR: st = launch_gemm<kModeTensor>(d, tA, tB, tSA, tSB, pb, stream); break;
        case FP8BS_SCALE_ROWWISE: st = launch_gemm<kModeRowwise>(d, tA, tB, tSA, tSB, pb, stream); break;
        case FP8BS_SCALE_BLOCK_1x128_128x128: st = launch_gemm<kModeBlock128>(d, tA, tB, tSA, tSB, pb, stream); break;
        case FP8BS_SCALE_BLOCK_1x128_1x128: st = launch_gemm<kModeBlock1x128>(d, tA, tB, tSA, tSB, pb, stream); break;
        }
    } else if (b_mn) {
        switch (mode) {
        case FP8BS_SCALE_TENSOR: st = launch_pair<kModeTensor, true>(d, tA, tB, tSA, tSB, pb, stream); break;
        case FP8BS_SCALE_ROWWISE: st = launch_pair<kModeRowwise, true>(d, tA, tB, tSA, tSB, pb, stream); break;
        default: st = launch_pair<kModeBlock128, true>(d, tA, tB, tSA, tSB, pb, stream); break;
        }
    } else {
        switch (mode) {
        case FP8BS_SCALE_TENSOR: st = launch_pair<kModeTensor, false>(d, tA, tB, tSA, tSB, pb, stream); break;
        case FP8BS_SCALE_ROWWISE: st = launch_pair<kModeRowwise, false>(d, tA, tB, tSA, tSB, pb, stream); break;
        case FP8BS_SCALE_BLOCK_1x128_128x128: st = launch_pair<kModeBlock128, false>(d, tA, tB, tSA, tSB, pb, stream); break;
        case FP8BS_SCALE_BLOCK_1x128_1x128: st = launch_pair<kModeBlock1x128, false>(d, tA, tB, tSA, tSB, pb, stream); break;
        }
    }
    if (st != FP8BS_OK) return st;
    if (plan.splits > 1) {
        const int64_t chunks = M * ((N + 3) / 4);
        const int grid = (int)std::max<int64_t>(
            1, std::min<int64_t>(cdiv(chunks, kReduceThreads), (int64_t)d->num_sms * 16));
        // programmatic dependent launch: the reduction's CTAs are scheduled
        // while the GEMM finishes and wait in-kernel for its completion
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid, 1, 1);
        cfg.blockDim = dim3(kReduceThreads, 1, 1);
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const float* wsp = p.ws;
        const int splits = plan.splits;
        const int64_t ldw = plan.ldw;
        const int out_f32 = p.out_f32;
        if (cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, wsp, splits, M, N, ldw, D, ldd, out_f32, vec_out) !=
            cudaSuccess)
            return FP8BS_ERR_CUDA;
        st = launch_status();
    }
    return st;
}

}  // namespace

extern "C" {

fp8bs_status fp8_scaled_gemm(int64_t M, int64_t N, int64_t K, const uint8_t* A, int64_t lda, const uint8_t* Bt,
                             int64_t ldb, const float* scale_a, int64_t ld_sa, const float* scale_b, int64_t ld_sb,
                             fp8bs_scale_mode mode, fp8bs_scale_layout layout, void* D, int64_t ldd,
                             fp8bs_dtype out_dtype, void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    if (D == nullptr) return FP8BS_ERR_INVALID_ARG;
    return scaled_gemm(M, N, K, A, lda, Bt, ldb, false, scale_a, ld_sa, scale_b, ld_sb, mode, layout, D, ldd,
                       out_dtype, workspace, workspace_bytes, QuantOut{}, stream);
}

fp8bs_status fp8_scaled_gemm_ex(int64_t M, int64_t N, int64_t K, const uint8_t* A, int64_t lda, const uint8_t* B,
                                int64_t ldb, fp8bs_major b_major, const float* scale_a, int64_t ld_sa,
                                const float* scale_b, int64_t ld_sb, fp8bs_scale_mode mode,
                                fp8bs_scale_layout layout, void* D, int64_t ldd, fp8bs_dtype out_dtype,
                                void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    if (D == nullptr) return FP8BS_ERR_INVALID_ARG;
    if (b_major != FP8BS_MAJOR_K && b_major != FP8BS_MAJOR_MN) return FP8BS_ERR_UNSUPPORTED;
    return scaled_gemm(M, N, K, A, lda, B, ldb, b_major == FP8BS_MAJOR_MN, scale_a, ld_sa, scale_b, ld_sb, mode,
                       layout, D, ldd, out_dtype, workspace, workspace_bytes, QuantOut{}, stream);
}

fp8bs_status fp8_scaled_gemm_quant(int64_t M, int64_t N, int64_t K, const uint8_t* A, int64_t lda, const uint8_t* Bt,
                                   int64_t ldb, const float* scale_a, int64_t ld_sa, const float* scale_b,
                                   int64_t ld_sb, fp8bs_scale_mode mode, fp8bs_scale_layout layout, void* D,
                                   int64_t ldd, uint8_t* q_out, int64_t ldq_out, float* scale_out,
                                   int64_t ld_scale_out, cudaStream_t stream)
{
    if (q_out == nullptr) return FP8BS_ERR_INVALID_ARG;
    QuantOut qo;
    qo.q = q_out;
    qo.ldq = ldq_out;
    qo.s = scale_out;
    qo.lds = ld_scale_out;
    return scaled_gemm(M, N, K, A, lda, Bt, ldb, false, scale_a, ld_sa, scale_b, ld_sb, mode, layout, D, ldd,
                       FP8BS_BF16, nullptr, 0, qo, stream);
}

fp8bs_status fp8_scaled_gemm_grouped(int64_t groups, const int64_t* group_rows, int64_t N, int64_t K,
                                     const uint8_t* A, int64_t lda, const uint8_t* Bt, int64_t ldb,
                                     const float* scale_a, int64_t ld_sa, const float* scale_b, int64_t ld_sb,
                                     int64_t sb_group_stride, fp8bs_scale_mode mode, fp8bs_scale_layout layout,
                                     void* D, int64_t ldd, fp8bs_dtype out_dtype, cudaStream_t stream)
{
    if (mode != FP8BS_SCALE_BLOCK_1x128_128x128 || layout != FP8BS_SCALE_COL_MAJOR || !valid_dtype(out_dtype))
        return FP8BS_ERR_UNSUPPORTED;
    if (groups < 1 || groups > kMaxGroups || group_rows == nullptr) return FP8BS_ERR_INVALID_ARG;
    if (N < 1 || K < 16 || N > INT32_MAX || K > INT32_MAX || groups * N > INT32_MAX) return FP8BS_ERR_INVALID_ARG;
    GemmParamsG p;
    std::memset(&p, 0, sizeof p);
    int64_t rows = 0, tiles = 0;
    const int64_t tiles_n = cdiv(N, kBN);
    for (int64_t g = 0; g < groups; ++g) {
        if (group_rows[g] < 0) return FP8BS_ERR_INVALID_ARG;
        p.row_start[g] = (int32_t)rows;
        p.tile_start[g] = (int32_t)tiles;
        rows += group_rows[g];
        tiles += cdiv(group_rows[g], kBM) * tiles_n;
        if (rows > INT32_MAX || tiles > INT32_MAX) return FP8BS_ERR_INVALID_ARG;
    }
    p.row_start[groups] = (int32_t)rows;
    p.tile_start[groups] = (int32_t)tiles;
    if (tiles == 0) return FP8BS_OK;             // every group empty: nothing to compute or write
    if (A == nullptr || Bt == nullptr || scale_a == nullptr || scale_b == nullptr || D == nullptr)
        return FP8BS_ERR_INVALID_ARG;
    const int64_t Kb = cdiv(K, kBK), Nb = cdiv(N, 128);
    if (lda < K || ldb < K || ldd < N || ld_sa < std::max<int64_t>(rows, 1) || ld_sb < Nb ||
        sb_group_stride < ld_sb * Kb)
        return FP8BS_ERR_INVALID_ARG;
    if (K % 16 || lda % 16 || ldb % 16 || ld_sa % 4 || ld_sb % 4) return FP8BS_ERR_ALIGNMENT;
    if (!aligned16(A) || !aligned16(Bt) || !aligned16(scale_a) || !aligned16(scale_b)) return FP8BS_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(D) % dtype_size(out_dtype)) return FP8BS_ERR_ALIGNMENT;
    DeviceInfo* d = nullptr;
    fp8bs_status st = get_device(&d);
    if (st != FP8BS_OK) return st;

    CUtensorMap tA, tB, tSA, tSB;
    std::memset(&tSA, 0, sizeof tSA);
    std::memset(&tSB, 0, sizeof tSB);
    if ((st = make_map(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, A, K, rows, lda, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_128B)) != FP8BS_OK)
        return st;
    if ((st = make_map(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Bt, K, groups * N, ldb, kBK, kBN, CU_TENSOR_MAP_SWIZZLE_128B)) != FP8BS_OK)
        return st;
    p.M = (int32_t)rows;
    p.N = (int32_t)N;
    p.K = (int32_t)K;
    p.Kb = (int32_t)Kb;
    p.tiles_m = (int32_t)std::max<int64_t>(1, tiles);   // only the K range of decode_unit is used
    p.tiles_n = (int32_t)tiles_n;
    p.splits = 1;
    p.group_m = 16;
    p.num_units = tiles;
    p.D = D;
    p.ldd = ldd;
    p.out_f32 = out_dtype == FP8BS_F32;
    p.vec_out = aligned16(D) && (ldd * (int64_t)dtype_size(out_dtype)) % 16 == 0;
    p.ws = nullptr;
    p.ldw = 0;
    p.sa = scale_a;
    p.sb = scale_b;
    p.ld_sa = ld_sa;
    p.ld_sb = ld_sb;
    p.err = d->err_ptr;
    p.groups = (int32_t)groups;
    p.sb_stride = sb_group_stride;
    return launch_gemm<kModeBlock128, false, true>(d, tA, tB, tSA, tSB, p, stream);
}

}  // extern "C"

// ---------------------------------------------------------------- self-test of the device timeout path

namespace {
// One thread waits, with the library's bounded wait, on an mbarrier phase
// that nothing will ever complete; when the limit runs out it raises the
// error flag exactly as a pipeline kernel does, and returns.
__global__ void selftest_wait_kernel(uint64_t limit_ns, int* err)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t a = smem_u32(&bar);
    mbar_init(a, 1);
    fence_barrier_init();
    if (!mbar_wait_bounded(a, 0, nullptr, limit_ns)) atomicOr(err, 1);
}
}  // namespace

extern "C" fp8bs_status fp8bs_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream)
{
    if (limit_ns == 0 || limit_ns > 10000000000ull) return FP8BS_ERR_INVALID_ARG;
    DeviceInfo* d = nullptr;
    fp8bs_status st = get_device(&d);
    if (st != FP8BS_OK) return st;
    selftest_wait_kernel<<<1, 1, 0, stream>>>(limit_ns, d->err_ptr);
    return launch_status();
}

// ---------------------------------------------------------------- per-tensor quantization without allocation
//
// fp8_quant_tensor needs a small device workspace for its per-CTA amax
// partials, which the caller allocates.  fp8_quant_tensor_noalloc runs the same
// two kernels with that scratch taken from a fixed array compiled into the
// library instead, so a caller that cannot allocate device memory at the point
// of the call still gets the quantization.  The array is 16 KB per GPU, held
// from the library's load on that GPU until the process exits.

namespace {
constexpr int kNoAllocPartials = 4096;                  // floats of scratch (16 KB)
constexpr int64_t kNoAllocMaxElems = int64_t(1) << 28;  // the documented size limit
std::atomic<float*> g_noalloc_scratch[kMaxDevices]{};   // device address of the array, per device
std::mutex g_noalloc_mutex;
}  // namespace

// The scratch itself.  In host code this name is only a host-side stand-in for
// the symbol: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) float g_noalloc_partials[kNoAllocPartials];

extern "C" fp8bs_status fp8_quant_tensor_noalloc(const void* x, fp8bs_dtype xt, int64_t n, uint8_t* q,
                                                 float* scale_inv, cudaStream_t stream)
{
    if (!valid_dtype(xt)) return FP8BS_ERR_UNSUPPORTED;
    if (x == nullptr || q == nullptr || scale_inv == nullptr || n < 1) return FP8BS_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scale_inv) & 3) || n % 16)
        return FP8BS_ERR_ALIGNMENT;
    if (n > kNoAllocMaxElems) return FP8BS_ERR_WORKSPACE;   // the built-in scratch covers at most this many
    DeviceInfo* d = nullptr;
    fp8bs_status st = get_device(&d);
    if (st != FP8BS_OK) return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FP8BS_ERR_CUDA;
    float* partial = g_noalloc_scratch[dev].load(std::memory_order_acquire);
    if (partial == nullptr) {
        // one-time set-up per device, with that device current
        std::lock_guard<std::mutex> lock(g_noalloc_mutex);
        partial = g_noalloc_scratch[dev].load(std::memory_order_relaxed);
        if (partial == nullptr) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_partials) != cudaSuccess || p == nullptr) return FP8BS_ERR_CUDA;
            partial = static_cast<float*>(p);
            g_noalloc_scratch[dev].store(partial, std::memory_order_release);
        }
    }
    // One amax partial per 8192 elements (as fp8_quant_tensor partitions the
    // tensor), at most one per scratch slot: the amax kernel's grid-stride loop
    // covers any n with any grid.  Every partial slot the second kernel reads is
    // written by the first one in this same call, so nothing left by an earlier
    // call needs clearing.
    const int parts = (int)std::max<int64_t>(1, std::min<int64_t>(kNoAllocPartials, cdiv(n, 8192)));
    const int64_t chunks = n / 8;
    if (xt == FP8BS_BF16) {
        tensor_amax_kernel<__nv_bfloat16><<<parts, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), n, partial);
        auto k = tensor_quant_kernel<__nv_bfloat16>;
        int g = persistent_grid(d, 6, k, cdiv(chunks, 256));
        k<<<g, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), n, partial, parts, q, scale_inv);
    } else {
        tensor_amax_kernel<float><<<parts, 256, 0, stream>>>(static_cast<const float*>(x), n, partial);
        auto k = tensor_quant_kernel<float>;
        int g = persistent_grid(d, 7, k, cdiv(chunks, 256));
        k<<<g, 256, 0, stream>>>(static_cast<const float*>(x), n, partial, parts, q, scale_inv);
    }
    return launch_status();
}
