// C ABI of libmacaq (declared in include/macaq.h): argument validation, launch
// planning and kernel launches for the MACaQ W4A4 linear layer on sm_100a.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include "macaq.h"
#include "flip_kernel.cuh"
#include "gemm_kernel.cuh"
#include "hessian_kernel.cuh"
#include "quant_kernel.cuh"
#include "selftest_kernel.cuh"

namespace macaq {

__device__ int g_device_error;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    bool supported = false;
    int num_sms = 0;
    int* err_ptr = nullptr;
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

macaq_status device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MACAQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo& d = g_devices[dev];
    if (!d.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MACAQ_ERR_CUDA;
        d.supported = (major == 10 && minor == 0);
        d.num_sms = sms;
        if (d.supported) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return MACAQ_ERR_CUDA;
            d.err_ptr = static_cast<int*>(p);
            if (g_encode == nullptr) {
                void* fn = nullptr;
                cudaDriverEntryPointQueryResult q;
                if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                        cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
                    return MACAQ_ERR_CUDA;
                g_encode = reinterpret_cast<EncodeTiledFn>(fn);
            }
        }
        d.ready = true;
    }
    if (!d.supported) return MACAQ_ERR_UNSUPPORTED_DEVICE;
    *out = &d;
    return MACAQ_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Limits that keep every index inside 32 bits where the kernels use int.
constexpr int64_t kMaxRows = (int64_t)1 << 30;
constexpr int64_t kMaxK = (int64_t)1 << 24;
constexpr int64_t kMaxFlipK = 8192;     // Flip-Refinement keeps a row's gradient in shared memory

// --------------------------------------------------------------------- quant ---

// Every kernel is launched with programmatic stream serialization: its launch and
// set-up may overlap the tail of the previous kernel on the stream, and each kernel
// executes griddepcontrol.wait before its first global memory access, so the order of
// memory effects is the same as with plain stream order.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

macaq_status launch_quant(const void* x, int64_t rows, int64_t K, int64_t ld, const float* mult,
                          uint8_t* codes, uint8_t* scales, const float* s_for_inv, float* inv_out,
                          cudaStream_t stream) {
    DeviceInfo* dev = nullptr;
    macaq_status st = device_info(&dev);
    if (st != MACAQ_OK) return st;
    QuantParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.mult = mult;
    p.codes = codes;
    p.scales = scales;
    p.s_for_inv = s_for_inv;
    p.inv_out = inv_out;
    p.rows = rows;
    p.K = K;
    p.ld = ld;
    p.rows_pad = round_up(rows, 128);
    p.kb_pad = round_up(K / 32, 8);
    p.chunks_per_row = cdiv(p.kb_pad, 32);
    // Every warp keeps one column chunk, so the grid's warp count is a multiple of the
    // chunks per row; no more warps than (chunk, row) pairs, and two CTAs per SM.
    const int64_t warps_per_cta = kQuantThreads / 32;
    const int64_t unit = std::max<int64_t>(1, std::lcm<int64_t>(warps_per_cta, p.chunks_per_row));
    const int64_t want = std::min<int64_t>((int64_t)dev->num_sms * 2 * warps_per_cta, p.rows_pad * p.chunks_per_row);
    const int64_t nwarps = std::max<int64_t>(unit, want / unit * unit);
    const int blocks = (int)(nwarps / warps_per_cta);
    static std::atomic<uint64_t> smem_set{0};
    int devid = 0;
    cudaGetDevice(&devid);
    if (!(smem_set.load() & (1ull << (devid & 63)))) {
        if (cudaFuncSetAttribute(quant_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kQuantSmemBytes) != cudaSuccess)
            return MACAQ_ERR_CUDA;
        smem_set.fetch_or(1ull << (devid & 63));
    }
    return launch_pdl(quant_rows_kernel, dim3(blocks), dim3(kQuantThreads), kQuantSmemBytes, stream, p) == cudaSuccess
               ? MACAQ_OK
               : MACAQ_ERR_CUDA;
}

// One launch of the grouped quantiser over every expert's padded rows (G > 0 experts
// with rows, table in device memory). Grid as launch_quant's; each warp then takes a
// contiguous range of rows_per_warp padded rows of its column chunk.
macaq_status launch_quant_grouped(const void* x, int64_t ld, int64_t K, const QuantGroup* table, int G,
                                  int64_t rows_pad, uint8_t* codes, uint8_t* scales, cudaStream_t stream) {
    DeviceInfo* dev = nullptr;
    macaq_status st = device_info(&dev);
    if (st != MACAQ_OK) return st;
    if (G < 1 || rows_pad < 128) return MACAQ_ERR_INVALID_ARG;
    GroupedQuantParams p{};
    p.x = static_cast<const uint16_t*>(x);
    p.codes = codes;
    p.scales = scales;
    p.groups = table;
    p.G = G;
    p.K = K;
    p.ld = ld;
    p.rows_pad = rows_pad;
    p.kb_pad = round_up(K / 32, 8);
    p.chunks_per_row = cdiv(p.kb_pad, 32);
    const int64_t warps_per_cta = kQuantThreads / 32;
    const int64_t unit = std::max<int64_t>(1, std::lcm<int64_t>(warps_per_cta, p.chunks_per_row));
    const int64_t want = std::min<int64_t>((int64_t)dev->num_sms * 2 * warps_per_cta, rows_pad * p.chunks_per_row);
    const int64_t nwarps = std::max<int64_t>(unit, want / unit * unit);
    p.rows_per_warp = (int32_t)cdiv(rows_pad, nwarps / p.chunks_per_row);
    const int blocks = (int)(nwarps / warps_per_cta);
    static std::atomic<uint64_t> smem_set{0};
    int devid = 0;
    cudaGetDevice(&devid);
    if (!(smem_set.load() & (1ull << (devid & 63)))) {
        if (cudaFuncSetAttribute(quant_grouped_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kQuantSmemBytes) != cudaSuccess)
            return MACAQ_ERR_CUDA;
        smem_set.fetch_or(1ull << (devid & 63));
    }
    return launch_pdl(quant_grouped_kernel, dim3(blocks), dim3(kQuantThreads), kQuantSmemBytes, stream, p) ==
                   cudaSuccess
               ? MACAQ_OK
               : MACAQ_ERR_CUDA;
}

macaq_status check_quant_args(const void* x, int64_t rows, int64_t K, int64_t ld, const void* mult,
                              const void* codes, const void* scales) {
    if (!x || !mult || !codes || !scales) return MACAQ_ERR_INVALID_ARG;
    if (rows < 1 || K < 32 || ld < K) return MACAQ_ERR_INVALID_ARG;
    if (K % 32 != 0 || rows > kMaxRows || K > kMaxK) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(mult) || !aligned16(codes) || !aligned16(scales) || ld % 8 != 0)
        return MACAQ_ERR_MISALIGNED;
    return MACAQ_OK;
}

// ---------------------------------------------------------------------- GEMM ---

struct GemmPlan {
    bool swap;        // P = weight, Q = activations, output written transposed
    bool pair;        // clusters of two CTAs, 256 x bn tiles (cta_group::2 MMAs)
    int split;        // > 1: clusters of `split` CTAs sharing each tile's K range
    int bn;
    int tiles_p, tiles_q, k_tiles;
    int sk_tile0;     // tiles below are whole units dealt round robin; the rest stream-K
    int64_t sk_iters; // K tiles of the stream-K tiles
    int sk_ctas;      // CTAs that share them (<= sk_iters)
    int group_p;
    int grid;
    bool sk() const { return sk_iters > 0; }
};

// Estimated SM cycles per 256-wide K tile of a 128 x bn tile: the four MMAs take about
// 2.4 bn cycles at the measured tensor rate, and a K tile costs ~400 cycles of copies,
// barriers and issue however narrow it is.
inline double ktile_cycles(int bn) { return std::max(400.0, 2.42 * bn); }


// Prefill products may run on CTA pairs: each pair computes 256 x 192 output tiles with
// cta_group::2 MMAs, each of its CTAs copying its own 128 activation rows and half of the
// 192 weight rows, so a CTA moves 28 KB of operands through shared memory per K tile
// instead of 40 KB. Measured per K tile: 0.95 of the single-CTA 128 x 192 tile's time
// (4096 x 14336 x 4096, the same 17 rounds of tiles either way: 102.1 against 107.2 us).
// A pair's tile is 256 rows, so ragged M costs it more rounds; the planner weighs both.
constexpr bool kPairPrefill = true;
// Largest K split over a cluster (the kernel's kMaxSplit), and the planner's estimate of
// what a split costs beside its share of the K tiles: a fixed part (the cluster launch
// and the exchange of partial slices: measured ~2-3 us more than one CTA per tile,
// outside the work itself) and a part per extra CTA. Measured at 256 rows: 5120 x 25600,
// split 2: 31.4 against 36.3 us; 1024 x 5120, split 4: 16.3 against 14.4 us; 5120 x 8192,
// split 2: 20.6 against 18.5 us.
constexpr int kSplitMax = kMaxSplit;
constexpr double kSplitFixedCycles = 6000.0;
constexpr double kSplitExchangeCycles = 600.0;

// Whether the ring of the K-split kernel of width bn (the instantiations launched:
// <128, 6>, <192, 5>) holds a CTA's parked partial tile and the slices it receives.
bool split_fits(int bn, int split) {
    return bn == 128 ? split_ring_fits<128>(split, 6 * (GemmShape<128, 6>::kPTileBytes + GemmShape<128, 6>::kQTileBytes))
                     : split_ring_fits<192>(split, 5 * (GemmShape<192, 5>::kPTileBytes + GemmShape<192, 5>::kQTileBytes));
}
constexpr double kPairKtileFactor = 0.95;

GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int num_sms, bool allow_sk = true, bool allow_pair = true) {
    GemmPlan best{};
    double best_cost = 0.0;
    const int k_tiles = (int)cdiv(K, 256);
    // Decode (M <= 128): weights take the MMA's 128-row side, the tokens its N.
    // Otherwise activations take the 128-row side and weights come in 128- or
    // 192-row tiles.
    const bool swap = M <= 128;
    int widths[2] = {0, 0};
    if (swap)
        widths[0] = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
    else if (N <= 128)
        widths[0] = 128;
    else {
        widths[0] = 192;
        widths[1] = 128;
    }
    const bool pair_ok = kPairPrefill && allow_pair && !swap && M > 128 && N > 128 && num_sms >= 2;
    for (int c = 0; c < 3; ++c) {
        // candidates: single CTAs with widths[0], widths[1] (each also with its K range
        // split over a cluster of 2 .. kSplitMax CTAs where every tile's cluster fits on
        // the SMs at once); then a pair of width 192
        const bool pair = c == 2;
        if (pair ? !pair_ok : widths[c] == 0) continue;
        for (int split = 1; split <= (pair || swap ? 1 : kSplitMax); ++split) {
            GemmPlan g{};
            g.swap = swap;
            g.pair = pair;
            g.split = split;
            g.k_tiles = k_tiles;
            g.bn = pair ? 192 : widths[c];
            g.tiles_p = (int)cdiv(swap ? N : M, pair ? 256 : 128);
            g.tiles_q = (int)cdiv(swap ? M : N, g.bn);
            const int64_t tiles = (int64_t)g.tiles_p * g.tiles_q;
            if (split > 1 &&
                (!allow_sk || g.bn < 128 || tiles * split > num_sms || k_tiles < 2 * split || !split_fits(g.bn, split)))
                continue;
            // time = rounds of tiles over the SMs (pairs) x K tiles per tile x cycles per K
            // tile; a split tile takes its share of the K tiles plus the exchange of one
            // partial tile per extra CTA through distributed shared memory
            const double cost = split > 1 ? (double)cdiv(k_tiles, split) * ktile_cycles(g.bn) + kSplitFixedCycles +
                                                (split - 1) * kSplitExchangeCycles
                                          : (double)cdiv(tiles, pair ? num_sms / 2 : num_sms) * k_tiles *
                                                ktile_cycles(g.bn) * (pair ? kPairKtileFactor : 1.0);
            g.sk_tile0 = (int)tiles;
            g.sk_iters = 0;
            g.grid = split > 1 ? (int)(tiles * split)
                     : pair    ? 2 * (int)std::min<int64_t>(tiles, num_sms / 2)
                               : (int)std::min<int64_t>(tiles, num_sms);
            if (best.bn == 0 || cost < best_cost * 0.98) {
                best = g;
                best_cost = cost;
            }
        }
    }
    // Decode: a weight-streaming product whose last round of tiles would leave SMs idle.
    // Each tile of that round is split in two halves of its K range, taken by two CTAs
    // before their whole tiles, so no CTA shares more than one tile and its fixup (one
    // exchange of partial tiles through L2) overlaps the MMAs of its whole tile. Needs
    // at most two halves per CTA: rest <= SMs / 2. Tiles up to 32 wide only: a wider
    // tile's exchange (its finisher reads the partner's partial tile 16 columns at a
    // time, each read an L2 round trip under a saturated HBM) costs more than the
    // balance buys (64 wide: 32.7 against 29.0 us on the 64 x 25600 x 5120 product).
    const int64_t tiles = (int64_t)best.tiles_p * best.tiles_q;
    if (allow_sk && best.swap && best.bn <= 32 && best.k_tiles >= 2) {
        const int64_t whole_rounds = tiles / num_sms;
        const int64_t rest = tiles - whole_rounds * num_sms;
        if (whole_rounds > 0 && rest > 0 && 2 * rest <= num_sms) {
            best.sk_tile0 = (int)(whole_rounds * num_sms);
            best.sk_iters = rest * best.k_tiles;
            best.grid = num_sms;
            best.sk_ctas = (int)(2 * rest);
        }
    }
    best.group_p = std::min(best.tiles_p, best.pair ? 8 : 16);   // raster groups of 16 x 128 rows
    return best;
}

// Stream-K workspace: two fp32 partial tiles per CTA (128 x bn each), then one 8-byte
// counter per tile.
struct SkWorkspace {
    size_t partial_bytes, counter_bytes;
};
SkWorkspace sk_workspace(const GemmPlan& g) {
    SkWorkspace w{0, 0};
    if (g.sk()) {
        w.partial_bytes = (size_t)round_up((int64_t)g.grid * 2 * 128 * g.bn * 4, 256);
        w.counter_bytes = (size_t)round_up((int64_t)g.tiles_p * g.tiles_q * 8, 256);
    }
    return w;
}

size_t gemm_workspace(int64_t M, int64_t N, int64_t K, int num_sms) {
    const SkWorkspace w = sk_workspace(plan_gemm(M, N, K, num_sms));
    return w.partial_bytes + w.counter_bytes;
}

// Stream-K counters carry a 48-bit tag unique to each call, so a count left by an
// earlier call (or whatever the workspace held) is never taken for a fresh one: a
// per-process salt from the clock and a call counter, mixed.
unsigned long long next_sk_tag() {
    static std::atomic<unsigned long long> counter{0};
    static const unsigned long long salt = [] {
        unsigned long long t = (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count();
        t ^= t >> 33;
        t *= 0xff51afd7ed558ccdull;
        t ^= t >> 33;
        return t;
    }();
    unsigned long long v = salt + 0x9e3779b97f4a7c15ull * (counter.fetch_add(1) + 1);
    v ^= v >> 29;
    return v & 0xFFFFFFFFFFFFull;
}

bool encode_codes_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K, int box_rows) {
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Output tensor map for the TMA-store epilogue: boxes of 32 rows x 64 bytes (32 bf16 or
// 16 fp32 columns), 64-byte swizzle.
bool encode_out_map(CUtensorMap* map, void* y, int64_t M, int64_t N, int64_t ldy, bool bf16) {
    const int64_t esz = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)(ldy * esz)};
    cuuint32_t box[2] = {(cuuint32_t)(64 / esz), 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, y, dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Largest dynamic shared memory of a CTA on sm_100.
constexpr int kMaxSmem = 232448;

template <int BN, int STAGES, int VAR = kVarPlain>
macaq_status launch_gemm_bn(const CUtensorMap& mp, const CUtensorMap& mq, const CUtensorMap& my,
                            const GemmParams& gp, int grid, cudaStream_t stream) {
    using L = GemmSmem<BN, STAGES, VAR == kVarFused>;
    static_assert(L::kAlloc <= kMaxSmem, "shared memory budget");
    const int smem = L::alloc(gp.k_tiles);
    if (smem > kMaxSmem) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    static std::atomic<uint64_t> configured_mask{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured_mask.load() & bit)) {
        if (cudaFuncSetAttribute(gemm_mxf4_kernel<BN, STAGES, VAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 VAR == kVarFused ? kMaxSmem : L::kAlloc) != cudaSuccess)
            return MACAQ_ERR_CUDA;
        configured_mask.fetch_or(bit);
    }
    return launch_pdl(gemm_mxf4_kernel<BN, STAGES, VAR>, dim3(grid), dim3(kGemmThreads), (size_t)smem, stream, mp, mq,
                      my, gp) == cudaSuccess
               ? MACAQ_OK
               : MACAQ_ERR_CUDA;
}

// Launch of the pair variant on clusters of two CTAs: one cluster per tile, at most as
// many clusters as fit on the device at once (looked up once per device and tile width:
// the kernel is persistent and its clusters share no waits, but a cluster's two CTAs
// are placed together).
template <int BN, int STAGES>
macaq_status launch_gemm_pair(const CUtensorMap& mp, const CUtensorMap& mq, const CUtensorMap& my,
                              const GemmParams& gp, int units, cudaStream_t stream) {
    using L = GemmSmem<BN, STAGES, false, true>;
    static_assert(L::kAlloc <= kMaxSmem, "shared memory budget");
    auto kernel = gemm_mxf4_kernel<BN, STAGES, kVarPair>;
    static std::mutex m;
    static int clusters[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MACAQ_ERR_CUDA;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = L::kAlloc;
    cfg.stream = stream;
    cfg.attrs = attr;
    {
        std::lock_guard<std::mutex> lock(m);
        if (clusters[dev] == 0) {
            if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
                return MACAQ_ERR_CUDA;
            int n = 0;
            cfg.gridDim = dim3(2);
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n < 1) return MACAQ_ERR_CUDA;
            clusters[dev] = n;
        }
    }
    cfg.gridDim = dim3(2 * std::min(units, clusters[dev]));
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, mp, mq, my, gp) == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

// Launch of the K-split variant: one cluster of `split` CTAs per tile. MACAQ_ERR_UNSUPPORTED_SHAPE
// (nothing launched) when not every tile's cluster fits on the device at once (looked up
// once per device, tile width and split); the caller then runs single CTAs.
template <int BN, int STAGES>
macaq_status launch_gemm_split(const CUtensorMap& mp, const CUtensorMap& mq, const CUtensorMap& my,
                               const GemmParams& gp, int units, int split, cudaStream_t stream) {
    using L = GemmSmem<BN, STAGES>;
    auto kernel = gemm_mxf4_kernel<BN, STAGES, kVarSplit>;
    static std::mutex m;
    static int clusters[kMaxDevices][kMaxSplit + 1] = {};
    int dev = 0;
    if (split < 2 || split > kMaxSplit) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MACAQ_ERR_CUDA;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = L::kAlloc;
    cfg.stream = stream;
    cfg.attrs = attr;
    {
        std::lock_guard<std::mutex> lock(m);
        if (clusters[dev][split] == 0) {
            if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
                return MACAQ_ERR_CUDA;
            int n = 0;
            cfg.gridDim = dim3(split);
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) return MACAQ_ERR_CUDA;
            clusters[dev][split] = n > 0 ? n : -1;
        }
    }
    if (units > clusters[dev][split]) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    cfg.gridDim = dim3(units * split);
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, mp, mq, my, gp) == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

// Whether the fused variant's persistent Q operand (every K tile of a bn-row tile) fits
// in shared memory beside its weight ring.
bool fused_fits(int bn, int k_tiles) {
    return bn == 16 ? GemmSmem<16, 8, true>::alloc(k_tiles) <= kMaxSmem
                    : GemmSmem<32, 6, true>::alloc(k_tiles) <= kMaxSmem;
}

macaq_status check_weight(const macaq_weight* w) {
    if (!w || !w->codes || !w->scales) return MACAQ_ERR_INVALID_ARG;
    if (w->N < 1 || w->K < 32) return MACAQ_ERR_INVALID_ARG;
    if (w->K % 32 != 0 || w->N > kMaxRows || w->K > kMaxK) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(w->codes) || !aligned16(w->scales)) return MACAQ_ERR_MISALIGNED;
    return MACAQ_OK;
}

// Activation transform fused into the GEMM kernel (decode): every CTA makes the MXFP4
// form of the whole activation (at most 32 rows) in shared memory before its main loop.
struct FusedAct {
    const void* x;
    int64_t ldx;
};
// Largest M the fused transform takes by default: every CTA repeats the transform of the
// whole activation, which costs less than the separate launch only for a row or two
// (measured on the Qwen3-32B up projection: fused 28.1 / 28.2 / 31.0 / 33.4 us against
// 29.3 / 29.7 / 29.2 / 29.6 us for M = 1 / 2 / 4 / 8). The kernel itself takes up to 32
// rows where their MXFP4 form fits in shared memory beside the weight ring.
constexpr int64_t kFusedMaxRows = 2;
constexpr int64_t kFusedKernelRows = 32;

// Output written to several destinations (the gathered output of a column-parallel
// layer): a device table of destination addresses, and whether all of them allow
// 16-byte vector stores.
struct GatherOut {
    const uint64_t* dest;          // host array, copied into the kernel's parameters
    int n;
    bool vec_ok;
};

macaq_status run_gemm(const uint8_t* a_codes, const uint8_t* a_scales, int64_t M,
                      const macaq_weight* w, void* y, int64_t ldy, macaq_out_dtype out,
                      void* workspace, size_t ws_bytes, cudaStream_t stream, const FusedAct* fa = nullptr,
                      const GatherOut* go = nullptr, bool after_own_quant = false) {
    DeviceInfo* dev = nullptr;
    macaq_status st = device_info(&dev);
    if (st != MACAQ_OK) return st;
    const int64_t N = w->N, K = w->K;
    // a gathered output: one CTA per tile, single CTAs
    GemmPlan g = go ? plan_gemm(M, N, K, dev->num_sms, false, false) : plan_gemm(M, N, K, dev->num_sms);
    const size_t need = gemm_workspace(M, N, K, dev->num_sms);
    if (need > 0 && (workspace == nullptr || ws_bytes < need)) return MACAQ_ERR_WORKSPACE;
    if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return MACAQ_ERR_MISALIGNED;

    const uint8_t* p_codes = g.swap ? w->codes : a_codes;
    const uint8_t* q_codes = g.swap ? a_codes : w->codes;
    const int64_t p_rows = g.swap ? N : M;
    const int64_t q_rows = g.swap ? M : N;
    CUtensorMap mp, mq;
    if (!encode_codes_map(&mp, p_codes, p_rows, K, 128) ||
        !encode_codes_map(&mq, q_codes, q_rows, K, g.pair ? g.bn / 2 : g.bn))
        return MACAQ_ERR_CUDA;

    GemmParams gp{};
    gp.sf_p = g.swap ? w->scales : a_scales;
    gp.sf_q = g.swap ? a_scales : w->scales;
    gp.p_rows = (int32_t)p_rows;
    gp.q_rows = (int32_t)q_rows;
    gp.k_tiles = g.k_tiles;
    gp.kb4_pad = (int32_t)(round_up(K / 32, 8) / 4);
    gp.tiles_p = g.tiles_p;
    gp.tiles_q = g.tiles_q;
    gp.total_units = g.tiles_p * g.tiles_q;
    gp.group_p = g.group_p;
    gp.transpose_out = g.swap ? 1 : 0;
    gp.err = dev->err_ptr;
    const int64_t esz = out == MACAQ_OUT_BF16 ? 2 : 4;
    gp.out = y;
    gp.ldo = ldy;
    gp.out_bf16 = out == MACAQ_OUT_BF16 ? 1 : 0;
    gp.vec_ok = (aligned16(y) && (ldy * esz) % 16 == 0) ? 1 : 0;
    // wide row-major tiles store through TMA when the output is aligned and its rows end
    // on a 16-byte boundary: a tensor store clips a box at the row's end only to whole
    // 16-byte pieces (a bf16 output of N = 700 got columns 700..703 written), so other
    // widths use direct stores, which check every column
    gp.tma_store = (!g.swap && g.bn >= 128 && gp.vec_ok && (N * esz) % 16 == 0) ? 1 : 0;
    if (go) {
        gp.n_dest = go->n;
        for (int d = 0; d < go->n; ++d) gp.dest[d] = go->dest[d];
        gp.vec_ok = go->vec_ok ? 1 : 0;
        gp.tma_store = 0;
    }
    gp.sk_tile0 = g.sk_tile0;
    gp.sk_iters = g.sk_iters;
    gp.sk_ctas = g.sk_ctas;
    if (g.sk()) {
        const SkWorkspace sw = sk_workspace(g);
        gp.sk_partials = static_cast<float*>(workspace);
        gp.sk_counters = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(workspace) + sw.partial_bytes);
        gp.sk_tag = next_sk_tag();
    }
    // after the library's own activation transform on this stream nothing still running
    // writes the weight, so its first tiles may be copied before the previous kernel ends
    gp.w_early = after_own_quant ? 1 : 0;
    const int grid = g.grid;
    if (fa) {
        // decode orientation only, one activation tile held whole in shared memory
        if (!g.swap || g.tiles_q != 1 || g.bn > 32 || !fused_fits(g.bn, g.k_tiles)) return MACAQ_ERR_UNSUPPORTED_SHAPE;
        gp.fx = static_cast<const uint16_t*>(fa->x);
        gp.fx_ld = fa->ldx;
        gp.f_mult = w->inv_s;
        gp.f_K = (int32_t)K;
    }
    CUtensorMap my;
    std::memset(&my, 0, sizeof(my));
    if (gp.tma_store && !encode_out_map(&my, y, M, N, ldy, out == MACAQ_OUT_BF16)) return MACAQ_ERR_CUDA;

    if (go) {
        switch (g.bn) {
            case 16: st = launch_gemm_bn<16, 8, kVarGather>(mp, mq, my, gp, grid, stream); break;
            case 32: st = launch_gemm_bn<32, 8, kVarGather>(mp, mq, my, gp, grid, stream); break;
            case 64: st = launch_gemm_bn<64, 8, kVarGather>(mp, mq, my, gp, grid, stream); break;
            case 128: st = launch_gemm_bn<128, 6, kVarGather>(mp, mq, my, gp, grid, stream); break;
            default: st = launch_gemm_bn<192, 5, kVarGather>(mp, mq, my, gp, grid, stream); break;
        }
        return st;
    }
    if (fa) {
        st = g.bn == 16 ? launch_gemm_bn<16, 8, kVarFused>(mp, mq, my, gp, grid, stream)
                        : launch_gemm_bn<32, 6, kVarFused>(mp, mq, my, gp, grid, stream);
    } else if (g.pair) {
        st = launch_gemm_pair<192, 5>(mp, mq, my, gp, gp.total_units, stream);
    } else if (g.split > 1) {
        gp.split = g.split;
        st = g.bn == 128 ? launch_gemm_split<128, 6>(mp, mq, my, gp, gp.total_units, g.split, stream)
                         : launch_gemm_split<192, 5>(mp, mq, my, gp, gp.total_units, g.split, stream);
        if (st == MACAQ_ERR_UNSUPPORTED_SHAPE) {
            // the clusters do not all fit at once: one CTA per tile
            gp.split = 1;
            const int grid1 = std::min(gp.total_units, dev->num_sms);
            st = g.bn == 128 ? launch_gemm_bn<128, 6>(mp, mq, my, gp, grid1, stream)
                             : launch_gemm_bn<192, 5>(mp, mq, my, gp, grid1, stream);
        }
    } else {
        switch (g.bn) {
            case 16: st = launch_gemm_bn<16, 8>(mp, mq, my, gp, grid, stream); break;
            case 32: st = launch_gemm_bn<32, 8>(mp, mq, my, gp, grid, stream); break;
            case 64: st = launch_gemm_bn<64, 8>(mp, mq, my, gp, grid, stream); break;
            case 128: st = launch_gemm_bn<128, 6>(mp, mq, my, gp, grid, stream); break;
            default: st = launch_gemm_bn<192, 5>(mp, mq, my, gp, grid, stream); break;
        }
    }
    return st;
}

macaq_status check_gemm_args(int64_t M, const macaq_weight* w, const void* y, int64_t ldy,
                             macaq_out_dtype out) {
    macaq_status st = check_weight(w);
    if (st != MACAQ_OK) return st;
    if (!y || M < 1 || ldy < w->N) return MACAQ_ERR_INVALID_ARG;
    if (out != MACAQ_OUT_F32 && out != MACAQ_OUT_BF16) return MACAQ_ERR_INVALID_ARG;
    if (M > kMaxRows || M * w->N > ((int64_t)1 << 40)) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    const uintptr_t esz = out == MACAQ_OUT_BF16 ? 2 : 4;
    if ((reinterpret_cast<uintptr_t>(y) & (esz - 1)) != 0) return MACAQ_ERR_MISALIGNED;
    return MACAQ_OK;
}

}  // namespace
}  // namespace macaq

using namespace macaq;

extern "C" {

size_t macaq_codes_bytes(int64_t rows, int64_t K) {
    if (rows < 0 || K < 0) return 0;
    return (size_t)(rows * (K / 2));
}

size_t macaq_scales_bytes(int64_t rows, int64_t K) {
    if (rows < 0 || K < 0) return 0;
    return (size_t)(round_up(rows, 128) * round_up(K / 32, 8));
}

size_t macaq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, macaq_out_dtype out) {
    (void)out;
    if (M < 1 || N < 1 || K < 32) return 0;
    DeviceInfo* dev = nullptr;
    int sms = 148;
    if (device_info(&dev) == MACAQ_OK) sms = dev->num_sms;
    return gemm_workspace(M, N, K, sms);
}

// macaq_linear_w4a4's workspace: activation codes | scales | the GEMM's own workspace,
// each 256-byte aligned.
static size_t linear_ws_parts(int64_t M, int64_t N, int64_t K, macaq_out_dtype out, size_t* off_scales,
                              size_t* off_gemm) {
    const size_t codes = (size_t)round_up((int64_t)macaq_codes_bytes(M, K), 256);
    const size_t scales = (size_t)round_up((int64_t)macaq_scales_bytes(M, K), 256);
    *off_scales = codes;
    *off_gemm = codes + scales;
    return *off_gemm + macaq_gemm_workspace_bytes(M, N, K, out);
}

size_t macaq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, macaq_out_dtype out) {
    if (M < 1 || N < 1 || K < 32) return 0;
    size_t a, b;
    return linear_ws_parts(M, N, K, out, &a, &b);
}

macaq_status macaq_prepare_weight(const void* W_bf16, int64_t N, int64_t K, int64_t ldw, const float* s,
                                  uint8_t* w_codes, uint8_t* w_scales, float* inv_s_out,
                                  macaq_stream stream) {
    macaq_status st = check_quant_args(W_bf16, N, K, ldw, s, w_codes, w_scales);
    if (st != MACAQ_OK) return st;
    if (!inv_s_out) return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(inv_s_out)) return MACAQ_ERR_MISALIGNED;
    return launch_quant(W_bf16, N, K, ldw, s, w_codes, w_scales, s, inv_s_out, (cudaStream_t)stream);
}

macaq_status macaq_quant_act(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, const float* inv_s,
                             uint8_t* a_codes, uint8_t* a_scales, macaq_stream stream) {
    macaq_status st = check_quant_args(x_bf16, M, K, ldx, inv_s, a_codes, a_scales);
    if (st != MACAQ_OK) return st;
    return launch_quant(x_bf16, M, K, ldx, inv_s, a_codes, a_scales, nullptr, nullptr, (cudaStream_t)stream);
}

macaq_status macaq_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_scales, int64_t M,
                              const macaq_weight* w, void* y, int64_t ldy, macaq_out_dtype out,
                              void* workspace, size_t ws_bytes, macaq_stream stream) {
    macaq_status st = check_gemm_args(M, w, y, ldy, out);
    if (st != MACAQ_OK) return st;
    if (!a_codes || !a_scales) return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(a_scales)) return MACAQ_ERR_MISALIGNED;
    return run_gemm(a_codes, a_scales, M, w, y, ldy, out, workspace, ws_bytes, (cudaStream_t)stream);
}

macaq_status macaq_linear_w4a4(const void* x_bf16, int64_t M, int64_t ldx, const macaq_weight* w, void* y,
                               int64_t ldy, macaq_out_dtype out, int fused, void* workspace, size_t ws_bytes,
                               macaq_stream stream) {
    macaq_status st = check_gemm_args(M, w, y, ldy, out);
    if (st != MACAQ_OK) return st;
    if (fused < 0 || fused > 2) return MACAQ_ERR_INVALID_ARG;
    if (!w->inv_s) return MACAQ_ERR_INVALID_ARG;
    st = check_quant_args(x_bf16, M, w->K, ldx, w->inv_s, w->codes, w->scales);
    if (st != MACAQ_OK) return st;
    size_t off_scales, off_gemm;
    const size_t need = linear_ws_parts(M, w->N, w->K, out, &off_scales, &off_gemm);
    if (!workspace || ws_bytes < need) return MACAQ_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return MACAQ_ERR_MISALIGNED;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* a_codes = ws;
    uint8_t* a_scales = ws + off_scales;
    const int64_t fused_rows = fused == 2 ? kFusedKernelRows : fused == 1 ? kFusedMaxRows : 0;
    if (M <= fused_rows && fused_fits(M <= 16 ? 16 : 32, (int)cdiv(w->K, 256))) {
        // one launch: the GEMM kernel makes the MXFP4 activations in shared memory itself
        // (the activation part of the workspace is not touched)
        const FusedAct fa{x_bf16, ldx};
        return run_gemm(a_codes, a_scales, M, w, y, ldy, out, ws + off_gemm, ws_bytes - off_gemm,
                        (cudaStream_t)stream, &fa);
    }
    st = launch_quant(x_bf16, M, w->K, ldx, w->inv_s, a_codes, a_scales, nullptr, nullptr, (cudaStream_t)stream);
    if (st != MACAQ_OK) return st;
    return run_gemm(a_codes, a_scales, M, w, y, ldy, out, ws + off_gemm, ws_bytes - off_gemm, (cudaStream_t)stream,
                    nullptr, nullptr, true);
}

size_t macaq_linear_gather_workspace_bytes(int64_t M, int64_t N, int64_t K, macaq_out_dtype out) {
    const size_t lin = macaq_linear_workspace_bytes(M, N, K, out);
    return lin;
}

macaq_status macaq_linear_w4a4_gather(const void* x_bf16, int64_t M, int64_t ldx, const macaq_weight* w,
                                      const uint64_t* dest, int n_dest, int64_t ldy, macaq_out_dtype out,
                                      void* workspace, size_t ws_bytes, macaq_stream stream) {
    if (!dest || n_dest < 1 || n_dest > kMaxGatherDest) return MACAQ_ERR_INVALID_ARG;
    const uintptr_t esz = out == MACAQ_OUT_BF16 ? 2 : 4;
    bool vec = (ldy * (int64_t)esz) % 16 == 0;
    for (int d = 0; d < n_dest; ++d) {
        macaq_status st = check_gemm_args(M, w, reinterpret_cast<const void*>(dest[d]), ldy, out);
        if (st != MACAQ_OK) return st;
        vec = vec && (dest[d] & 15) == 0;
    }
    if (!w->inv_s) return MACAQ_ERR_INVALID_ARG;
    macaq_status st = check_quant_args(x_bf16, M, w->K, ldx, w->inv_s, w->codes, w->scales);
    if (st != MACAQ_OK) return st;
    size_t off_scales, off_gemm;
    const size_t lin = linear_ws_parts(M, w->N, w->K, out, &off_scales, &off_gemm);
    const size_t need = macaq_linear_gather_workspace_bytes(M, w->N, w->K, out);
    if (!workspace || ws_bytes < need) return MACAQ_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return MACAQ_ERR_MISALIGNED;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    st = launch_quant(x_bf16, M, w->K, ldx, w->inv_s, ws, ws + off_scales, nullptr, nullptr, (cudaStream_t)stream);
    if (st != MACAQ_OK) return st;
    const GatherOut go{dest, n_dest, vec};
    return run_gemm(ws, ws + off_scales, M, w, nullptr, ldy, out, ws + off_gemm, lin - off_gemm,
                    (cudaStream_t)stream, nullptr, &go, true);
}

}  // extern "C"

// Scratch of macaq_linear_w4a4_noalloc: one static array per device that loads the
// library. Host code must not pass the symbol itself to a kernel (on the host it names
// a stand-in, not device memory); its device address is looked up once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MACAQ_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[macaq::kMaxDevices];
}  // namespace

extern "C" {

macaq_status macaq_linear_w4a4_noalloc(const void* x_bf16, int64_t M, int64_t ldx, const macaq_weight* w,
                                       void* y, int64_t ldy, macaq_out_dtype out, macaq_stream stream) {
    macaq_status st = check_gemm_args(M, w, y, ldy, out);
    if (st != MACAQ_OK) return st;
    if (macaq_linear_workspace_bytes(M, w->N, w->K, out) > MACAQ_NOALLOC_SCRATCH_BYTES)
        return MACAQ_ERR_WORKSPACE;
    DeviceInfo* info = nullptr;
    st = device_info(&info);
    if (st != MACAQ_OK) return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MACAQ_ERR_CUDA;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mutex);
        if (g_noalloc_ptr[dev] == nullptr) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
                return MACAQ_ERR_CUDA;
            g_noalloc_ptr[dev] = p;
        }
        scratch = g_noalloc_ptr[dev];
    }
    return macaq_linear_w4a4(x_bf16, M, ldx, w, y, ldy, out, 0, scratch, MACAQ_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"

// ------------------------------------------- grouped layers (MoE, shared input) ---

namespace macaq {

// Per-call tables (tensor maps, group descriptors) reach the device inside kernel
// parameters: one small kernel per chunk writes its bytes to the workspace. Parameters
// are copied when the kernel is enqueued, so the call neither waits for the stream nor
// reads host memory after it returns.
constexpr uint32_t kUploadChunkBytes = 16384;
struct UploadChunk {
    uint4* dst;
    uint32_t words;                       // 16-byte words in data
    uint4 data[kUploadChunkBytes / 16];
};

__global__ void __launch_bounds__(256) upload_kernel(const __grid_constant__ UploadChunk c) {
    ptx::griddep_wait();                  // the stream's earlier kernels may still read dst
    ptx::griddep_launch_dependents();
    for (uint32_t i = threadIdx.x; i < c.words; i += blockDim.x) c.dst[i] = c.data[i];
}

// Enqueue the upload of `bytes` (a multiple of 16) from host memory to device `dst`.
macaq_status upload(void* dst, const void* src, size_t bytes, cudaStream_t stream) {
    const uint8_t* s = static_cast<const uint8_t*>(src);
    for (size_t off = 0; off < bytes; off += kUploadChunkBytes) {
        const size_t n = std::min<size_t>(kUploadChunkBytes, bytes - off);
        UploadChunk c;
        c.dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(dst) + off);
        c.words = (uint32_t)(n / 16);
        std::memcpy(c.data, s + off, n);
        if (launch_pdl(upload_kernel, dim3(1), dim3(256), 0, stream, c) != cudaSuccess) return MACAQ_ERR_CUDA;
    }
    return MACAQ_OK;
}

}  // namespace macaq

namespace {

// One group of a grouped layer: rows x_row .. x_row + rows - 1 of x through weight w into
// rows row_y .. of y (row stride ldy).
struct GroupSpec {
    int64_t x_row, rows;
    const macaq_weight* w;
    void* y;
    int64_t row_y, ldy;
};

// Workspace of a grouped layer: the activation codes and scales of every group, each
// group padded to whole 128-row scale slabs, then the tables (tensor maps, group
// descriptors, the quantiser's table), each part 256-byte aligned.
struct GroupedLayout {
    int64_t rows_pad_total = 0;
    size_t off_scales = 0, off_tmaps = 0, off_desc = 0, off_qtab = 0, total = 0;
};

bool grouped_layout(const int64_t* rows, int64_t G, int64_t K, GroupedLayout* L) {
    if (!rows || G < 1 || G > 4096 || K < 32 || K % 32 != 0) return false;
    int64_t total = 0;
    for (int64_t g = 0; g < G; ++g) {
        if (rows[g] < 0) return false;
        total += round_up(rows[g], 128);
    }
    if (total > kMaxRows) return false;
    L->rows_pad_total = total;
    const size_t codes = (size_t)round_up(std::max<int64_t>(total, 128) * (K / 2), 256);
    const size_t scales = (size_t)round_up(std::max<int64_t>(total, 128) * round_up(K / 32, 8), 256);
    L->off_scales = codes;
    L->off_tmaps = codes + scales;
    L->off_desc = L->off_tmaps + (size_t)round_up(G * (int64_t)sizeof(CUtensorMap), 256);
    L->off_qtab = L->off_desc + (size_t)round_up(G * (int64_t)sizeof(GemmGroup), 256);
    L->total = L->off_qtab + (size_t)round_up(G * (int64_t)sizeof(QuantGroup), 256);
    return true;
}

// The grouped layer (arguments validated by the caller): one quantiser launch puts every
// group's rows through the activation transform with its own weight's inv_s, one GEMM
// launch covers every group's tiles (prefill orientation, 128- or 192-wide weight tiles,
// direct stores). The tables reach the workspace through kernel parameters.
macaq_status run_grouped(const void* x, int64_t ldx, int64_t K, const std::vector<GroupSpec>& gs,
                         macaq_out_dtype out, const GroupedLayout& GL, uint8_t* ws, cudaStream_t cs) {
    DeviceInfo* dev = nullptr;
    macaq_status st = device_info(&dev);
    if (st != MACAQ_OK) return st;
    const int64_t G = (int64_t)gs.size();
    const int64_t esz = out == MACAQ_OUT_BF16 ? 2 : 4;
    int64_t n_max = 0;
    for (const GroupSpec& g : gs) n_max = std::max(n_max, g.w->N);
    // tile width: the fewer rounds of tiles over the SMs, then the narrower tiles' cost
    int bn = 128;
    if (n_max > 128) {
        double best = 0.0;
        for (int cand : {192, 128}) {
            int64_t units = 0;
            for (const GroupSpec& g : gs) units += cdiv(g.rows, 128) * cdiv(g.w->N, cand);
            const double cost = (double)cdiv(units, dev->num_sms) * ktile_cycles(cand);
            if (best == 0.0 || cost < best * 0.98) {
                best = cost;
                bn = cand;
            }
        }
    }
    std::vector<CUtensorMap> maps((size_t)G);
    std::vector<GemmGroup> desc((size_t)G);
    std::vector<QuantGroup> qtab;
    int64_t units = 0, row_p = 0;
    bool vec = true;
    for (int64_t g = 0; g < G; ++g) {
        const GroupSpec& q = gs[(size_t)g];
        if (q.rows > 0) qtab.push_back(QuantGroup{q.x_row, (int32_t)q.rows, (int32_t)row_p, q.w->inv_s});
        if (!encode_codes_map(&maps[g], q.w->codes, q.w->N, K, bn)) return MACAQ_ERR_CUDA;
        GemmGroup& d = desc[(size_t)g];
        d.unit_begin = (int32_t)units;
        d.rows = (int32_t)q.rows;
        d.row_p = (int32_t)row_p;
        d.row_y = (int32_t)q.row_y;
        d.q_rows = (int32_t)q.w->N;
        d.tiles_q = (int32_t)cdiv(q.w->N, bn);
        d.sf_q = q.w->scales;
        d.out = q.y;
        d.ldo = q.ldy;
        vec = vec && aligned16(q.y) && (q.ldy * esz) % 16 == 0;
        units += cdiv(q.rows, 128) * d.tiles_q;
        row_p += round_up(q.rows, 128);
    }
    if (units > INT32_MAX) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    {
        // one contiguous image of the three tables, in their workspace layout
        std::vector<uint8_t> image(GL.total - GL.off_tmaps, 0);
        std::memcpy(image.data(), maps.data(), maps.size() * sizeof(CUtensorMap));
        std::memcpy(image.data() + (GL.off_desc - GL.off_tmaps), desc.data(), desc.size() * sizeof(GemmGroup));
        std::memcpy(image.data() + (GL.off_qtab - GL.off_tmaps), qtab.data(), qtab.size() * sizeof(QuantGroup));
        st = upload(ws + GL.off_tmaps, image.data(), image.size(), cs);
        if (st != MACAQ_OK) return st;
    }
    uint8_t* a_codes = ws;
    uint8_t* a_scales = ws + GL.off_scales;
    if (!qtab.empty()) {
        st = launch_quant_grouped(x, ldx, K, reinterpret_cast<const QuantGroup*>(ws + GL.off_qtab), (int)qtab.size(),
                                  GL.rows_pad_total, a_codes, a_scales, cs);
        if (st != MACAQ_OK) return st;
    }
    if (units == 0) return MACAQ_OK;
    CUtensorMap mp, mq, my;
    std::memset(&mq, 0, sizeof(mq));
    std::memset(&my, 0, sizeof(my));
    if (!encode_codes_map(&mp, a_codes, std::max<int64_t>(GL.rows_pad_total, 1), K, 128)) return MACAQ_ERR_CUDA;
    GemmParams gp{};
    gp.sf_p = a_scales;
    gp.sf_q = gs[0].w->scales;
    gp.out = gs[0].y;
    gp.ldo = gs[0].ldy;
    gp.p_rows = (int32_t)GL.rows_pad_total;
    gp.q_rows = (int32_t)n_max;
    gp.k_tiles = (int32_t)cdiv(K, 256);
    gp.kb4_pad = (int32_t)(round_up(K / 32, 8) / 4);
    gp.tiles_p = 1;
    gp.tiles_q = (int32_t)cdiv(n_max, bn);
    gp.total_units = (int32_t)units;
    gp.sk_tile0 = (int32_t)units;
    gp.group_p = 1;
    gp.out_bf16 = out == MACAQ_OUT_BF16 ? 1 : 0;
    gp.vec_ok = vec ? 1 : 0;
    gp.err = dev->err_ptr;
    gp.groups = (int32_t)G;
    gp.g_desc = reinterpret_cast<const GemmGroup*>(ws + GL.off_desc);
    gp.g_tmaps = reinterpret_cast<const CUtensorMap*>(ws + GL.off_tmaps);
    // the tables' upload kernels and the grouped quantiser run before this GEMM on the
    // stream, each starting its work only after everything before it has completed: when
    // the GEMM starts, the tables and every weight are final
    gp.w_early = qtab.empty() ? 0 : 1;
    // few tiles for the SMs (the shared-input q/k/v projections): K split over clusters,
    // as for a single layer (plan_gemm)
    const int k_tiles = (int)cdiv(K, 256);
    // (by the same cost model: one round of the tiles' K tiles against a split's share plus
    // its fixed and per-CTA costs)
    if (2 * units <= dev->num_sms && k_tiles >= 4) {
        int split = (int)std::min<int64_t>(std::min<int64_t>(kSplitMax, dev->num_sms / units), k_tiles / 2);
        while (split >= 2 && (double)cdiv(k_tiles, split) * ktile_cycles(bn) + kSplitFixedCycles +
                                     (split - 1) * kSplitExchangeCycles >=
                                 0.98 * (double)k_tiles * ktile_cycles(bn))
            --split;
        while (split >= 2 && !split_fits(bn, split)) --split;
        if (split >= 2) {
            gp.split = split;
            st = bn == 128 ? launch_gemm_split<128, 6>(mp, mq, my, gp, (int)units, split, cs)
                           : launch_gemm_split<192, 5>(mp, mq, my, gp, (int)units, split, cs);
            if (st != MACAQ_ERR_UNSUPPORTED_SHAPE) return st;
            gp.split = 1;
        }
    }
    const int grid = (int)std::min<int64_t>(units, dev->num_sms);
    return bn == 128 ? launch_gemm_bn<128, 6>(mp, mq, my, gp, grid, cs) : launch_gemm_bn<192, 5>(mp, mq, my, gp, grid, cs);
}

// Group rows of the MoE layer from its offsets (false if they are not valid).
bool moe_rows(const int64_t* offsets, int64_t G, std::vector<int64_t>* rows) {
    if (!offsets || G < 1 || G > 4096 || offsets[0] != 0) return false;
    rows->resize((size_t)G);
    for (int64_t g = 0; g < G; ++g) {
        (*rows)[(size_t)g] = offsets[g + 1] - offsets[g];
        if ((*rows)[(size_t)g] < 0) return false;
    }
    return true;
}

}  // namespace

extern "C" {

size_t macaq_grouped_linear_workspace_bytes(const int64_t* offsets, int64_t G, int64_t K) {
    std::vector<int64_t> rows;
    GroupedLayout L;
    return moe_rows(offsets, G, &rows) && grouped_layout(rows.data(), G, K, &L) ? L.total : 0;
}

macaq_status macaq_grouped_linear_w4a4(const void* x_bf16, int64_t ldx, const int64_t* offsets, int64_t G,
                                       const macaq_weight* weights, void* y, int64_t ldy, macaq_out_dtype out,
                                       void* workspace, size_t ws_bytes, macaq_stream stream) {
    if (!x_bf16 || !offsets || !weights || !y) return MACAQ_ERR_INVALID_ARG;
    if (G < 1 || !weights[0].codes) return MACAQ_ERR_INVALID_ARG;
    const int64_t N = weights[0].N, K = weights[0].K;
    std::vector<int64_t> rows;
    GroupedLayout GL;
    if (!moe_rows(offsets, G, &rows) || !grouped_layout(rows.data(), G, K, &GL)) return MACAQ_ERR_INVALID_ARG;
    const int64_t M = offsets[G];
    if (M < 1) return MACAQ_ERR_INVALID_ARG;
    for (int64_t g = 0; g < G; ++g) {
        macaq_status st = check_weight(&weights[g]);
        if (st != MACAQ_OK) return st;
        if (weights[g].N != N || weights[g].K != K || !weights[g].inv_s) return MACAQ_ERR_INVALID_ARG;
        if (!aligned16(weights[g].inv_s)) return MACAQ_ERR_MISALIGNED;
    }
    macaq_status st = check_gemm_args(M, &weights[0], y, ldy, out);
    if (st != MACAQ_OK) return st;
    st = check_quant_args(x_bf16, M, K, ldx, weights[0].inv_s, weights[0].codes, weights[0].scales);
    if (st != MACAQ_OK) return st;
    if (!workspace || ws_bytes < GL.total) return MACAQ_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return MACAQ_ERR_MISALIGNED;
    std::vector<GroupSpec> gs((size_t)G);
    for (int64_t g = 0; g < G; ++g)
        gs[(size_t)g] = GroupSpec{offsets[g], rows[(size_t)g], &weights[g], y, offsets[g], ldy};
    return run_grouped(x_bf16, ldx, K, gs, out, GL, static_cast<uint8_t*>(workspace), (cudaStream_t)stream);
}

size_t macaq_multi_linear_workspace_bytes(int64_t M, int64_t K, int64_t G) {
    if (M < 1 || G < 1 || G > 4096) return 0;
    std::vector<int64_t> rows((size_t)G, M);
    GroupedLayout L;
    return grouped_layout(rows.data(), G, K, &L) ? L.total : 0;
}

macaq_status macaq_multi_linear_w4a4(const void* x_bf16, int64_t M, int64_t ldx, const macaq_weight* weights,
                                     int64_t G, void* const* y, const int64_t* ldy, macaq_out_dtype out,
                                     void* workspace, size_t ws_bytes, macaq_stream stream) {
    if (!x_bf16 || !weights || !y || !ldy || G < 1 || G > 4096 || M < 1) return MACAQ_ERR_INVALID_ARG;
    const int64_t K = weights[0].K;
    for (int64_t g = 0; g < G; ++g) {
        macaq_status st = check_gemm_args(M, &weights[g], y[g], ldy[g], out);
        if (st != MACAQ_OK) return st;
        if (weights[g].K != K || !weights[g].inv_s) return MACAQ_ERR_INVALID_ARG;
        if (!aligned16(weights[g].inv_s)) return MACAQ_ERR_MISALIGNED;
    }
    macaq_status st = check_quant_args(x_bf16, M, K, ldx, weights[0].inv_s, weights[0].codes, weights[0].scales);
    if (st != MACAQ_OK) return st;
    std::vector<int64_t> rows((size_t)G, M);
    GroupedLayout GL;
    if (!grouped_layout(rows.data(), G, K, &GL)) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    if (!workspace || ws_bytes < GL.total) return MACAQ_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return MACAQ_ERR_MISALIGNED;
    std::vector<GroupSpec> gs((size_t)G);
    for (int64_t g = 0; g < G; ++g) gs[(size_t)g] = GroupSpec{0, M, &weights[g], y[g], 0, ldy[g]};
    return run_grouped(x_bf16, ldx, K, gs, out, GL, static_cast<uint8_t*>(workspace), (cudaStream_t)stream);
}

size_t macaq_hessian_bytes(int64_t K) {
    if (K < 32 || K % 32 != 0) return 0;
    return (size_t)(K / 32) * 32 * 32 * sizeof(double);
}

macaq_status macaq_hessian_blocks(const void* x_bf16, int64_t T, int64_t K, int64_t ldx, const float* s, double* H,
                                  macaq_stream stream) {
    if (!x_bf16 || !s || !H) return MACAQ_ERR_INVALID_ARG;
    if (T < 1 || K < 32 || ldx < K) return MACAQ_ERR_INVALID_ARG;
    if (K % 32 != 0 || T > kMaxRows || K > kMaxK) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(s) || !aligned16(H) || ldx % 8 != 0) return MACAQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    macaq_status st = device_info(&dev);
    if (st != MACAQ_OK) return st;
    HessianParams hp{static_cast<const uint16_t*>(x_bf16), s, H, T, K, ldx};
    return launch_pdl(hessian_blocks_kernel, dim3((unsigned)(K / 32)), dim3(1024), 0, (cudaStream_t)stream, hp) ==
                   cudaSuccess
               ? MACAQ_OK
               : MACAQ_ERR_CUDA;
}

macaq_status macaq_prepare_weight_hessian(const void* W_bf16, int64_t N, int64_t K, int64_t ldw, const float* s,
                                          const double* H, uint8_t* w_codes, uint8_t* w_scales, float* inv_s_out,
                                          macaq_stream stream) {
    macaq_status st = check_quant_args(W_bf16, N, K, ldw, s, w_codes, w_scales);
    if (st != MACAQ_OK) return st;
    if (!H || !inv_s_out) return MACAQ_ERR_INVALID_ARG;
    if (!aligned16(H) || !aligned16(inv_s_out)) return MACAQ_ERR_MISALIGNED;
    const int64_t slabs = round_up(N, 128) / 128;
    if (slabs > 65535) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    DeviceInfo* dev = nullptr;
    st = device_info(&dev);
    if (st != MACAQ_OK) return st;
    HessianPrepParams hp{static_cast<const uint16_t*>(W_bf16), s, H, w_codes, w_scales, inv_s_out, N, K, ldw,
                         round_up(K / 32, 8)};
    const dim3 grid((unsigned)hp.kb_pad, (unsigned)slabs);
    return launch_pdl(prepare_weight_hessian_kernel, grid, dim3(128), 0, (cudaStream_t)stream, hp) == cudaSuccess
               ? MACAQ_OK
               : MACAQ_ERR_CUDA;
}

size_t macaq_hessian_full_workspace_bytes(int64_t T, int64_t K) {
    if (T < 1 || K < 32 || K % 32 != 0) return 0;
    return (size_t)round_up(T * K * 4, 256);
}

macaq_status macaq_hessian_full(const void* x_bf16, int64_t T, int64_t K, int64_t ldx, const float* s, double* H,
                                void* workspace, size_t ws_bytes, macaq_stream stream) {
    if (!x_bf16 || !s || !H) return MACAQ_ERR_INVALID_ARG;
    if (T < 1 || K < 32 || ldx < K) return MACAQ_ERR_INVALID_ARG;
    if (K % 32 != 0 || T > kMaxRows || K > kMaxFlipK) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(s) || !aligned16(H) || ldx % 8 != 0) return MACAQ_ERR_MISALIGNED;
    const size_t need = macaq_hessian_full_workspace_bytes(T, K);
    if (!workspace || ws_bytes < need) return MACAQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MACAQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    macaq_status st = device_info(&dev);
    if (st != MACAQ_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    float* xt = static_cast<float*>(workspace);
    TransformParams tp{static_cast<const uint16_t*>(x_bf16), s, xt, T, K, ldx, 1};
    const int64_t blocks = std::min<int64_t>(cdiv(T * (K / 32), 128), (int64_t)dev->num_sms * 16);
    if (launch_pdl(transform_rows_kernel, dim3((unsigned)blocks), dim3(128), 0, cs, tp) != cudaSuccess)
        return MACAQ_ERR_CUDA;
    const int64_t nb = K / 32;
    GramParams gp{xt, H, T, K};
    if (launch_pdl(gram_tile_kernel, dim3((unsigned)(nb * (nb + 1) / 2)), dim3(1024), 0, cs, gp) != cudaSuccess)
        return MACAQ_ERR_CUDA;
    return MACAQ_OK;
}

size_t macaq_flip_workspace_bytes(int64_t N, int64_t K) {
    if (N < 1 || K < 32 || K % 32 != 0) return 0;
    return (size_t)round_up(N * K * 4, 256) + (size_t)round_up(N * K * 8, 256);
}

macaq_status macaq_flip_refine(const void* W_bf16, int64_t N, int64_t K, int64_t ldw, const float* s, const double* H,
                               uint8_t* w_codes, const uint8_t* w_scales, int max_rounds, int32_t* moves,
                               void* workspace, size_t ws_bytes, macaq_stream stream) {
    macaq_status st = check_quant_args(W_bf16, N, K, ldw, s, w_codes, w_scales);
    if (st != MACAQ_OK) return st;
    if (!H || !moves || max_rounds < 0) return MACAQ_ERR_INVALID_ARG;
    if (K > kMaxFlipK || cdiv(N, 64) > 65535) return MACAQ_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(H) || !aligned16(moves)) return MACAQ_ERR_MISALIGNED;
    const size_t need = macaq_flip_workspace_bytes(N, K);
    if (!workspace || ws_bytes < need) return MACAQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MACAQ_ERR_MISALIGNED;
    DeviceInfo* dev = nullptr;
    st = device_info(&dev);
    if (st != MACAQ_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    float* wv = static_cast<float*>(workspace);
    double* G = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + round_up(N * K * 4, 256));
    const int64_t kb_pad = round_up(K / 32, 8);
    TransformParams tp{static_cast<const uint16_t*>(W_bf16), s, wv, N, K, ldw, 0};
    const int64_t blocks = std::min<int64_t>(cdiv(N * (K / 32), 128), (int64_t)dev->num_sms * 16);
    if (launch_pdl(transform_rows_kernel, dim3((unsigned)blocks), dim3(128), 0, cs, tp) != cudaSuccess)
        return MACAQ_ERR_CUDA;
    FlipGradParams fg{wv, w_codes, w_scales, H, G, N, K, kb_pad};
    if (launch_pdl(flip_gradient_kernel, dim3((unsigned)cdiv(K, 64), (unsigned)cdiv(N, 64)), dim3(256), 0, cs, fg) !=
        cudaSuccess)
        return MACAQ_ERR_CUDA;
    const size_t smem = flip_rounds_smem(K);
    static std::atomic<uint64_t> configured{0};
    int devid = 0;
    cudaGetDevice(&devid);
    if (!(configured.load() & (1ull << (devid & 63)))) {
        if (cudaFuncSetAttribute(flip_rounds_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)flip_rounds_smem(kMaxFlipK)) != cudaSuccess)
            return MACAQ_ERR_CUDA;
        configured.fetch_or(1ull << (devid & 63));
    }
    FlipRoundParams fr{wv, w_codes, w_scales, H, G, moves, N, K, kb_pad, max_rounds};
    if (launch_pdl(flip_rounds_kernel, dim3((unsigned)N), dim3(kFlipThreads), smem, cs, fr) != cudaSuccess)
        return MACAQ_ERR_CUDA;
    return MACAQ_OK;
}

}  // extern "C"

namespace {
// Results of macaq_selftest_wait_timeout (the device error word is not used).
__device__ long long g_selftest_out[macaq::kSelftestWords];
}  // namespace

extern "C" {

macaq_status macaq_selftest_wait_timeout(uint32_t limit_us, int64_t* result, macaq_stream stream) {
    if (!result || limit_us < 1 || limit_us > 1000000) return MACAQ_ERR_INVALID_ARG;
    DeviceInfo* dev = nullptr;
    const macaq_status st = device_info(&dev);
    if (st != MACAQ_OK) return st;
    void* out = nullptr;
    if (cudaGetSymbolAddress(&out, g_selftest_out) != cudaSuccess) return MACAQ_ERR_CUDA;
    wait_selftest_kernel<<<2, 96, 0, stream>>>((uint64_t)limit_us * 1000u, static_cast<long long*>(out));
    if (cudaGetLastError() != cudaSuccess) return MACAQ_ERR_CUDA;
    long long host[kSelftestWords];
    if (cudaMemcpyAsync(host, out, sizeof host, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return MACAQ_ERR_CUDA;
    for (int i = 0; i < kSelftestWords; ++i) result[i] = host[i];
    return MACAQ_OK;
}

macaq_status macaq_get_device_error(void) {
    DeviceInfo* dev = nullptr;
    macaq_status st = device_info(&dev);
    if (st != MACAQ_OK) return st;
    if (cudaDeviceSynchronize() != cudaSuccess) return MACAQ_ERR_CUDA;
    int v = 0, zero = 0;
    if (cudaMemcpy(&v, dev->err_ptr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MACAQ_ERR_CUDA;
    if (v != 0 && cudaMemcpy(dev->err_ptr, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
        return MACAQ_ERR_CUDA;
    return v != 0 ? MACAQ_ERR_DEVICE_TIMEOUT : MACAQ_OK;
}

const char* macaq_status_string(macaq_status s) {
    switch (s) {
        case MACAQ_OK: return "MACAQ_OK";
        case MACAQ_ERR_INVALID_ARG: return "MACAQ_ERR_INVALID_ARG";
        case MACAQ_ERR_MISALIGNED: return "MACAQ_ERR_MISALIGNED";
        case MACAQ_ERR_UNSUPPORTED_SHAPE: return "MACAQ_ERR_UNSUPPORTED_SHAPE";
        case MACAQ_ERR_UNSUPPORTED_DEVICE: return "MACAQ_ERR_UNSUPPORTED_DEVICE";
        case MACAQ_ERR_CUDA: return "MACAQ_ERR_CUDA";
        case MACAQ_ERR_DEVICE_TIMEOUT: return "MACAQ_ERR_DEVICE_TIMEOUT";
        case MACAQ_ERR_WORKSPACE: return "MACAQ_ERR_WORKSPACE";
        case MACAQ_ERR_UNSUPPORTED: return "MACAQ_ERR_UNSUPPORTED";
    }
    return "MACAQ_ERR_UNKNOWN";
}

int macaq_version(void) { return MACAQ_VERSION; }

}  // extern "C"
