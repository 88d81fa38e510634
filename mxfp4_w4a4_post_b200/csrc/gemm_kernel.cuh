// Block-scaled FP4 GEMM for the MACaQ W4A4 layer on Blackwell tensor cores (sm_100a).
//
//   D[p, q] = sum_b 2^(e_P[p,b] + e_Q[q,b]) * sum_{k in block b} dec(P[p,k]) dec(Q[q,k])
//
// P (the "M-slot" operand, 128-row tiles) and Q (the "N-slot" operand, BN-row tiles)
// are MXFP4: packed E2M1 codes, K-major, plus E8M0 scales in the 128x4 atom layout.
// For prefill P = activations and Q = weights, D = y. For decode the roles swap
// (P = weights, so the 128-wide MMA M dimension covers output features and the few
// tokens become the MMA N dimension), and the epilogue writes D transposed.
//
// One persistent CTA per SM, warp-specialised:
//   warp 0      TMA producer: codes via 2D tensor maps with the 128-byte swizzle (one
//               256-element K tile = 128 bytes per row), scale atoms via bulk copies.
//               The producer and the MMA issuer run their loops on the whole warp, so
//               every address and descriptor is a warp-uniform value, and one elected
//               lane issues.
//   warp 1      TMEM owner and single-thread MMA issuer: four tcgen05.mma
//               kind::mxf4.block_scale (K = 64 each) per K tile into an fp32 TMEM
//               accumulator (for narrow tiles, into 2 or 4 partial accumulators in
//               turn, summed by the epilogue)
//   warps 2-5   epilogue: tcgen05.ld the accumulator (each warp owns one 32-lane TMEM
//               subpartition), convert, and either stage 32-row boxes in shared memory
//               for TMA tensor stores (wide row-major tiles) or store directly (decode's
//               transposed tiles, unaligned outputs). With split K every split adds its
//               fp32 partial into a workspace accumulator (zeroed by the kernel itself)
//               with vector reductions; a small kernel then writes y from it.
//   warps 6-13  scale-factor writers, two sets of four taking alternate K tiles: each
//               warp reads the scale atoms of a K tile from shared memory and writes
//               them into its TMEM subpartition with tcgen05.st, so the tensor pipe
//               executes nothing but MMAs
// Accumulators are double-buffered in TMEM when they fit, so the epilogue of one tile
// overlaps the MMAs of the next. Every mbarrier wait is bounded by a wall-clock limit;
// a kernel that gives up records an error code, drains what it issued, frees its TMEM
// and returns. The one split-K wait (for every CTA to have zeroed its slice of the
// workspace, done first thing) always ends: all CTAs are resident at once (grid <= SMs,
// one CTA per SM). It is bounded all the same.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "quant_kernel.cuh"

namespace macaq {

// One group of a grouped GEMM: its P rows, its own weight (tensor map alongside, scale
// atoms sf_q) with q_rows rows, and its own output (row row_y of out, row stride ldo).
struct GemmGroup {
    int32_t unit_begin, rows, row_p, row_y;
    int32_t q_rows, tiles_q;
    const uint8_t* sf_q;
    void* out;
    int64_t ldo;
};

// Largest number of destinations of a gathered output.
constexpr int kMaxGatherDest = 64;

struct GemmParams {
    const uint8_t* sf_p;     // scale atoms of P
    const uint8_t* sf_q;     // scale atoms of Q
    void* out;               // y
    int64_t ldo;             // leading dimension of out, elements
    int32_t p_rows, q_rows;  // logical rows of P and Q
    int32_t k_tiles;         // ceil(K / 256)
    int32_t kb4_pad;         // scale atoms per 128-row slab along K
    int32_t tiles_p, tiles_q;
    int32_t total_units;     // tiles (grouped: every group's tiles)
    int32_t group_p;         // raster group height (in P tiles)
    int32_t out_bf16;        // 1: bf16 output, 0: fp32
    int32_t transpose_out;   // 1: out[q * ldo + p], 0: out[p * ldo + q]
    int32_t vec_ok;          // 1: out and ldo allow 16-byte vector stores
    int32_t tma_store;       // 1: epilogue stages 32 x 32 output boxes in shared memory and
                             //    writes them with TMA stores (row-major tiles, vec_ok)
    int* err;                // device error word
    // Schedule (ungrouped). Tiles [0, sk_tile0) are whole units dealt round robin: CTA c
    // takes tiles c, c + G, .. (G = gridDim.x). The K tiles of tiles [sk_tile0,
    // total_units), tile after tile, form one sequence of sk_iters iterations that is
    // split evenly over the CTAs (stream-K): CTA c takes iterations [c I / G, (c + 1) I / G)
    // of it (G = sk_ctas, I = sk_iters), before its whole tiles, so a CTA's share of the
    // grid's work differs from another's by at most one K tile. A tile whose K tiles fall to several CTAs is
    // finished by the last of them to arrive: each writes its fp32 partial tile into its
    // own slot of sk_partials (two per CTA: the first and the last tile of its stream-K
    // range), counts itself in on the tile's counter, and the one that completes the count
    // adds the partials in the order of their K ranges and writes y. No CTA ever waits for
    // another, and as the stream-K tiles come first, a finisher's epilogue runs while its
    // MMAs go on with its whole tiles. A counter holds the call's tag in its upper 48
    // bits, so counts left by earlier calls (or whatever the workspace held) read as zero.
    int32_t sk_tile0;                // first stream-K tile (total_units: none)
    int32_t sk_ctas;                 // CTAs 0 .. sk_ctas - 1 share the stream-K iterations
                                     // (at most sk_iters: every share is non-empty)
    int64_t sk_iters;                // (total_units - sk_tile0) * k_tiles
    float* sk_partials;              // [G][2][128 x BN] fp32
    unsigned long long* sk_counters; // [total_units]
    unsigned long long sk_tag;       // 48-bit tag unique to the call
    // Fused activation transform (the kernel's FUSED instantiation; decode, Q =
    // activations, one Q tile): the scale-factor warps transform the bf16 activation K
    // tile themselves (per-channel multiplier, block Hadamard, E8M0 exponent, E2M1 codes)
    // and write the codes into the stage's Q buffer and the scales into its Q scale
    // chunk, in the layouts the TMA would have written; only the weight side is copied.
    const uint16_t* fx;              // bf16 activations [q_rows x f_K], row stride fx_ld
    int64_t fx_ld;
    const float* f_mult;             // inv_s [f_K]
    int32_t f_K;
    // Grouped GEMM (groups > 0; prefill orientation, every tile whole): group g multiplies
    // its rows activation rows starting at P row row_p (a multiple of 128: groups sit in
    // whole scale slabs) by its own weight (tensor map g_tmaps[g], q_rows rows, scale atoms
    // sf_q) and writes rows row_y .. of its own output; its units are unit_begin ..
    // unit_begin + ceil(rows / 128) * tiles_q - 1, P tiles fastest.
    int32_t groups;
    const GemmGroup* g_desc;         // [groups]
    const CUtensorMap* g_tmaps;      // [groups], 64-byte aligned
    // Gathered output (column-parallel layers; the kernel's GATHER instantiation): every
    // output element goes to each of dest[0 .. n_dest - 1] (device addresses of the
    // destinations' first column for this weight, the same row stride ldo) instead of to
    // out, with direct stores (no TMA store, no stream-K schedule). The addresses travel
    // in the kernel's parameters.
    int32_t n_dest;
    unsigned long long dest[kMaxGatherDest];
    // 1: the producer may copy the weight side of its first fills before waiting for the
    // previous kernel on the stream (set by the layer entry points, which launch their
    // own activation transform just before the GEMM)
    int32_t w_early;
    // K split over a cluster (the kernel's SPLIT instantiation): `split` CTAs per cluster,
    // one output tile per cluster, CTA r accumulating K tiles [r k / split, (r + 1) k /
    // split) of it; CTA 0 adds the others' partial tiles, read from their shared memory.
    int32_t split;
};

enum : int {
    kErrTimeoutProducer = 1,
    kErrTimeoutMma = 2,
    kErrTimeoutEpilogue = 3,
    kErrSfOffset = 4,
    kErrTimeoutSet = 5,
    kErrPlan = 6              // a cluster launch the K-split kernel is not planned for
};

template <int BN, int STAGES>
struct GemmShape {
    // Q tiles start on a 64-row boundary of the 128-row scale slabs (offset 0 or 2 TMEM
    // columns), the only scale-factor column offsets the MMA is given.
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128 || BN == 192,
                  "unsupported tile width");
    static constexpr int kBM = 128;
    static constexpr int kBKBytes = 128;                    // 256 FP4 elements per row
    static constexpr int kPTileBytes = kBM * kBKBytes;      // 16 KB
    static constexpr int kQTileBytes = BN * kBKBytes;
    static constexpr int kSfChunkBytes = 1024;              // 128 rows x 8 scale blocks
    // 128-row scale slabs a Q tile can touch (a 192-row tile may start 64 rows into one)
    static constexpr int kQChunks = (BN <= 128) ? 1 : 2;
    static constexpr int kSfCols = 8 + 8 * kQChunks;        // 4 columns per atom, 2 atoms per tile
    // Narrow tiles split each accumulator into kSub independent partial sums: the four
    // MMAs of a K tile rotate over them, so consecutive MMAs do not wait on one another's
    // result (a 128 x BN x 64 MMA is short next to its latency when BN is small), and the
    // epilogue adds the partial sums.
    static constexpr int kSub = BN <= 32 ? 4 : BN == 64 ? 2 : 1;
    // TMEM: two fp32 accumulators of kSub x BN columns side by side, then one
    // scale-factor slot per pipeline stage (the K tile in stage s uses slot s).
    static constexpr int kNumAcc = 2;
    static constexpr int kAccStride = kSub * BN;
    static constexpr int kSfBase = kNumAcc * kAccStride;
    static constexpr int kTmemNeed = kSfBase + STAGES * kSfCols;
    static_assert(kTmemNeed <= 512, "tensor memory budget");
    static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64
                                   : kTmemNeed <= 128 ? 128 : kTmemNeed <= 256 ? 256 : 512;
    static constexpr int kChunkCols = BN <= 64 ? 16 : 32;   // epilogue TMEM load width
    // Output staging for TMA stores (wide tiles only): one box of 32 rows x 64 bytes
    // (32 bf16 or 16 fp32 columns) per epilogue warp.
    static constexpr int kStageBoxBytes = 32 * 64;
    static constexpr int kStagingBytes = BN >= 128 ? 4 * kStageBoxBytes : 0;
};

template <int BN, int STAGES, bool FUSED = false, bool PAIR = false>
struct GemmSmem {
    using S = GemmShape<BN, STAGES>;
    // the fused variant keeps its Q operand for every K tile in one persistent region
    // after the fixed layout instead of in the stage ring
    static constexpr int kQRing = FUSED ? 0 : 1;
    // a CTA of a pair holds half of the Q tile's rows (and the scales of all of them)
    static constexpr int kQStageBytes = PAIR ? S::kQTileBytes / 2 : S::kQTileBytes;
    static constexpr int kOffP = 0;
    static constexpr int kOffQ = kOffP + STAGES * S::kPTileBytes;
    static constexpr int kOffSfP = kOffQ + kQRing * STAGES * kQStageBytes;
    static constexpr int kOffSfQ = kOffSfP + STAGES * S::kSfChunkBytes;
    static constexpr int kOffStaging = kOffSfQ + kQRing * STAGES * S::kQChunks * S::kSfChunkBytes;   // 1 KB aligned
    static constexpr int kOffBar = kOffStaging + S::kStagingBytes;
    static constexpr int kNumBars = 3 * STAGES + 4 + 1 + 2;    // ..., sf_full[STAGES], part_full, ring_free
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffMisc + 16;
    // fused: Q codes of K tile kt at kOffPersist + kt * BN * 128 (128-byte swizzle, as the
    // copies of the plain kernel lay them out), then its scale atoms (1 KB per K tile)
    static constexpr int kOffPersist = (kBytes + 1023) / 1024 * 1024;
    static constexpr int kPersistPerKt = S::kQTileBytes + S::kSfChunkBytes;
    static constexpr int kAlloc = kBytes + 1024;            // slack to align the base to 1 KB
    static constexpr int alloc(int k_tiles) { return FUSED ? kOffPersist + k_tiles * kPersistPerKt + 1024 : kAlloc; }
};

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Longest a kernel waits on one barrier or flag before it gives up.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __noinline__ bool wait_or_abort_slow(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                int* err, int code, uint64_t limit_ns);

// Wait for `parity` on `bar`, giving up after limit_ns (or as soon as another role of
// the CTA has given up). On give-up record `code`, raise the CTA abort flag, return
// false. mbarrier.try_wait suspends the thread in hardware until the phase completes or
// a short hardware time limit passes, so the loop just polls again; the wall clock and
// the abort flag are read every 16 polls.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort,
                                              int* err, int code, uint64_t limit_ns = kWaitLimitNs) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    return wait_or_abort_slow(bar, parity, abort, err, code, limit_ns);
}

__device__ __noinline__ bool wait_or_abort_slow(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                int* err, int code, uint64_t limit_ns) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 0) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                atomicExch(err, code);
                *abort = 1;
                return false;
            }
        }
    }
}

// The CTA abort flag as a warp-uniform value.
__device__ __forceinline__ bool cta_aborted(volatile int* abort) { return __any_sync(0xffffffffu, *abort != 0); }

// wait_or_abort by every lane of a warp, with a warp-uniform result: false if any lane
// gave up.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* err,
                                          int code, uint64_t limit_ns = kWaitLimitNs) {
    return __all_sync(0xffffffffu, wait_or_abort(bar, parity, abort, err, code, limit_ns));
}

// Named barrier `id` over `nthreads` threads (whole warps) that also returns, to every
// thread, whether `v` held in all of them.
__device__ __forceinline__ bool bar_and(int id, int nthreads, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

struct Unit {
    int tile, tp, tq, kt_begin, kt_end;
    int p_row0;                    // first P row of the tile in the P tensor map
    int out_row0;                  // output row of the tile's P row 0
    int rows;                      // valid P rows from p_row0 on (the tile's group)
    int q_rows;                    // rows of the tile's Q operand (its group's)
    const CUtensorMap* tmap_q;     // Q tensor map of the tile
    const uint8_t* sf_q;           // Q scale atoms of the tile
    void* out;                     // the tile's output and its row stride
    int64_t ldo;
};

// The units a CTA works through, in order: its stream-K tiles sk_first .. sk_first +
// n_sk - 1 (the tiles that hold iterations [i0, i1) of the stream-K sequence, each
// clipped to the K tiles in that range), then its whole tiles blockIdx.x, blockIdx.x + G,
// .. below sk_tile0 (grouped GEMM: every tile is whole).
struct Sched {
    int n_sk, sk_first, n_units;
    int base, stride;            // whole tiles base, base + stride, ..
    int64_t i0, i1;
    __device__ __forceinline__ int unit(int j) const {
        return j < n_sk ? sk_first + j : base + (j - n_sk) * stride;
    }
};

__device__ __forceinline__ int64_t sk_start(const GemmParams& p, int c) {
    return (int64_t)c * p.sk_iters / p.sk_ctas;
}

// cluster > 1: the CTAs of a cluster work through the same units (G = gridDim.x /
// cluster).
__device__ __forceinline__ Sched cta_sched(const GemmParams& p, int cluster = 1) {
    Sched s;
    const int whole = p.groups > 0 ? p.total_units : p.sk_tile0;
    s.base = (int)blockIdx.x / cluster;
    s.stride = (int)gridDim.x / cluster;
    s.i0 = 0;
    s.i1 = 0;
    s.n_sk = 0;
    s.sk_first = 0;
    if (p.groups == 0 && p.sk_iters > 0 && (int)blockIdx.x < p.sk_ctas) {
        s.i0 = sk_start(p, blockIdx.x);
        s.i1 = sk_start(p, blockIdx.x + 1);
        if (s.i1 > s.i0) {
            s.sk_first = p.sk_tile0 + (int)(s.i0 / p.k_tiles);
            s.n_sk = p.sk_tile0 + (int)((s.i1 - 1) / p.k_tiles) + 1 - s.sk_first;
        }
    }
    const int n_whole = s.base < whole ? (whole - 1 - s.base) / s.stride + 1 : 0;
    s.n_units = s.n_sk + n_whole;
    return s;
}

// The CTA whose stream-K range holds iteration j: the largest c with c I / G <= j (every
// range is non-empty, as G <= I, so the CTAs from the holder of a tile's first K tile to
// the holder of its last are exactly its contributors).
__device__ __forceinline__ int sk_cta_of(const GemmParams& p, int64_t j) {
    return (int)(((j + 1) * p.sk_ctas - 1) / p.sk_iters);
}

// rank >= 0: CTA `rank` of a pair, whose unit is a 256-row tile (tp counts 256 rows) of
// which this CTA holds rows 128 rank .. 128 rank + 127; or, with p.split > 1, CTA `rank`
// of a K-split cluster, which has the whole tile and its share of the K tiles.
__device__ __forceinline__ Unit decode_unit(const GemmParams& p, int u, const CUtensorMap* tmap_q, const Sched& sc,
                                            int rank = -1) {
    if (p.groups > 0) {
        // the group whose units contain u: binary search over the unit offsets
        int lo = 0, hi = p.groups - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.g_desc[mid].unit_begin <= u) lo = mid; else hi = mid - 1;
        }
        const GemmGroup gd = p.g_desc[lo];
        const int tiles_p = (gd.rows + 127) >> 7;
        const int lu = u - gd.unit_begin;
        Unit x;
        x.tile = u;
        x.tp = lu % tiles_p;
        x.tq = lu / tiles_p;
        x.kt_begin = 0;
        x.kt_end = p.k_tiles;
        x.p_row0 = gd.row_p + x.tp * 128;
        x.out_row0 = gd.row_y + x.tp * 128;
        x.rows = gd.rows - x.tp * 128;
        x.q_rows = gd.q_rows;
        x.tmap_q = p.g_tmaps + lo;
        x.sf_q = gd.sf_q;
        x.out = gd.out;
        x.ldo = gd.ldo;
        if (p.split > 1 && rank >= 0) {
            x.kt_begin = rank * p.k_tiles / p.split;
            x.kt_end = (rank + 1) * p.k_tiles / p.split;
        }
        return x;
    }
    const int tile = u;
    const int per_group = p.group_p * p.tiles_q;
    const int g = tile / per_group;
    const int r = tile - g * per_group;
    const int gp = min(p.group_p, p.tiles_p - g * p.group_p);
    Unit x;
    x.tile = tile;
    x.tp = g * p.group_p + r % gp;
    x.tq = r / gp;
    x.kt_begin = 0;
    x.kt_end = p.k_tiles;
    if (tile >= p.sk_tile0) {
        // a stream-K tile: the K tiles of it in this CTA's range
        const int64_t t0 = (int64_t)(tile - p.sk_tile0) * p.k_tiles;
        x.kt_begin = (int)(max(sc.i0, t0) - t0);
        x.kt_end = (int)(min(sc.i1, t0 + p.k_tiles) - t0);
    }
    if (p.split > 1 && rank >= 0) {
        // a K-split cluster: every CTA has the whole tile, and its share of the K range
        x.kt_begin = rank * p.k_tiles / p.split;
        x.kt_end = (rank + 1) * p.k_tiles / p.split;
        rank = -1;
    }
    x.p_row0 = rank >= 0 ? x.tp * 256 + rank * 128 : x.tp * 128;
    x.out_row0 = x.p_row0;
    x.rows = p.p_rows - x.p_row0;
    x.q_rows = p.q_rows;
    x.tmap_q = tmap_q;
    x.sf_q = p.sf_q;
    x.out = p.out;
    x.ldo = p.ldo;
    return x;
}

// Stream-K: count this CTA in on a tile's counter; returns the count including this
// arrival (1 for the first arrival of the call). Lock-free: the compare-and-swap loop
// only retries when another contributor of the same tile arrived in between.
__device__ __forceinline__ uint32_t sk_arrive(unsigned long long* ctr, unsigned long long tag) {
    // first guess: no arrival of this call yet (saves a read before the swap)
    unsigned long long cur = tag << 16;
    for (;;) {
        const uint32_t n = (cur >> 16) == tag ? (uint32_t)(cur & 0xFFFFu) : 0u;
        const unsigned long long next = (tag << 16) | (unsigned long long)(n + 1);
        const unsigned long long prev = atomicCAS(ctr, cur, next);
        if (prev == cur) return n + 1;
        cur = prev;
    }
}

// Writes one chunk of output row `prow` (a P row; the output column of it when
// transposed) if `valid`, into `out` with row stride ldo and q_rows columns (rows when
// transposed).
template <int CW>
__device__ __forceinline__ void store_chunk(const GemmParams& p, void* out, int64_t ldo, int q_rows, int prow,
                                            bool valid, int q_base, const uint32_t (&r)[CW]) {
    if (!valid) return;
    if (p.transpose_out) {
        // out[q, prow]: for each column the 32 lanes of the warp write consecutive prow
        if (p.out_bf16) {
            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
#pragma unroll
            for (int j = 0; j < CW; ++j) {
                const int q = q_base + j;
                if (q < q_rows) o[(int64_t)q * ldo + prow] = __float2bfloat16_rn(__uint_as_float(r[j]));
            }
        } else {
            float* o = reinterpret_cast<float*>(out);
#pragma unroll
            for (int j = 0; j < CW; ++j) {
                const int q = q_base + j;
                if (q < q_rows) o[(int64_t)q * ldo + prow] = __uint_as_float(r[j]);
            }
        }
        return;
    }
    const bool full = q_base + CW <= q_rows && p.vec_ok;
    if (p.out_bf16) {
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + (int64_t)prow * ldo + q_base;
        if (full) {
#pragma unroll
            for (int j = 0; j < CW; j += 8) {
                uint4 v;
                __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(r[j + 0]), __uint_as_float(r[j + 1]));
                __nv_bfloat162 h1 = __floats2bfloat162_rn(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[j + 4]), __uint_as_float(r[j + 5]));
                __nv_bfloat162 h3 = __floats2bfloat162_rn(__uint_as_float(r[j + 6]), __uint_as_float(r[j + 7]));
                v.x = *reinterpret_cast<uint32_t*>(&h0);
                v.y = *reinterpret_cast<uint32_t*>(&h1);
                v.z = *reinterpret_cast<uint32_t*>(&h2);
                v.w = *reinterpret_cast<uint32_t*>(&h3);
                *reinterpret_cast<uint4*>(o + j) = v;
            }
        } else {
#pragma unroll
            for (int j = 0; j < CW; ++j)
                if (q_base + j < q_rows) o[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
        }
    } else {
        float* o = reinterpret_cast<float*>(out) + (int64_t)prow * ldo + q_base;
        if (full) {
#pragma unroll
            for (int j = 0; j < CW; j += 4)
                *reinterpret_cast<float4*>(o + j) =
                    make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
        } else {
#pragma unroll
            for (int j = 0; j < CW; ++j)
                if (q_base + j < q_rows) o[j] = __uint_as_float(r[j]);
        }
    }
}

template <int CW>
__device__ __forceinline__ void tmem_load_chunk(uint32_t taddr, uint32_t (&r)[CW]);

template <>
__device__ __forceinline__ void tmem_load_chunk<32>(uint32_t taddr, uint32_t (&r)[32]) {
    ptx::tmem_ld_32x32b_x32(taddr, r);
}

template <>
__device__ __forceinline__ void tmem_load_chunk<16>(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

constexpr int kSfWarpSets = 2;                                // scale-writer sets
constexpr int kGemmThreads = 32 * (6 + 4 * kSfWarpSets);

// Kernel variants, each its own instantiation so that the ordinary kernels keep their
// registers: kVarGather writes the output to p.dest[0 .. p.n_dest - 1]; kVarFused makes
// the Q operand (the activations) from bf16 inside the kernel; kVarPair runs on clusters
// of two CTAs, each pair computing 256 x BN tiles with cta_group::2 MMAs (prefill);
// kVarSplit runs on clusters of p.split CTAs that share one tile's K range.
enum : int { kVarPlain = 0, kVarGather = 1, kVarFused = 2, kVarPair = 3, kVarSplit = 4 };

// Largest K split over a cluster.
constexpr int kMaxSplit = 4;

// Whether a ring of `ring_bytes` holds what a K-split CTA keeps there: its parked partial
// tile (128 x BN fp32) and the other split - 1 CTAs' slices of its own output chunks
// (ceil(NCH / split) chunks of 128 x 32 fp32 at most).
template <int BN>
__host__ __device__ constexpr bool split_ring_fits(int split, int ring_bytes) {
    constexpr int kChunks = BN / 32;
    return split >= 2 && 128 * BN * 4 + (split - 1) * ((kChunks + split - 1) / split) * 128 * 32 * 4 <= ring_bytes;
}

// The fused variant's Q operand, made once per CTA before its main loop by warps 2-13
// (the epilogue and scale-factor warps; the producer starts streaming the weight tiles
// meanwhile and the MMA warp waits for its first scale slot): the MXFP4 form of the
// activation's q_rows (<= BN) rows for every K tile, with the quantiser's own block
// routine, written where the copies of the plain kernel would have put each K tile:
// codes at kOffPersist + kt * BN * 128 in the 128-byte swizzle (16-byte piece j of row r
// at j ^ (r % 8)), scales in a 1 KB atom chunk per K tile after them. Rows past the last
// activation row get zero codes, blocks past K zero codes and scale byte 0 (what the
// zero-filled copies give). Item i = (K tile, row, block) goes to thread i % 384 of the
// warps, so four consecutive lanes hold the four blocks of one scale word.
constexpr int kFusedThreads = 32 * (4 + 4 * kSfWarpSets);

template <int BN, int STAGES>
__device__ __forceinline__ void fused_transform(const GemmParams& p, uint8_t* smem) {
    using S = GemmShape<BN, STAGES>;
    using L = GemmSmem<BN, STAGES, true>;
    const int tt = (int)threadIdx.x - 64;              // 0 .. kFusedThreads - 1
    const int rows = p.q_rows;
    const int kb = p.f_K >> 5;
    const uint32_t qp = ptx::smem_u32(smem + L::kOffPersist);
    const uint32_t sp = qp + p.k_tiles * S::kQTileBytes;
    const int zero_items = (BN - rows) * 8;            // 16-byte pieces of rows past the last
    for (int i = tt; i < p.k_tiles * zero_items; i += kFusedThreads) {
        const int kt = i / zero_items, rem = i - kt * zero_items;
        ptx::sts128(qp + kt * S::kQTileBytes + (rows + rem / 8) * 128 + (rem % 8) * 16, 0u, 0u, 0u, 0u);
    }
    for (int i = tt; i < p.k_tiles * S::kSfChunkBytes / 16; i += kFusedThreads) ptx::sts128(sp + 16 * i, 0u, 0u, 0u, 0u);
    asm volatile("bar.sync 2, %0;" ::"n"(kFusedThreads) : "memory");   // zeros before scale words
    const int total = p.k_tiles * rows * 8;
    // item i -> (K tile, row, block); the activation load of a thread's next item is
    // issued before its current item is encoded, so its latency overlaps the encoding
    auto item = [&](int i, int& kt, int& r, int& j) {
        kt = i / (rows * 8);
        const int rem = i - kt * rows * 8;
        r = rem >> 3;
        j = rem & 7;
    };
    auto load_x = [&](int i, uint4 (&xv)[4]) {
        int kt, r, j;
        item(i, kt, r, j);
        const int b = kt * 8 + j;
        if (i < total && b < kb) {
            const uint4* xs = reinterpret_cast<const uint4*>(p.fx + (int64_t)r * p.fx_ld + (int64_t)b * 32);
#pragma unroll
            for (int c = 0; c < 4; ++c) xv[c] = __ldg(xs + c);
        }
    };
    uint4 nx[4];
    load_x(tt, nx);
    for (int base = 0; base < total; base += kFusedThreads) {
        const int i = base + tt;
        const bool live = i < total;
        int kt = 0, r = 0, j = 0;
        if (live) item(i, kt, r, j);
        uint4 xv[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) xv[c] = nx[c];
        load_x(i + kFusedThreads, nx);
        const int b = kt * 8 + j;
        uint32_t sbyte = 0;
        if (live) {
            uint32_t packed[4] = {0u, 0u, 0u, 0u};
            if (b < kb) {
                const float4* ms = reinterpret_cast<const float4*>(p.f_mult + (int64_t)b * 32);
                float4 mv[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) mv[c] = __ldg(ms + c);
                uint64_t T[16];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t w[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
                    const uint64_t mm[4] = {pk(mv[2 * c].x, mv[2 * c].y), pk(mv[2 * c].z, mv[2 * c].w),
                                            pk(mv[2 * c + 1].x, mv[2 * c + 1].y), pk(mv[2 * c + 1].z, mv[2 * c + 1].w)};
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        T[4 * c + q] =
                            mul2(pk(__uint_as_float(w[q] << 16), __uint_as_float(w[q] & 0xFFFF0000u)), mm[q]);
                }
                sbyte = encode_block(T, packed);
            }
            ptx::sts128(qp + kt * S::kQTileBytes + r * 128 + ((j ^ (r & 7)) << 4), packed[0], packed[1], packed[2],
                        packed[3]);
        }
        const uint32_t s1 = __shfl_down_sync(0xffffffffu, sbyte, 1);
        const uint32_t s2 = __shfl_down_sync(0xffffffffu, sbyte, 2);
        const uint32_t s3 = __shfl_down_sync(0xffffffffu, sbyte, 3);
        if (live && (j & 3) == 0)
            ptx::sts32(sp + kt * S::kSfChunkBytes + 512 * (j >> 2) + (r & 31) * 16 + ((r >> 5) & 3) * 4,
                       sbyte | (s1 << 8) | (s2 << 16) | (s3 << 24));
    }
    // the MMAs read the codes through the async proxy; the scale-factor warps read the
    // scale words after this barrier
    ptx::fence_proxy_async_smem();
    asm volatile("bar.sync 2, %0;" ::"n"(kFusedThreads) : "memory");
}

template <int BN, int STAGES, int VAR = kVarPlain>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_mxf4_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
    constexpr bool GATHER = VAR == kVarGather;
    constexpr bool FUSED = VAR == kVarFused;
    constexpr bool PAIR = VAR == kVarPair;
    constexpr bool SPLIT = VAR == kVarSplit;
    // The fused variant covers Q tiles of at most 32 rows (one 128-row scale slab).
    static_assert(!FUSED || BN <= 32, "fused transform tile");
    // A pair splits its Q tile in two halves of whole 8-row swizzle atoms; prefill only.
    static_assert(!PAIR || BN == 128 || BN == 192, "pair tile");
    using S = GemmShape<BN, STAGES>;
    using L = GemmSmem<BN, STAGES, FUSED, PAIR>;
    // A K-split CTA parks its fp32 partial tile in its pipeline ring once its MMAs are done
    // (wide tiles only: one accumulator per tile, no partial sums to add first).
    static_assert(!SPLIT || (BN >= 128 && 128 * BN * 4 <= STAGES * (S::kPTileBytes + S::kQTileBytes)),
                  "split partial tile");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* acc_full = bars + 2 * STAGES;
    uint64_t* acc_empty = bars + 2 * STAGES + 2;
    uint64_t* drain = bars + 2 * STAGES + 4;
    uint64_t* sf_full = bars + 2 * STAGES + 5;    // [STAGES]: scale-factor slot written
    uint64_t* part_full = bars + 3 * STAGES + 5;  // K split: the other CTAs' slices of this CTA's columns in
    uint64_t* ring_free = bars + 3 * STAGES + 6;  // K split: every other CTA's ring may take slices
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // CTA pair: rank 0 issues the MMAs of both; rank 1's scale-factor writers and
    // epilogue signal rank 0's sf_full and acc_empty barriers remotely, and rank 0's
    // commits arrive on both CTAs' stage and accumulator barriers.
    const int rank = PAIR || SPLIT ? (int)ptx::cluster_ctarank() : -1;
    constexpr uint32_t kPeerArrivals = PAIR ? 2 : 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&acc_full[a], 1);
            ptx::mbar_init(&acc_empty[a], 4 * kPeerArrivals);
        }
        ptx::mbar_init(drain, 1);
        for (int s = 0; s < STAGES; ++s) ptx::mbar_init(&sf_full[s], 4 * kPeerArrivals);
        // K split: a CTA arrives once on its own part_full (with the bytes the others copy
        // in), and once on every other CTA's ring_free
        ptx::mbar_init(part_full, 1);
        ptx::mbar_init(ring_free, SPLIT && p.split > 1 ? p.split - 1 : 1);
        *abort = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
        ptx::prefetch_tensormap(&tmap_p);
        if (p.groups == 0) ptx::prefetch_tensormap(&tmap_q);
        if (S::kStagingBytes > 0 && p.tma_store) ptx::prefetch_tensormap(&tmap_y);
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            ptx::tmem_alloc_pair(tmem_slot, S::kTmemCols);
            ptx::tmem_relinquish_pair();
        } else {
            ptx::tmem_alloc(tmem_slot, S::kTmemCols);
            ptx::tmem_relinquish();
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    // the other CTAs of a cluster signal this CTA's barriers only after they are set up
    if constexpr (PAIR || SPLIT) ptx::cluster_sync();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    Sched sc = cta_sched(p, PAIR ? 2 : SPLIT ? p.split : 1);
    if constexpr (SPLIT) {
        // planned: clusters of p.split CTAs (<= kMaxSplit), at most one tile per cluster
        // (partial tiles live in the rings after the MMAs), CTA 0's ring large enough for
        // the others' partial tiles; otherwise do nothing
        if ((int)ptx::cluster_nctarank() != p.split || p.split < 2 || p.split > kMaxSplit || sc.n_units > 1 ||
            !split_ring_fits<BN>(p.split, STAGES * (S::kPTileBytes + S::kQTileBytes))) {
            if (threadIdx.x == 0) atomicExch(p.err, kErrPlan);
            sc.n_units = 0;
        }
    }
    // Set-up above overlaps the previous kernel's tail; operands are read only after it.
    // (With w_early the producer copies the weight side of its first fills first and
    // waits after that.)
    if (warp != 0 || !p.w_early) ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    if constexpr (FUSED) {
        if (warp >= 2) fused_transform<BN, STAGES>(p, smem);
    }

    if (warp == 0) {
        // ------------------------------------------------------------ producer ---
        // The whole warp runs the loop, so addresses and coordinates are warp-uniform
        // values; one elected lane issues the copies.
        const bool leader = ptx::elect_one();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued_mask = 0, issued_phase = 0;
        // Q side of one fill: codes tile and scale chunks
        auto issue_q = [&](const Unit& t, int st, int kt, int q0, int slab0, int nchunks) {
            // a pair's CTA copies its half of the Q tile's rows, and the scales of all
            ptx::tma_load_2d(smem + L::kOffQ + st * L::kQStageBytes, t.tmap_q, &full[st], kt * S::kBKBytes,
                             PAIR ? q0 + rank * (BN / 2) : q0);
            for (int c = 0; c < nchunks; ++c)
                ptx::bulk_load(smem + L::kOffSfQ + (st * S::kQChunks + c) * S::kSfChunkBytes,
                               t.sf_q + ((int64_t)(slab0 + c) * p.kb4_pad + 2 * kt) * 512, S::kSfChunkBytes,
                               &full[st]);
        };
        // w_early: no kernel still running on the stream writes the weight (the library
        // launched its own activation transform just before, and that kernel starts its
        // work only after everything before it has completed), so the weight side of the
        // first fills, whose stages are still free, is copied before the wait for the
        // previous kernel; their activation side follows in the loop below. The weight is
        // P for decode's swapped tiles, Q otherwise. The main loop is instantiated twice so
        // that the one without early fills is the plain loop (a test per K tile in it cost
        // ~4% of the prefill GEMM).
        const bool p_is_weight = p.transpose_out != 0;
        int n_early = 0;
        if (p.w_early) {
            for (int uj = 0; uj < sc.n_units && n_early < STAGES; ++uj) {
                const Unit t = decode_unit(p, sc.unit(uj), &tmap_q, sc, rank);
                const int q0 = t.tq * BN;
                const int slab0 = q0 / 128;
                const int nchunks = min(S::kQChunks, (t.q_rows + 127) / 128 - slab0);
                const int slab_p = t.rows > 0 ? (t.p_row0 >> 7) : 0;
                const uint32_t bytes = FUSED ? S::kPTileBytes + S::kSfChunkBytes
                                             : S::kPTileBytes + L::kQStageBytes + S::kSfChunkBytes * (1 + nchunks);
                for (int kt = t.kt_begin; kt < t.kt_end && n_early < STAGES; ++kt, ++n_early) {
                    if (leader) {
                        ptx::mbar_arrive_expect_tx(&full[n_early], bytes);
                        if (p_is_weight) {
                            ptx::tma_load_2d(smem + L::kOffP + n_early * S::kPTileBytes, &tmap_p, &full[n_early],
                                             kt * S::kBKBytes, t.p_row0);
                            ptx::bulk_load(smem + L::kOffSfP + n_early * S::kSfChunkBytes,
                                           p.sf_p + ((int64_t)slab_p * p.kb4_pad + 2 * kt) * 512, S::kSfChunkBytes,
                                           &full[n_early]);
                        } else if constexpr (!FUSED) {
                            issue_q(t, n_early, kt, q0, slab0, nchunks);
                        }
                    }
                    __syncwarp();
                }
            }
            ptx::griddep_wait();
        }
        auto main_loop = [&](auto has_early) {
            constexpr bool kEarly = decltype(has_early)::value;
            int fills = 0;
            for (int uj = 0; uj < sc.n_units; ++uj) {
                const int u = sc.unit(uj);
                if (cta_aborted(abort)) break;
                const Unit t = decode_unit(p, u, &tmap_q, sc, rank);
                const int q0 = t.tq * BN;
                const int slab0 = q0 / 128;
                const int nchunks = min(S::kQChunks, (t.q_rows + 127) / 128 - slab0);   // scale slabs of the Q rows
                // P scale slab of the tile; a pair's second CTA past the last P row (its rows
                // are all zero-filled codes, and their results are never stored) reads slab 0
                const int slab_p = t.rows > 0 ? (t.p_row0 >> 7) : 0;
                // the fused variant copies only the weight side; its Q side is made in place
                const uint32_t bytes = FUSED ? S::kPTileBytes + S::kSfChunkBytes
                                             : S::kPTileBytes + L::kQStageBytes + S::kSfChunkBytes * (1 + nchunks);
                bool ok = true;
                for (int kt = t.kt_begin; kt < t.kt_end; ++kt) {
                    if (kEarly && fills < n_early) {
                        // an early fill: its activation side
                        if (leader) {
                            if (!p_is_weight) {
                                ptx::tma_load_2d(smem + L::kOffP + stage * S::kPTileBytes, &tmap_p, &full[stage],
                                                 kt * S::kBKBytes, t.p_row0);
                                ptx::bulk_load(smem + L::kOffSfP + stage * S::kSfChunkBytes,
                                               p.sf_p + ((int64_t)slab_p * p.kb4_pad + 2 * kt) * 512,
                                               S::kSfChunkBytes, &full[stage]);
                            } else if constexpr (!FUSED) {
                                issue_q(t, stage, kt, q0, slab0, nchunks);
                            }
                        }
                    } else {
                        if (!warp_wait(&empty[stage], phase ^ 1, abort, p.err, kErrTimeoutProducer)) {
                            ok = false;
                            break;
                        }
                        if (leader) {
                            ptx::mbar_arrive_expect_tx(&full[stage], bytes);
                            ptx::tma_load_2d(smem + L::kOffP + stage * S::kPTileBytes, &tmap_p, &full[stage],
                                             kt * S::kBKBytes, t.p_row0);
                            ptx::bulk_load(smem + L::kOffSfP + stage * S::kSfChunkBytes,
                                           p.sf_p + ((int64_t)slab_p * p.kb4_pad + 2 * kt) * 512, S::kSfChunkBytes,
                                           &full[stage]);
                            if constexpr (!FUSED) issue_q(t, stage, kt, q0, slab0, nchunks);
                        }
                    }
                    __syncwarp();
                    if constexpr (kEarly) ++fills;
                    issued_mask |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
        };
        if (n_early > 0) main_loop(std::true_type{});
        else main_loop(std::false_type{});
        if (cta_aborted(abort) && leader) {
            // let copies already in flight land before the CTA can exit: wait
            // (bounded) for the phase of the latest fill of every stage
            for (int s = 0; s < STAGES; ++s) {
                if (!((issued_mask >> s) & 1)) continue;
                const uint32_t ph = (issued_phase >> s) & 1;
                const uint64_t t0 = global_timer_ns();
                while (!ptx::mbar_try_wait(&full[s], ph) && global_timer_ns() - t0 < 100000000ull) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1 && (!PAIR || rank == 0)) {
        // -------------------------------------------------------------- MMA -----
        // (a pair's MMAs are issued by its rank-0 CTA alone; they wait for both CTAs'
        // scale slots and accumulators, and their commits arrive in both CTAs)
        // Whole-warp loop with warp-uniform descriptors; the elected lane issues the
        // MMAs and the commits (a commit tracks the MMAs of the thread that issues it).
        // A K tile is ready once its scale-factor slot is: the scale-factor warps arrive
        // on sf_full only after they have waited for the same fill's full barrier.
        const bool leader = ptx::elect_one();
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool issued = false;
        for (int uj = 0; uj < sc.n_units; ++uj) {
            const int u = sc.unit(uj);
            if (cta_aborted(abort)) break;
            const Unit t = decode_unit(p, u, &tmap_q, sc, rank);
            const uint32_t q_off = (uint32_t)((t.tq * BN) % 128) / 32;
            if ((q_off & 1) != 0 || q_off * 32 + (BN < 32 ? 32 : BN) > 128 * S::kQChunks) {
                // never planned: a scale-factor column offset the MMA is not given
                if (leader) {
                    atomicExch(p.err, kErrSfOffset);
                    *abort = 1;
                }
                __syncwarp();
                break;
            }
            if (!warp_wait(&acc_empty[acc], acc_phase ^ 1, abort, p.err, kErrTimeoutMma)) break;
            ptx::tc_fence_after();
            const uint32_t d_tmem = tmem + acc * S::kAccStride;
            bool ok = true;
            for (int kt = t.kt_begin; kt < t.kt_end; ++kt) {
                if (!warp_wait(&sf_full[stage], phase, abort, p.err, kErrTimeoutMma)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t sf_base = tmem + S::kSfBase + stage * S::kSfCols;
                const uint64_t adesc = ptx::smem_desc_sw128(ptx::smem_u32(smem + L::kOffP + stage * S::kPTileBytes));
                const uint64_t bdesc = ptx::smem_desc_sw128(ptx::smem_u32(
                    FUSED ? smem + L::kOffPersist + kt * S::kQTileBytes : smem + L::kOffQ + stage * L::kQStageBytes));
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t a = kk >> 1;
                        const uint32_t sfid = (kk & 1) * 2;
                        const uint32_t sfa = (sf_base + 4 * a) | (sfid << 30);
                        const uint32_t sfb = (sf_base + 8 + a * 4 * S::kQChunks + q_off) | (sfid << 30);
                        const uint32_t acc_in = (kt > t.kt_begin || kk >= S::kSub) ? 1u : 0u;
                        if constexpr (PAIR)
                            ptx::mma_mxf4_pair(d_tmem, adesc + 2 * kk, bdesc + 2 * kk,
                                               ptx::idesc_mxf4(BN, sfid, sfid, 256), sfa, sfb, acc_in);
                        else
                            ptx::mma_mxf4(d_tmem + (kk % S::kSub) * BN, adesc + 2 * kk, bdesc + 2 * kk,
                                          ptx::idesc_mxf4(BN, sfid, sfid), sfa, sfb, acc_in);
                    }
                    if constexpr (PAIR) ptx::tc_commit_pair(&empty[stage], 3);
                    else ptx::tc_commit(&empty[stage]);
                }
                __syncwarp();
                issued = true;
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
            if (leader) {
                if constexpr (PAIR) ptx::tc_commit_pair(&acc_full[acc], 3);
                else ptx::tc_commit(&acc_full[acc]);
            }
            __syncwarp();
            if (S::kNumAcc == 2) {
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            } else {
                acc_phase ^= 1;
            }
        }
        if (cta_aborted(abort) && issued && leader) {
            // wait (bounded) for every MMA this thread issued before TMEM is freed
            if constexpr (PAIR) ptx::tc_commit_pair(drain, 1);
            else ptx::tc_commit(drain);
            const uint64_t t0 = global_timer_ns();
            while (!ptx::mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 100000000ull) {
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // rank 1 of a pair: no MMAs of its own to issue (rank 0 issues the pair's)
    } else if (warp >= 6) {
        // ------------------------------------------------- scale-factor writers ---
        // Warp q' (= warp % 4) owns TMEM lanes 32q'..32q'+31. In the 128x4 scale atom,
        // the 16 bytes of shared-memory row l hold, as word w, the four block scales of
        // matrix row l + 32w. The MMA's subpartition q reads the P scales of its rows
        // 32q + l from column (atom base + q) and the Q scales of Q row l + 32w from
        // column (atom base + w) of every subpartition.
        const int quad = warp & 3;
        const int set = (warp - 6) >> 2;          // this set writes K tiles with count % sets == set
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        int stage = 0;
        uint32_t phase = 0;
        uint32_t kt_count = 0;
        for (int uj = 0; uj < sc.n_units && !*abort; ++uj) {
            const int u = sc.unit(uj);
            const Unit t = decode_unit(p, u, &tmap_q, sc, rank);
            bool ok = true;
            for (int kt = t.kt_begin; kt < t.kt_end; ++kt, ++kt_count) {
                // Every set waits for every fill, in order, even those it does not
                // write: a fill's barrier can then never be more than one phase ahead
                // of the parity waited for, so a wait cannot match an older phase.
                // Slot `stage` was last read by the MMAs of the previous fill of this
                // stage; the producer waited for their completion before refilling the
                // stage, so once the new fill has landed the slot is free.
                if (!wait_or_abort(&full[stage], phase, abort, p.err, kErrTimeoutMma)) { ok = false; break; }
                if ((int)(kt_count % kSfWarpSets) != set) {
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                    continue;
                }
                ptx::tc_fence_after();
                const uint32_t col = lane_base + S::kSfBase + stage * S::kSfCols;
                const uint32_t sfp_s = ptx::smem_u32(smem + L::kOffSfP + stage * S::kSfChunkBytes) + lane * 16;
                const uint32_t sfq_s =
                    ptx::smem_u32(FUSED ? smem + L::kOffPersist + p.k_tiles * S::kQTileBytes + kt * S::kSfChunkBytes
                                        : smem + L::kOffSfQ + stage * S::kQChunks * S::kSfChunkBytes) +
                    lane * 16;
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    ptx::tmem_st_32x32b_x1(col + 4 * a + quad, ptx::lds32(sfp_s + 512 * a + 4 * quad));
#pragma unroll
                    for (int c = 0; c < S::kQChunks; ++c) {
                        const uint4 v = ptx::lds128(sfq_s + 1024 * c + 512 * a);
                        ptx::tmem_st_32x32b_x4(col + 8 + a * 4 * S::kQChunks + 4 * c, v.x, v.y, v.z, v.w);
                    }
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR && rank > 0) ptx::mbar_arrive_remote(ptx::mapa_shared(&sf_full[stage], 0));
                    else ptx::mbar_arrive(&sf_full[stage]);
                }
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
        }
    } else {
        // ----------------------------------------------------------- epilogue ---
        const int quad = warp & 3;                 // TMEM subpartition this warp may read
        int acc = 0;
        uint32_t acc_phase = 0;
        constexpr int CW = S::kChunkCols;
        constexpr int NCH = BN / CW;
        const bool via_tma = S::kStagingBytes > 0 && p.tma_store;
        const uint32_t staging = ptx::smem_u32(smem + L::kOffStaging) + quad * S::kStageBoxBytes;
        volatile int* sk_last = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 8);
        constexpr bool kSkWidth = BN <= 32 && !GATHER;
        // The four epilogue warps leave the loop together: a stream-K tile synchronises
        // them on a named barrier, which a warp that had left alone would hold forever.
        for (int uj = 0; uj < sc.n_units; ++uj) {
            const int u = sc.unit(uj);
            const Unit t = decode_unit(p, u, &tmap_q, sc, rank);
            if (!bar_and(1, 128, wait_or_abort(&acc_full[acc], acc_phase, abort, p.err, kErrTimeoutEpilogue))) break;
            ptx::tc_fence_after();
            const int prow = t.out_row0 + quad * 32 + lane;      // output row (transposed: column)
            const bool row_ok = quad * 32 + lane < t.rows;
            const uint32_t taddr = tmem + acc * S::kAccStride + ((uint32_t)(quad * 32) << 16);
            // stream-K (planned for decode tiles of width <= 32 only): this CTA holds only
            // part of the tile's K range
            const bool partial = kSkWidth && (t.kt_begin > 0 || t.kt_end < p.k_tiles);
            // write chunk c of y from registers: staged TMA store or direct stores
            auto emit = [&](int c, uint32_t (&r)[CW]) {
                if constexpr (GATHER) {
                    for (int d = 0; d < p.n_dest; ++d)
                        store_chunk<CW>(p, reinterpret_cast<void*>(p.dest[d]), p.ldo, p.q_rows, prow, row_ok,
                                        t.tq * BN + c * CW, r);
                    return;
                }
                if constexpr (S::kStagingBytes > 0) {
                    if (via_tma) {
                        // Stage this warp's box of 32 rows x 64 bytes in shared memory in the
                        // tensor map's 64-byte-swizzled layout (row = lane; 16-byte piece j of
                        // the row at j ^ ((row >> 1) & 3)), then one lane stores the box. The
                        // buffer is rewritten only after the previous store from it has been
                        // read out.
                        const int boxes = p.out_bf16 ? 1 : 2;     // 32 columns = 64 or 128 bytes
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            if (h >= boxes) break;
                            const int bx = t.tq * BN + c * CW + 16 * h, by = t.out_row0 + quad * 32;
                            if (bx >= p.q_rows || by >= p.p_rows) break;   // box wholly outside y
                            if (lane == 0) ptx::bulk_wait_group_read<0>();
                            __syncwarp();
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                uint32_t w[4];
                                if (p.out_bf16) {
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        __nv_bfloat162 v = __floats2bfloat162_rn(
                                            __uint_as_float(r[8 * j + 2 * e]), __uint_as_float(r[8 * j + 2 * e + 1]));
                                        w[e] = *reinterpret_cast<uint32_t*>(&v);
                                    }
                                } else {
#pragma unroll
                                    for (int e = 0; e < 4; ++e) w[e] = r[16 * h + 4 * j + e];
                                }
                                ptx::sts128(staging + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4), w[0], w[1], w[2],
                                            w[3]);
                            }
                            ptx::fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                ptx::tma_store_2d(&tmap_y, staging, bx, by);
                                ptx::bulk_commit_group();
                            }
                        }
                        return;
                    }
                }
                store_chunk<CW>(p, t.out, t.ldo, t.q_rows, prow, row_ok, t.tq * BN + c * CW, r);
            };
            if constexpr (SPLIT) {
                // K split over the cluster, finished as a reduce-scatter by columns: CTA s owns
                // output chunks [s NCH / split, (s + 1) NCH / split). Every CTA parks, in its
                // own ring (its MMAs have read their last stage, and it has no further tile),
                // the chunks of its partial tile that other CTAs own, as float4 columns of
                // 128 rows (columns 4j .. 4j + 3 of row i at float4 j * 128 + i: chunk c is
                // 16 KB at 16 KB c, and a warp's accesses are 512 contiguous bytes); once
                // every other CTA's MMAs are done too (ring_free), it copies each CTA's chunks
                // into that CTA's ring after the parked tile (bulk copies completing on that
                // CTA's part_full). Each CTA then adds, for its own chunks, the partial tiles
                // of all CTAs in the order of their K ranges (its own from TMEM) and writes
                // them to y. The CTAs leave together (cluster barrier at the end), so no
                // CTA's shared memory goes while a copy may still read or write it.
                constexpr uint32_t kChunkBytes = 128 * CW * 4;
                constexpr uint32_t kPartBytes = NCH * kChunkBytes;
                const int nsplit = p.split;
                auto chunk0 = [&](int q) { return q * NCH / nsplit; };     // first chunk CTA q owns
                const int my0 = chunk0(rank), my1 = chunk0(rank + 1);
                const int row = quad * 32 + lane;
                float4* part = reinterpret_cast<float4*>(smem);
#pragma unroll 1
                for (int c = 0; c < NCH; ++c) {
                    if (c >= my0 && c < my1) continue;
                    uint32_t r[CW];
                    tmem_load_chunk<CW>(taddr + c * CW, r);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < CW; j += 4)
                        part[((c * CW + j) >> 2) * 128 + row] =
                            make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                        __uint_as_float(r[j + 3]));
                }
                ptx::fence_proxy_async_smem();             // the copies read through the async proxy
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (threadIdx.x == 64) {
                    // the slices of this CTA's chunks that the others send: expected bytes,
                    // then this CTA's ring is free for them
                    ptx::mbar_arrive_expect_tx(part_full, (uint32_t)(nsplit - 1) * (my1 - my0) * kChunkBytes);
                    for (int q = 0; q < nsplit; ++q)
                        if (q != rank) ptx::mbar_arrive_remote(ptx::mapa_shared(ring_free, (uint32_t)q));
                    if (wait_or_abort(ring_free, 0, abort, p.err, kErrTimeoutEpilogue)) {
                        // CTA q's chunks go to its ring, slot of this CTA among its senders
                        for (int q = 0; q < nsplit; ++q) {
                            if (q == rank) continue;
                            const int q0 = chunk0(q), q1 = chunk0(q + 1);
                            const uint32_t slot = (uint32_t)(rank < q ? rank : rank - 1);
                            const uint32_t dst = kPartBytes + slot * (uint32_t)(q1 - q0) * kChunkBytes;
                            const uint32_t mbar = ptx::mapa_shared(part_full, (uint32_t)q);
                            for (int c = q0; c < q1; ++c)
                                ptx::bulk_copy_to_cluster(
                                    ptx::mapa_shared(smem + dst + (uint32_t)(c - q0) * kChunkBytes, (uint32_t)q),
                                    smem + (uint32_t)c * kChunkBytes, kChunkBytes, mbar);
                        }
                    }
                }
                if (!bar_and(1, 128, wait_or_abort(part_full, 0, abort, p.err, kErrTimeoutEpilogue))) break;
#pragma unroll 1
                for (int c = my0; c < my1; ++c) {
                    uint32_t r[CW];
#pragma unroll 1
                    for (int q = 0; q < nsplit; ++q) {
                        // partial of CTA q (K order): this CTA's from TMEM, others from the ring
                        uint32_t v[CW];
                        if (q == rank) {
                            tmem_load_chunk<CW>(taddr + c * CW, v);
                            ptx::tmem_ld_wait();
                        } else {
                            const uint32_t slot = (uint32_t)(q < rank ? q : q - 1);
                            const float4* src = part + (kPartBytes + slot * (uint32_t)(my1 - my0) * kChunkBytes +
                                                        (uint32_t)(c - my0) * kChunkBytes) / 16 + row;
#pragma unroll
                            for (int j = 0; j < CW / 4; ++j) {
                                const float4 f = src[j * 128];
                                v[4 * j] = __float_as_uint(f.x);
                                v[4 * j + 1] = __float_as_uint(f.y);
                                v[4 * j + 2] = __float_as_uint(f.z);
                                v[4 * j + 3] = __float_as_uint(f.w);
                            }
                        }
#pragma unroll
                        for (int j = 0; j < CW; ++j)
                            r[j] = q == 0 ? v[j] : __float_as_uint(__fadd_rn(__uint_as_float(r[j]), __uint_as_float(v[j])));
                    }
                    emit(c, r);
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&acc_empty[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
                continue;
            }
            // this thread's row of the CTA's partial-tile slot (the first or the last tile of
            // its stream-K range)
            const int64_t slot_row = ((int64_t)blockIdx.x * 2 + (u == sc.sk_first ? 0 : 1)) * (128 * BN) +
                                     (int64_t)(quad * 32 + lane) * BN;
#pragma unroll 1
            for (int c = 0; c < NCH; ++c) {
                uint32_t r[CW];
                tmem_load_chunk<CW>(taddr + c * CW, r);
                if (S::kSub > 1) {
                    uint32_t r2[CW];
#pragma unroll
                    for (int sub = 1; sub < S::kSub; ++sub) {
                        tmem_load_chunk<CW>(taddr + sub * BN + c * CW, r2);
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < CW; ++j)
                            r[j] = __float_as_uint(__uint_as_float(r[j]) + __uint_as_float(r2[j]));
                    }
                }
                ptx::tmem_ld_wait();
                if (c == NCH - 1) {
                    // the accumulator is in registers: hand it back to the MMA warp now
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (PAIR && rank > 0) ptx::mbar_arrive_remote(ptx::mapa_shared(&acc_empty[acc], 0));
                        else ptx::mbar_arrive(&acc_empty[acc]);
                    }
                }
                if (!partial) {
                    emit(c, r);
                } else {
                    float4* dst = reinterpret_cast<float4*>(p.sk_partials + slot_row + c * CW);
#pragma unroll
                    for (int j = 0; j < CW; j += 4)
                        dst[j / 4] = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                                 __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                }
            }
            if constexpr (kSkWidth) if (partial) {
                // Count the CTA in once all four warps' rows are written; the arrival that
                // completes the count finishes the tile.
                const int64_t t0 = (int64_t)(u - p.sk_tile0) * p.k_tiles;
                const int c_lo = sk_cta_of(p, t0), c_hi = sk_cta_of(p, t0 + p.k_tiles - 1);
                __threadfence();
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (threadIdx.x == 64)
                    *sk_last = sk_arrive(p.sk_counters + u, p.sk_tag) == (uint32_t)(c_hi - c_lo + 1) ? 1 : 0;
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (*sk_last) {
                    __threadfence();
                    // y = the contributors' partial tiles added in the order of their K
                    // ranges, 16 columns at a time; the loads of two contributors are issued
                    // together (decode tiles: transposed direct stores)
                    const int64_t row_off = (int64_t)(quad * 32 + lane) * BN;
#pragma unroll 1
                    for (int c16 = 0; c16 < BN / 16; ++c16) {
                        uint32_t r[16];
#pragma unroll 1
                        for (int k0 = c_lo; k0 <= c_hi; k0 += 2) {
                            float4 v[2][4];
#pragma unroll
                            for (int g = 0; g < 2; ++g) {
                                const int k = k0 + g;
                                if (k <= c_hi) {
                                    const int slot = u == p.sk_tile0 + (int)(sk_start(p, k) / p.k_tiles) ? 0 : 1;
                                    const float4* src = reinterpret_cast<const float4*>(
                                        p.sk_partials + ((int64_t)k * 2 + slot) * (128 * BN) + row_off + c16 * 16);
#pragma unroll
                                    for (int j = 0; j < 4; ++j) v[g][j] = __ldcg(src + j);
                                }
                            }
#pragma unroll
                            for (int g = 0; g < 2; ++g) {
                                if (k0 + g > c_hi) break;
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const float f[4] = {v[g][j].x, v[g][j].y, v[g][j].z, v[g][j].w};
#pragma unroll
                                    for (int e = 0; e < 4; ++e)
                                        r[4 * j + e] = k0 + g == c_lo ? __float_as_uint(f[e])
                                                                      : __float_as_uint(__fadd_rn(__uint_as_float(r[4 * j + e]), f[e]));
                                }
                            }
                        }
                        store_chunk<16>(p, t.out, t.ldo, t.q_rows, prow, row_ok, t.tq * BN + c16 * 16, r);
                    }
                }
            }
            if (S::kNumAcc == 2) {
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            } else {
                acc_phase ^= 1;
            }
        }
        // the staging buffers must outlive the stores that read them
        if (via_tma && lane == 0) ptx::bulk_wait_group_all();
        __syncwarp();
    }

    ptx::tc_fence_before();
    __syncthreads();
    // a cluster's CTAs leave together: none frees its TMEM or shared memory while another
    // may still signal it, read it or (pair) write there with its MMAs
    if constexpr (PAIR || SPLIT) ptx::cluster_sync();
    if (warp == 1) {
        ptx::tc_fence_after();
        if constexpr (PAIR) ptx::tmem_dealloc_pair(tmem, S::kTmemCols);
        else ptx::tmem_dealloc(tmem, S::kTmemCols);
    }
}

}  // namespace macaq
