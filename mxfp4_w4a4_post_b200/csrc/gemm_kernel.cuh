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
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "quant_kernel.cuh"

namespace macaq {

struct GemmGroup {
    int32_t unit_begin, rows, row_p, row_y;
    const uint8_t* sf_q;
    int64_t pad;
};

struct GemmParams {
    const uint8_t* sf_p;     // scale atoms of P
    const uint8_t* sf_q;     // scale atoms of Q
    void* out;               // y, or the fp32 split-K accumulator when atomic
    int64_t ldo;             // leading dimension of out, elements
    int32_t p_rows, q_rows;  // logical rows of P and Q
    int32_t k_tiles;         // ceil(K / 256)
    int32_t kb4_pad;         // scale atoms per 128-row slab along K
    int32_t tiles_p, tiles_q;
    int32_t splits, k_tiles_per_split;
    int32_t total_units;     // tiles_p * tiles_q * splits
    int32_t group_p;         // raster group height (in P tiles)
    int32_t out_bf16;        // 1: bf16 output, 0: fp32 (ignored when atomic)
    int32_t atomic;          // 1: split K, fp32 vector reductions into out
    int32_t transpose_out;   // 1: out[q * ldo + p], 0: out[p * ldo + q]
    int32_t vec_ok;          // 1: out and ldo allow 16-byte vector stores
    int32_t tma_store;       // 1: epilogue stages 32 x 32 output boxes in shared memory and
                             //    writes them with TMA stores (row-major tiles, vec_ok)
    int* err;                // device error word
    // Split K (atomic): the accumulator `out` starts at zero without a separate memset.
    // First thing, the epilogue warps of every CTA zero their slice of it and set their
    // CTA's flag to `epoch` (a value unique to the call, so flags left by earlier calls
    // never match); before its first reduction a CTA waits until every flag is set.
    int64_t zero_vec4;               // 16-byte words of the accumulator
    unsigned long long* cta_flags;   // [gridDim.x]
    unsigned long long epoch;
    // Fused activation transform (decode, Q = activations): first thing, the epilogue
    // warps of every CTA quantise their share of the activation blocks into the Q codes
    // and scales (the transform and encoding of macaq_quant_act) and then set the CTA's
    // flag as above; the producer issues the Q side of its copies only once every flag
    // is set (the weight side of its first fills goes ahead meanwhile).
    int32_t fused;
    const uint16_t* fx;              // bf16 activations [f_rows x f_K], row stride fx_ld
    int64_t fx_ld;
    const float* f_mult;             // inv_s [f_K]
    uint8_t* f_codes;                // [f_rows x f_K/2]
    uint8_t* f_scales;               // atom layout, 128-row slabs x f_kb_pad blocks
    int32_t f_rows, f_K, f_kb_pad;
    // Grouped GEMM (groups > 0; prefill orientation, no split K): group g multiplies the
    // g_rows[g] activation rows starting at P row g_row_p[g] (a multiple of 128: groups
    // sit in whole scale slabs) by its own weight (tensor map g_tmaps[g], scale atoms
    // g_sf_q[g]) and writes y rows g_row_y[g] ..; its units are g_unit_begin[g] ..
    // g_unit_begin[g + 1] - 1, P tiles fastest.
    int32_t groups;
    const GemmGroup* g_desc;         // [groups]
    const CUtensorMap* g_tmaps;      // [groups], 64-byte aligned
    // Gathered output (column-parallel layers; the kernel's GATHER instantiation): every
    // output element goes to each of dest[0 .. n_dest - 1] (device addresses of the
    // destinations' first column for this weight, the same row stride ldo) instead of to
    // out, with direct stores (no TMA store, no split K).
    int32_t n_dest;
    const unsigned long long* dest;  // [n_dest], device memory
};

enum : int {
    kErrTimeoutProducer = 1,
    kErrTimeoutMma = 2,
    kErrTimeoutEpilogue = 3,
    kErrSfOffset = 4,
    kErrTimeoutSplit = 5
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
    static constexpr int kChunkCols = BN <= 32 ? 16 : 32;   // epilogue TMEM load width
    // Output staging for TMA stores (wide tiles only): one box of 32 rows x 64 bytes
    // (32 bf16 or 16 fp32 columns) per epilogue warp.
    static constexpr int kStageBoxBytes = 32 * 64;
    static constexpr int kStagingBytes = BN >= 128 ? 4 * kStageBoxBytes : 0;
};

template <int BN, int STAGES>
struct GemmSmem {
    using S = GemmShape<BN, STAGES>;
    static constexpr int kOffP = 0;
    static constexpr int kOffQ = kOffP + STAGES * S::kPTileBytes;
    static constexpr int kOffSfP = kOffQ + STAGES * S::kQTileBytes;
    static constexpr int kOffSfQ = kOffSfP + STAGES * S::kSfChunkBytes;
    static constexpr int kOffStaging = kOffSfQ + STAGES * S::kQChunks * S::kSfChunkBytes;   // 1 KB aligned
    static constexpr int kOffBar = kOffStaging + S::kStagingBytes;
    static constexpr int kNumBars = 3 * STAGES + 4 + 1;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;            // slack to align the base to 1 KB
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

struct Unit {
    int tile, split, tp, tq, kt_begin, kt_end;
    int p_row0;                    // first P row of the tile in the P tensor map
    int out_row0;                  // output row of the tile's P row 0
    int rows;                      // valid P rows from p_row0 on (the tile's group)
    const CUtensorMap* tmap_q;     // Q tensor map of the tile
    const uint8_t* sf_q;           // Q scale atoms of the tile
};

__device__ __forceinline__ Unit decode_unit(const GemmParams& p, int u, const CUtensorMap* tmap_q) {
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
        x.split = 0;
        x.tp = lu % tiles_p;
        x.tq = lu / tiles_p;
        x.kt_begin = 0;
        x.kt_end = p.k_tiles;
        x.p_row0 = gd.row_p + x.tp * 128;
        x.out_row0 = gd.row_y + x.tp * 128;
        x.rows = gd.rows - x.tp * 128;
        x.tmap_q = p.g_tmaps + lo;
        x.sf_q = gd.sf_q;
        return x;
    }
    const int tile = u / p.splits;
    const int split = u - tile * p.splits;
    const int per_group = p.group_p * p.tiles_q;
    const int g = tile / per_group;
    const int r = tile - g * per_group;
    const int gp = min(p.group_p, p.tiles_p - g * p.group_p);
    Unit x;
    x.tile = tile;
    x.split = split;
    x.tp = g * p.group_p + r % gp;
    x.tq = r / gp;
    x.kt_begin = split * p.k_tiles_per_split;
    x.kt_end = min(p.k_tiles, x.kt_begin + p.k_tiles_per_split);
    x.p_row0 = x.tp * 128;
    x.out_row0 = x.tp * 128;
    x.rows = p.p_rows - x.tp * 128;
    x.tmap_q = tmap_q;
    x.sf_q = p.sf_q;
    return x;
}

// Writes one chunk of output row `prow` (a P row; the output column of it when
// transposed) if `valid`.
template <int CW>
__device__ __forceinline__ void store_chunk(const GemmParams& p, void* out, int prow, bool valid, int q_base,
                                            const uint32_t (&r)[CW]) {
    if (!valid) return;
    if (p.transpose_out) {
        // out[q, prow]: for each column the 32 lanes of the warp write consecutive prow
        if (p.atomic) {
            float* o = reinterpret_cast<float*>(out);
#pragma unroll
            for (int j = 0; j < CW; ++j) {
                const int q = q_base + j;
                if (q < p.q_rows) atomicAdd(o + (int64_t)q * p.ldo + prow, __uint_as_float(r[j]));
            }
        } else if (p.out_bf16) {
            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
#pragma unroll
            for (int j = 0; j < CW; ++j) {
                const int q = q_base + j;
                if (q < p.q_rows) o[(int64_t)q * p.ldo + prow] = __float2bfloat16_rn(__uint_as_float(r[j]));
            }
        } else {
            float* o = reinterpret_cast<float*>(out);
#pragma unroll
            for (int j = 0; j < CW; ++j) {
                const int q = q_base + j;
                if (q < p.q_rows) o[(int64_t)q * p.ldo + prow] = __uint_as_float(r[j]);
            }
        }
        return;
    }
    const bool full = q_base + CW <= p.q_rows && p.vec_ok;
    if (p.atomic) {
        float* o = reinterpret_cast<float*>(out) + (int64_t)prow * p.ldo + q_base;
        if (full) {
#pragma unroll
            for (int j = 0; j < CW; j += 4)
                atomicAdd(reinterpret_cast<float4*>(o + j),
                          make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                      __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3])));
        } else {
#pragma unroll
            for (int j = 0; j < CW; ++j)
                if (q_base + j < p.q_rows) atomicAdd(o + j, __uint_as_float(r[j]));
        }
    } else if (p.out_bf16) {
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out) + (int64_t)prow * p.ldo + q_base;
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
                if (q_base + j < p.q_rows) o[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
        }
    } else {
        float* o = reinterpret_cast<float*>(out) + (int64_t)prow * p.ldo + q_base;
        if (full) {
#pragma unroll
            for (int j = 0; j < CW; j += 4)
                *reinterpret_cast<float4*>(o + j) =
                    make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
        } else {
#pragma unroll
            for (int j = 0; j < CW; ++j)
                if (q_base + j < p.q_rows) o[j] = __uint_as_float(r[j]);
        }
    }
}

// Split-K zeroing protocol (gpu scope): a CTA zeroes its slice, fences, and one thread
// releases its flag; the epilogue lanes acquire every CTA's flag before reducing.
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* f) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(f) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u64(unsigned long long* f, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(f), "l"(v) : "memory");
}
// Wait (bounded, ~2 s) until *flag == epoch. On give-up record kErrTimeoutSplit, raise
// the CTA abort flag and return false. Polls sleep briefly: the flag lives in L2.
__device__ __noinline__ bool wait_split_flag(const unsigned long long* flag, unsigned long long epoch,
                                             volatile int* abort, int* err, uint64_t limit_ns = kWaitLimitNs) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (ld_acquire_u64(flag) == epoch) return true;
        if ((it & 15) == 15) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                atomicExch(err, kErrTimeoutSplit);
                *abort = 1;
                return false;
            }
        }
        __nanosleep(128);
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

// This CTA's share of the fused activation transform: one 32-element block per thread
// and step over the 128-row slab(s) x f_kb_pad blocks of the Q operand. Blocks of real
// rows and columns get codes and their scale byte; padding blocks get scale byte 0.
__device__ __forceinline__ void fused_quant_share(const GemmParams& p, int et) {
    const int kb = p.f_K >> 5;
    const int64_t rows_pad = ((int64_t)p.f_rows + 127) / 128 * 128;
    const int64_t total = rows_pad * p.f_kb_pad;
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    const int64_t b0 = (int64_t)blockIdx.x * per, b1 = min(total, b0 + per);
    for (int64_t i = b0 + et; i < b1; i += 128) {
        const int row = (int)(i / p.f_kb_pad);
        const int b = (int)(i - (int64_t)row * p.f_kb_pad);
        uint32_t sbyte = 0;
        if (row < p.f_rows && b < kb) {
            const uint4* xs = reinterpret_cast<const uint4*>(p.fx + (int64_t)row * p.fx_ld + (int64_t)b * 32);
            const float4* ms = reinterpret_cast<const float4*>(p.f_mult + (int64_t)b * 32);
            uint64_t T[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 v = __ldg(xs + j);
                const float4 m0 = __ldg(ms + 2 * j), m1 = __ldg(ms + 2 * j + 1);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                const uint64_t mm[4] = {pk(m0.x, m0.y), pk(m0.z, m0.w), pk(m1.x, m1.y), pk(m1.z, m1.w)};
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    T[4 * j + q] = mul2(pk(__uint_as_float(w[q] << 16), __uint_as_float(w[q] & 0xFFFF0000u)), mm[q]);
            }
            uint32_t packed[4];
            sbyte = encode_block(T, packed);
            *reinterpret_cast<uint4*>(p.f_codes + (int64_t)row * (p.f_K >> 1) + (int64_t)b * 16) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
        const int64_t o = ((int64_t)(row >> 7) * (p.f_kb_pad >> 2) + (b >> 2)) * 512 + (row & 31) * 16 +
                          ((row >> 5) & 3) * 4 + (b & 3);
        p.f_scales[o] = (uint8_t)sbyte;
    }
}

constexpr int kSfWarpSets = 2;                                // scale-writer sets
constexpr int kGemmThreads = 32 * (6 + 4 * kSfWarpSets);

// GATHER: the output goes to p.dest[0 .. p.n_dest - 1] (a separate instantiation, so
// that the ordinary kernels keep their registers).
template <int BN, int STAGES, bool GATHER = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_mxf4_kernel(const __grid_constant__ CUtensorMap tmap_p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
    using S = GemmShape<BN, STAGES>;
    using L = GemmSmem<BN, STAGES>;
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
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kOffMisc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&acc_full[a], 1);
            ptx::mbar_init(&acc_empty[a], 4);
        }
        ptx::mbar_init(drain, 1);
        for (int s = 0; s < STAGES; ++s) ptx::mbar_init(&sf_full[s], 4);
        *abort = 0;
        ptx::fence_mbar_init();
        ptx::fence_proxy_async_smem();
        ptx::prefetch_tensormap(&tmap_p);
        if (p.groups == 0) ptx::prefetch_tensormap(&tmap_q);
        if (S::kStagingBytes > 0 && p.tma_store) ptx::prefetch_tensormap(&tmap_y);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, S::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Set-up above overlaps the previous kernel's tail; operands are read only after it.
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer ---
        // The whole warp runs the loop, so addresses and coordinates are warp-uniform
        // values; one elected lane issues the copies.
        const bool leader = ptx::elect_one();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued_mask = 0, issued_phase = 0;
        const int q_slabs = (p.q_rows + 127) / 128;
        // Q side of one fill: codes tile and scale chunks
        auto issue_q = [&](const Unit& t, int st, int kt, int q0, int slab0, int nchunks) {
            ptx::tma_load_2d(smem + L::kOffQ + st * S::kQTileBytes, t.tmap_q, &full[st], kt * S::kBKBytes, q0);
            for (int c = 0; c < nchunks; ++c)
                ptx::bulk_load(smem + L::kOffSfQ + (st * S::kQChunks + c) * S::kSfChunkBytes,
                               t.sf_q + ((int64_t)(slab0 + c) * p.kb4_pad + 2 * kt) * 512, S::kSfChunkBytes,
                               &full[st]);
        };
        bool q_ready = !p.fused;
        int deferred = 0;                   // fills of the first unit still without their Q side
        for (int u = blockIdx.x; u < p.total_units; u += gridDim.x) {
            if (cta_aborted(abort)) break;
            const Unit t = decode_unit(p, u, &tmap_q);
            const int q0 = t.tq * BN;
            const int slab0 = q0 / 128;
            const int nchunks = min(S::kQChunks, q_slabs - slab0);
            const uint32_t bytes = S::kPTileBytes + S::kQTileBytes + S::kSfChunkBytes * (1 + nchunks);
            bool ok = true;
            for (int kt = t.kt_begin; kt < t.kt_end; ++kt) {
                if (!warp_wait(&empty[stage], phase ^ 1, abort, p.err, kErrTimeoutProducer)) { ok = false; break; }
                if (leader) {
                    ptx::mbar_arrive_expect_tx(&full[stage], bytes);
                    ptx::tma_load_2d(smem + L::kOffP + stage * S::kPTileBytes, &tmap_p, &full[stage],
                                     kt * S::kBKBytes, t.p_row0);
                    ptx::bulk_load(smem + L::kOffSfP + stage * S::kSfChunkBytes,
                                   p.sf_p + ((int64_t)(t.p_row0 >> 7) * p.kb4_pad + 2 * kt) * 512,
                                   S::kSfChunkBytes, &full[stage]);
                    if (q_ready) issue_q(t, stage, kt, q0, slab0, nchunks);
                }
                __syncwarp();
                issued_mask |= 1u << stage;
                issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
                if (!q_ready && (++deferred == STAGES || kt + 1 == t.kt_end)) {
                    // every CTA's share of the quantised activations is in memory: give
                    // the deferred fills (stages 0.. of the first unit) their Q side
                    bool fl = true;
                    for (int i = lane; i < (int)gridDim.x && fl; i += 32)
                        fl = wait_split_flag(p.cta_flags + i, p.epoch, abort, p.err);
                    if (!__all_sync(0xffffffffu, fl)) { ok = false; break; }
                    ptx::fence_proxy_async_global();
                    if (leader)
                        for (int d = 0; d < deferred; ++d) issue_q(t, d, t.kt_begin + d, q0, slab0, nchunks);
                    __syncwarp();
                    q_ready = true;
                }
            }
            if (!ok) break;
        }
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
    } else if (warp == 1) {
        // -------------------------------------------------------------- MMA -----
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
        for (int u = blockIdx.x; u < p.total_units; u += gridDim.x) {
            if (cta_aborted(abort)) break;
            const Unit t = decode_unit(p, u, &tmap_q);
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
                const uint64_t bdesc = ptx::smem_desc_sw128(ptx::smem_u32(smem + L::kOffQ + stage * S::kQTileBytes));
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t a = kk >> 1;
                        const uint32_t sfid = (kk & 1) * 2;
                        const uint32_t sfa = (sf_base + 4 * a) | (sfid << 30);
                        const uint32_t sfb = (sf_base + 8 + a * 4 * S::kQChunks + q_off) | (sfid << 30);
                        ptx::mma_mxf4(d_tmem + (kk % S::kSub) * BN, adesc + 2 * kk, bdesc + 2 * kk,
                                      ptx::idesc_mxf4(BN, sfid, sfid), sfa, sfb,
                                      (kt > t.kt_begin || kk >= S::kSub) ? 1u : 0u);
                    }
                    ptx::tc_commit(&empty[stage]);
                }
                __syncwarp();
                issued = true;
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
            if (leader) ptx::tc_commit(&acc_full[acc]);
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
            ptx::tc_commit(drain);
            const uint64_t t0 = global_timer_ns();
            while (!ptx::mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 100000000ull) {
            }
        }
        __syncwarp();
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
        for (int u = blockIdx.x; u < p.total_units && !*abort; u += gridDim.x) {
            const Unit t = decode_unit(p, u, &tmap_q);
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
                    ptx::smem_u32(smem + L::kOffSfQ + stage * S::kQChunks * S::kSfChunkBytes) + lane * 16;
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
                if (lane == 0) ptx::mbar_arrive(&sf_full[stage]);
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
        bool zeroed = false;
        if (p.atomic || p.fused) {
            const int et = threadIdx.x - 64;                     // 0..127 over warps 2-5
            if (p.atomic) {
                // zero this CTA's slice of the split-K accumulator
                const int64_t per = (p.zero_vec4 + gridDim.x - 1) / gridDim.x;
                const int64_t b0 = (int64_t)blockIdx.x * per, b1 = min(p.zero_vec4, b0 + per);
                float4* z = reinterpret_cast<float4*>(p.out);
                for (int64_t i = b0 + et; i < b1; i += 128) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            if (p.fused) fused_quant_share(p, et);
            ptx::fence_proxy_async_global();
            __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (et == 0) st_release_u64(p.cta_flags + blockIdx.x, p.epoch);
        }
        for (int u = blockIdx.x; u < p.total_units && !*abort; u += gridDim.x) {
            const Unit t = decode_unit(p, u, &tmap_q);
            if (!wait_or_abort(&acc_full[acc], acc_phase, abort, p.err, kErrTimeoutEpilogue)) break;
            ptx::tc_fence_after();
            const int prow = t.out_row0 + quad * 32 + lane;      // output row (transposed: column)
            const bool row_ok = quad * 32 + lane < t.rows;
            const uint32_t taddr = tmem + acc * S::kAccStride + ((uint32_t)(quad * 32) << 16);
            if (p.atomic && !zeroed) {
                // once per kernel: every CTA has zeroed its slice of the accumulator
                bool ok = true;
                for (int i = lane; i < (int)gridDim.x && ok; i += 32)
                    ok = wait_split_flag(p.cta_flags + i, p.epoch, abort, p.err);
                if (!__all_sync(0xffffffffu, ok)) break;
                zeroed = true;
            }
            // write chunk c of y from registers: staged TMA store or direct stores
            auto emit = [&](int c, uint32_t (&r)[CW]) {
                if constexpr (GATHER) {
                    for (int d = 0; d < p.n_dest; ++d)
                        store_chunk<CW>(p, reinterpret_cast<void*>(p.dest[d]), prow, row_ok, t.tq * BN + c * CW, r);
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
                store_chunk<CW>(p, p.out, prow, row_ok, t.tq * BN + c * CW, r);
            };
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
                    if (lane == 0) ptx::mbar_arrive(&acc_empty[acc]);
                }
                emit(c, r);
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
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, S::kTmemCols);
    }
}

}  // namespace macaq
