// MACaQ online activation transform / offline weight preparation kernel (sm_100a).
//
// Per row r and 32-element block b (MACaQ pages: per-channel scale then block
// Hadamard rotation aligned to the MXFP4 group, openai-hub.com article; MXFP4 = E2M1
// elements + one E8M0 scale per 32):
//   u   = fp32(x[r, k]) * mult[k]                      (mult = 1/s or s)
//   t   = FWHT32(u)    stages h = 1,2,4,8,16, pair (a+b, a-b), a the lower index
//   v   = c * t        c = fp32(1/sqrt(32))
//   e   = max(floor(log2 max|v|) - 2, -127)             (0 for an all-zero block)
//   q   = v * 2^-e  ->  E2M1 round-to-nearest-even, saturating, sign kept
//
// One thread owns one block; a warp covers 32 consecutive blocks (1024 elements) of a
// row and keeps that column chunk for all its rows, so its 32 multipliers stay in
// registers. Activation bytes move global -> shared with per-thread cp.async (16 bytes
// each, 4 per block), STAGES - 1 rows ahead of the one being computed; each thread
// reads back only what it copied, so a wait_group is the only synchronisation. The
// first copies are issued before the multipliers are fetched, so the two latencies
// overlap. The four 16-byte pieces of a block sit XOR-swizzled in the thread's 64-byte
// slot (piece j at (j ^ ((lane >> 1) & 3))), which keeps both the copies and the reads
// free of bank conflicts. The butterfly runs in registers, no shuffles; max |t| is a
// three-level tree of 3-input maxima rather than a 32-long chain. Every fp32 step uses
// the explicit round-to-nearest intrinsics, so nothing is contracted.
//
// Two exact shortcuts, each giving the same bits as the steps above:
//  - max|v| = fl(c * max|t|): rounding is monotone and c > 0.
//  - for -123 <= e <= 123, q = fl(t * (c * 2^-e)) with c * 2^-e an exact normal fp32:
//    whenever fl(c t) is normal, fl(c t) * 2^-e is exact, so both round c t 2^-e once;
//    whenever it is not, |q| < 2^-3 and both give a zero code of the same sign. Outside
//    that range the two multiplies are done one after the other.
// E2M1 encoding uses cvt.rn.satfinite.e2m1x2.f32 (round to nearest even, saturating to
// +-6, sign of zero kept), two elements per instruction, element 2j in the low nibble.
//
// Scales: one byte per thread; the four threads of blocks 4g..4g+3 combine them into
// one 32-bit word of the 128-row x 4-block atom layout. Padding rows (up to a multiple
// of 128) and padding blocks (up to a multiple of 8) get scale byte 0.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"

namespace macaq {

struct QuantParams {
    const uint16_t* x;       // bf16 bits [rows x K], row stride ld
    const float* mult;       // [K]
    uint8_t* codes;          // [rows x K/2]
    uint8_t* scales;         // atom layout, rows_pad x kb_pad bytes
    const float* s_for_inv;  // non-null: also write inv_out[k] = 1/s[k]
    float* inv_out;
    int64_t rows, K, ld;
    int64_t rows_pad;        // round_up(rows, 128)
    int64_t kb_pad;          // round_up(K/32, 8)
    int64_t chunks_per_row;  // ceil(kb_pad / 32): warp-sized groups of blocks per row
};

// Eight fp32 values -> eight E2M1 codes in one 32-bit word, value i in nibble i.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&a)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]), "f"(a[7]));
    return out;
}

// Packed fp32 pairs (sm_100 f32x2 instructions): each half is an independent IEEE
// round-to-nearest operation, bit-identical to the scalar one.
__device__ __forceinline__ uint64_t pk(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void upk(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// Eight fp32 values held as four pairs -> eight E2M1 codes, value i in nibble i.
__device__ __forceinline__ uint32_t cvt_e2m1x8(uint64_t p0, uint64_t p1, uint64_t p2, uint64_t p3) {
    float a[8];
    upk(p0, a[0], a[1]);
    upk(p1, a[2], a[3]);
    upk(p2, a[4], a[5]);
    upk(p3, a[6], a[7]);
    return cvt_e2m1x8(a);
}

__device__ __forceinline__ float absmax3(float a, float b, float c) { return max3(fabsf(a), fabsf(b), fabsf(c)); }

// The block transform and encoding for one block held as T[j] = elements (2j, 2j+1)
// of u = x * mult: the butterfly, the shared exponent and the E2M1 codes (element i in nibble i % 8 of
// packed[i / 8]). Returns the scale byte e + 127. T is overwritten.
// The unnormalised 32-point butterfly on T[j] = elements (2j, 2j+1): stages
// h = 1, 2, 4, 8, 16, pairs (a + b, a - b) with a at the lower index, fp32 round to
// nearest at every step.
__device__ __forceinline__ void butterfly_block(uint64_t (&T)[16]) {
    // stage h = 1 combines the two halves of each pair
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        float a, d;
        upk(T[j], a, d);
        T[j] = pk(__fadd_rn(a, d), __fsub_rn(a, d));
    }
    // stages h = 2, 4, 8, 16 pair T[j] with T[j + h/2], two elements per instruction
#pragma unroll
    for (int hp = 1; hp < 16; hp <<= 1) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (j & hp) continue;
            const uint64_t A = T[j], B = T[j + hp];
            T[j] = add2(A, B);
            T[j + hp] = sub2(A, B);
        }
    }
}

__device__ __forceinline__ uint32_t encode_block(uint64_t (&T)[16], uint32_t (&packed)[4]) {
    const float c = __uint_as_float(0x3E3504F3u);        // nearest fp32 to 1/sqrt(32)
    butterfly_block(T);

    // max |t| as a three-level tree (the order of a max does not change its value)
    float a[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) upk(T[j], a[2 * j], a[2 * j + 1]);
    float m[11];
#pragma unroll
    for (int i = 0; i < 10; ++i) m[i] = absmax3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
    m[10] = fmaxf(fabsf(a[30]), fabsf(a[31]));
    const float tmax = max3(max3(m[0], m[1], m[2]), max3(m[3], m[4], m[5]),
                            max3(max3(m[6], m[7], m[8]), m[9], m[10]));
    const float amax = __fmul_rn(tmax, c);
    const int biased = (int)(__float_as_uint(amax) >> 23);
    const int e = max(biased - 129, -127);        // biased == 0 (zero / subnormal) -> -127
    if (e >= -123 && e <= 123) {
        const float k = __uint_as_float(0x3E3504F3u - ((uint32_t)e << 23));   // c * 2^-e
        const uint64_t kk = pk(k, k);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            packed[i] = cvt_e2m1x8(mul2(T[4 * i], kk), mul2(T[4 * i + 1], kk), mul2(T[4 * i + 2], kk),
                                   mul2(T[4 * i + 3], kk));
    } else {
        const float inv = __uint_as_float((uint32_t)(127 - e) << 23);      // 2^-e
        const uint64_t cc = pk(c, c), ii = pk(inv, inv);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            packed[i] = cvt_e2m1x8(mul2(mul2(T[4 * i], cc), ii), mul2(mul2(T[4 * i + 1], cc), ii),
                                   mul2(mul2(T[4 * i + 2], cc), ii), mul2(mul2(T[4 * i + 3], cc), ii));
    }
    return (uint32_t)(e + 127);
}

constexpr int kQuantThreads = 256;
// Two stages: one row in flight while the current one is encoded. Deeper prefetch
// puts more rows in the first burst of requests that all warps issue at once, and a
// warp's first row then arrives later (every warp waits on its oldest copy, which the
// memory system does not serve first); one row ahead already keeps HBM busy in the
// steady state with 16 warps per SM.
constexpr int kQuantStages = 2;
constexpr uint32_t kQuantStageBytes = kQuantThreads * 64;
constexpr int kQuantSmemBytes = kQuantStages * kQuantStageBytes;

// 16-byte global -> shared copy; src_bytes = 0 reads nothing and writes 16 zero bytes.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(kQuantThreads, 2) quant_rows_kernel(QuantParams p) {
    extern __shared__ __align__(16) uint8_t qsmem[];
    const uint32_t lane = threadIdx.x & 31;
    // grid sizes are small (a few thousand warps): 32-bit warp and row indices
    const int gw = (int)((blockIdx.x * kQuantThreads + threadIdx.x) >> 5);
    const int nwarps = (int)((gridDim.x * kQuantThreads) >> 5);
    const int cpr = (int)p.chunks_per_row;
    // the host makes nwarps a multiple of chunks_per_row: every warp keeps one chunk
    const int chunk = gw % cpr;
    const int row_step = nwarps / cpr;
    const int row0 = gw / cpr;
    const int rows = (int)p.rows, rows_pad = (int)p.rows_pad;
    const int b = chunk * 32 + lane;                     // block index in the row
    const bool col_live = b < (int)(p.K >> 5);

    // Copy pipeline. Rows past the end and blocks past K are zero-filled instead of
    // branched around: they give zero blocks, whose scale byte 0 is exactly what the
    // padding of the scale layout needs, and their codes are never stored.
    const uint32_t swz16 = ((lane >> 1) & 3) << 4;
    uint32_t off[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) off[j] = (uint32_t)(16 * j) ^ swz16;
    const uint32_t slot0 = (uint32_t)__cvta_generic_to_shared(qsmem) + threadIdx.x * 64;
    const uint32_t slot_end = slot0 + kQuantStages * kQuantStageBytes;
    const uint8_t* xbase = reinterpret_cast<const uint8_t*>(p.x);
    const int64_t ld_bytes = p.ld * 2;
    const uint8_t* isrc = xbase + (int64_t)row0 * ld_bytes + (int64_t)b * 64;
    const int64_t istep = (int64_t)row_step * ld_bytes;
    int irow = row0;
    uint32_t islot = slot0;
    auto issue = [&]() {
        const bool v = col_live && irow < rows;
        const uint8_t* src = v ? isrc : xbase;
        const uint32_t n = v ? 16u : 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) cp_async_16(islot + off[j], src + 16 * j, n);
        cp_async_commit();
        irow += row_step;
        isrc += istep;
        islot += kQuantStageBytes;
        if (islot == slot_end) islot = slot0;
    };
    // Nothing global is touched before the previous kernel on the stream has finished.
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
#pragma unroll
    for (int s = 0; s < kQuantStages - 1; ++s) issue();

    if (p.s_for_inv != nullptr && row0 == 0 && col_live) {
        const float4* sp = reinterpret_cast<const float4*>(p.s_for_inv + b * 32);
        float4* ip = reinterpret_cast<float4*>(p.inv_out + b * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 v = __ldg(sp + i);
            ip[i] = make_float4(__fdiv_rn(1.0f, v.x), __fdiv_rn(1.0f, v.y), __fdiv_rn(1.0f, v.z),
                                __fdiv_rn(1.0f, v.w));
        }
    }

    uint64_t mult[16];                                   // multiplier pairs (2j, 2j+1)
    if (col_live) {
        const float4* mp = reinterpret_cast<const float4*>(p.mult + b * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 m = __ldg(mp + i);
            mult[2 * i] = pk(m.x, m.y);
            mult[2 * i + 1] = pk(m.z, m.w);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) mult[i] = 0;
    }


    uint32_t rslot = slot0;
    uint8_t* cdst = p.codes + (int64_t)row0 * (p.K >> 1) + (int64_t)b * 16;
    const int64_t cstep = (int64_t)row_step * (p.K >> 1);
    const int kb_pad = (int)p.kb_pad;
    const int64_t kb4 = p.kb_pad >> 2;
    for (int row = row0; row < rows_pad; row += row_step) {
        issue();
        cp_async_wait<kQuantStages - 1>();

        // T[j] holds elements (2j, 2j+1) of the block
        uint64_t T[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t w[4];
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                         : "r"(rslot + off[j]));
#pragma unroll
            for (int q = 0; q < 4; ++q)
                T[4 * j + q] = mul2(pk(__uint_as_float(w[q] << 16), __uint_as_float(w[q] & 0xFFFF0000u)),
                                    mult[4 * j + q]);
        }
        rslot += kQuantStageBytes;
        if (rslot == slot_end) rslot = slot0;

        uint32_t packed[4];
        const uint32_t sbyte = encode_block(T, packed);

        if (col_live && row < rows)
            *reinterpret_cast<uint4*>(cdst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        cdst += cstep;
        // four consecutive blocks -> one scale word (lanes 4g .. 4g+3 of the warp)
        const uint32_t s1 = __shfl_down_sync(0xffffffffu, sbyte, 1);
        const uint32_t s2 = __shfl_down_sync(0xffffffffu, sbyte, 2);
        const uint32_t s3 = __shfl_down_sync(0xffffffffu, sbyte, 3);
        if ((lane & 3) == 0 && b < kb_pad) {
            const int64_t o = ((int64_t)(row >> 7) * kb4 + (b >> 2)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4;
            *reinterpret_cast<uint32_t*>(p.scales + o) = sbyte | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
    }
    cp_async_wait<0>();
}

// ---------------------------------------------------------------------------------
// Grouped activation transform (MoE experts): one launch for every expert's rows.
//
// Expert g's rows x_row .. x_row + rows - 1 of x go through the transform with its own
// multipliers and land at padded rows row_p .. row_p + rows - 1 of one grouped output,
// each expert on a 128-row boundary; rows row_p + rows .. up to the next boundary are
// padding (scale byte 0, codes not written). Only experts with rows > 0 are listed,
// in increasing row_p. A warp keeps one column chunk and walks a contiguous range of
// padded rows, so it changes expert (and reloads its 32 multipliers) at most a few
// times. Per block the arithmetic is the same encode_block as quant_rows_kernel.

struct QuantGroup {
    int64_t x_row;        // first row of the expert in x
    int32_t rows;         // its row count (> 0)
    int32_t row_p;        // its first padded row in the grouped output (multiple of 128)
    const float* mult;    // its multipliers [K]
};

struct GroupedQuantParams {
    const uint16_t* x;    // bf16 bits, row stride ld
    uint8_t* codes;       // [rows_pad x K/2]
    uint8_t* scales;      // atom layout, rows_pad x kb_pad bytes
    const QuantGroup* groups;
    int32_t G;
    int32_t rows_per_warp;
    int64_t K, ld;
    int64_t rows_pad;     // sum over experts of round_up(rows, 128)
    int64_t kb_pad;
    int64_t chunks_per_row;
};

// Index of the expert whose padded rows contain r (largest g with row_p <= r).
__device__ __forceinline__ int find_group(const QuantGroup* t, int G, int r) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (t[mid].row_p <= r) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kQuantThreads, 2) quant_grouped_kernel(GroupedQuantParams p) {
    extern __shared__ __align__(16) uint8_t qsmem[];
    const uint32_t lane = threadIdx.x & 31;
    const int gw = (int)((blockIdx.x * kQuantThreads + threadIdx.x) >> 5);
    const int cpr = (int)p.chunks_per_row;
    const int chunk = gw % cpr;
    const int r_begin = (gw / cpr) * p.rows_per_warp;
    const int r_end = min(r_begin + p.rows_per_warp, (int)p.rows_pad);
    const int b = chunk * 32 + lane;
    const bool col_live = b < (int)(p.K >> 5);
    const int G = p.G;
    const QuantGroup* tab = p.groups;

    const uint32_t swz16 = ((lane >> 1) & 3) << 4;
    uint32_t off[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) off[j] = (uint32_t)(16 * j) ^ swz16;
    const uint32_t slot0 = (uint32_t)__cvta_generic_to_shared(qsmem) + threadIdx.x * 64;
    const uint32_t slot_end = slot0 + kQuantStages * kQuantStageBytes;
    const uint8_t* xbase = reinterpret_cast<const uint8_t*>(p.x);

    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    if (r_begin >= r_end) return;                        // warp-uniform

    // copy side: the expert of the row being fetched
    int irow = r_begin;
    int ig = find_group(tab, G, r_begin);
    int i_rowp = tab[ig].row_p, i_rows = tab[ig].rows;
    int64_t i_xrow = tab[ig].x_row;
    int i_next = ig + 1 < G ? tab[ig + 1].row_p : INT32_MAX;
    uint32_t islot = slot0;
    auto issue = [&]() {
        if (irow >= i_next) {
            ++ig;
            i_rowp = tab[ig].row_p;
            i_rows = tab[ig].rows;
            i_xrow = tab[ig].x_row;
            i_next = ig + 1 < G ? tab[ig + 1].row_p : INT32_MAX;
        }
        const int local = irow - i_rowp;
        const bool v = col_live && irow < r_end && local < i_rows;
        const uint8_t* src = v ? xbase + (i_xrow + local) * p.ld * 2 + (int64_t)b * 64 : xbase;
        const uint32_t n = v ? 16u : 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) cp_async_16(islot + off[j], src + 16 * j, n);
        cp_async_commit();
        ++irow;
        islot += kQuantStageBytes;
        if (islot == slot_end) islot = slot0;
    };
#pragma unroll
    for (int s = 0; s < kQuantStages - 1; ++s) issue();

    // compute side: the expert of the row being encoded, and its multipliers
    int cg = find_group(tab, G, r_begin);
    int c_rowp = tab[cg].row_p, c_rows = tab[cg].rows;
    int c_next = cg + 1 < G ? tab[cg + 1].row_p : INT32_MAX;
    uint64_t mult[16];
    auto load_mult = [&]() {
        if (col_live) {
            const float4* mp = reinterpret_cast<const float4*>(tab[cg].mult + b * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 m = __ldg(mp + i);
                mult[2 * i] = pk(m.x, m.y);
                mult[2 * i + 1] = pk(m.z, m.w);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) mult[i] = 0;
        }
    };
    load_mult();

    uint32_t rslot = slot0;
    const int64_t half_k = p.K >> 1;
    const int kb_pad = (int)p.kb_pad;
    const int64_t kb4 = p.kb_pad >> 2;
    for (int row = r_begin; row < r_end; ++row) {
        issue();
        if (row >= c_next) {
            ++cg;
            c_rowp = tab[cg].row_p;
            c_rows = tab[cg].rows;
            c_next = cg + 1 < G ? tab[cg + 1].row_p : INT32_MAX;
            load_mult();
        }
        cp_async_wait<kQuantStages - 1>();

        uint64_t T[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t w[4];
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                         : "r"(rslot + off[j]));
#pragma unroll
            for (int q = 0; q < 4; ++q)
                T[4 * j + q] = mul2(pk(__uint_as_float(w[q] << 16), __uint_as_float(w[q] & 0xFFFF0000u)),
                                    mult[4 * j + q]);
        }
        rslot += kQuantStageBytes;
        if (rslot == slot_end) rslot = slot0;

        uint32_t packed[4];
        const uint32_t sbyte = encode_block(T, packed);

        if (col_live && row - c_rowp < c_rows)
            *reinterpret_cast<uint4*>(p.codes + (int64_t)row * half_k + (int64_t)b * 16) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
        const uint32_t s1 = __shfl_down_sync(0xffffffffu, sbyte, 1);
        const uint32_t s2 = __shfl_down_sync(0xffffffffu, sbyte, 2);
        const uint32_t s3 = __shfl_down_sync(0xffffffffu, sbyte, 3);
        if ((lane & 3) == 0 && b < kb_pad) {
            const int64_t o = ((int64_t)(row >> 7) * kb4 + (b >> 2)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4;
            *reinterpret_cast<uint32_t*>(p.scales + o) = sbyte | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
    }
    cp_async_wait<0>();
}

}  // namespace macaq
