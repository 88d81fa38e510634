// MACaQ online activation transform / offline weight preparation kernel (sm_100a).
//
// Per row r and 32-element block b (MACaQ pages: per-channel scale then block
// Hadamard "micro-rotation" aligned to the MXFP4 group, openai-hub.com article;
// MXFP4 = E2M1 elements + one E8M0 scale per 32):
//   u   = fp32(x[r, k]) * mult[k]                      (mult = 1/s or s)
//   v   = c * FWHT32(u)   stages h = 1,2,4,8,16, (a+b, a-b), c = fp32(1/sqrt(32))
//   e   = max(floor(log2 max|v|) - 2, -127)             (0 for an all-zero block)
//   q   = v * 2^-e  ->  E2M1 round-to-nearest-even, saturating, sign kept
//
// Mapping: one warp handles a 256-element chunk of one row (8 blocks); lane l holds
// elements 8*(l%4) .. 8*(l%4)+7 of block l/4, loaded with one 16-byte load. Butterfly
// stages h = 1, 2, 4 stay inside a lane, h = 8 and 16 use xor-shuffles over lane bits
// 0 and 1. Every arithmetic step uses the explicit round-to-nearest intrinsics, so the
// compiler cannot contract a multiply into an add.
//
// Output: the lane's 8 codes as one 32-bit word (nibble t = element t), and one 32-bit
// word of four consecutive block scales per 4 blocks, placed in the 128-row x 4-block
// atom layout of the tensor-core scale factors. Padding rows (up to a multiple of 128)
// and padding blocks (up to a multiple of 8) get scale byte 0.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace macaq {

struct QuantParams {
    const uint16_t* x;     // bf16 bits [rows x K], row stride ld
    const float* mult;     // [K]
    uint8_t* codes;        // [rows x K/2]
    uint8_t* scales;       // atom layout, rows_pad x kb_pad bytes
    const float* s_for_inv;  // non-null: also write inv_out[k] = 1/s[k]
    float* inv_out;
    int64_t rows, K, ld;
    int64_t rows_pad;      // round_up(rows, 128)
    int64_t kb_pad;        // round_up(K/32, 8)
    int64_t chunks_per_row;  // kb_pad / 8
    int64_t items;         // rows_pad * chunks_per_row
};

__device__ __forceinline__ uint32_t e2m1_code(float q) {
    // Count of rounding thresholds exceeded: 0.25 and 1.25, 2.5 and 5 are ties that go
    // down (to the even mantissa), 0.75, 1.75 and 3.5 ties that go up.
    const float a = fabsf(q);
    uint32_t idx = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
                   (a >= 3.5f) + (a > 5.0f);
    return ((__float_as_uint(q) >> 31) << 3) | idx;
}

// Quantise the lane's 8 values; returns the packed codes and, through `sbyte`, the
// block's scale byte (identical in the 4 lanes of the block).
__device__ __forceinline__ uint32_t transform_and_encode(float (&v)[8], uint32_t lane,
                                                         uint32_t& sbyte) {
    // in-lane butterfly stages h = 1, 2, 4
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i & h) continue;
            const float a = v[i], b = v[i + h];
            v[i] = __fadd_rn(a, b);
            v[i + h] = __fsub_rn(a, b);
        }
    }
    // cross-lane stages h = 8 (lane bit 0) and h = 16 (lane bit 1)
#pragma unroll
    for (int bit = 1; bit <= 2; bit <<= 1) {
        const bool upper = (lane & bit) != 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float p = __shfl_xor_sync(0xffffffffu, v[i], bit);
            // lower position keeps a + b, upper keeps a - b, a being the lower one
            v[i] = upper ? __fsub_rn(p, v[i]) : __fadd_rn(v[i], p);
        }
    }
    const float c = __uint_as_float(0x3E3504F3u);  // nearest fp32 to 1/sqrt(32)
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[i] = __fmul_rn(v[i], c);
        amax = fmaxf(amax, fabsf(v[i]));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));

    // floor(log2 amax) from the exponent field; any amax below 2^-124 (subnormals
    // included) lands on the clamp e = -127.
    const int biased = (int)(__float_as_uint(amax) >> 23);
    int e = biased - 127 - 2;
    if (biased == 0) e = -127;
    e = max(e, -127);
    sbyte = (uint32_t)(e + 127);
    const float inv = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, exact

    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) word |= e2m1_code(__fmul_rn(v[i], inv)) << (4 * i);
    return word;
}

template <int UNROLL>
__global__ void __launch_bounds__(256) quant_rows_kernel(QuantParams p) {
    const uint32_t lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t kb = p.K >> 5;
    const uint32_t blk_in_chunk = lane >> 2;   // 0..7
    const uint32_t quarter = lane & 3;         // which 8 elements of the block

    for (int64_t base = warp; base < p.items; base += nwarps * UNROLL) {
        uint4 raw[UNROLL];
        float4 m0[UNROLL], m1[UNROLL];
        bool valid[UNROLL];
        int64_t row[UNROLL], k0[UNROLL];
        // issue every load of the unrolled items first
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t item = base + (int64_t)u * nwarps;
            row[u] = item / p.chunks_per_row;
            const int64_t chunk = item - row[u] * p.chunks_per_row;
            const int64_t blk = chunk * 8 + blk_in_chunk;
            k0[u] = blk * 32 + quarter * 8;
            valid[u] = item < p.items && row[u] < p.rows && blk < kb;
            raw[u] = make_uint4(0, 0, 0, 0);
            m0[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            m1[u] = m0[u];
            if (valid[u]) {
                raw[u] = __ldg(reinterpret_cast<const uint4*>(p.x + row[u] * p.ld + k0[u]));
                m0[u] = __ldg(reinterpret_cast<const float4*>(p.mult + k0[u]));
                m1[u] = __ldg(reinterpret_cast<const float4*>(p.mult + k0[u] + 4));
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t item = base + (int64_t)u * nwarps;
            if (item >= p.items) break;   // warp-uniform
            const float mm[8] = {m0[u].x, m0[u].y, m0[u].z, m0[u].w,
                                 m1[u].x, m1[u].y, m1[u].z, m1[u].w};
            const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
            float v[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), mm[2 * i]);
                v[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), mm[2 * i + 1]);
            }
            uint32_t sbyte;
            const uint32_t word = transform_and_encode(v, lane, sbyte);
            if (valid[u]) {
                *reinterpret_cast<uint32_t*>(p.codes + row[u] * (p.K >> 1) + (k0[u] >> 1)) = word;
                if (p.s_for_inv != nullptr && row[u] == 0) {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        p.inv_out[k0[u] + i] = __fdiv_rn(1.0f, p.s_for_inv[k0[u] + i]);
                }
            }
            // gather the scale bytes of blocks 4g .. 4g+3 (lanes 16g, 16g+4, ...)
            const uint32_t b0 = __shfl_sync(0xffffffffu, sbyte, (lane & 16) + 0);
            const uint32_t b1 = __shfl_sync(0xffffffffu, sbyte, (lane & 16) + 4);
            const uint32_t b2 = __shfl_sync(0xffffffffu, sbyte, (lane & 16) + 8);
            const uint32_t b3 = __shfl_sync(0xffffffffu, sbyte, (lane & 16) + 12);
            if ((lane & 15) == 0) {
                const int64_t r = row[u];
                const int64_t chunk = item - r * p.chunks_per_row;
                const int64_t j = chunk * 8 + (lane >> 2);   // multiple of 4
                const int64_t off = ((r >> 7) * (p.kb_pad >> 2) + (j >> 2)) * 512 +
                                    (r & 31) * 16 + ((r >> 5) & 3) * 4;
                *reinterpret_cast<uint32_t*>(p.scales + off) = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
            }
        }
    }
}

}  // namespace macaq
