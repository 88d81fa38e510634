// Hessian exponent search for MXFP4 weight blocks (sm_100a).
//
// The ablation paragraph of the openai-hub.com MACaQ article lists a "Hessian exponent
// search" step between round-to-nearest and the micro-rotation; the Flip-Refinement
// paragraphs of the zicq.com articles give its error model, the second-order form
//   dL ~ 1/2 (w - w_hat)^T H (w - w_hat),  H from the layer's input distribution.
// Here H is the Gram matrix of calibration activations in the transformed basis (the
// fp32 values the online transform hands to the quantiser), restricted to its 32 x 32
// diagonal blocks, and each weight block keeps, among the exponents e0 (the floor rule),
// e0 + 1 and e0 - 1, the one whose round-to-nearest codes give the smallest d^T H_b d,
// d = w' - dec(codes) 2^e. Only weight scale bytes (and the codes under them) change;
// the GEMM is the same.
//
// hessian_blocks_kernel: one CTA per 32-column block b, 1024 threads, thread (i, j)
// owns H_b[i][j]. Four warps transform 128 calibration rows at a time into shared
// memory (the same fp32 transform as the quantiser: x * (1/s), butterfly, times
// fp32(1/sqrt(32))), then every thread adds v[i] * v[j] for those rows in ascending
// order. The product of two fp32 values is exact in fp64, so the fused multiply-add
// rounds exactly like a multiply followed by an add: only the running sum rounds.
//
// prepare_weight_hessian_kernel: one thread per weight block (CTA = 128 rows of one
// block column, H_b in shared memory). Each candidate exponent is evaluated as
//   sum_i d_i * r_i,  r_i = sum_j H_ij * d_j   (i, j ascending, fp64, each product and
// sum rounded on its own), d exact in fp64; a later candidate (order e0, e0+1, e0-1)
// replaces the choice only when strictly smaller. Codes under an exponent are those of
// fp32(v * 2^-e) by cvt.rn.satfinite.e2m1x2.f32, as in the quantiser. Padding rows
// (to a multiple of 128) and padding blocks (to a multiple of 8) get scale byte 0.
#pragma once

#include <cstdint>

#include "quant_kernel.cuh"

namespace macaq {

constexpr int kHessRows = 128;                 // calibration rows transformed per step

struct HessianParams {
    const uint16_t* x;     // bf16 calibration activations [T x K], row stride ld
    const float* s;        // per-channel scale [K]; the transform multiplies by RN32(1/s)
    double* H;             // [K/32][32][32]
    int64_t T, K, ld;
};

// fp32 transformed block: v = c * butterfly(x * mult) for one 32-element block.
__device__ __forceinline__ void transform_block_f32(const uint16_t* xb, const float* mult, float (&v)[32]) {
    const uint4* xs = reinterpret_cast<const uint4*>(xb);
    uint64_t T[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 w4 = __ldg(xs + j);
        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
            T[4 * j + q] = mul2(pk(__uint_as_float(w[q] << 16), __uint_as_float(w[q] & 0xFFFF0000u)),
                                pk(mult[8 * j + 2 * q], mult[8 * j + 2 * q + 1]));
    }
    butterfly_block(T);
    const float c = __uint_as_float(0x3E3504F3u);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        float a, d;
        upk(T[j], a, d);
        v[2 * j] = __fmul_rn(a, c);
        v[2 * j + 1] = __fmul_rn(d, c);
    }
}

__global__ void __launch_bounds__(1024, 1) hessian_blocks_kernel(HessianParams p) {
    __shared__ float vs[kHessRows][33];
    __shared__ float inv[32];
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    const int b = blockIdx.x;
    const int i = threadIdx.x >> 5, j = threadIdx.x & 31;
    if (threadIdx.x < 32) inv[threadIdx.x] = __fdiv_rn(1.0f, p.s[32 * b + threadIdx.x]);
    __syncthreads();
    double acc = 0.0;
    for (int64_t t0 = 0; t0 < p.T; t0 += kHessRows) {
        const int64_t left = p.T - t0;
        const int n = left < kHessRows ? (int)left : kHessRows;
        if (threadIdx.x < n) {
            float v[32];
            transform_block_f32(p.x + (t0 + threadIdx.x) * p.ld + 32 * b, inv, v);
#pragma unroll
            for (int k = 0; k < 32; ++k) vs[threadIdx.x][k] = v[k];
        }
        __syncthreads();
        for (int r = 0; r < n; ++r) acc = __fma_rn((double)vs[r][i], (double)vs[r][j], acc);
        __syncthreads();
    }
    p.H[(int64_t)b * 1024 + i * 32 + j] = acc;
}

struct HessianPrepParams {
    const uint16_t* W;     // bf16 [N x K], row stride ld
    const float* s;        // [K]
    const double* H;       // [K/32][32][32]
    uint8_t* codes;        // [N x K/2]
    uint8_t* scales;       // atom layout, round_up(N, 128) x kb_pad
    float* inv_out;        // [K]: RN32(1/s)
    int64_t N, K, ld, kb_pad;
};

// The E2M1 value of a code (sign in bit 3).
__device__ __forceinline__ double e2m1_value(uint32_t code) {
    const uint32_t m = code & 7u;
    const double mag = m < 4 ? 0.5 * m : (m == 4 ? 2.0 : (m == 5 ? 3.0 : (m == 6 ? 4.0 : 6.0)));
    return (code & 8u) ? -mag : mag;
}

__global__ void __launch_bounds__(128) prepare_weight_hessian_kernel(HessianPrepParams p) {
    __shared__ double Hs[32 * 32];
    __shared__ double ds[128][33];
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    const int b = blockIdx.x;
    const int kb = (int)(p.K >> 5);
    const int64_t n = (int64_t)blockIdx.y * 128 + threadIdx.x;
    const bool live = b < kb && n < p.N;
    if (b < kb) {
        for (int k = threadIdx.x; k < 1024; k += 128) Hs[k] = p.H[(int64_t)b * 1024 + k];
        if (blockIdx.y == 0 && threadIdx.x < 32)
            p.inv_out[32 * b + threadIdx.x] = __fdiv_rn(1.0f, p.s[32 * b + threadIdx.x]);
    }
    __syncthreads();
    uint32_t sbyte = 0;
    if (live) {
        float v[32];
        transform_block_f32(p.W + n * p.ld + 32 * b, p.s + 32 * b, v);
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < 32; ++k) amax = fmaxf(amax, fabsf(v[k]));
        const int e0 = max((int)(__float_as_uint(amax) >> 23) - 129, -127);
        int best_e = e0;
        double best = 0.0;
        uint32_t best_codes[4] = {0, 0, 0, 0};
        bool have = false;
#pragma unroll 1
        for (int ci = 0; ci < 3; ++ci) {
            const int e = ci == 0 ? e0 : (ci == 1 ? e0 + 1 : e0 - 1);
            if (e < -127 || e > 126) continue;
            const float inv_step = __uint_as_float((uint32_t)(127 - e) << 23);           // 2^-e
            const double step = __longlong_as_double((long long)(1023 + e) << 52);       // 2^e
            uint32_t codes[4];
            double d[32];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                float q[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) q[k] = __fmul_rn(v[8 * w + k], inv_step);   // fp32(v 2^-e)
                codes[w] = cvt_e2m1x8(q);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    d[8 * w + k] = __dsub_rn((double)v[8 * w + k],
                                             __dmul_rn(e2m1_value((codes[w] >> (4 * k)) & 15u), step));
                    ds[threadIdx.x][8 * w + k] = d[8 * w + k];
                }
            }
            double err = 0.0;
#pragma unroll 1
            for (int i = 0; i < 32; ++i) {
                double r = 0.0;
#pragma unroll
                for (int j = 0; j < 32; ++j) r = __dadd_rn(r, __dmul_rn(Hs[i * 32 + j], d[j]));
                err = __dadd_rn(err, __dmul_rn(ds[threadIdx.x][i], r));
            }
            if (!have || err < best) {
                have = true;
                best = err;
                best_e = e;
#pragma unroll
                for (int w = 0; w < 4; ++w) best_codes[w] = codes[w];
            }
        }
        *reinterpret_cast<uint4*>(p.codes + n * (p.K >> 1) + 16 * b) =
            make_uint4(best_codes[0], best_codes[1], best_codes[2], best_codes[3]);
        sbyte = (uint32_t)(best_e + 127);
    }
    // every (row, block) of the padded scale layout, padding included, gets its byte
    if (b < p.kb_pad) {
        const int64_t o = ((n >> 7) * (p.kb_pad >> 2) + (b >> 2)) * 512 + (n & 31) * 16 + ((n >> 5) & 3) * 4 + (b & 3);
        p.scales[o] = (uint8_t)sbyte;
    }
}

}  // namespace macaq
