// Flip-Refinement of MXFP4 weight codes (sm_100a).
//
// The Flip-Refinement paragraphs of the zicq.com MACaQ articles (and of the
// openai-hub.com article): after quantisation, for every output row, each round moves
// the one code whose step to an adjacent representable value lowers the second-order
// error dL ~ 1/2 (w - w_hat)^T H (w - w_hat) most; a row stops when no step lowers it;
// gradients are kept up to date incrementally. Here, per weight row n:
//   e = w' - w_hat            (transformed fp32 weights minus dequantised codes, exact in fp64)
//   g = H e                   (H: full K x K Gram matrix of transformed calibration rows)
//   dE(k, +-) = delta^2 H_kk - 2 delta g_k,   delta = neighbour value - value (times 2^scale)
//   take the smallest dE < 0 (ties: lowest k, then the lower neighbour), then
//   e_k -= delta, g -= delta H[k, :]
// Block scales stay fixed. fp64 throughout, with one fixed arithmetic so that every
// integer decision matches the definition bit for bit:
//   g_j = fma chain over k ascending of H[j][k] * e_k, from 0
//   dE  = (delta * delta) * H_kk - (2 delta) * g_k, each product and the difference rounded
//   g_j = fma(-delta, H[k][j], g_j)
//
// Kernels:
//   transform_rows_kernel   fp32 transformed rows (x * mult -> butterfly -> times c)
//   gram_tile_kernel        one 32 x 32 tile of X'^T X' per CTA (upper triangle, mirrored;
//                           rows of X' in ascending order, exact products, fma sums)
//   flip_gradient_kernel    G = E H for all rows (64 x 64 output tile per CTA, K in order)
//   flip_rounds_kernel      one CTA per row: the greedy rounds on g in shared memory (only
//                           g and the codes change; the error e itself is never needed)
#pragma once

#include <cstdint>

#include "hessian_kernel.cuh"

namespace macaq {

// ---------------------------------------------------------------- transform rows ---

struct TransformParams {
    const uint16_t* x;     // bf16 [rows x K], row stride ld
    const float* s;        // [K]
    float* out;            // fp32 [rows x K]
    int64_t rows, K, ld;
    int32_t invert;        // 1: multiplier RN32(1/s) (activations), 0: s (weights)
};

__global__ void __launch_bounds__(128) transform_rows_kernel(TransformParams p) {
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    const int64_t kb = p.K >> 5;
    const int64_t total = p.rows * kb;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / kb, b = i - r * kb;
        float mult[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const float sv = p.s[32 * b + k];
            mult[k] = p.invert ? __fdiv_rn(1.0f, sv) : sv;
        }
        float v[32];
        transform_block_f32(p.x + r * p.ld + 32 * b, mult, v);
        float4* o = reinterpret_cast<float4*>(p.out + r * p.K + 32 * b);
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    }
}

// ------------------------------------------------------------------ Gram tiles ---

struct GramParams {
    const float* xt;       // transformed calibration rows [T x K]
    double* H;             // [K x K]
    int64_t T, K;
};

// CTA (bi, bj) with bj >= bi: thread (i, j) sums xt[t][32 bi + i] * xt[t][32 bj + j] over t
// ascending; the tile and its mirror get the same values.
__global__ void __launch_bounds__(1024, 1) gram_tile_kernel(GramParams p) {
    __shared__ float a[kHessRows][33];
    __shared__ float b[kHessRows][33];
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    const int nb = (int)(p.K >> 5);
    // blockIdx.x enumerates the upper triangle row by row
    int bi = 0, rem = blockIdx.x;
    while (rem >= nb - bi) {
        rem -= nb - bi;
        ++bi;
    }
    const int bj = bi + rem;
    const int i = threadIdx.x >> 5, j = threadIdx.x & 31;
    double acc = 0.0;
    for (int64_t t0 = 0; t0 < p.T; t0 += kHessRows) {
        const int64_t left = p.T - t0;
        const int n = left < kHessRows ? (int)left : kHessRows;
        for (int q = threadIdx.x; q < n * 32; q += 1024) {
            const int r = q >> 5, c = q & 31;
            a[r][c] = p.xt[(t0 + r) * p.K + 32 * bi + c];
            b[r][c] = p.xt[(t0 + r) * p.K + 32 * bj + c];
        }
        __syncthreads();
        for (int r = 0; r < n; ++r) acc = __fma_rn((double)a[r][i], (double)b[r][j], acc);
        __syncthreads();
    }
    p.H[(32 * (int64_t)bi + i) * p.K + 32 * bj + j] = acc;
    p.H[(32 * (int64_t)bj + j) * p.K + 32 * bi + i] = acc;
}

// -------------------------------------------------------------- gradient G = E H ---

struct FlipGradParams {
    const float* wv;       // transformed weight rows [N x K]
    const uint8_t* codes;  // [N x K/2]
    const uint8_t* scales; // atom layout
    const double* H;       // [K x K]
    double* G;             // [N x K]
    int64_t N, K, kb_pad;
};

__device__ __forceinline__ double e2m1_signed(uint32_t code) { return e2m1_value(code); }

__device__ __forceinline__ int64_t scale_offset(int64_t r, int64_t b, int64_t kb_pad) {
    return ((r >> 7) * (kb_pad >> 2) + (b >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3);
}

// e[n][k] = wv[n][k] - value(code) * 2^(scale - 127), exact in fp64
__device__ __forceinline__ double flip_error(const FlipGradParams& p, int64_t n, int64_t k) {
    const uint8_t byte = p.codes[n * (p.K >> 1) + (k >> 1)];
    const uint32_t code = (k & 1) ? (byte >> 4) : (byte & 15u);
    const int sc = (int)p.scales[scale_offset(n, k >> 5, p.kb_pad)] - 127;
    const double step = __longlong_as_double((long long)(1023 + sc) << 52);
    return __dsub_rn((double)p.wv[n * p.K + k], __dmul_rn(e2m1_signed(code), step));
}

// CTA: 64 rows x 64 columns of G, 256 threads of 4 x 4 outputs; K in chunks of 16,
// every output's fma chain in ascending k.
__global__ void __launch_bounds__(256) flip_gradient_kernel(FlipGradParams p) {
    __shared__ double Es[16][64 + 1];      // [k][row]
    __shared__ double Hs[16][64 + 1];      // [k][col]
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    const int64_t n0 = (int64_t)blockIdx.y * 64, j0 = (int64_t)blockIdx.x * 64;
    const int tr = threadIdx.x >> 4, tc = threadIdx.x & 15;   // 16 x 16 threads
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = 0.0;
    for (int64_t k0 = 0; k0 < p.K; k0 += 16) {
        for (int q = threadIdx.x; q < 16 * 64; q += 256) {
            const int kk = q >> 6, rr = q & 63;
            const int64_t n = n0 + rr, k = k0 + kk;
            Es[kk][rr] = n < p.N ? flip_error(p, n, k) : 0.0;
            const int64_t jj = j0 + rr;
            Hs[kk][rr] = jj < p.K ? p.H[k * p.K + jj] : 0.0;   // H[j][k] = H[k][j] (H symmetric)
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < 16; ++kk) {
            double ev[4], hv[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) ev[a] = Es[kk][tr + 16 * a];
#pragma unroll
            for (int c = 0; c < 4; ++c) hv[c] = Hs[kk][tc + 16 * c];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[a][c] = __fma_rn(hv[c], ev[a], acc[a][c]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int64_t n = n0 + tr + 16 * a, j = j0 + tc + 16 * c;
            if (n < p.N && j < p.K) p.G[n * p.K + j] = acc[a][c];
        }
}

// ------------------------------------------------------------------ the rounds ---

struct FlipRoundParams {
    const float* wv;       // [N x K]
    uint8_t* codes;        // [N x K/2], refined in place
    const uint8_t* scales; // atom layout
    const double* H;       // [K x K]
    const double* G;       // [N x K] initial gradients
    int32_t* moves;        // [N]
    int64_t N, K, kb_pad;
    int32_t max_rounds;
};

constexpr int kFlipThreads = 256;

// Grid positions of the 15 signed E2M1 values (index 7 = 0) and back.
__device__ __forceinline__ int flip_index_of(uint32_t code) {
    const int m = (int)(code & 7u);
    if (m == 0) return 7;
    return (code & 8u) ? 7 - m : 7 + m;
}
__device__ __forceinline__ uint32_t flip_code_of(int index) {
    if (index == 7) return 0;
    return index > 7 ? (uint32_t)(index - 7) : (8u | (uint32_t)(7 - index));
}
__device__ __forceinline__ double flip_grid(int index) {
    const int m = index >= 7 ? index - 7 : 7 - index;
    const double mag = m < 4 ? 0.5 * m : (m == 4 ? 2.0 : (m == 5 ? 3.0 : (m == 6 ? 4.0 : 6.0)));
    return index >= 7 ? mag : -mag;
}

// Candidate order key: smaller dE first, then lower k, then the lower neighbour.
struct FlipBest {
    double dE;
    int key;               // 2 k + (upper neighbour ? 1 : 0), INT_MAX for none
};
__device__ __forceinline__ bool flip_better(double dE, int key, const FlipBest& b) {
    return dE < b.dE || (dE == b.dE && key < b.key);
}

// Dynamic shared memory: g [K] and the diagonal of H [K] (doubles), the 2^scale step of
// every block [K/32] (doubles), the row's code bytes [K/2] and grid positions [K].
inline size_t flip_rounds_smem(int64_t K) { return (size_t)K * 16 + (size_t)(K / 32) * 8 + (size_t)K / 2 + (size_t)K; }

__global__ void __launch_bounds__(kFlipThreads) flip_rounds_kernel(FlipRoundParams p) {
    extern __shared__ __align__(16) uint8_t fsmem[];
    double* g = reinterpret_cast<double*>(fsmem);
    double* hdiag = g + p.K;
    double* step = hdiag + p.K;
    uint8_t* cbytes = reinterpret_cast<uint8_t*>(step + (p.K >> 5));
    uint8_t* idx = cbytes + (p.K >> 1);
    __shared__ double red_dE[kFlipThreads / 32];
    __shared__ int red_key[kFlipThreads / 32];
    __shared__ int s_key;
    ptx::griddep_wait();
    ptx::griddep_launch_dependents();
    const int64_t n = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    for (int64_t b = tid; b < (p.K >> 5); b += kFlipThreads) {
        const int sc = (int)p.scales[scale_offset(n, b, p.kb_pad)] - 127;
        step[b] = __longlong_as_double((long long)(1023 + sc) << 52);
    }
    for (int64_t q = tid; q < (p.K >> 1); q += kFlipThreads) {
        const uint8_t byte = p.codes[n * (p.K >> 1) + q];
        cbytes[q] = byte;
        idx[2 * q] = (uint8_t)flip_index_of(byte & 15u);
        idx[2 * q + 1] = (uint8_t)flip_index_of(byte >> 4);
    }
    for (int64_t k = tid; k < p.K; k += kFlipThreads) {
        g[k] = p.G[n * p.K + k];
        hdiag[k] = p.H[k * p.K + k];
    }
    __syncthreads();
    int moves = 0;
    for (int round = 0; round < p.max_rounds; ++round) {
        FlipBest best{0.0, 0x7FFFFFFF};
        for (int64_t k = tid; k < p.K; k += kFlipThreads) {
            const int ix = idx[k];
            const double st = step[k >> 5], hkk = hdiag[k], gk = g[k];
#pragma unroll
            for (int d = 0; d < 2; ++d) {
                const int ni = ix + (d ? 1 : -1);
                if (ni < 0 || ni > 14) continue;
                const double delta = __dmul_rn(__dsub_rn(flip_grid(ni), flip_grid(ix)), st);   // exact
                const double dE = __dsub_rn(__dmul_rn(__dmul_rn(delta, delta), hkk), __dmul_rn(2.0 * delta, gk));
                if (dE < 0.0 && flip_better(dE, (int)(2 * k + d), best)) best = FlipBest{dE, (int)(2 * k + d)};
            }
        }
        // block argmin under the candidate order
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const double od = __shfl_down_sync(0xffffffffu, best.dE, off);
            const int ok = __shfl_down_sync(0xffffffffu, best.key, off);
            if (flip_better(od, ok, best)) best = FlipBest{od, ok};
        }
        if (lane == 0) {
            red_dE[wid] = best.dE;
            red_key[wid] = best.key;
        }
        __syncthreads();
        if (tid == 0) {
            FlipBest b{red_dE[0], red_key[0]};
            for (int w = 1; w < kFlipThreads / 32; ++w)
                if (flip_better(red_dE[w], red_key[w], b)) b = FlipBest{red_dE[w], red_key[w]};
            s_key = b.key;
        }
        __syncthreads();
        const int key = s_key;
        if (key == 0x7FFFFFFF) break;                  // no move lowers the error
        const int64_t bk = key >> 1;
        const int ix = idx[bk];
        const int ni = ix + ((key & 1) ? 1 : -1);
        const double delta = __dmul_rn(__dsub_rn(flip_grid(ni), flip_grid(ix)), step[bk >> 5]);
        __syncthreads();                               // idx[bk] read by everyone before it changes
        for (int64_t j = tid; j < p.K; j += kFlipThreads) g[j] = __fma_rn(-delta, p.H[bk * p.K + j], g[j]);
        if (tid == 0) {
            idx[bk] = (uint8_t)ni;
            const uint32_t nc = flip_code_of(ni);      // a move to 0 writes +0
            uint8_t& byte = cbytes[bk >> 1];
            byte = (bk & 1) ? (uint8_t)((byte & 0x0Fu) | (nc << 4)) : (uint8_t)((byte & 0xF0u) | nc);
        }
        ++moves;
        __syncthreads();
    }
    for (int64_t q = tid; q < (p.K >> 1); q += kFlipThreads) p.codes[n * (p.K >> 1) + q] = cbytes[q];
    if (tid == 0) p.moves[n] = moves;
}

}  // namespace macaq
