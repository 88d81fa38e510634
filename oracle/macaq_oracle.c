/*
 * Test infrastructure: plain, slow CPU oracle of the MACaQ W4A4 linear layer.
 * Scalar loops only; no blocking, fusion or reordering beyond what each definition
 * states. Build with -O2 -ffp-contract=off -fno-fast-math so every fp32 operation is
 * a single IEEE round-to-nearest-even step (see oracle/build_oracle.py).
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may use this.
 *
 * Rows are independent in quant_rows, dequant_rows and gemm_fp64; their row loops
 * carry OpenMP pragmas so that a second build (-fopenmp) can time the oracle on all
 * host cores. The default build ignores the pragmas; either way every row is computed
 * by the same scalar code in the same order, so the results are identical.
 *
 * Sources, by page and section:
 *  - Layer identity y = xW^T rewritten with an online per-channel scale and block
 *    Hadamard on the activation, inverse folded into the weight: zicq.com English
 *    article "MACaQ Enables Streaming W4A4 Quantization", section "Quantization
 *    mechanism" (and its Chinese twin, section 量化机制); abstract on the Hugging Face
 *    papers mirror.
 *  - 32-element Hadamard blocks matching the MXFP4 group: openai-hub.com article
 *    "华为开源MACaQ", paragraph on the Hadamard rotation.
 *  - MXFP4 = 32-element groups, shared E8M0 scale, E2M1 elements: same article,
 *    paragraph defining MXFP4.
 *  - Round-to-nearest as the base rounding: "Flip-Refinement" sections of both
 *    zicq.com articles.
 * The pages are silent on the following; the readings taken here are:
 *  - activations are divided by s (multiplied by fp32 1/s), weights multiplied by s,
 *    and the scale is applied before the rotation;
 *  - H32 is in natural Sylvester order, normalised by fp32(1/sqrt(32)) after the
 *    butterfly, with no random sign flips;
 *  - butterfly stages in ascending h, pair (a + b, a - b), a at the lower index;
 *  - shared exponent 2^(floor(log2 amax) - 2) clamped to [-127, 127], 0 for amax = 0;
 *  - E2M1 rounding ties to the even mantissa bit, saturating, sign of zero kept;
 *  - element 2j in the low nibble of byte j;
 *  - scales in the 128-row x 4-block atom order of the Blackwell block-scaled MMA.
 */
#include "macaq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- helpers --- */

static uint32_t f32_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

static float bits_f32(uint32_t u) {
    float f;
    memcpy(&f, &u, 4);
    return f;
}

int oracle_hadamard_entry(int i, int j) {
    /* Sylvester construction H_{2n} = [[H_n, H_n], [H_n, -H_n]] gives
     * H[i][j] = (-1)^(number of bit positions set in both i and j). */
    int both = i & j;
    int parity = 0;
    while (both) {
        parity ^= (both & 1);
        both >>= 1;
    }
    return parity ? -1 : 1;
}

float oracle_bf16_to_f32(uint16_t b) {
    /* bf16 is the upper half of an fp32 bit pattern. */
    return bits_f32(((uint32_t)b) << 16);
}

/* ------------------------------------------------------- transform (fp32) --- */

void oracle_fwht32_f32(float v[32]) {
    /* Fast Walsh-Hadamard transform in natural (Sylvester) order. Stage h combines
     * positions i and i + h for every i with bit h clear. */
    for (int h = 1; h < 32; h <<= 1) {
        for (int i = 0; i < 32; ++i) {
            if (i & h) continue;
            float a = v[i];
            float b = v[i + h];
            v[i] = a + b;
            v[i + h] = a - b;
        }
    }
    /* Normalisation by the fp32 value nearest to 1/sqrt(32) = 2^-2.5. */
    const float c = bits_f32(0x3E3504F3u);
    for (int i = 0; i < 32; ++i) v[i] = v[i] * c;
}

/* ------------------------------------------------------------- MXFP4 codec --- */

int oracle_e8m0_exponent(float amax) {
    uint32_t u = f32_bits(amax) & 0x7FFFFFFFu;
    if (u == 0) return -127;
    int biased = (int)(u >> 23);
    int E;
    if (biased > 0) {
        E = biased - 127; /* normal: floor(log2) is the unbiased exponent */
    } else {
        /* subnormal: value = m * 2^-149, floor(log2) = (index of top set bit of m) - 149 */
        uint32_t m = u & 0x7FFFFFu;
        int top = 31;
        while (!(m & (1u << top))) --top;
        E = top - 149;
    }
    int e = E - 2; /* largest E2M1 magnitude 6 lies in [4, 8) = 2^2 .. 2^3 */
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

uint8_t oracle_e2m1_encode(float q) {
    uint8_t sign = (f32_bits(q) >> 31) ? 0x8 : 0x0;
    float a = fabsf(q);
    uint8_t idx;
    /* Magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 -> index 0..7. Midpoints break toward the
     * value whose mantissa bit is 0 (indices 0, 2, 4, 6); above 5 saturates at 6. */
    if (a <= 0.25f)      idx = 0;
    else if (a < 0.75f)  idx = 1;
    else if (a <= 1.25f) idx = 2;
    else if (a < 1.75f)  idx = 3;
    else if (a <= 2.5f)  idx = 4;
    else if (a < 3.5f)   idx = 5;
    else if (a <= 5.0f)  idx = 6;
    else                 idx = 7;
    return (uint8_t)(sign | idx);
}

double oracle_e2m1_decode(uint8_t code) {
    /* E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit; exponent field 0 is
     * subnormal (0 or 0.5). */
    int s = (code >> 3) & 1;
    int ex = (code >> 1) & 3;
    int m = code & 1;
    double mag = (ex == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, ex - 1);
    return s ? -mag : mag;
}

void oracle_e2m1_encode_array(const float* q, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_encode(q[i]);
}

void oracle_e8m0_exponent_array(const float* amax, int64_t n, int32_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e8m0_exponent(amax[i]);
}

/* --------------------------------------------------------------- rows ------ */

static void quant_block(const float v[32], uint8_t* codes16, uint8_t* scale) {
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    int e = oracle_e8m0_exponent(amax);
    /* q = v * 2^-e is exact: a power-of-two scaling of a value that stays normal. */
    float inv = ldexpf(1.0f, -e);
    for (int j = 0; j < 16; ++j) {
        uint8_t lo = oracle_e2m1_encode(v[2 * j] * inv);
        uint8_t hi = oracle_e2m1_encode(v[2 * j + 1] * inv);
        codes16[j] = (uint8_t)(lo | (hi << 4));
    }
    *scale = (uint8_t)(e + 127);
}

void oracle_quant_rows(const uint16_t* x, int64_t rows, int64_t K, int64_t ld,
                       const float* mult, uint8_t* codes, uint8_t* scales) {
    int64_t Kb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < Kb; ++b) {
            float v[32];
            for (int i = 0; i < 32; ++i) {
                int64_t k = 32 * b + i;
                v[i] = oracle_bf16_to_f32(x[r * ld + k]) * mult[k];
            }
            oracle_fwht32_f32(v);
            quant_block(v, codes + r * (K / 2) + 16 * b, scales + r * Kb + b);
        }
    }
}

/* inv_s = RN32(1 / s), one IEEE fp32 division per channel. */
static void inverse_scales(const float* s, int64_t K, float* inv_s) {
    for (int64_t k = 0; k < K; ++k) inv_s[k] = 1.0f / s[k];
}

void oracle_prepare_weight(const uint16_t* W, int64_t N, int64_t K, int64_t ld,
                           const float* s, uint8_t* codes, uint8_t* scales, float* inv_s) {
    inverse_scales(s, K, inv_s);
    oracle_quant_rows(W, N, K, ld, s, codes, scales);
}

/* -------------------------------------------------------- scale layout ----- */

int64_t oracle_scale_rows_padded(int64_t rows) { return (rows + 127) / 128 * 128; }

int64_t oracle_scale_blocks_padded(int64_t K) { return (K / 32 + 7) / 8 * 8; }

int64_t oracle_scale_offset(int64_t r, int64_t j, int64_t K) {
    /* One atom = 128 rows x 4 consecutive scale blocks = 512 bytes. Inside it, row r
     * sits at (r % 32) * 16 + ((r / 32) % 4) * 4 and block j at j % 4. Atoms of one
     * 128-row slab follow each other along K. */
    int64_t atoms_per_slab = oracle_scale_blocks_padded(K) / 4;
    int64_t atom = (r / 128) * atoms_per_slab + j / 4;
    return atom * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (j % 4);
}

void oracle_swizzle_scales(const uint8_t* rowmajor, int64_t rows, int64_t K, uint8_t* atom) {
    int64_t Kb = K / 32;
    int64_t bytes = oracle_scale_rows_padded(rows) * oracle_scale_blocks_padded(K);
    memset(atom, 0, (size_t)bytes);
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < Kb; ++j)
            atom[oracle_scale_offset(r, j, K)] = rowmajor[r * Kb + j];
}

void oracle_unswizzle_scales(const uint8_t* atom, int64_t rows, int64_t K, uint8_t* rowmajor) {
    int64_t Kb = K / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < Kb; ++j)
            rowmajor[r * Kb + j] = atom[oracle_scale_offset(r, j, K)];
}

/* ------------------------------------------------------------ GEMM (fp64) -- */

void oracle_dequant_rows(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K,
                         double* out) {
    int64_t Kb = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            uint8_t code = (k & 1) ? (byte >> 4) : (byte & 0xF);
            int e = (int)scales[r * Kb + k / 32] - 127;
            out[r * K + k] = ldexp(oracle_e2m1_decode(code), e);
        }
    }
}

void oracle_gemm_fp64(const uint8_t* a_codes, const uint8_t* a_scales, int64_t M,
                      const uint8_t* w_codes, const uint8_t* w_scales, int64_t N, int64_t K,
                      const int64_t* rows, int64_t n_rows, double* y) {
    (void)M;
    double* wdec = (double*)malloc(sizeof(double) * (size_t)(N * K));
    if (!wdec) return;
    oracle_dequant_rows(w_codes, w_scales, N, K, wdec);
    int64_t count = rows ? n_rows : M;
#pragma omp parallel
    {
        /* one decoded activation row per thread (one in all without OpenMP) */
        double* adec = (double*)malloc(sizeof(double) * (size_t)K);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < count; ++i) {
            if (!adec) continue;
            int64_t m = rows ? rows[i] : i;
            oracle_dequant_rows(a_codes + m * (K / 2), a_scales + m * (K / 32), 1, K, adec);
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                const double* wr = wdec + n * K;
                for (int64_t k = 0; k < K; ++k) acc += adec[k] * wr[k];
                y[i * N + n] = acc;
            }
        }
        free(adec);
    }
    free(wdec);
}

/* ------------------------------------------------ exact algebra (fp64) ----- */

void oracle_transform_rows_f64(const double* x, int64_t rows, int64_t K, const double* mult,
                               double norm, double* out) {
    /* Row vector times the block-diagonal matrix: out[32b + j] =
     * sum_i x[32b + i] * mult[32b + i] * H32[i][j] / norm. */
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < K / 32; ++b) {
            for (int j = 0; j < 32; ++j) {
                double acc = 0.0;
                for (int i = 0; i < 32; ++i) {
                    int64_t k = 32 * b + i;
                    acc += x[r * K + k] * mult[k] * (double)oracle_hadamard_entry(i, j);
                }
                out[r * K + 32 * b + j] = acc / norm;
            }
        }
    }
}

/* ----------------------------------------- Hessian exponent search ---------- */

void oracle_transform_block_f32(const uint16_t* x_row, const float* mult, int64_t b, float v[32]) {
    for (int i = 0; i < 32; ++i) {
        int64_t k = 32 * b + i;
        v[i] = oracle_bf16_to_f32(x_row[k]) * mult[k];
    }
    oracle_fwht32_f32(v);
}

void oracle_hessian_blocks(const uint16_t* x, int64_t T, int64_t K, int64_t ld, const float* inv_s,
                           double* H) {
    int64_t Kb = K / 32;
    memset(H, 0, (size_t)(Kb * 32 * 32) * sizeof(double));
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t b = 0; b < Kb; ++b) {
            float v[32];
            oracle_transform_block_f32(x + t * ld, inv_s, b, v);
            double* Hb = H + b * 32 * 32;
            for (int i = 0; i < 32; ++i)
                for (int j = 0; j < 32; ++j) Hb[i * 32 + j] += (double)v[i] * (double)v[j];
        }
    }
}

double oracle_block_error(const double d[32], const double H[32 * 32]) {
    double err = 0.0;
    for (int i = 0; i < 32; ++i) {
        double r = 0.0;
        for (int j = 0; j < 32; ++j) r += H[i * 32 + j] * d[j];
        err += d[i] * r;
    }
    return err;
}

double oracle_block_error_at(const float v[32], int e, const double H[32 * 32], uint8_t codes16[16]) {
    float inv = ldexpf(1.0f, -e);
    double d[32];
    for (int j = 0; j < 16; ++j) {
        uint8_t lo = oracle_e2m1_encode(v[2 * j] * inv);
        uint8_t hi = oracle_e2m1_encode(v[2 * j + 1] * inv);
        codes16[j] = (uint8_t)((hi << 4) | lo);             /* element 2j in the low nibble */
        d[2 * j] = (double)v[2 * j] - ldexp(oracle_e2m1_decode(lo), e);
        d[2 * j + 1] = (double)v[2 * j + 1] - ldexp(oracle_e2m1_decode(hi), e);
    }
    return oracle_block_error(d, H);
}

void oracle_search_block(const float v[32], const double H[32 * 32], uint8_t codes16[16], uint8_t* scale) {
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    int e0 = oracle_e8m0_exponent(amax);
    int cand[3] = {e0, e0 + 1, e0 - 1};
    int best_e = e0;
    double best = 0.0;
    int have = 0;
    for (int c = 0; c < 3; ++c) {
        int e = cand[c];
        if (e < -127 || e > 127) continue;
        uint8_t tmp[16];
        double err = oracle_block_error_at(v, e, H, tmp);
        if (!have || err < best) {
            best = err;
            best_e = e;
            memcpy(codes16, tmp, 16);
            have = 1;
        }
    }
    *scale = (uint8_t)(best_e + 127);
}

void oracle_prepare_weight_hessian(const uint16_t* W, int64_t N, int64_t K, int64_t ld, const float* s,
                                   const double* H, uint8_t* codes, uint8_t* scales, float* inv_s) {
    int64_t Kb = K / 32;
    inverse_scales(s, K, inv_s);
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < Kb; ++b) {
            float v[32];
            oracle_transform_block_f32(W + n * ld, s, b, v);
            oracle_search_block(v, H + b * 32 * 32, codes + n * (K / 2) + 16 * b, scales + n * Kb + b);
        }
    }
}

/* ----------------------------------------------------- Flip-Refinement ------ */

void oracle_hessian_full(const uint16_t* x, int64_t T, int64_t K, int64_t ld, const float* inv_s, double* H) {
    int64_t Kb = K / 32;
    float* v = (float*)malloc((size_t)K * sizeof(float));
    memset(H, 0, (size_t)(K * K) * sizeof(double));
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t b = 0; b < Kb; ++b) oracle_transform_block_f32(x + t * ld, inv_s, b, v + 32 * b);
        for (int64_t i = 0; i < K; ++i)
            for (int64_t j = 0; j < K; ++j) H[i * K + j] += (double)v[i] * (double)v[j];
    }
    free(v);
}

/* The 15 signed E2M1 values in increasing order; index 7 is zero. */
static const double kFlipGrid[15] = {-6.0, -4.0, -3.0, -2.0, -1.5, -1.0, -0.5, 0.0,
                                     0.5,  1.0,  1.5,  2.0,  3.0,  4.0,  6.0};

static int flip_index(uint8_t code) {
    int m = code & 7;
    if (m == 0) return 7;
    return (code & 8) ? 7 - m : 7 + m;
}

static uint8_t flip_code(int index) {
    if (index == 7) return 0;
    return index > 7 ? (uint8_t)(index - 7) : (uint8_t)(8 | (7 - index));
}

int oracle_flip_refine_row(const float* wv, const double* H, int64_t K, uint8_t* codes, const uint8_t* scales_row,
                           int max_rounds) {
    double* e = (double*)malloc((size_t)K * sizeof(double));
    double* g = (double*)malloc((size_t)K * sizeof(double));
    int* idx = (int*)malloc((size_t)K * sizeof(int));
    for (int64_t k = 0; k < K; ++k) {
        uint8_t byte = codes[k / 2];
        uint8_t code = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
        idx[k] = flip_index(code);
        e[k] = (double)wv[k] - ldexp(kFlipGrid[idx[k]], (int)scales_row[k / 32] - 127);
    }
    for (int64_t j = 0; j < K; ++j) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc = fma(H[j * K + k], e[k], acc);
        g[j] = acc;
    }
    int moves = 0;
    for (int round = 0; round < max_rounds; ++round) {
        double best = 0.0;
        int64_t bk = -1;
        int bdir = 0;
        double bdelta = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            int sc = (int)scales_row[k / 32] - 127;
            for (int dir = -1; dir <= 1; dir += 2) {
                int ni = idx[k] + dir;
                if (ni < 0 || ni > 14) continue;
                double delta = ldexp(kFlipGrid[ni] - kFlipGrid[idx[k]], sc);
                double a = delta * delta;
                double b2 = a * H[k * K + k];
                double c = (2.0 * delta) * g[k];
                double dE = b2 - c;
                if (dE < best) {
                    best = dE;
                    bk = k;
                    bdir = dir;
                    bdelta = delta;
                }
            }
        }
        if (bk < 0) break;
        idx[bk] += bdir;
        uint8_t nc = flip_code(idx[bk]);
        uint8_t* byte = &codes[bk / 2];
        *byte = (bk & 1) ? (uint8_t)((*byte & 0x0F) | (nc << 4)) : (uint8_t)((*byte & 0xF0) | nc);
        e[bk] -= bdelta;
        for (int64_t j = 0; j < K; ++j) g[j] = fma(-bdelta, H[bk * K + j], g[j]);
        ++moves;
    }
    free(idx);
    free(g);
    free(e);
    return moves;
}

void oracle_flip_refine(const uint16_t* W, int64_t N, int64_t K, int64_t ld, const float* s, const double* H,
                        uint8_t* codes, const uint8_t* scales, int max_rounds, int32_t* moves) {
    int64_t Kb = K / 32;
    float* wv = (float*)malloc((size_t)K * sizeof(float));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < Kb; ++b) oracle_transform_block_f32(W + n * ld, s, b, wv + 32 * b);
        moves[n] = oracle_flip_refine_row(wv, H, K, codes + n * (K / 2), scales + n * Kb, max_rounds);
    }
    free(wv);
}
