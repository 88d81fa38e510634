/*
 * Test infrastructure: the CPU oracle of the MACaQ W4A4 linear layer.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may load this
 * library. The product path (the CUDA library and its Python binding) never calls it,
 * and the two share no code, header, table or constant generator.
 *
 * What it computes (MACaQ pages: "Quantization mechanism" of the zicq.com English
 * article, equation y = xW^T and the garbled transformed form; openai-hub.com
 * article, paragraphs on MXFP4 and on the block Hadamard "micro-rotation"):
 *
 *   y = x W^T = (x D^-1 Hb) (Hb D W^T),   D = diag(s),
 *   Hb = block-diag(H32 / sqrt(32)), H32 the Sylvester Hadamard matrix,
 *
 * with both factors quantised to OCP MXFP4 (E2M1 elements, one E8M0 scale per 32).
 *
 * Precision: the quantisation steps run in IEEE fp32 with round-to-nearest-even,
 * no FMA contraction, in the fixed butterfly order given below,
 * because the fp32 result decides integer codes. The GEMM reference and the
 * exact-algebra helpers run in fp64.
 *
 * Parity status: every function below is pinned by tests in tests/test_oracle_*.py
 * against closed forms, library routines (scipy's Hadamard, numpy matmul) or brute
 * force; none is "parity unpinned".
 */
#ifndef MACAQ_ORACLE_H
#define MACAQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* (-1)^popcount(i & j): entry (i, j) of the natural-order Sylvester matrix H_n. */
int oracle_hadamard_entry(int i, int j);

/* Widen a bf16 bit pattern to fp32 (exact: bf16 is the upper half of an fp32). */
float oracle_bf16_to_f32(uint16_t b);

/* In-place 32-point Walsh-Hadamard butterfly in fp32, stages h = 1,2,4,8,16,
 * pair (a, b) -> (a + b, a - b) with a at the lower index, then every element is
 * multiplied by c = fp32(1/sqrt(32)) (bit pattern 0x3E3504F3). */
void oracle_fwht32_f32(float v[32]);

/* Shared-exponent rule: e = max(floor(log2 amax) - 2, -127); amax == 0 gives -127.
 * floor(log2) is read exactly from the fp32 bit pattern. Returns e in [-127, 125]. */
int oracle_e8m0_exponent(float amax);

/* E2M1 round-to-nearest, ties to the even mantissa bit, saturating at +-6.
 * Returns the 4-bit code (sign << 3 | index into {0,.5,1,1.5,2,3,4,6}); the sign of
 * q is kept, so -0 and tiny negatives encode as 0x8. */
uint8_t oracle_e2m1_encode(float q);

/* Decode a 4-bit E2M1 code to its value. */
double oracle_e2m1_decode(uint8_t code);

/* Element-wise loops over the two scalar rules above, for sweeps from tests. */
void oracle_e2m1_encode_array(const float* q, int64_t n, uint8_t* out);
void oracle_e8m0_exponent_array(const float* amax, int64_t n, int32_t* out);

/* Quantise rows of a bf16 matrix through the MACaQ transform.
 *   x      : bf16 bits, rows x K, row stride ld (elements)
 *   mult   : K fp32 multipliers (inv_s for activations, s for weights)
 *   codes  : rows x K/2 bytes, element 2j in the low nibble of byte j
 *   scales : rows x K/32 bytes, row-major E8M0 (value 2^(byte - 127))
 * K must be a multiple of 32. */
void oracle_quant_rows(const uint16_t* x, int64_t rows, int64_t K, int64_t ld,
                       const float* mult, uint8_t* codes, uint8_t* scales);

/* Offline weight preparation: W' = W D Hb quantised like the activations
 * (multiplier s), and inv_s[k] = 1.0f / s[k] in IEEE fp32. */
void oracle_prepare_weight(const uint16_t* W, int64_t N, int64_t K, int64_t ld,
                           const float* s, uint8_t* codes, uint8_t* scales, float* inv_s);

/* Padded geometry of the tensor-core scale layout: rows rounded up to 128, scale
 * blocks per row rounded up to 8 (a whole number of 4-block atoms per 256-wide
 * K tile). */
int64_t oracle_scale_rows_padded(int64_t rows);
int64_t oracle_scale_blocks_padded(int64_t K);

/* Byte offset of scale (r, j) in the 128-row x 4-block atom layout consumed by the
 * Blackwell block-scaled MMA. */
int64_t oracle_scale_offset(int64_t r, int64_t j, int64_t K);

/* Row-major [rows x K/32] scales -> atom layout (padding bytes set to 0), and back. */
void oracle_swizzle_scales(const uint8_t* rowmajor, int64_t rows, int64_t K, uint8_t* atom);
void oracle_unswizzle_scales(const uint8_t* atom, int64_t rows, int64_t K, uint8_t* rowmajor);

/* y[m, n] = sum_k dec(a[m,k]) 2^ea[m,k/32] * dec(w[n,k]) 2^ew[n,k/32], summed in fp64.
 * Codes as produced by oracle_quant_rows, scales row-major. Rows of A listed in
 * `rows` (or all M rows if rows == NULL), output row i is y + i * N. */
void oracle_gemm_fp64(const uint8_t* a_codes, const uint8_t* a_scales, int64_t M,
                      const uint8_t* w_codes, const uint8_t* w_scales, int64_t N, int64_t K,
                      const int64_t* rows, int64_t n_rows, double* y);

/* Dequantise MXFP4 rows to fp64 (value = dec(code) * 2^e). */
void oracle_dequant_rows(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K,
                         double* out);

/* Exact-algebra transform in fp64 with the dense block matrix (no butterfly, no
 * quantisation): out[r, :] = (x[r, :] * mult) Hb_unnormalised / norm, where
 * Hb_unnormalised has +-1 entries and norm is a caller-chosen divisor (sqrt(32) for
 * the orthonormal transform, 1 for the raw +-1 product). */
void oracle_transform_rows_f64(const double* x, int64_t rows, int64_t K, const double* mult,
                               double norm, double* out);

/* ------------------------------------------------------------------------------
 * Hessian exponent search for weight blocks (the "Hessian exponent search" step of the
 * ablation paragraph of the openai-hub.com article, between round-to-nearest and the
 * micro-rotation; its error model is the second-order form
 *   dL ~ 1/2 (w - w_hat)^T H (w - w_hat)
 * of the Flip-Refinement paragraph of the zicq.com articles). Reading taken: H is the
 * Gram matrix X'^T X' of calibration activations in the transformed basis (the fp32
 * values oracle_quant_rows quantises), restricted to its 32 x 32 diagonal blocks, and
 * each weight block keeps the exponent, among e0 (the floor rule), e0 + 1 and e0 - 1,
 * with the smallest d^T H_b d, d = w' - dec(codes) 2^e.
 * ---------------------------------------------------------------------------- */

/* The transformed block v (32 fp32 values) of row r, block b: fwht32 of x * mult. */
void oracle_transform_block_f32(const uint16_t* x_row, const float* mult, int64_t b, float v[32]);

/* H[b][i][j] = sum_t v_t[i] v_t[j] over the calibration rows t = 0 .. T-1 (ascending),
 * v_t the transformed block b of row t under multiplier inv_s. fp64: each product of
 * two fp32 values is exact, so only the running sum rounds. H: [K/32][32][32]. */
void oracle_hessian_blocks(const uint16_t* x, int64_t T, int64_t K, int64_t ld, const float* inv_s,
                           double* H);

/* d^T H d for one block, fp64: sum over i ascending of d[i] * r[i], where
 * r[i] = sum over j ascending of H[i][j] * d[j]; every product and sum rounded on its own. */
double oracle_block_error(const double d[32], const double H[32 * 32]);

/* Encode v under exponent e (codes of v * 2^-e, as the floor-rule path encodes) and
 * return d^T H d with d = v - dec(codes) * 2^e (exact in fp64). */
double oracle_block_error_at(const float v[32], int e, const double H[32 * 32], uint8_t codes16[16]);

/* One block of the search: candidates e0, e0 + 1, e0 - 1 (those within [-127, 127]), in
 * that order; a candidate replaces the current choice only with a strictly smaller
 * error. Writes the 16 code bytes and the scale byte e + 127. */
void oracle_search_block(const float v[32], const double H[32 * 32], uint8_t codes16[16], uint8_t* scale);

/* Weight preparation with the exponent search: as oracle_prepare_weight, with every
 * block of every row chosen by oracle_search_block under H[b]. */
void oracle_prepare_weight_hessian(const uint16_t* W, int64_t N, int64_t K, int64_t ld, const float* s,
                                   const double* H, uint8_t* codes, uint8_t* scales, float* inv_s);

/* ------------------------------------------------------------------------------
 * Flip-Refinement of weight codes (the Flip-Refinement paragraphs of the zicq.com
 * articles and of the openai-hub.com article: starting from quantised weights, each
 * round moves, for every output row, the one code whose move to an adjacent
 * representable value lowers the second-order error most; a row stops when no such move
 * lowers it). Reading taken: the error of row n is E = e^T H e, e = w' - w_hat (the
 * transformed weight row minus its dequantised codes), H the full K x K Gram matrix of
 * the transformed calibration rows; block scales stay fixed; the representable values of
 * a coordinate are the 15 signed E2M1 values times its block scale. With g = H e, moving
 * coordinate k by delta changes E by delta^2 H_kk - 2 delta g_k, and g then changes by
 * -delta H[k, :].
 * ---------------------------------------------------------------------------- */

/* H[i][j] = sum_t v_t[i] v_t[j] over all K columns (t ascending), fp64, K x K. */
void oracle_hessian_full(const uint16_t* x, int64_t T, int64_t K, int64_t ld, const float* inv_s, double* H);

/* One row. wv: the K transformed fp32 weight values; codes: K/2 bytes, refined in place;
 * scales_row: K/32 E8M0 bytes (row-major); at most max_rounds moves. fp64 throughout:
 *   e_k = wv_k - value(code_k) 2^(scale - 127)                   (exact)
 *   g_j = fma chain over k ascending of H[j][k] * e_k, from 0
 *   for each k ascending, first the lower then the higher neighbour value:
 *     delta = (neighbour - value) 2^(scale - 127)                 (exact)
 *     dE = (delta * delta) * H[k][k] - (2 delta) * g_k           (each op rounded)
 *   the first strictly smallest dE < 0 is taken (none: the row stops);
 *   then e_k -= delta and g_j = fma(-delta, H[k][j], g_j) for every j.
 * A move to the value 0 writes code 0 (+0). Returns the number of moves. */
int oracle_flip_refine_row(const float* wv, const double* H, int64_t K, uint8_t* codes, const uint8_t* scales_row,
                           int max_rounds);

/* Every row of a prepared weight: wv from W and s by the weight transform, codes
 * (N x K/2) refined in place, scales row-major (N x K/32); moves[n] receives the count. */
void oracle_flip_refine(const uint16_t* W, int64_t N, int64_t K, int64_t ld, const float* s, const double* H,
                        uint8_t* codes, const uint8_t* scales, int max_rounds, int32_t* moves);

#ifdef __cplusplus
}
#endif

#endif
