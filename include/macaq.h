/*
 * libmacaq: MACaQ W4A4 linear layer on NVIDIA B200 (sm_100a), C ABI.
 *
 * The layer (MACaQ pages: zicq.com "MACaQ Enables Streaming W4A4 Quantization",
 * section "Quantization mechanism", equation y = xW^T and its transformed form;
 * abstract on the Hugging Face papers mirror; openai-hub.com "华为开源MACaQ",
 * paragraphs on MXFP4 and on the 32-element block Hadamard rotation):
 *
 *     y = x W^T = (x D^-1 Hb) (Hb D W^T),   D = diag(s),
 *
 * Hb block-diagonal with 32x32 Sylvester Hadamard blocks scaled by 1/sqrt(32), the
 * blocks aligned with the 32-element MXFP4 groups. The weight factor Hb D W^T is
 * computed once, ahead of inference; at inference the activation is scaled, rotated
 * and quantised online, then both MXFP4 operands meet in a block-scaled FP4 GEMM.
 *
 * Conventions shared by every entry point:
 *  - Pointers marked "device" are CUDA device pointers of the current device; the
 *    caller allocates and owns every buffer. The library allocates no memory. Its only
 *    state is static: one device-side error word per device, the scratch array of
 *    macaq_linear_w4a4_noalloc, the self-test's result words, and per-device host
 *    facts (SM count, symbol addresses) looked up on first use.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *    A returned MACAQ_OK means the work was validated and enqueued. Host arrays passed
 *    in (offsets, weight descriptors, destination addresses) are read before the call
 *    returns and may be reused at once: per-call tables reach the device inside kernel
 *    parameters, never through a copy that waits for the stream. Exceptions:
 *    macaq_selftest_wait_timeout and macaq_get_device_error synchronise.
 *  - The library looks up, once per device, the device addresses of its static arrays
 *    (the error word, the no-allocation scratch) and keeps them for the life of the
 *    process: do not keep using it on a device after cudaDeviceReset.
 *  - Arguments are validated on the host before any launch; a failed check returns an
 *    error code and enqueues nothing. Nothing throws or aborts across the ABI.
 *  - Only devices of compute capability 10.0 (B200, sm_100a) are supported.
 *  - Inputs must be finite, and scaled/rotated values must stay finite in fp32;
 *    anything else is out of contract.
 *
 * MXFP4 storage, 4.25 bits per element (the storage figure per weight in the
 * openai-hub.com article's FLUX comparison paragraph):
 *  - codes : rows x K/2 bytes, row stride K/2; element 2j of a row in the low nibble of
 *            byte j; E2M1 code = sign<<3 | {0,.5,1,1.5,2,3,4,6} index.
 *  - scales: E8M0 bytes (value 2^(byte-127)), one per 32 elements, in the tensor-core
 *            atom layout: rows padded to a multiple of 128, scale blocks per row
 *            padded to a multiple of 8; scale (r, j) at byte
 *              ((r/128) * (Kb_pad/4) + j/4) * 512 + (r%32)*16 + ((r/32)%4)*4 + j%4
 *            with Kb_pad = round_up(K/32, 8). Padding bytes are 0.
 */
#ifndef MACAQ_H
#define MACAQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MACAQ_VERSION 1

/* Same object as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* macaq_stream;

typedef enum {
    MACAQ_OK = 0,
    MACAQ_ERR_INVALID_ARG = 1,        /* null pointer, non-positive size, bad enum */
    MACAQ_ERR_MISALIGNED = 2,         /* pointer or leading dimension not aligned */
    MACAQ_ERR_UNSUPPORTED_SHAPE = 3,  /* K % 32 != 0, sizes beyond the documented limits */
    MACAQ_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not compute capability 10.0 */
    MACAQ_ERR_CUDA = 5,               /* a CUDA runtime/driver call or launch failed */
    MACAQ_ERR_DEVICE_TIMEOUT = 6,     /* a kernel gave up a bounded wait (see below) */
    MACAQ_ERR_WORKSPACE = 7,          /* workspace pointer null or smaller than required */
    MACAQ_ERR_UNSUPPORTED = 8         /* a documented option that is not built */
} macaq_status;

typedef enum { MACAQ_OUT_F32 = 0, MACAQ_OUT_BF16 = 1 } macaq_out_dtype;

/* Prepared weight (the offline artefact): codes/scales of W' = W D Hb, plus the
 * activation multiplier inv_s = 1/s. All three device pointers, owned by the caller. */
typedef struct {
    const uint8_t* codes;  /* device, N x K/2 bytes, 16-byte aligned */
    const uint8_t* scales; /* device, macaq_scales_bytes(N, K) bytes, 16-byte aligned */
    const float* inv_s;    /* device, K floats, 16-byte aligned */
    int64_t N;             /* output features */
    int64_t K;             /* input features, multiple of 32 */
} macaq_weight;

/* ------------------------------------------------------------- sizes ---------- */

/* Bytes of the packed E2M1 codes of a rows x K matrix: rows * K / 2. */
size_t macaq_codes_bytes(int64_t rows, int64_t K);

/* Bytes of the padded scale layout of a rows x K matrix:
 * round_up(rows, 128) * round_up(K/32, 8). */
size_t macaq_scales_bytes(int64_t rows, int64_t K);

/* Device workspace macaq_gemm_mxfp4 needs for an M x N x K product with output
 * `out`: when the library runs the product on its stream-K schedule (decode shapes,
 * M <= 32, whose last round of weight tiles would leave SMs idle: each tile of that
 * round is split in two halves of its K range taken by two CTAs), two fp32 partial
 * tiles per CTA and an arrival counter per output tile; 0 otherwise. Its contents need
 * no clearing. */
size_t macaq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, macaq_out_dtype out);

/* Device workspace macaq_linear_w4a4 needs: the activation codes and scales, then the
 * GEMM workspace, each 256-byte aligned. */
size_t macaq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, macaq_out_dtype out);

/* ------------------------------------------------------------ compute --------- */

/* Offline weight preparation (pages: the weight factor is folded in before
 * quantisation; round-to-nearest baseline of the ablation in the openai-hub.com
 * article). For each row n of W: w = fp32(W[n,:]) * s (fp32, per channel), then per
 * 32-block the normalised Hadamard butterfly, the E8M0 exponent
 * e = max(floor(log2 amax) - 2, -127) and round-to-nearest-even E2M1 codes.
 * Also writes inv_s[k] = 1.0f / s[k] (IEEE fp32 division).
 *   W_bf16    device bf16 [N x K], row stride ldw elements (ldw >= K, ldw % 8 == 0),
 *             16-byte aligned
 *   s         device fp32 [K], 16-byte aligned, finite and non-zero
 *   w_codes   device, macaq_codes_bytes(N, K), 16-byte aligned
 *   w_scales  device, macaq_scales_bytes(N, K), 16-byte aligned (padding written 0)
 *   inv_s_out device fp32 [K], 16-byte aligned
 * K % 32 == 0, N >= 1. */
macaq_status macaq_prepare_weight(const void* W_bf16, int64_t N, int64_t K, int64_t ldw,
                                  const float* s, uint8_t* w_codes, uint8_t* w_scales,
                                  float* inv_s_out, macaq_stream stream);

/* Online activation transform (pages: per-channel scale and block Hadamard applied
 * online to each layer's activation, then MXFP4): for each row m,
 * u = fp32(x[m,:]) * inv_s, then the same block transform and encoding as above.
 *   x_bf16   device bf16 [M x K], row stride ldx elements (ldx >= K, ldx % 8 == 0),
 *            16-byte aligned
 *   inv_s    device fp32 [K] (normally macaq_weight.inv_s), 16-byte aligned
 *   a_codes  device, macaq_codes_bytes(M, K); a_scales device, macaq_scales_bytes(M, K)
 * Results are bit-identical to the CPU definition for every finite input. */
macaq_status macaq_quant_act(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                             const float* inv_s, uint8_t* a_codes, uint8_t* a_scales,
                             macaq_stream stream);

/* Block-scaled FP4 GEMM on pre-quantised operands (pages: the FP4 matrix product
 * that follows the activation transform; W4A4 definition in the openai-hub.com
 * article):
 *   y[m, n] = sum_b 2^(ea[m,b] + ew[n,b]) * sum_{k in b} dec(a[m,k]) * dec(w[n,k]),
 * fp32 accumulation on the tensor cores (tcgen05 kind::mxf4). Large prefill products
 * run on clusters of two CTAs (256-row tiles, cta_group::2 MMAs), products with few
 * long-K tiles on clusters of 2-4 CTAs that share each tile's K range, the rest on single
 * CTAs; the choice is the library's and does not change the result's tolerance. Every
 * plan gives the same y for the same inputs, call after call.
 *   a_codes/a_scales device, as written by macaq_quant_act for M rows
 *   w        prepared weight (inv_s unused here)
 *   y        device [M x N] fp32 or bf16, row stride ldy elements (ldy >= N), aligned
 *            to its element size (16-byte alignment of y and of ldy * element size
 *            enables vector stores)
 *   workspace device, >= macaq_gemm_workspace_bytes(M, N, K, out), 256-byte aligned
 *            (may be NULL when that size is 0). Contents are scratch and need no
 *            clearing: a stream-K product's CTAs never wait for one another; the last
 *            contributor to a shared output tile adds the partial tiles, in the order
 *            of their K ranges, and writes it, and each call tags its arrival counters
 *            with a value unique to the call. Two calls that may run at the same time
 *            must not share it.
 * M >= 1. Also the entry point for externally refined weight codes/scales. */
macaq_status macaq_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_scales, int64_t M,
                              const macaq_weight* w, void* y, int64_t ldy, macaq_out_dtype out,
                              void* workspace, size_t ws_bytes, macaq_stream stream);

/* The whole online layer: the activation transform of macaq_quant_act into the
 * workspace, then the GEMM of macaq_gemm_mxfp4.
 *   fused     0: two launches (macaq_quant_act's kernel, then the GEMM).
 *             1: one launch where that is the faster form: for M <= 2 (decode) the GEMM
 *             kernel makes the MXFP4 activations itself, before its main loop, in the
 *             shared memory its tensor-core MMAs read them from (the per-channel
 *             multiplier, block Hadamard, E8M0 exponent and E2M1 encoding of
 *             macaq_quant_act, bit for bit), while the weight tiles stream in; every CTA
 *             repeats that transform, so for more rows two launches are faster and are
 *             used. y is bit-identical to fused = 0, and the activation part of the
 *             workspace is not written.
 *             2: as 1, for every M <= 32 whose MXFP4 activations fit in shared memory
 *             beside the weight ring (K <= 7680 for M <= 16, K <= 6400 for M <= 32);
 *             for callers that want a single launch whatever it costs. Other shapes as 0.
 *             Other values return MACAQ_ERR_INVALID_ARG.
 *   workspace device, >= macaq_linear_workspace_bytes(M, N, K, out), 256-byte aligned;
 *             it starts with the activation codes (macaq_codes_bytes(M, K) bytes) and,
 *             256-byte aligned after them, the scales (macaq_scales_bytes(M, K) bytes)
 * Other arguments as for macaq_quant_act / macaq_gemm_mxfp4. */
macaq_status macaq_linear_w4a4(const void* x_bf16, int64_t M, int64_t ldx, const macaq_weight* w,
                               void* y, int64_t ldy, macaq_out_dtype out, int fused,
                               void* workspace, size_t ws_bytes, macaq_stream stream);

/* ------------------------------- gathered output (column-parallel layers) ----- */

/* macaq_linear_w4a4 for one rank of a column-parallel layer (the pages have no
 * tensor parallelism; the cut follows from the layer being row-wise in W', whose
 * quantisation is row by row): the GEMM's epilogue writes this rank's y columns
 * straight into each of n_dest full-width outputs (every rank's y, when the caller maps
 * the other GPUs' buffers into this process), so no separate all-gather is needed.
 *   dest      host [n_dest] device addresses: dest[d] is the address of row 0, column
 *             n0 of destination d (n0 = this rank's first output column); each
 *             destination has row stride ldy elements (ldy >= w->N) and room for M rows
 *             of w->N columns from there; aligned to the element size. Memory of another
 *             GPU must be accessible from this device (peer access or an IPC mapping).
 *   n_dest    1 .. 64
 *   workspace >= macaq_linear_gather_workspace_bytes(M, N, K, out) (the same size as
 *             macaq_linear_w4a4's), 256-byte aligned. The destination addresses travel in
 *             the GEMM kernel's parameters.
 * Every destination receives the same values that macaq_linear_w4a4 (fused = 0) would
 * write to y, except that every output tile is computed by one CTA over its whole K
 * range (no stream-K schedule, no K split over a cluster, no CTA pairs), so sums may
 * round differently. Completion of the writes into another
 * GPU's memory is ordered for that GPU only by the caller (for example a barrier on
 * both streams after the call). */
size_t macaq_linear_gather_workspace_bytes(int64_t M, int64_t N, int64_t K, macaq_out_dtype out);
macaq_status macaq_linear_w4a4_gather(const void* x_bf16, int64_t M, int64_t ldx, const macaq_weight* w,
                                      const uint64_t* dest, int n_dest, int64_t ldy, macaq_out_dtype out,
                                      void* workspace, size_t ws_bytes, macaq_stream stream);

/* --------------------------------------------- grouped layer (MoE experts) ----- */

/* The layer for the routed experts of a mixture-of-experts block (the pages' remark that
 * MACaQ targets MoE models and a grouped matmul kernel, openai-hub.com article): the
 * tokens arrive sorted by expert; expert g owns rows offsets[g] .. offsets[g+1] - 1 of x
 * and y and its own prepared weight weights[g] (own s, so its own online transform).
 * One quantiser launch puts every group's rows through the activation transform with
 * its own weights[g].inv_s, then one GEMM launch covers every group's tiles (prefill
 * orientation, 128- or 192-wide weight tiles).
 *   offsets   host [G + 1], offsets[0] == 0, non-decreasing (empty groups allowed)
 *   weights   host [G], all with the same N and K
 *   x_bf16    device bf16 [offsets[G] x K], row stride ldx; y device [offsets[G] x N]
 *   workspace >= macaq_grouped_linear_workspace_bytes(offsets, G, K), 256-byte aligned:
 *             activation codes and scales with every group padded to 128 rows, the
 *             per-group tables of the GEMM and the quantiser's table of non-empty groups
 *             (built on the host and written by small kernels that carry them in their
 *             parameters, 16 KB per launch, ahead of the two compute launches)
 * G <= 4096. */
size_t macaq_grouped_linear_workspace_bytes(const int64_t* offsets, int64_t G, int64_t K);
macaq_status macaq_grouped_linear_w4a4(const void* x_bf16, int64_t ldx, const int64_t* offsets, int64_t G,
                                       const macaq_weight* weights, void* y, int64_t ldy, macaq_out_dtype out,
                                       void* workspace, size_t ws_bytes, macaq_stream stream);

/* ----------------------------------- layers that share one input (one launch each) --- */

/* Several MACaQ layers that read the same activation x: the q, k and v projections of
 * an attention block, or the gate and up projections of an MLP (the pages apply the
 * per-channel scale and block Hadamard to each linear layer's input separately; each
 * weight carries its own s, so x goes through each weight's own online transform). One
 * quantiser launch transforms x once per weight, with weights[g].inv_s, and one GEMM
 * launch covers every weight's output tiles (prefill orientation, 128- or 192-wide
 * weight tiles); y[g] = the layer of weights[g] applied to x, exactly what
 * macaq_linear_w4a4 gives up to the order of fp32 sums.
 *   x_bf16    device bf16 [M x K], row stride ldx (ldx >= K, ldx % 8 == 0), 16-byte
 *             aligned
 *   weights   host [G], all with the same K (N may differ)
 *   y         host [G] device pointers: y[g] is [M x weights[g].N], fp32 or bf16 per
 *             `out`, row stride ldy[g] (host [G]), aligned to the element size
 *   workspace >= macaq_multi_linear_workspace_bytes(M, K, G), 256-byte aligned: the
 *             activation codes and scales of every weight's transform (each padded to
 *             128 rows), then the GEMM's tables (written by small kernels that carry
 *             them in their parameters)
 * 1 <= G <= 4096. */
size_t macaq_multi_linear_workspace_bytes(int64_t M, int64_t K, int64_t G);
macaq_status macaq_multi_linear_w4a4(const void* x_bf16, int64_t M, int64_t ldx, const macaq_weight* weights,
                                     int64_t G, void* const* y, const int64_t* ldy, macaq_out_dtype out,
                                     void* workspace, size_t ws_bytes, macaq_stream stream);

/* ------------------------------------------ Hessian exponent search (offline) --- */

/* The "Hessian exponent search" step of the ablation paragraph of the openai-hub.com
 * article, with the second-order error model dL ~ 1/2 (w - w_hat)^T H (w - w_hat) of the
 * Flip-Refinement paragraphs of the zicq.com articles. H is taken as the Gram matrix
 * of calibration activations in the transformed basis, restricted to its 32 x 32
 * diagonal blocks; each weight block keeps, of the exponents e0 (the floor rule), e0 + 1
 * and e0 - 1, the one with the smallest d^T H_b d. Only the weight bytes change: the
 * result feeds macaq_gemm_mxfp4 / macaq_linear_w4a4 like macaq_prepare_weight's. */

/* Bytes of the H block array for K: (K/32) * 32 * 32 doubles (0 if K % 32 != 0). */
size_t macaq_hessian_bytes(int64_t K);

/* H[b][i][j] = sum over t = 0 .. T-1 (in that order) of v_t[32b+i] * v_t[32b+j], fp64,
 * where v_t is calibration row t after the online transform of macaq_quant_act with
 * inv_s = RN32(1/s) (the fp32 values before quantisation). Each product of two fp32
 * values is exact in fp64, so only the running sum rounds: the result is bit-identical
 * to that sequential definition.
 *   x_bf16  device bf16 [T x K], row stride ldx (ldx >= K, ldx % 8 == 0), 16-byte aligned
 *   s       device fp32 [K], 16-byte aligned
 *   H       device fp64, macaq_hessian_bytes(K), 16-byte aligned, row-major [K/32][32][32]
 * T >= 1, K % 32 == 0. */
macaq_status macaq_hessian_blocks(const void* x_bf16, int64_t T, int64_t K, int64_t ldx, const float* s, double* H,
                                  macaq_stream stream);

/* macaq_prepare_weight with the exponent search: for every 32-block of every row of
 * W' = W diag(s) Hb, candidates e0, e0 + 1, e0 - 1 (within [-127, 127]); for each, the
 * round-to-nearest codes of fp32(v * 2^-e) and d = v - dec(codes) 2^e (exact in fp64);
 * error = sum_i d_i * (sum_j H_b[i][j] * d_j), i and j ascending, every fp64 product and
 * sum rounded on its own; a later candidate replaces the choice only when its error is
 * strictly smaller. Codes, scales (same layout and padding as macaq_prepare_weight) and
 * inv_s are written; bit-identical to that definition.
 *   H       device fp64 [K/32][32][32] (from macaq_hessian_blocks or the caller)
 * Other arguments as for macaq_prepare_weight. */
macaq_status macaq_prepare_weight_hessian(const void* W_bf16, int64_t N, int64_t K, int64_t ldw, const float* s,
                                          const double* H, uint8_t* w_codes, uint8_t* w_scales, float* inv_s_out,
                                          macaq_stream stream);

/* ------------------------------------------------ Flip-Refinement (offline) ----- */

/* The Flip-Refinement paragraphs of the zicq.com and openai-hub.com articles: after
 * quantisation, each round moves, for every output row, the one code whose step to an
 * adjacent representable value lowers the second-order error most; a row stops when no
 * step lowers it. Error of row n: e^T H e, e = w' - w_hat (transformed weights minus the
 * dequantised codes), H the full K x K Gram matrix of transformed calibration rows
 * (macaq_hessian_full). Block scales stay fixed; codes move along the 15 signed E2M1
 * values. Only weight codes change: the result feeds the same GEMM. */

/* Workspace of macaq_hessian_full: the fp32 transformed calibration rows (T x K). */
size_t macaq_hessian_full_workspace_bytes(int64_t T, int64_t K);

/* H[i][j] = sum over t = 0 .. T-1 (in that order) of v_t[i] * v_t[j], fp64, K x K,
 * v_t calibration row t after the online transform with inv_s = RN32(1/s); exactly
 * symmetric (both halves from the same products). Bit-identical to that sequential
 * definition (products of two fp32 values are exact in fp64).
 *   x_bf16 [T x K] (ldx >= K, ldx % 8 == 0), s [K], H [K x K] fp64: device, 16-byte aligned
 *   workspace >= macaq_hessian_full_workspace_bytes(T, K), 16-byte aligned
 * K % 32 == 0, K <= 8192. */
macaq_status macaq_hessian_full(const void* x_bf16, int64_t T, int64_t K, int64_t ldx, const float* s, double* H,
                                void* workspace, size_t ws_bytes, macaq_stream stream);

/* Workspace of macaq_flip_refine: transformed weight rows (fp32) and their initial
 * gradients (fp64), N x K each. */
size_t macaq_flip_workspace_bytes(int64_t N, int64_t K);

/* Flip-Refinement of a prepared weight's codes, in place, rows in parallel. Per row, fp64:
 *   e_k = w'_k - dec(code_k) 2^(scale - 127) (exact); g_j = fma chain over k ascending
 *   of H[j][k] e_k from 0; per round, for k ascending, lower then higher neighbour:
 *   delta = (neighbour - value) 2^(scale - 127), dE = (delta delta) H_kk - (2 delta) g_k
 *   (each operation rounded); the first strictly smallest dE < 0 is applied (code
 *   changed, a move to 0 writing +0), then g_j = fma(-delta, H[k][j], g_j); the row stops
 *   when no dE < 0 remains or after max_rounds moves. Bit-identical to that definition.
 *   W_bf16, s      the weight and channel scales macaq_prepare_weight(_hessian) was given
 *   H              device fp64 [K x K], symmetric (as macaq_hessian_full writes it)
 *   w_codes        device [N x K/2], refined in place; w_scales: its scale atoms
 *   moves          device int32 [N]: the number of moves made in each row
 *   workspace      >= macaq_flip_workspace_bytes(N, K), 16-byte aligned
 * K % 32 == 0, K <= 8192, max_rounds >= 0. */
macaq_status macaq_flip_refine(const void* W_bf16, int64_t N, int64_t K, int64_t ldw, const float* s, const double* H,
                               uint8_t* w_codes, const uint8_t* w_scales, int max_rounds, int32_t* moves,
                               void* workspace, size_t ws_bytes, macaq_stream stream);

/* Largest scratch the no-allocation variant below can use: 16 MiB, held in a static
 * device array on every GPU that loads this library, for as long as it stays loaded. */
#define MACAQ_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* macaq_linear_w4a4 for callers that cannot allocate device memory. (The paper has no
 * counterpart: this is a deployment convenience of this library.)
 *
 * Some callers cannot call cudaMalloc or hand the library a workspace: code embedded in
 * a serving runtime or plugin host that owns the whole device memory pool and gives
 * libraries none of it, and latency-critical loops where allocating or freeing would
 * stall the device (cudaFree synchronises it) or could fail under memory pressure in the
 * middle of serving. This entry point takes no workspace: the activation codes, scales
 * and stream-K partial tiles live in one file-scope static device array of
 * MACAQ_NOALLOC_SCRATCH_BYTES. The caller still passes x, the prepared weight and y,
 * with the same meaning, layout and alignment rules as macaq_linear_w4a4 (fused = 0).
 *
 * - Sizes whose workspace (macaq_linear_workspace_bytes(M, N, K, out)) exceeds
 *   MACAQ_NOALLOC_SCRATCH_BYTES are rejected with MACAQ_ERR_WORKSPACE; nothing is
 *   enqueued.
 * - The first call on each device looks up the array's device address (once per device,
 *   with that device current); make that first call before any stream capture.
 * - Every call on a device shares the one array, and the array keeps the last call's
 *   contents. Nothing in it needs to start at zero: every call overwrites what it reads
 *   and tags its stream-K counters with a value unique to the call. Calls whose executions
 *   overlap on the GPU (other streams, or no ordering between them) race on the array
 *   and give undefined results: order them on one stream.
 * - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine. */
macaq_status macaq_linear_w4a4_noalloc(const void* x_bf16, int64_t M, int64_t ldx,
                                       const macaq_weight* w, void* y, int64_t ldy,
                                       macaq_out_dtype out, macaq_stream stream);

/* ------------------------------------------------------------ status ---------- */

/* Every wait inside the GEMM kernel is bounded. A kernel that gives up a wait records
 * a code in a device-side word and returns early (its output is then undefined); so does
 * a kernel launched in a way it is not planned for (a scale-factor offset or a cluster
 * size the plan never gives).
 * This call synchronises the current device, reads the word, clears it, and returns
 * MACAQ_ERR_DEVICE_TIMEOUT if it was set (MACAQ_OK otherwise, MACAQ_ERR_CUDA if the
 * read fails). */
macaq_status macaq_get_device_error(void);

/* Self-test of the bounded device waits (failure detection; the pages have no
 * counterpart). Launches on `stream` a 2-CTA kernel that runs the GEMM kernel's own
 * wait routines against waits that cannot succeed, then synchronises `stream` and
 * copies the outcome into result[0..9] (host memory, caller-owned):
 *   [0] wait on an mbarrier nothing arrives at, limit limit_us: 1 completed, 0 gave up
 *   [1] a second wait in the same CTA, normal 2 s limit: 0 if it left on the CTA's
 *       abort flag
 *   [2] a wait on a barrier the warp completes itself: 1
 *   [3] the CTA's recorded error code (1: producer-wait timeout)
 *   [4] [5] time spent in waits [0] and [1], ns, by the device clock
 *   [6] a group of three warps, one of whose waits (limit limit_us) cannot succeed,
 *       agreeing at its named barrier whether to go on, as the kernel's warp groups
 *       do: 0 (all leave together, none is held at the barrier)
 *   [7] that CTA's recorded error code (5: a warp group's wait timed out)
 *   [8] time spent in the wait that gave up, ns
 *   [9] another member's own wait (on a barrier that completes): 1
 * limit_us must be in [1, 1000000] (else MACAQ_ERR_INVALID_ARG). A kernel that gives
 * up returns normally, so the context stays usable; the device error word read by
 * macaq_get_device_error is not touched. MACAQ_ERR_CUDA if the launch or copy fails. */
macaq_status macaq_selftest_wait_timeout(uint32_t limit_us, int64_t* result, macaq_stream stream);

/* Static, human-readable name of a status code. */
const char* macaq_status_string(macaq_status status);

/* MACAQ_VERSION of the built library. */
int macaq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MACAQ_H */
