/*
 * nvfp4.h — C ABI of libnvfp4.so: NVFP4 scale calibration on B200 (sm_100a).
 *
 * NVFP4 stores a tensor as 4-bit E2M1 codes in blocks of 16 consecutive
 * values of a row, one FP8 E4M3 scale per block and one FP32 scale per
 * tensor.  This library computes, on the GPU:
 *   - the FP32 tensor scale,
 *   - the block-diagonal Gram matrix of calibration activations,
 *   - the per-block FP8 scale by the max, MSE or Local-Hessian rule,
 *   - E2M1 quantisation with packing, dequantisation,
 *   - dynamic (per call) activation fake-quantisation for W4A4.
 *
 * Sources (page title, section):
 *   [BT]  Baseten engineering blog, "What makes high-quality NVFP4":
 *         "Why do we need scales?" (E2M1 value set, FP32 tensor scale),
 *         "Block scaling: one scale per 16 values", "Why blocks?" (worked
 *         example, max / 6), "Calibration" (activation block scales).
 *   [LH]  "4 比特量化到底让模型笨了多少？" (write-up of NVIDIA Model
 *         Optimizer's "Improving NVFP4 Accuracy with Local-Hessian Weight
 *         Scales"): "The NVFP4 structure" (FP8 block scale, max scaling,
 *         MSE over 126 candidates), "A different objective" (E(s) =
 *         ||delta X||^2 = tr(delta X X^T delta^T), 16x16 block-diagonal
 *         approximation, exhaustive candidate search).
 *   [QAD] "為什么NVFP4推理精度會掉以及QAD到底在修什么": 2.1 (round to the
 *         nearest E2M1 value), 2.3 (step = block max / 6), 3.2 (fake-quant
 *         forward: block max / 6, quantise, multiply back), 4.2 (clamp the
 *         scale to the FP8 maximum).
 *
 * Conventions shared by every entry point:
 *   - bf16 tensors are passed as uint16_t bit patterns; every pointer is a
 *     DEVICE pointer owned by the caller unless stated otherwise; nothing is
 *     freed or retained by the library.
 *   - Matrices are row-major.  A weight W is [R, C] (C = input channels);
 *     activations X are [tokens, C].  Blocks are 16 consecutive elements of
 *     a row, so C must be a multiple of 16 (else NVFP4_ERR_SHAPE).
 *   - bf16 and packed-code pointers must be 16-byte aligned, float pointers
 *     4-byte aligned (else NVFP4_ERR_MISALIGNED).  Block-code (uint8) arrays
 *     have no alignment requirement.
 *   - `batch` >= 1 stacks independent tensors (e.g. MoE experts) with a
 *     contiguous batch stride; each has its own FP32 scale s_g[batch].
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work on it and return without synchronising, except the status
 *     and statistics reads (nvfp4_get_device_status, nvfp4_search_evaluations,
 *     nvfp4_search_rescores).  Argument errors are detected on the host
 *     before anything is enqueued; a failed launch returns NVFP4_ERR_CUDA.
 *   - Stream order holds between calls and with the caller's own work: a
 *     call's first kernel starts after everything enqueued before it.  The
 *     later kernels of a call are launched with programmatic stream
 *     serialisation (their launch overlaps the previous kernel's tail; each
 *     waits for it before touching memory).
 *   - A CUDA device must be current; all pointers must belong to it.
 *
 * Block-scale codes are E4M3 (FN variant) bit patterns, 0x00..0x7E.  The
 * effective scale of a block is s_eff = fl32(s_g * e4m3(code)).  E2M1 codes
 * are sign<<3 | k with magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}[k]; element 2j
 * of a row is the low nibble of byte j of its packed row.  Rounding is to
 * nearest, ties to even, decided on the exact quotient |x| / s_eff, and
 * saturates at 6; a negative input that rounds to zero keeps its sign.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nvfp4_status {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,     /* null pointer, negative size, batch or group count < 1 */
    NVFP4_ERR_SHAPE = 2,           /* C not a multiple of 16, or sizes overflow */
    NVFP4_ERR_MISALIGNED = 3,      /* pointer alignment rule above violated */
    NVFP4_ERR_NONFINITE = 4,       /* NaN or Inf met in an input (device-side report) */
    NVFP4_ERR_CUDA = 5,            /* a CUDA runtime call or launch failed */
    NVFP4_ERR_NOT_IMPLEMENTED = 6,
    NVFP4_ERR_TOO_LARGE = 7,       /* request beyond a documented maximum */
    NVFP4_ERR_DEVICE_TIMEOUT = 8,  /* a Gram kernel gave up waiting (one second) for its
                                      own tile copies (device-side report).  H is left
                                      as it was by that call, and by every later Gram
                                      call until nvfp4_get_device_status has read and
                                      cleared this status */
    NVFP4_ERR_NOT_POSITIVE_DEFINITE = 9, /* a dampened Hessian had a non-positive (or
                                           non-finite) Cholesky pivot; the GPTQ output
                                           is not usable (device-side report) */
    NVFP4_ERR_DEVICE_UNDRAINED = 10 /* after such a timeout, copies still in flight did
                                       not land within ten more seconds and the kernel
                                       returned anyway: shared memory of its SM may
                                       still receive them, so results of later kernels
                                       are not trustworthy; end the process (device-side
                                       report, as NVFP4_ERR_DEVICE_TIMEOUT otherwise) */
} nvfp4_status;

/* Human-readable name of a status code (static string, never NULL). */
const char *nvfp4_status_string(nvfp4_status st);

/*
 * FP32 tensor scale per batch element ([BT] "Why do we need scales?": NVFP4
 * has a tensor-level FP32 scale besides the block scales; the formula is
 * this library's reading): s_g[i] = fl32(amax_i / 2688) with amax_i the
 * largest |x| of batch element i and 2688 = 6 * 448, so that the largest
 * E4M3 scale maps the tensor maximum onto E2M1's 6.  amax = 0 gives 1.
 *   x        [batch, n_per_batch] bf16, n_per_batch a multiple of 8.
 *   s_g      [batch] float, written.  If an element is NaN/Inf, its s_g is
 *            set to NaN and the device status becomes NVFP4_ERR_NONFINITE
 *            (see nvfp4_get_device_status).
 */
nvfp4_status nvfp4_global_scale(const uint16_t *x, int64_t batch, int64_t n_per_batch,
                                float *s_g, void *stream);

/*
 * Block-diagonal Gram accumulation over calibration tokens ([LH] "A
 * different objective": H = X X^T restricted to its 16x16 diagonal blocks):
 *   H[j] += sum_t x[t, 16j:16j+16]^T x[t, 16j:16j+16],  j = 0..C/16-1.
 *   x   [n_tok, C] bf16 (n_tok >= 0; 0 is a no-op).
 *   H   [C/16, 16, 16] float, read and written (accumulated in place, so a
 *       calibration set can be streamed in chunks).
 * Products of bf16 values are exact in fp32 and accumulate in fp32 on the
 * tensor cores; partial sums over token ranges are combined in a fixed
 * order, so the result is bitwise reproducible for a given shape.  Uses a
 * stream-ordered scratch buffer from a library-owned memory pool.
 */
nvfp4_status nvfp4_hessian_accumulate(const uint16_t *x, int64_t n_tok, int64_t C, float *H,
                                      void *stream);

/*
 * The same accumulation as nvfp4_hessian_accumulate, for callers that may not
 * allocate device memory: applications that give all of HBM to their own
 * allocator or work under a fixed memory budget, and loops that cannot take an
 * allocation's latency or implicit synchronisation.  The pages have no
 * counterpart to this call; it is a property of this library only.
 * Partial sums go to one 16 MiB device array inside the library (held by each
 * device that loads it until exit) instead of the memory pool, so nothing is
 * allocated.  C must not exceed 262,144 (else NVFP4_ERR_TOO_LARGE, nothing
 * launched).  All calls on a device share that array: calls that overlap on
 * the GPU race and must be serialised by the caller.  The first call on a
 * device looks up the array's address with that device current; make it
 * before any stream capture.  Results agree with nvfp4_hessian_accumulate up
 * to fp32 summation order.
 */
nvfp4_status nvfp4_hessian_accumulate_noalloc(const uint16_t *x, int64_t n_tok, int64_t C,
                                              float *H, void *stream);

/*
 * Grouped form for experts: tokens are sorted by group; group g owns rows
 * offsets[g] .. offsets[g+1]-1 of x and accumulates into H[g].
 *   x         [n_tok_total, C] bf16
 *   offsets   DEVICE int64 [G+1], non-decreasing, offsets[0] = 0,
 *             offsets[G] = n_tok_total (the host passes n_tok_total so that no
 *             device value has to be read back).  Offsets outside
 *             [0, n_tok_total] are clamped on the device.
 *   H         [G, C/16, 16, 16] float, accumulated.
 * n_tok_total above 2^30 returns NVFP4_ERR_TOO_LARGE (tile row coordinates
 * of the tile copies are 32-bit; split such a set into calls).
 */
nvfp4_status nvfp4_hessian_accumulate_grouped(const uint16_t *x, const int64_t *offsets,
                                              int64_t G, int64_t n_tok_total, int64_t C,
                                              float *H, void *stream);

/*
 * Max rule ([QAD] 2.3 and 4.2, [BT] "Why blocks?", [LH] "The NVFP4
 * structure"): code = E4M3 round-to-nearest-even, saturating at 448, of the
 * exact quotient amax_b / (6 * s_g); an all-zero block gets code 0.
 *   w            [batch, R, C] bf16
 *   s_g          DEVICE [batch] float, positive and finite
 *   scale_codes  [batch, R, C/16] uint8, written
 */
nvfp4_status nvfp4_scale_search_max(const uint16_t *w, int64_t batch, int64_t R, int64_t C,
                                    const float *s_g, uint8_t *scale_codes, void *stream);

/*
 * Four Over Six ([LH] "The NVFP4 structure": the rule picks one of two
 * candidate scales per block).  The two are not named on the pages; the
 * reading: the max-rule code (block amax onto E2M1's 6) and the code of
 * amax_b / (4 * s_g) (block amax onto 4), both rounded as the max rule
 * rounds; the one with the smaller block MSE sum_i (w_i - v(q_i) s_eff)^2
 * wins, the smaller code on a tie; an all-zero block gets code 0.  The
 * choice is the one the two objectives give when evaluated in fp64 with the
 * definition's operations in its order: an fp32 screen decides only when
 * they differ by more than its error bound (2^-16 relative plus 2^-130),
 * otherwise that fp64 comparison decides.  Arguments as
 * nvfp4_scale_search_max.
 */
nvfp4_status nvfp4_scale_search_four_over_six(const uint16_t *w, int64_t batch, int64_t R,
                                              int64_t C, const float *s_g, uint8_t *scale_codes,
                                              void *stream);

/*
 * MSE rule ([LH] "The NVFP4 structure"): for every block, the code in
 * 1..126 minimising sum_i (w_i - v(q_i) s_eff)^2, q_i the E2M1 code of w_i at
 * s_eff; the smallest code wins a tie.  Candidates are screened in fp32 and
 * near-ties (best two within 2^-12 relative plus 2^-130, in the screen's
 * units) are re-scored in fp64.  Range:
 * the screen works on each row scaled by a power of two, so tiny and huge
 * weights alike stay in fp32's normal range; the codes follow the
 * definition for every tensor scale s_g; outside [2^-100, 2^100) (tensor
 * maxima below about 2^-88.6 or above 2^111.4) every block is re-scored in
 * fp64 over all 126 candidates, which is exact but slower.
 *   best_obj     optional [batch, R, C/16] float, the winning objective
 *                (0 or inf where it leaves fp32's range).
 */
nvfp4_status nvfp4_scale_search_mse(const uint16_t *w, int64_t batch, int64_t R, int64_t C,
                                    const float *s_g, uint8_t *scale_codes, float *best_obj,
                                    void *stream);

/*
 * Local-Hessian rule ([LH] "A different objective"): for every block b of
 * every row, the code in 1..126 minimising E = delta H_b delta^T, with
 * delta_i = w_i - v(q_i) s_eff and H_b the 16x16 Gram block of the block's
 * columns (shared by all rows); the smallest code wins a tie.  H_b is
 * factored once per column block (fp64 Cholesky, semidefinite pivots
 * dropped) and candidates are screened in fp32 as ||L^T delta||^2 with the
 * 16x16 product on the tensor cores; every block whose best two the
 * screen's error bound cannot separate -- 2^-12 relative plus an absolute
 * term that grows with ||L^T w|| (the f16 split of L and the MMA's fp32
 * accumulation, assumed to err by at most 2^-18 of the sum of its addends'
 * magnitudes; see nvfp4_self_test_mma) and with any dropped pivot -- is
 * re-scored in fp64 from H, so the codes are the definition's.
 * Range as nvfp4_scale_search_mse; the tensor-core screen holds each row in
 * f16 at its own power-of-two scale, so a row keeps full precision whatever
 * the other rows of its 16-row tile hold.
 *   H            [batch, C/16, 16, 16] float (e.g. from
 *                nvfp4_hessian_accumulate), symmetric positive semidefinite
 *   best_obj     optional [batch, R, C/16] float, the winning objective.
 */
nvfp4_status nvfp4_scale_search_local_hessian(const uint16_t *w, int64_t batch, int64_t R,
                                              int64_t C, const float *s_g, const float *H,
                                              uint8_t *scale_codes, float *best_obj,
                                              void *stream);

/*
 * E2M1 quantisation and packing given block codes ([BT] "Why do we need
 * scales?", "Block scaling"; [QAD] 2.1).  Two codes per byte, element 2j in
 * the low nibble.  A block with code 0 has s_eff = 0 and encodes as
 * (signed) zeros.
 *   packed  [batch, R, C/2] uint8, written (16-byte aligned)
 */
nvfp4_status nvfp4_quantize_pack(const uint16_t *w, int64_t batch, int64_t R, int64_t C,
                                 const float *s_g, const uint8_t *scale_codes, uint8_t *packed,
                                 void *stream);

/*
 * Dequantisation ([QAD] 3.2: the quantised value times its scale):
 * out = bf16_rn(fl32(v(q) * s_eff)).
 *   out   [batch, R, C] bf16, written
 */
nvfp4_status nvfp4_dequantize(const uint8_t *packed, const uint8_t *scale_codes,
                              const float *s_g, int64_t batch, int64_t R, int64_t C,
                              uint16_t *out, void *stream);

/*
 * Dynamic W4A4 activation fake-quant ([BT] "Calibration"; [QAD] 3.2):
 * s_g from the whole x (as nvfp4_global_scale), then per block the max rule,
 * E2M1 encode and dequantise, fused in one pass over x.
 *   x       [rows, C] bf16
 *   out     [rows, C] bf16, written (may not alias x)
 *   packed  optional [rows, C/2] uint8 (NULL to skip)
 *   scale_codes optional [rows, C/16] uint8 (NULL to skip)
 *   s_g     DEVICE float [1], written
 */
nvfp4_status nvfp4_fake_quant(const uint16_t *x, int64_t rows, int64_t C, uint16_t *out,
                              uint8_t *packed, uint8_t *scale_codes, float *s_g, void *stream);

/*
 * Activation-range calibration ([BT] "Calibration": the clipping range of an
 * activation tensor comes from calibration data; the maximum avoids
 * clipping, percentile-, histogram- and error-based ranges clip a few
 * outliers so that typical values are represented more finely).  The range
 * sets a static tensor scale s_g = fl32(clip / 2688) (1 for clip 0) used by
 * nvfp4_fake_quant_static; block scales still follow each block's maximum,
 * so values beyond 6 * 448 * s_g saturate.
 *
 * nvfp4_abs_histogram: hist[|x| bf16 magnitude pattern] += count, exact, over
 * the 32768 patterns; call once per calibration chunk.
 *   x     [n] bf16 (16-byte aligned);  hist  DEVICE uint64 [32768], accumulated
 */
nvfp4_status nvfp4_abs_histogram(const uint16_t *x, int64_t n, uint64_t *hist, void *stream);

/*
 * The p-quantile (0 < p <= 1) of the counted magnitudes -- the smallest
 * bf16 magnitude m with at least ceil(p * N) of the N values at or below it
 * (p = 1: the maximum) -- as the static tensor scale s_g = fl32(m / 2688).
 * An empty histogram gives s_g = 1; a quantile on a non-finite pattern sets
 * s_g to NaN and the device status to NVFP4_ERR_NONFINITE.
 *   hist  DEVICE uint64 [32768];  s_g  DEVICE float [1], written
 */
nvfp4_status nvfp4_static_scale_from_histogram(const uint64_t *hist, double p, float *s_g,
                                               void *stream);

/*
 * nvfp4_fake_quant with a given (static, calibrated) tensor scale instead of
 * the tensor's own maximum.  Arguments as nvfp4_fake_quant; s_g is read.
 */
nvfp4_status nvfp4_fake_quant_static(const uint16_t *x, int64_t rows, int64_t C, const float *s_g,
                                     uint16_t *out, uint8_t *packed, uint8_t *scale_codes,
                                     void *stream);

/*
 * Quantisation error of nvfp4_fake_quant_static at s_g: sum over x of
 * (x - y)^2, y the bf16 fake-quant output, in fp64 (per-CTA partials added
 * in a fixed order: reproducible for a shape) -- the measure an error-based
 * range minimises over candidate clips.
 *   err  DEVICE double [1], written
 */
nvfp4_status nvfp4_quant_error(const uint16_t *x, int64_t rows, int64_t C, const float *s_g,
                               double *err, void *stream);

/*
 * Reads and clears the device-side status of the current device after
 * synchronising `stream`.  *out is NVFP4_OK, NVFP4_ERR_NONFINITE,
 * NVFP4_ERR_DEVICE_TIMEOUT, NVFP4_ERR_DEVICE_UNDRAINED or
 * NVFP4_ERR_NOT_POSITIVE_DEFINITE.
 */
nvfp4_status nvfp4_get_device_status(void *stream, nvfp4_status *out);

/*
 * NVFP4 x NVFP4 matrix product on the tensor cores (W4A4: weights and
 * activations both NVFP4 -- the consumer of nvfp4_quantize_pack /
 * nvfp4_fake_quant outputs):
 *   out[m][n] = bf16_rn(s_ga s_gb sum_k (v(a_mk) e4m3(ca_m,k/16))
 *                                      (v(b_nk) e4m3(cb_n,k/16)))
 * accumulated in fp32 (the tensor cores' block-scaled E2M1 MMA; the
 * products are exact, the sum is fp32), s_ga s_gb rounded to fp32.
 *   a_packed [M, K/2] uint8 and a_codes [M, K/16] uint8 (A row-major, K
 *            contiguous: e.g. activations), a_sg DEVICE float [1]
 *   b_packed [N, K/2], b_codes [N, K/16] (B row-major: e.g. weights
 *            [out, in], so out = A B^T), b_sg DEVICE float [1]
 *   out      [M, N] bf16, written (16-byte aligned)
 * K must be a multiple of 32 and N of 8 (NVFP4_ERR_SHAPE); packed operands
 * and out 16-byte aligned.  The block codes are copied into the scale layout
 * the MMA reads (stream-ordered scratch from the library pool).  Returns
 * NVFP4_ERR_NOT_IMPLEMENTED if the kernel cannot take the shape.
 */
nvfp4_status nvfp4_gemm(const uint8_t *a_packed, const uint8_t *a_codes, const float *a_sg,
                        const uint8_t *b_packed, const uint8_t *b_codes, const float *b_sg,
                        int64_t M, int64_t N, int64_t K, uint16_t *out, void *stream);

/*
 * Full Gram accumulation ([LH] "A different objective": the output-error
 * Hessian is X X^T; "Trying it": GPTQ, combined there with Local-Hessian
 * scales, needs all of it):
 *   H[a][b] += sum_t x[t][a] x[t][b]   for all a, b < C
 * on the tensor cores (bf16 products, fp32 accumulation and sum into H).
 *   x  [n_tok, C] bf16 (tokens by channels), 16-byte aligned
 *   H  [C, C] float, row-major, accumulated in place (16-byte aligned)
 * C must be a multiple of 16 (NVFP4_ERR_SHAPE).  Workspace, if the kernel
 * needs any, is stream-ordered scratch from the library pool.  Returns
 * NVFP4_ERR_NOT_IMPLEMENTED if the kernel cannot take the shape.
 */
nvfp4_status nvfp4_hessian_full_accumulate(const uint16_t *x, int64_t n_tok, int64_t C, float *H,
                                           void *stream);

/*
 * GPTQ rounding at given block scales (GPTQ: Frantar et al., "GPTQ: Accurate
 * Post-Training Quantization for Generative Pre-trained Transformers";
 * [LH] "Trying it": Local-Hessian chooses the scales, GPTQ the rounding).
 * The columns of each row are rounded in order (E2M1 nearest-even at the
 * block's s_eff, exact), and every column not yet rounded first moves by
 * the rounding errors of the earlier ones so that ||(W - Q) X||^2 stays
 * least, through the dampened Hessian H + lambda I, lambda = damp *
 * mean(diag H).  All of it in fp64.
 *   w            [batch, R, C] bf16 (16-byte aligned)
 *   s_g          DEVICE [batch] float
 *   scale_codes  [batch, R, C/16] uint8, E4M3 codes 0..126 (any scale rule)
 *   H            [batch, C, C] float (e.g. from nvfp4_hessian_full_accumulate);
 *                only its lower triangle is read
 *   damp         >= 0 (the GPTQ paper uses 0.01)
 *   packed       [batch, R, C/2] uint8, written (nibble order of
 *                nvfp4_quantize_pack)
 * Scratch (stream-ordered, library pool): batch (C^2 + R C + 128^2) doubles.  A
 * Hessian that is not positive definite after dampening sets the device
 * status NVFP4_ERR_NOT_POSITIVE_DEFINITE (see nvfp4_get_device_status).
 */
nvfp4_status nvfp4_gptq(const uint16_t *w, int64_t batch, int64_t R, int64_t C, const float *s_g,
                        const uint8_t *scale_codes, const float *H, double damp,
                        uint8_t *packed, void *stream);

/*
 * Work statistic of the scale searches (the pages have no counterpart; it
 * measures how much of the 126-candidate search the exact pruning leaves):
 * out[0] and out[1] receive the number of (block, candidate) objective
 * evaluations of the fp32 screen made by nvfp4_scale_search_mse and by
 * nvfp4_scale_search_local_hessian on the current device since the last
 * reset (the fp64 re-scores of near ties are not counted); between 1 and 126
 * per block searched.  Synchronises `stream` first, so calls queued on it
 * are included; calls still running on other streams may be partly
 * included.  `reset` != 0 zeroes every search statistic afterwards (these
 * counters and those of nvfp4_search_rescores).
 *   out   [2] uint64, HOST, written
 */
nvfp4_status nvfp4_search_evaluations(void *stream, int reset, uint64_t *out);

/*
 * Second statistic of the scale searches (no counterpart on the pages): how
 * many rows the fp32 screen could not decide and sent to the fp64 re-score,
 * since the last reset, on the current device: out[0] MSE rows re-scored over
 * their best two candidates, out[1] MSE rows re-scored over all 126, out[2]
 * and out[3] the same for nvfp4_scale_search_local_hessian.  Synchronises
 * `stream` first; `reset` != 0 zeroes every search statistic afterwards.
 *   out   [4] uint64, HOST, written
 */
nvfp4_status nvfp4_search_rescores(void *stream, int reset, uint64_t *out);

/*
 * Diagnostic of the failure path of the kernels that wait on their own tile
 * copies (the pages have no counterpart): enqueues one warp that waits on an
 * mbarrier nothing arrives on.  Its wait gives up after about one second and
 * sets the device status to NVFP4_ERR_DEVICE_TIMEOUT, which the next
 * nvfp4_get_device_status reports; the context stays usable.  No data is
 * touched, but until that status is read, Gram calls leave H unchanged (as
 * after a real timeout).
 */
nvfp4_status nvfp4_self_test_device_timeout(void *stream);

/*
 * Diagnostic of the scale search's error bound (the pages have no
 * counterpart): runs each tile through the same tensor-core instruction the
 * Local-Hessian screen uses, a 16x8x16 MMA of f16 operands with fp32
 * accumulation, so that a test can check on the device the accumulation
 * error the screen's bound assumes (at most 2^-18 of the sum of the
 * magnitudes of the products and of c).
 *   a  [n_tiles, 16, 16] f16 bit patterns (rows m, columns k), 2-byte aligned
 *   b  [n_tiles, 16, 8] f16 (rows k, columns n), 2-byte aligned
 *   c  [n_tiles, 16, 8] float, read;  d  [n_tiles, 16, 8] float, written:
 *      d = a b + c per tile
 */
nvfp4_status nvfp4_self_test_mma(const uint16_t *a, const uint16_t *b, const float *c, float *d,
                                 int64_t n_tiles, void *stream);

/* Releases the library's memory pool on every device it touched.  No call
 * may be in flight. */
void nvfp4_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
