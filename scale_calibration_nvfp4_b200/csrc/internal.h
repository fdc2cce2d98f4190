// Launchers behind the C ABI (arguments already validated by api.cu).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

int sm_count();

cudaError_t launch_global_scale(const uint16_t *x, int64_t batch, int64_t n_per_batch,
                                float *s_g, cudaStream_t st);
cudaError_t launch_scale_max(const uint16_t *w, int64_t batch, int64_t nblk, const float *s_g,
                             uint8_t *codes, cudaStream_t st);
cudaError_t launch_four_over_six(const uint16_t *w, int64_t batch, int64_t nblk,
                                 const float *s_g, uint8_t *codes, cudaStream_t st);
cudaError_t launch_pack(const uint16_t *w, int64_t batch, int64_t nblk, const float *s_g,
                        const uint8_t *codes, uint8_t *packed, cudaStream_t st);
cudaError_t launch_dequant(const uint8_t *packed, const uint8_t *codes, const float *s_g,
                           int64_t batch, int64_t nblk, uint16_t *out, cudaStream_t st);
cudaError_t launch_fake_quant(const uint16_t *x, int64_t rows, int64_t C, uint16_t *out,
                              uint8_t *packed, uint8_t *codes, float *s_g, cudaStream_t st);
cudaError_t read_and_clear_device_status(cudaStream_t st, int *out);

// Scale search: objective 0 = MSE, 1 = Local-Hessian (H required).
cudaError_t launch_scale_search(const uint16_t *w, int64_t batch, int64_t R, int64_t C,
                                const float *s_g, const float *H, uint8_t *codes,
                                float *best_obj, int local_hessian, cudaStream_t st);

// Copies the search's evaluation counters ([0] MSE, [1] Local-Hessian) to
// the host after the work queued on `st`, optionally zeroing them.
// all six search statistics (see g_search_evals in search.cu)
cudaError_t read_search_evaluations(cudaStream_t st, unsigned long long out[6], bool reset);
cudaError_t launch_mma_probe(const uint16_t *a, const uint16_t *b, const float *c, float *d,
                             int64_t n, cudaStream_t st);

// Gram accumulation.  `offsets` == nullptr: one group of n_tok tokens.
cudaError_t launch_gram(const uint16_t *x, const int64_t *offsets, int64_t G, int64_t n_tok,
                        int64_t C, float *H, cudaStream_t st);

// Gram accumulation with its partial sums in a fixed device array (no
// allocation); C up to gram_noalloc_max_channels().
cudaError_t launch_gram_noalloc(const uint16_t *x, int64_t n_tok, int64_t C, float *H,
                                cudaStream_t st);
int64_t gram_noalloc_max_channels();

// Copies the Gram kernels' device status to *out after the work queued on
// `st`, and clears it.
cudaError_t read_and_clear_gram_status(cudaStream_t st, int *out);

// One warp whose bounded mbarrier wait runs out (about one second), setting
// the device timeout status.
cudaError_t launch_wait_timeout_probe(cudaStream_t st);

// NVFP4 x NVFP4 product Y[M, N] (bf16) of A [M, K] and B [N, K] given as
// packed codes, row-major block codes and device tensor scales.
cudaError_t launch_gemm_fp4(const uint8_t *a_packed, const uint8_t *a_codes, const float *a_sg,
                            const uint8_t *b_packed, const uint8_t *b_codes, const float *b_sg,
                            int64_t M, int64_t N, int64_t K, uint16_t *out, cudaStream_t st);

// Activation-range calibration: exact |x| histogram (uint64 [32768],
// accumulated), its p-quantile as a static tensor scale, fake-quant at a
// given tensor scale, and the quantisation error at a given tensor scale.
cudaError_t launch_abs_histogram(const uint16_t *x, int64_t n, uint64_t *hist, cudaStream_t st);
cudaError_t launch_quantile_scale(const uint64_t *hist, double p, float *s_g, cudaStream_t st);
cudaError_t launch_fake_quant_static(const uint16_t *x, int64_t rows, int64_t C, const float *s_g,
                                     uint16_t *out, uint8_t *packed, uint8_t *codes,
                                     cudaStream_t st);
cudaError_t launch_quant_error(const uint16_t *x, int64_t rows, int64_t C, const float *s_g,
                               double *err, cudaStream_t st);
cudaError_t read_and_clear_calib_status(cudaStream_t st, int *out);

// Full Gram H [C, C] += X^T X on the tensor cores.
cudaError_t launch_gram_full(const uint16_t *x, int64_t n_tok, int64_t C, float *H,
                             cudaStream_t st);

// GPTQ rounding of W [batch, R, C] at the given block codes with the
// Hessians H [batch, C, C]; packed [batch, R, C/2].
cudaError_t launch_gptq(const uint16_t *w, int64_t batch, int64_t R, int64_t C, const float *s_g,
                        const uint8_t *codes, const float *H, double damp, uint8_t *packed,
                        cudaStream_t st);
cudaError_t read_and_clear_gptq_status(cudaStream_t st, int *out);

// Stream-ordered scratch from the library's pool on the current device.
cudaError_t scratch_alloc(void **p, size_t bytes, cudaStream_t st);
cudaError_t scratch_free(void *p, cudaStream_t st);
void scratch_release_all();

}  // namespace nvfp4
