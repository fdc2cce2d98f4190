// C ABI of libnvfp4.so (declared in include/nvfp4.h): argument validation on
// the host, then launches on the caller's stream.  Nothing here computes on
// the data.
#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/nvfp4.h"
#include "internal.h"

namespace nvfp4 {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_pool_mu;
cudaMemPool_t g_pools[kMaxDevices] = {};

cudaError_t pool_for_current(cudaMemPool_t *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_pool_mu);
  if (!g_pools[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    e = cudaMemPoolCreate(&g_pools[dev], &props);
    if (e != cudaSuccess) {
      g_pools[dev] = nullptr;
      return e;
    }
    // keep freed scratch cached in the pool between calls
    uint64_t keep = UINT64_MAX;
    cudaMemPoolSetAttribute(g_pools[dev], cudaMemPoolAttrReleaseThreshold, &keep);
  }
  *out = g_pools[dev];
  return cudaSuccess;
}

}  // namespace

cudaError_t scratch_alloc(void **p, size_t bytes, cudaStream_t st) {
  cudaMemPool_t pool;
  cudaError_t e = pool_for_current(&pool);
  if (e != cudaSuccess) return e;
  return cudaMallocFromPoolAsync(p, bytes < 256 ? 256 : bytes, pool, st);
}

cudaError_t scratch_free(void *p, cudaStream_t st) { return p ? cudaFreeAsync(p, st) : cudaSuccess; }

void scratch_release_all() {
  std::lock_guard<std::mutex> lk(g_pool_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (int d = 0; d < kMaxDevices; ++d) {
    if (!g_pools[d]) continue;
    cudaSetDevice(d);
    cudaDeviceSynchronize();
    cudaMemPoolDestroy(g_pools[d]);
    g_pools[d] = nullptr;
  }
  cudaSetDevice(cur);
}

}  // namespace nvfp4

namespace {

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// a * b * c without overflow past INT64_MAX / 8 (room for byte offsets)
inline bool fits(int64_t a, int64_t b, int64_t c = 1) {
  const int64_t lim = INT64_MAX / 8;
  if (a < 0 || b < 0 || c < 0) return false;
  if (a && b > lim / a) return false;
  const int64_t ab = a * b;
  if (ab && c > lim / ab) return false;
  return true;
}

inline nvfp4_status map_cuda(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

nvfp4_status check_weight_args(const uint16_t *w, int64_t batch, int64_t R, int64_t C,
                               const float *s_g, const void *codes) {
  if (batch < 1 || R < 0 || C < 0) return NVFP4_ERR_INVALID_ARG;
  if (!w || !s_g || !codes) return NVFP4_ERR_INVALID_ARG;
  if (C % 16) return NVFP4_ERR_SHAPE;
  if (!fits(batch, R, C)) return NVFP4_ERR_SHAPE;
  if (batch > 65535 || C / 16 > 65535) return NVFP4_ERR_TOO_LARGE;
  if (!aligned(w, 16) || !aligned(s_g, 4)) return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

}  // namespace

extern "C" {

const char *nvfp4_status_string(nvfp4_status st) {
  switch (st) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
    case NVFP4_ERR_SHAPE: return "NVFP4_ERR_SHAPE";
    case NVFP4_ERR_MISALIGNED: return "NVFP4_ERR_MISALIGNED";
    case NVFP4_ERR_NONFINITE: return "NVFP4_ERR_NONFINITE";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
    case NVFP4_ERR_NOT_IMPLEMENTED: return "NVFP4_ERR_NOT_IMPLEMENTED";
    case NVFP4_ERR_TOO_LARGE: return "NVFP4_ERR_TOO_LARGE";
    case NVFP4_ERR_DEVICE_TIMEOUT: return "NVFP4_ERR_DEVICE_TIMEOUT";
    case NVFP4_ERR_NOT_POSITIVE_DEFINITE: return "NVFP4_ERR_NOT_POSITIVE_DEFINITE";
    case NVFP4_ERR_DEVICE_UNDRAINED: return "NVFP4_ERR_DEVICE_UNDRAINED";
  }
  return "NVFP4_ERR_UNKNOWN";
}

nvfp4_status nvfp4_global_scale(const uint16_t *x, int64_t batch, int64_t n_per_batch,
                                float *s_g, void *stream) {
  if (batch < 1 || n_per_batch < 0 || !s_g || (n_per_batch > 0 && !x))
    return NVFP4_ERR_INVALID_ARG;
  if (n_per_batch % 8 || !fits(batch, n_per_batch)) return NVFP4_ERR_SHAPE;
  if (batch > 65535) return NVFP4_ERR_TOO_LARGE;
  if ((x && !aligned(x, 16)) || !aligned(s_g, 4)) return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_global_scale(x, batch, n_per_batch, s_g, as_stream(stream)));
}

nvfp4_status nvfp4_hessian_accumulate(const uint16_t *x, int64_t n_tok, int64_t C, float *H,
                                      void *stream) {
  if (n_tok < 0 || C < 0 || !H || (n_tok > 0 && !x)) return NVFP4_ERR_INVALID_ARG;
  if (C % 16 || !fits(n_tok, C)) return NVFP4_ERR_SHAPE;
  if (C / 16 > 8 * 65535) return NVFP4_ERR_TOO_LARGE;
  if ((x && !aligned(x, 16)) || !aligned(H, 4)) return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_gram(x, nullptr, 1, n_tok, C, H, as_stream(stream)));
}

nvfp4_status nvfp4_hessian_full_accumulate(const uint16_t *x, int64_t n_tok, int64_t C,
                                           float *H, void *stream) {
  if (n_tok < 0 || C < 0 || !H || (n_tok > 0 && !x)) return NVFP4_ERR_INVALID_ARG;
  if (C % 16 || !fits(n_tok, C) || !fits(C, C)) return NVFP4_ERR_SHAPE;
  if (C > INT32_MAX || n_tok > INT32_MAX) return NVFP4_ERR_TOO_LARGE;
  if ((x && !aligned(x, 16)) || !aligned(H, 16)) return NVFP4_ERR_MISALIGNED;
  const cudaError_t e = nvfp4::launch_gram_full(x, n_tok, C, H, as_stream(stream));
  if (e == cudaErrorNotSupported) return NVFP4_ERR_NOT_IMPLEMENTED;
  return map_cuda(e);
}

nvfp4_status nvfp4_hessian_accumulate_noalloc(const uint16_t *x, int64_t n_tok, int64_t C,
                                              float *H, void *stream) {
  if (n_tok < 0 || C < 0 || !H || (n_tok > 0 && !x)) return NVFP4_ERR_INVALID_ARG;
  if (C % 16 || !fits(n_tok, C)) return NVFP4_ERR_SHAPE;
  if (C > nvfp4::gram_noalloc_max_channels()) return NVFP4_ERR_TOO_LARGE;
  if ((x && !aligned(x, 16)) || !aligned(H, 4)) return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_gram_noalloc(x, n_tok, C, H, as_stream(stream)));
}

nvfp4_status nvfp4_hessian_accumulate_grouped(const uint16_t *x, const int64_t *offsets,
                                              int64_t G, int64_t n_tok_total, int64_t C,
                                              float *H, void *stream) {
  if (G < 1 || n_tok_total < 0 || C < 0 || !H || !offsets || (n_tok_total > 0 && !x))
    return NVFP4_ERR_INVALID_ARG;
  if (C % 16 || !fits(n_tok_total, C) || !fits(G, C, 16)) return NVFP4_ERR_SHAPE;
  if (C / 16 > 8 * 65535 || n_tok_total > ((int64_t)1 << 30) || n_tok_total / 2048 + G > INT32_MAX)
    return NVFP4_ERR_TOO_LARGE;
  if ((x && !aligned(x, 16)) || !aligned(H, 4) || !aligned(offsets, 8))
    return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_gram(x, offsets, G, n_tok_total, C, H, as_stream(stream)));
}

nvfp4_status nvfp4_scale_search_max(const uint16_t *w, int64_t batch, int64_t R, int64_t C,
                                    const float *s_g, uint8_t *scale_codes, void *stream) {
  nvfp4_status st = check_weight_args(w, batch, R, C, s_g, scale_codes);
  if (st != NVFP4_OK) return st;
  return map_cuda(nvfp4::launch_scale_max(w, batch, R * C / 16, s_g, scale_codes,
                                          as_stream(stream)));
}

nvfp4_status nvfp4_scale_search_four_over_six(const uint16_t *w, int64_t batch, int64_t R,
                                              int64_t C, const float *s_g, uint8_t *scale_codes,
                                              void *stream) {
  nvfp4_status st = check_weight_args(w, batch, R, C, s_g, scale_codes);
  if (st != NVFP4_OK) return st;
  return map_cuda(nvfp4::launch_four_over_six(w, batch, R * C / 16, s_g, scale_codes,
                                              as_stream(stream)));
}

nvfp4_status nvfp4_scale_search_mse(const uint16_t *w, int64_t batch, int64_t R, int64_t C,
                                    const float *s_g, uint8_t *scale_codes, float *best_obj,
                                    void *stream) {
  nvfp4_status st = check_weight_args(w, batch, R, C, s_g, scale_codes);
  if (st != NVFP4_OK) return st;
  if (best_obj && !aligned(best_obj, 4)) return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_scale_search(w, batch, R, C, s_g, nullptr, scale_codes, best_obj,
                                             0, as_stream(stream)));
}

nvfp4_status nvfp4_scale_search_local_hessian(const uint16_t *w, int64_t batch, int64_t R,
                                              int64_t C, const float *s_g, const float *H,
                                              uint8_t *scale_codes, float *best_obj,
                                              void *stream) {
  nvfp4_status st = check_weight_args(w, batch, R, C, s_g, scale_codes);
  if (st != NVFP4_OK) return st;
  if (!H) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(H, 4) || (best_obj && !aligned(best_obj, 4))) return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_scale_search(w, batch, R, C, s_g, H, scale_codes, best_obj, 1,
                                             as_stream(stream)));
}

nvfp4_status nvfp4_quantize_pack(const uint16_t *w, int64_t batch, int64_t R, int64_t C,
                                 const float *s_g, const uint8_t *scale_codes, uint8_t *packed,
                                 void *stream) {
  nvfp4_status st = check_weight_args(w, batch, R, C, s_g, scale_codes);
  if (st != NVFP4_OK) return st;
  if (!packed) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(packed, 16)) return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_pack(w, batch, R * C / 16, s_g, scale_codes, packed,
                                     as_stream(stream)));
}

nvfp4_status nvfp4_dequantize(const uint8_t *packed, const uint8_t *scale_codes,
                              const float *s_g, int64_t batch, int64_t R, int64_t C,
                              uint16_t *out, void *stream) {
  if (!packed || !scale_codes || !s_g || !out || batch < 1 || R < 0 || C < 0)
    return NVFP4_ERR_INVALID_ARG;
  if (C % 16 || !fits(batch, R, C)) return NVFP4_ERR_SHAPE;
  if (batch > 65535) return NVFP4_ERR_TOO_LARGE;
  if (!aligned(packed, 16) || !aligned(out, 16) || !aligned(s_g, 4)) return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_dequant(packed, scale_codes, s_g, batch, R * C / 16, out,
                                        as_stream(stream)));
}

nvfp4_status nvfp4_fake_quant(const uint16_t *x, int64_t rows, int64_t C, uint16_t *out,
                              uint8_t *packed, uint8_t *scale_codes, float *s_g, void *stream) {
  if (!x || !out || !s_g || rows < 0 || C < 0) return NVFP4_ERR_INVALID_ARG;
  if (C % 16 || !fits(rows, C)) return NVFP4_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(out, 16) || !aligned(s_g, 4) ||
      (packed && !aligned(packed, 16)))
    return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_fake_quant(x, rows, C, out, packed, scale_codes, s_g,
                                           as_stream(stream)));
}

nvfp4_status nvfp4_abs_histogram(const uint16_t *x, int64_t n, uint64_t *hist, void *stream) {
  if (!hist || n < 0 || (n > 0 && !x)) return NVFP4_ERR_INVALID_ARG;
  if (!fits(n, 1)) return NVFP4_ERR_SHAPE;
  if ((x && !aligned(x, 16)) || !aligned(hist, 8)) return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_abs_histogram(x, n, hist, as_stream(stream)));
}

nvfp4_status nvfp4_static_scale_from_histogram(const uint64_t *hist, double p, float *s_g,
                                               void *stream) {
  if (!hist || !s_g || !(p > 0.0) || !(p <= 1.0)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(hist, 8) || !aligned(s_g, 4)) return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_quantile_scale(hist, p, s_g, as_stream(stream)));
}

nvfp4_status nvfp4_fake_quant_static(const uint16_t *x, int64_t rows, int64_t C, const float *s_g,
                                     uint16_t *out, uint8_t *packed, uint8_t *scale_codes,
                                     void *stream) {
  if (!x || !out || !s_g || rows < 0 || C < 0) return NVFP4_ERR_INVALID_ARG;
  if (C % 16 || !fits(rows, C)) return NVFP4_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(out, 16) || !aligned(s_g, 4) ||
      (packed && !aligned(packed, 16)))
    return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_fake_quant_static(x, rows, C, s_g, out, packed, scale_codes,
                                                  as_stream(stream)));
}

nvfp4_status nvfp4_quant_error(const uint16_t *x, int64_t rows, int64_t C, const float *s_g,
                               double *err, void *stream) {
  if (!x || !s_g || !err || rows < 0 || C < 0) return NVFP4_ERR_INVALID_ARG;
  if (C % 16 || !fits(rows, C)) return NVFP4_ERR_SHAPE;
  if (!aligned(x, 16) || !aligned(s_g, 4) || !aligned(err, 8)) return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_quant_error(x, rows, C, s_g, err, as_stream(stream)));
}

nvfp4_status nvfp4_get_device_status(void *stream, nvfp4_status *out) {
  if (!out) return NVFP4_ERR_INVALID_ARG;
  int v = 0;
  cudaError_t e = nvfp4::read_and_clear_device_status(as_stream(stream), &v);
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  *out = (nvfp4_status)v;
  return NVFP4_OK;
}

nvfp4_status nvfp4_gptq(const uint16_t *w, int64_t batch, int64_t R, int64_t C, const float *s_g,
                        const uint8_t *scale_codes, const float *H, double damp,
                        uint8_t *packed, void *stream) {
  const nvfp4_status st = check_weight_args(w, batch, R, C, s_g, scale_codes);
  if (st != NVFP4_OK) return st;
  if (!H || !packed || !(damp >= 0.0) || !(damp < INFINITY)) return NVFP4_ERR_INVALID_ARG;
  if (!fits(batch, C, C) || !fits(batch, R, C)) return NVFP4_ERR_SHAPE;
  if ((R + 63) / 64 > 65535) return NVFP4_ERR_TOO_LARGE;
  if (!aligned(H, 4)) return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_gptq(w, batch, R, C, s_g, scale_codes, H, damp, packed,
                                     as_stream(stream)));
}

nvfp4_status nvfp4_search_evaluations(void *stream, int reset, uint64_t *out) {
  if (!out) return NVFP4_ERR_INVALID_ARG;
  unsigned long long v[6] = {0, 0, 0, 0, 0, 0};
  cudaError_t e = nvfp4::read_search_evaluations(as_stream(stream), v, reset != 0);
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  out[0] = v[0];
  out[1] = v[1];
  return NVFP4_OK;
}

nvfp4_status nvfp4_search_rescores(void *stream, int reset, uint64_t *out) {
  if (!out) return NVFP4_ERR_INVALID_ARG;
  unsigned long long v[6] = {0, 0, 0, 0, 0, 0};
  cudaError_t e = nvfp4::read_search_evaluations(as_stream(stream), v, reset != 0);
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  for (int i = 0; i < 4; ++i) out[i] = v[2 + i];
  return NVFP4_OK;
}

nvfp4_status nvfp4_gemm(const uint8_t *a_packed, const uint8_t *a_codes, const float *a_sg,
                        const uint8_t *b_packed, const uint8_t *b_codes, const float *b_sg,
                        int64_t M, int64_t N, int64_t K, uint16_t *out, void *stream) {
  if (!a_packed || !a_codes || !a_sg || !b_packed || !b_codes || !b_sg || !out)
    return NVFP4_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
  if (K % 32 || N % 8) return NVFP4_ERR_SHAPE;
  if (M > INT32_MAX / 2 || N > INT32_MAX / 2 || K > INT32_MAX / 2 || !fits(M, K) || !fits(N, K) ||
      !fits(M, N))
    return NVFP4_ERR_TOO_LARGE;
  if (!aligned(a_packed, 16) || !aligned(b_packed, 16) || !aligned(out, 16) ||
      !aligned(a_sg, 4) || !aligned(b_sg, 4))
    return NVFP4_ERR_MISALIGNED;
  const cudaError_t e = nvfp4::launch_gemm_fp4(a_packed, a_codes, a_sg, b_packed, b_codes, b_sg,
                                               M, N, K, out, as_stream(stream));
  if (e == cudaErrorNotSupported) return NVFP4_ERR_NOT_IMPLEMENTED;
  return map_cuda(e);
}

nvfp4_status nvfp4_self_test_device_timeout(void *stream) {
  return map_cuda(nvfp4::launch_wait_timeout_probe(as_stream(stream)));
}

nvfp4_status nvfp4_self_test_mma(const uint16_t *a, const uint16_t *b, const float *c, float *d,
                                 int64_t n_tiles, void *stream) {
  if (n_tiles < 0 || (n_tiles > 0 && (!a || !b || !c || !d))) return NVFP4_ERR_INVALID_ARG;
  if (n_tiles > ((int64_t)1 << 31) * 4 - 4) return NVFP4_ERR_TOO_LARGE;
  if (!aligned(a, 2) || !aligned(b, 2) || !aligned(c, 4) || !aligned(d, 4))
    return NVFP4_ERR_MISALIGNED;
  return map_cuda(nvfp4::launch_mma_probe(a, b, c, d, n_tiles, as_stream(stream)));
}

void nvfp4_shutdown(void) { nvfp4::scratch_release_all(); }

}  // extern "C"
