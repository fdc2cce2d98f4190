// Activation-range calibration (Baseten, "What makes high-quality NVFP4",
// "Calibration": the clipping range of an activation tensor comes from
// calibration data; the maximum avoids clipping but lets rare outliers widen
// the range, while percentile-, histogram- and error-based ranges clip a few
// outliers so that the typical values are represented more finely).  The
// range sets the static tensor scale s_g = fl32(clip / 2688) used by the
// static fake-quant; block scales still follow each block's maximum.
//
//  - abs_histogram_kernel: exact counts of |x| over the 32768 bf16
//    magnitude patterns (one CTA per SM, a 128 KiB shared-memory histogram,
//    shared atomics, non-zero bins flushed to the global uint64 histogram);
//  - quantile_scale_kernel: one CTA scans the histogram for the p-quantile
//    magnitude (the smallest m with at least ceil(p N) values at or below
//    it) and writes s_g;
//  - quant_error_kernel + error_reduce_kernel: the sum of (x - y)^2 over a
//    tensor for the bf16 fake-quant output y at a given s_g, in fp64, per-CTA
//    partials added in a fixed order (the measure an error-based range
//    minimises over candidate clips).
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "../../include/nvfp4.h"

namespace nvfp4 {

// Sticky status of the calibration kernels (a quantile on a non-finite
// value), read with the library status.
__device__ int g_calib_status = 0;

namespace {

constexpr int kBins = 32768;
constexpr int kHistThreads = 1024;
constexpr int kHistSmem = kBins * (int)sizeof(uint32_t);  // 128 KiB

__global__ void __launch_bounds__(kHistThreads)
    abs_histogram_kernel(const uint16_t *__restrict__ x, int64_t n, uint64_t *__restrict__ hist) {
  extern __shared__ uint32_t sh[];
  for (int i = threadIdx.x; i < kBins; i += kHistThreads) sh[i] = 0u;
  __syncthreads();
  const int64_t nv = n / 8;  // whole 8-value vectors
  const uint4 *xv = reinterpret_cast<const uint4 *>(x);
  for (int64_t i = (int64_t)blockIdx.x * kHistThreads + threadIdx.x; i < nv;
       i += (int64_t)gridDim.x * kHistThreads) {
    const uint4 v = ld_stream_v4(xv + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      atomicAdd(&sh[w[j] & 0x7FFFu], 1u);
      atomicAdd(&sh[(w[j] >> 16) & 0x7FFFu], 1u);
    }
  }
  // the tail past the last whole vector
  if (blockIdx.x == 0)
    for (int64_t i = nv * 8 + threadIdx.x; i < n; i += kHistThreads)
      atomicAdd(&sh[x[i] & 0x7FFFu], 1u);
  __syncthreads();
  for (int i = threadIdx.x; i < kBins; i += kHistThreads)
    if (sh[i]) atomicAdd(reinterpret_cast<unsigned long long *>(hist + i),
                         (unsigned long long)sh[i]);
}

// One CTA of 1024 threads, 32 bins each.
__global__ void __launch_bounds__(kHistThreads)
    quantile_scale_kernel(const uint64_t *__restrict__ hist, double p, float *__restrict__ s_g) {
  constexpr int kPer = kBins / kHistThreads;
  __shared__ unsigned long long part[kHistThreads];
  __shared__ int found;
  const int t = threadIdx.x;
  unsigned long long local = 0;
  for (int j = 0; j < kPer; ++j) local += hist[t * kPer + j];
  part[t] = local;
  if (t == 0) found = kBins;
  __syncthreads();
  // inclusive scan of the per-thread sums (Hillis-Steele)
  for (int o = 1; o < kHistThreads; o <<= 1) {
    const unsigned long long v = t >= o ? part[t - o] : 0ull;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  const unsigned long long total = part[kHistThreads - 1];
  unsigned long long need = (unsigned long long)ceil(p * (double)total);
  if (need < 1ull) need = 1ull;
  const unsigned long long before = t ? part[t - 1] : 0ull;
  if (total > 0 && before < need && part[t] >= need) {
    unsigned long long acc = before;
    for (int j = 0; j < kPer; ++j) {
      acc += hist[t * kPer + j];
      if (acc >= need) {
        found = t * kPer + j;
        break;
      }
    }
  }
  __syncthreads();
  if (t == 0) {
    if (total == 0 || found >= kBins) {
      *s_g = 1.0f;
      return;
    }
    const float m = __uint_as_float((uint32_t)found << 16);
    if (!isfinite(m)) {
      atomicExch(&g_calib_status, (int)NVFP4_ERR_NONFINITE);
      *s_g = __int_as_float(0x7FC00000);
    } else {
      *s_g = m == 0.0f ? 1.0f : __fdiv_rn(m, 2688.0f);
    }
  }
}

std::mutex g_attr_mu;
bool g_hist_attr[64] = {};

cudaError_t ensure_hist_attr() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (!g_hist_attr[dev]) {
    e = cudaFuncSetAttribute(abs_histogram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kHistSmem);
    if (e != cudaSuccess) return e;
    g_hist_attr[dev] = true;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_abs_histogram(const uint16_t *x, int64_t n, uint64_t *hist, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  cudaError_t e = ensure_hist_attr();
  if (e != cudaSuccess) return e;
  int64_t ctas = (n / 8 + kHistThreads - 1) / kHistThreads;
  if (ctas > sm_count()) ctas = sm_count();
  if (ctas < 1) ctas = 1;
  abs_histogram_kernel<<<(unsigned)ctas, kHistThreads, kHistSmem, st>>>(x, n, hist);
  return cudaGetLastError();
}

cudaError_t launch_quantile_scale(const uint64_t *hist, double p, float *s_g, cudaStream_t st) {
  quantile_scale_kernel<<<1, kHistThreads, 0, st>>>(hist, p, s_g);
  return cudaGetLastError();
}

cudaError_t read_and_clear_calib_status(cudaStream_t st, int *out) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_calib_status, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && *out != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_calib_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice,
                                st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  }
  return e;
}

}  // namespace nvfp4
