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
//  - quantile_scale_kernel: one CTA finds the p-quantile magnitude (the
//    smallest m with at least ceil(p N) values at or below it) -- per-warp
//    chunk totals read coalesced, then the one warp whose chunk holds it
//    walks that chunk -- and writes s_g;
//  - quant_error_kernel + error_reduce_kernel: the sum of (x - y)^2 over a
//    tensor for the bf16 fake-quant output y at a given s_g, in fp64, per-CTA
//    partials added in a fixed order (the measure an error-based range
//    minimises over candidate clips).
#include <cmath>
#include <mutex>

#include "chained.cuh"
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
  chained_entry(x);  // the shared histogram was cleared before the wait
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

// One CTA of 32 warps; warp w owns bins [1024 w, 1024 w + 1024), read
// coalesced (lane l takes bins 1024 w + 32 j + l).
__global__ void __launch_bounds__(kHistThreads)
    quantile_scale_kernel(const uint64_t *__restrict__ hist, double p, float *__restrict__ s_g) {
  chained_entry();
  constexpr int kWarpBins = kBins / (kHistThreads / 32);  // 1024
  __shared__ unsigned long long warp_total[kHistThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint64_t *h = hist + (size_t)warp * kWarpBins;
  unsigned long long sum = 0;
#pragma unroll 8
  for (int j = 0; j < kWarpBins / 32; ++j) sum += h[j * 32 + lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  if (lane == 0) warp_total[warp] = sum;
  __syncthreads();
  // totals before this warp's chunk, and over all chunks (fixed order)
  unsigned long long before = 0, total = 0;
  for (int w = 0; w < kHistThreads / 32; ++w) {
    if (w < warp) before += warp_total[w];
    total += warp_total[w];
  }
  unsigned long long need = (unsigned long long)ceil(p * (double)total);
  if (need < 1ull) need = 1ull;
  // the warp whose chunk holds the quantile walks it again in bin order
  if (total > 0 && before < need && before + warp_total[warp] >= need) {
    unsigned long long acc = before;
    int found = -1;
#pragma unroll 1
    for (int j = 0; j < kWarpBins / 32 && found < 0; ++j) {
      // inclusive prefix over the 32 bins of step j (bin order = lane order)
      unsigned long long v = h[j * 32 + lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += u;
      }
      const uint32_t hit = __ballot_sync(0xFFFFFFFFu, acc + v >= need);
      if (hit) found = j * 32 + __ffs(hit) - 1;
      acc += __shfl_sync(0xFFFFFFFFu, v, 31);
    }
    if (lane == 0) {
      const float m = __uint_as_float((uint32_t)(warp * kWarpBins + found) << 16);
      if (!isfinite(m)) {
        atomicExch(&g_calib_status, (int)NVFP4_ERR_NONFINITE);
        *s_g = __int_as_float(0x7FC00000);
      } else {
        *s_g = m == 0.0f ? 1.0f : __fdiv_rn(m, 2688.0f);
      }
    }
  } else if (total == 0 && threadIdx.x == 0) {
    *s_g = 1.0f;
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
  return launch_first(abs_histogram_kernel, dim3((unsigned)ctas), dim3(kHistThreads), kHistSmem,
                        st, x, n, hist);
}

cudaError_t launch_quantile_scale(const uint64_t *hist, double p, float *s_g, cudaStream_t st) {
  return launch_first(quantile_scale_kernel, dim3(1), dim3(kHistThreads), 0, st, hist, p, s_g);
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
