// Streaming NVFP4 kernels: tensor amax -> FP32 tensor scale, max-rule block
// scales, E2M1 quantise + pack, dequantise, and the fused dynamic activation
// fake-quant.  All are HBM-bound: one thread owns one 16-value block
// (32 bytes of bf16, two 128-bit loads), consecutive threads own consecutive
// blocks, so every warp moves 1 KiB of contiguous input per step.
//
// Method sources: Baseten, "What makes high-quality NVFP4" ("Why do we need
// scales?", "Block scaling", "Why blocks?", "Calibration"); the QAD article
// "為什么NVFP4推理精度會掉以及QAD到底在修什么" (2.1, 2.3, 3.2, 4.2).
#include "common.cuh"
#include "internal.h"
#include "../../include/nvfp4.h"

namespace nvfp4 {

// Sticky device status (NVFP4_OK or NVFP4_ERR_NONFINITE), read and cleared
// by nvfp4_get_device_status.
__device__ int g_device_status = 0;

namespace {

constexpr int kThreads = 256;
constexpr uint32_t kMagMask = 0x7FFF7FFFu;

// ---------------------------------------------------------------- amax
// Largest bf16 magnitude of batch element blockIdx.y, merged with
// atomicMax into amax_bits[b] (magnitudes order like unsigned integers;
// NaN/Inf patterns compare above every finite value).
__global__ void __launch_bounds__(kThreads) amax_kernel(const uint16_t *__restrict__ x,
                                                        int64_t n_per_batch,
                                                        uint32_t *__restrict__ amax_bits) {
  const int64_t b = blockIdx.y;
  const uint4 *xb = reinterpret_cast<const uint4 *>(x + b * n_per_batch);
  const int64_t nv = n_per_batch / 8;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  uint32_t m = 0;
  for (; i + 3 * stride < nv; i += 4 * stride) {
    uint4 v0 = ld_stream_v4(xb + i);
    uint4 v1 = ld_stream_v4(xb + i + stride);
    uint4 v2 = ld_stream_v4(xb + i + 2 * stride);
    uint4 v3 = ld_stream_v4(xb + i + 3 * stride);
    uint32_t a = __vmaxu2(__vmaxu2(v0.x & kMagMask, v0.y & kMagMask),
                          __vmaxu2(v0.z & kMagMask, v0.w & kMagMask));
    uint32_t c = __vmaxu2(__vmaxu2(v1.x & kMagMask, v1.y & kMagMask),
                          __vmaxu2(v1.z & kMagMask, v1.w & kMagMask));
    uint32_t d = __vmaxu2(__vmaxu2(v2.x & kMagMask, v2.y & kMagMask),
                          __vmaxu2(v2.z & kMagMask, v2.w & kMagMask));
    uint32_t e = __vmaxu2(__vmaxu2(v3.x & kMagMask, v3.y & kMagMask),
                          __vmaxu2(v3.z & kMagMask, v3.w & kMagMask));
    m = __vmaxu2(m, __vmaxu2(__vmaxu2(a, c), __vmaxu2(d, e)));
  }
  for (; i < nv; i += stride) {
    uint4 v = ld_stream_v4(xb + i);
    m = __vmaxu2(m, __vmaxu2(__vmaxu2(v.x & kMagMask, v.y & kMagMask),
                             __vmaxu2(v.z & kMagMask, v.w & kMagMask)));
  }
  uint32_t mm = max(m & 0xFFFFu, m >> 16);
  mm = __reduce_max_sync(0xFFFFFFFFu, mm);
  __shared__ uint32_t warp_max[kThreads / 32];
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = mm;
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t v = threadIdx.x < kThreads / 32 ? warp_max[threadIdx.x] : 0u;
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    if (threadIdx.x == 0 && v) atomicMax(amax_bits + b, v);
  }
}

// s_g = fl32(amax / 2688), 1 for amax = 0, NaN (and a NONFINITE report) when
// the tensor held NaN/Inf.  The amax bits were accumulated in place.
__global__ void global_scale_finish_kernel(float *s_g, int64_t batch) {
  const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= batch) return;
  const uint32_t bits = reinterpret_cast<const uint32_t *>(s_g)[b];
  float r;
  if (bits >= 0x7F80u) {
    r = __uint_as_float(0x7FC00000u);
    atomicExch(&g_device_status, (int)NVFP4_ERR_NONFINITE);
  } else if (bits == 0u) {
    r = 1.0f;
  } else {
    r = __fdiv_rn(__uint_as_float(bits << 16), 2688.0f);
  }
  s_g[b] = r;
}

// ------------------------------------------------------------ block helpers
__device__ __forceinline__ void load_block(const uint16_t *p, uint32_t w[8]) {
  const uint4 *q = reinterpret_cast<const uint4 *>(p);
  uint4 v0 = ld_stream_v4(q), v1 = ld_stream_v4(q + 1);
  w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
  w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
}

// Eight packed bytes (two signed E2M1 codes each) of one block at scale s.
// s = 0 (code 0) encodes every value as a signed zero.
__device__ __forceinline__ void encode_block(const uint32_t w[8], float s, uint32_t bytes[8]) {
  if (s > 0.0f) {
    const ScaleRecip r = make_recip(s);
    uint32_t mismatch = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      bytes[j] = e2m1_pair_bracket(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j])), r, mismatch);
    if (mismatch) {  // some |x|/s within rounding distance of a midpoint
#pragma unroll
      for (int j = 0; j < 8; ++j)
        bytes[j] = e2m1_mag_exact(fabsf(bf16_lo(w[j])), s) |
                   (e2m1_mag_exact(fabsf(bf16_hi(w[j])), s) << 4);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) bytes[j] = 0u;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) bytes[j] |= ((w[j] >> 12) & 0x8u) | ((w[j] >> 24) & 0x80u);
}

__device__ __forceinline__ uint2 pack8(const uint32_t bytes[8]) {
  return make_uint2(bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24),
                    bytes[4] | (bytes[5] << 8) | (bytes[6] << 16) | (bytes[7] << 24));
}

// bf16 pair of v(q) * s for one packed byte: fp32 product, then bf16 RN.
__device__ __forceinline__ uint32_t dequant_byte(uint32_t byte, float s) {
  const uint32_t h2 = cvt_f16x2_from_e2m1x2(byte);
  const float y0 = __fmul_rn(f16_lo_to_float(h2), s);
  const float y1 = __fmul_rn(f16_hi_to_float(h2), s);
  __nv_bfloat162 p = __floats2bfloat162_rn(y0, y1);
  return *reinterpret_cast<uint32_t *>(&p);
}

__device__ __forceinline__ void store_dequant(uint16_t *out, const uint32_t bytes[8], float s) {
  uint4 o0, o1;
  o0.x = dequant_byte(bytes[0], s); o0.y = dequant_byte(bytes[1], s);
  o0.z = dequant_byte(bytes[2], s); o0.w = dequant_byte(bytes[3], s);
  o1.x = dequant_byte(bytes[4], s); o1.y = dequant_byte(bytes[5], s);
  o1.z = dequant_byte(bytes[6], s); o1.w = dequant_byte(bytes[7], s);
  uint4 *q = reinterpret_cast<uint4 *>(out);
  st_stream_v4(q, o0);
  st_stream_v4(q + 1, o1);
}

// --------------------------------------------------------------- kernels
// grid: (x: block-strided CTAs, y: batch element)
__global__ void __launch_bounds__(kThreads) max_rule_kernel(const uint16_t *__restrict__ w,
                                                            int64_t nblk,
                                                            const float *__restrict__ s_g,
                                                            uint8_t *__restrict__ codes) {
  const int64_t b = blockIdx.y;
  const float sg = s_g[b];
  w += b * nblk * kBlock;
  codes += b * nblk;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nblk;
       i += (int64_t)gridDim.x * kThreads) {
    uint32_t v[8];
    load_block(w + i * kBlock, v);
    const float amax = __uint_as_float(amax_bits8(v) << 16);
    codes[i] = (uint8_t)max_rule_code(amax, sg);
  }
}

__global__ void __launch_bounds__(kThreads) pack_kernel(const uint16_t *__restrict__ w,
                                                        int64_t nblk,
                                                        const float *__restrict__ s_g,
                                                        const uint8_t *__restrict__ codes,
                                                        uint8_t *__restrict__ packed) {
  const int64_t b = blockIdx.y;
  const float sg = s_g[b];
  w += b * nblk * kBlock;
  codes += b * nblk;
  packed += b * nblk * (kBlock / 2);
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nblk;
       i += (int64_t)gridDim.x * kThreads) {
    uint32_t v[8], bytes[8];
    load_block(w + i * kBlock, v);
    const float s = effective_scale(sg, codes[i]);
    encode_block(v, s, bytes);
    st_stream_v2(packed + i * 8, pack8(bytes));
  }
}

__global__ void __launch_bounds__(kThreads) dequant_kernel(const uint8_t *__restrict__ packed,
                                                           const uint8_t *__restrict__ codes,
                                                           const float *__restrict__ s_g,
                                                           int64_t nblk,
                                                           uint16_t *__restrict__ out) {
  const int64_t b = blockIdx.y;
  const float sg = s_g[b];
  packed += b * nblk * (kBlock / 2);
  codes += b * nblk;
  out += b * nblk * kBlock;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nblk;
       i += (int64_t)gridDim.x * kThreads) {
    const uint2 p = __ldcs(reinterpret_cast<const uint2 *>(packed) + i);
    const float s = effective_scale(sg, codes[i]);
    const uint32_t bytes[8] = {p.x & 0xFFu, (p.x >> 8) & 0xFFu, (p.x >> 16) & 0xFFu, p.x >> 24,
                               p.y & 0xFFu, (p.y >> 8) & 0xFFu, (p.y >> 16) & 0xFFu, p.y >> 24};
    store_dequant(out + i * kBlock, bytes, s);
  }
}

// Fused fake-quant pass (after the tensor scale is known): max rule, encode,
// dequantise; optional packed codes and block codes.
__global__ void __launch_bounds__(kThreads) fake_quant_kernel(const uint16_t *__restrict__ x,
                                                              int64_t nblk,
                                                              const float *__restrict__ s_g,
                                                              uint16_t *__restrict__ out,
                                                              uint8_t *__restrict__ packed,
                                                              uint8_t *__restrict__ codes) {
  const float sg = *s_g;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nblk;
       i += (int64_t)gridDim.x * kThreads) {
    uint32_t v[8], bytes[8];
    load_block(x + i * kBlock, v);
    const float amax = __uint_as_float(amax_bits8(v) << 16);
    const uint32_t code = max_rule_code(amax, sg);
    const float s = effective_scale(sg, code);
    encode_block(v, s, bytes);
    store_dequant(out + i * kBlock, bytes, s);
    if (packed) st_stream_v2(packed + i * 8, pack8(bytes));
    if (codes) codes[i] = (uint8_t)code;
  }
}

int g_sm_count = 0;

int grid_for(int64_t work_items, int max_ctas_per_sm) {
  if (g_sm_count == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (g_sm_count <= 0) g_sm_count = 148;
  }
  int64_t need = (work_items + kThreads - 1) / kThreads;
  int64_t cap = (int64_t)g_sm_count * max_ctas_per_sm;
  if (need < 1) need = 1;
  return (int)(need < cap ? need : cap);
}

}  // namespace

int sm_count() {
  grid_for(1, 1);
  return g_sm_count;
}

cudaError_t launch_global_scale(const uint16_t *x, int64_t batch, int64_t n_per_batch,
                                float *s_g, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(s_g, 0, sizeof(float) * batch, st);
  if (e != cudaSuccess) return e;
  if (n_per_batch > 0) {
    const int64_t nv = n_per_batch / 8;
    int gx = grid_for(nv / 4 + 1, 8);
    const int64_t per_batch_cap = ((int64_t)sm_count() * 8 + batch - 1) / batch;
    if (gx > per_batch_cap) gx = (int)(per_batch_cap > 0 ? per_batch_cap : 1);
    amax_kernel<<<dim3(gx, (unsigned)batch), kThreads, 0, st>>>(
        x, n_per_batch, reinterpret_cast<uint32_t *>(s_g));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  global_scale_finish_kernel<<<(unsigned)((batch + 127) / 128), 128, 0, st>>>(s_g, batch);
  return cudaGetLastError();
}

cudaError_t launch_scale_max(const uint16_t *w, int64_t batch, int64_t nblk, const float *s_g,
                             uint8_t *codes, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  int gx = grid_for(nblk, 16);
  max_rule_kernel<<<dim3(gx, (unsigned)batch), kThreads, 0, st>>>(w, nblk, s_g, codes);
  return cudaGetLastError();
}

cudaError_t launch_pack(const uint16_t *w, int64_t batch, int64_t nblk, const float *s_g,
                        const uint8_t *codes, uint8_t *packed, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  int gx = grid_for(nblk, 16);
  pack_kernel<<<dim3(gx, (unsigned)batch), kThreads, 0, st>>>(w, nblk, s_g, codes, packed);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t *packed, const uint8_t *codes, const float *s_g,
                           int64_t batch, int64_t nblk, uint16_t *out, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  int gx = grid_for(nblk, 16);
  dequant_kernel<<<dim3(gx, (unsigned)batch), kThreads, 0, st>>>(packed, codes, s_g, nblk,
                                                                  out);
  return cudaGetLastError();
}

cudaError_t launch_fake_quant(const uint16_t *x, int64_t rows, int64_t C, uint16_t *out,
                              uint8_t *packed, uint8_t *codes, float *s_g, cudaStream_t st) {
  const int64_t n = rows * C;
  cudaError_t e = launch_global_scale(x, 1, n, s_g, st);
  if (e != cudaSuccess || n == 0) return e;
  const int64_t nblk = n / kBlock;
  int gx = grid_for(nblk, 16);
  fake_quant_kernel<<<gx, kThreads, 0, st>>>(x, nblk, s_g, out, packed, codes);
  return cudaGetLastError();
}

cudaError_t read_and_clear_device_status(cudaStream_t st, int *out) {
  int zero = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(out, g_device_status, sizeof(int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
}

}  // namespace nvfp4
