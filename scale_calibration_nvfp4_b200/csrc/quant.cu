// Streaming NVFP4 kernels: tensor amax -> FP32 tensor scale, max-rule block
// scales, E2M1 quantise + pack, dequantise, and the fused dynamic activation
// fake-quant.  All are HBM-bound: one thread owns one 16-value block
// (32 bytes of bf16, two 128-bit loads), consecutive threads own consecutive
// blocks, so every warp moves 1 KiB of contiguous input per step.
//
// Method sources: Baseten, "What makes high-quality NVFP4" ("Why do we need
// scales?", "Block scaling", "Why blocks?", "Calibration"); the QAD article
// "為什么NVFP4推理精度會掉以及QAD到底在修什么" (2.1, 2.3, 3.2, 4.2).
#include <algorithm>

#include "chained.cuh"
#include "common.cuh"
#include "internal.h"
#include "../../include/nvfp4.h"

namespace nvfp4 {

// Sticky device status of the streaming kernels (NVFP4_OK or
// NVFP4_ERR_NONFINITE), read and cleared by nvfp4_get_device_status.
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
  chained_entry(x);
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

// n words set to zero
__global__ void zero_words_kernel(uint32_t *p, int64_t n) {
  chained_entry();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = 0u;
}

// s_g = fl32(amax / 2688), 1 for amax = 0, NaN (and a NONFINITE report) when
// the tensor held NaN/Inf.  The amax bits were accumulated in place.
__global__ void global_scale_finish_kernel(float *s_g, int64_t batch) {
  chained_entry();
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

// ------------------------------------------------------- exact block encode
//
// Exact rounding of a quotient q by the hardware nearest-even conversions.
// The E4M3 max-rule code rounds t (within one float of q) and t_alt, the
// neighbouring float on the other side of q (chosen by the exact sign of a
// residual); the two can only disagree when one of them is a rounding
// midpoint, q then lies strictly on the other one's side, and the correct
// code is the odd one of the two (the tie went to the even one).  The E2M1
// encode below needs the residual only for a t that could be a midpoint.

// Four e2m1x2 conversions into one word: byte i = (code(h_i) << 4) | code(l_i),
// signed inputs give signed codes (a negative value rounding to 0 gives -0).
__device__ __forceinline__ uint32_t cvt4_e2m1(float h0, float l0, float h1, float l1, float h2,
                                              float l2, float h3, float l3) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %1, %2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %3, %4;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %5, %6;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %7, %8;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(r)
      : "f"(h0), "f"(l0), "f"(h1), "f"(l1), "f"(h2), "f"(l2), "f"(h3), "f"(l3));
  return r;
}

// Adjacent float of t towards the side given by the residual (same sign as
// q - t); t itself when the residual is zero (q == t exactly), of either sign
// (t = +0 with rho = -0 must not step towards zero into a NaN).
__device__ __forceinline__ float toward(float t, float rho) {
  const int rb = __float_as_int(rho);
  const int dir = ((rb ^ __float_as_int(t)) >> 31) | 1;  // +1 away from 0, -1 towards
  return __int_as_float(__float_as_int(t) + ((__float_as_uint(rho) << 1) != 0u ? dir : 0));
}

// Packed signed E2M1 codes of 8 consecutive elements (4 bf16 pairs) at scale
// s > 0 with r_hi + r_lo = 1/s (r_lo >= 0).  t = x (r_hi + r_lo) rounds
// once from a value within 2^-45 (relative) of q = x / s, so it is one of the
// two floats around q, and no float lies strictly between t and q.  Every
// rounding midpoint (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) is a float, so
// when t is not one of them, rounding t to nearest-even gives q's code.
// Midpoints have at most 3 significant bits; only a t with 21 zero low
// mantissa bits (rare: an exact or nearly exact quotient) is stepped to its
// neighbour across q by the exact sign of the residual x - t s (one fma),
// which is t itself when q == t.  That neighbour has 24 significant bits, so
// it is no midpoint and rounds like q: to the odd code when t was a midpoint
// and q lies off it, to the even one on an exact tie.
__device__ __forceinline__ uint32_t encode_word(const uint32_t *w, float s, float r_hi,
                                                float r_lo) {
  float t[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float x = (e & 1) ? bf16_hi(w[e >> 1]) : bf16_lo(w[e >> 1]);
    t[e] = fmaf(x, r_hi, x * r_lo);
  }
#pragma unroll
  for (int p = 0; p < 8; p += 2) {
    const bool n0 = (__float_as_uint(t[p]) & 0x1FFFFFu) == 0u;
    const bool n1 = (__float_as_uint(t[p + 1]) & 0x1FFFFFu) == 0u;
    if (n0 || n1) {
      const float x0 = bf16_lo(w[p >> 1]), x1 = bf16_hi(w[p >> 1]);
      const float a0 = toward(t[p], fmaf(-t[p], s, x0));
      const float a1 = toward(t[p + 1], fmaf(-t[p + 1], s, x1));
      t[p] = n0 ? a0 : t[p];
      t[p + 1] = n1 ? a1 : t[p + 1];
    }
  }
  return cvt4_e2m1(t[1], t[0], t[3], t[2], t[5], t[4], t[7], t[6]);
}

__device__ __forceinline__ uint2 encode_block(const uint32_t w[8], float s, float r_hi,
                                              float r_lo) {
  return make_uint2(encode_word(w, s, r_hi, r_lo), encode_word(w + 4, s, r_hi, r_lo));
}

// Packed codes by the exact fp64 midpoint test (s = 0: signed zeros).
__device__ __forceinline__ uint2 encode_block_exact(const uint32_t w[8], float s) {
  uint32_t bytes[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    bytes[j] = (s > 0.0f ? (e2m1_mag_exact(fabsf(bf16_lo(w[j])), s) |
                            (e2m1_mag_exact(fabsf(bf16_hi(w[j])), s) << 4))
                         : 0u) |
               ((w[j] >> 12) & 0x8u) | ((w[j] >> 24) & 0x80u);
  }
  return make_uint2(bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24),
                    bytes[4] | (bytes[5] << 8) | (bytes[6] << 16) | (bytes[7] << 24));
}

// E4M3 code (0..0x7E) -> fp32 value, branch-free.
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const float sub = (float)c * 0x1p-9f;
  const float nor = __uint_as_float((c << 20) + (120u << 23));
  return c < 8u ? sub : nor;
}

// Everything a block's encode needs from its scale, computed once per code
// and CTA: s_eff and its reciprocal split (r_hi rounded down, so r_lo >= 0 and
// x = -0 keeps its sign in t), or 0 for scales outside [2^-100, 2^100) (below,
// the reciprocal may overflow; above, r_lo is subnormal and too coarse near
// the top of the fp32 range), zero or NaN, which take the exact fp64 encode.
struct __align__(16) ScaleEntry {  // one 128-bit shared-memory load
  float s, r_hi, r_lo;
  uint32_t exact64;
};
__device__ __forceinline__ ScaleEntry make_scale_entry(float s) {
  ScaleEntry e;
  e.s = s;
  e.r_hi = 0.0f;
  e.r_lo = 0.0f;
  e.exact64 = 1u;
  if (s >= 0x1p-100f && s < 0x1p100f) {
    e.r_hi = __frcp_rd(s);
    e.r_lo = fmaf(-s, e.r_hi, 1.0f) * e.r_hi;
    e.exact64 = 0u;
  }
  return e;
}
__device__ __forceinline__ uint2 encode_block_entry(const uint32_t w[8], const ScaleEntry &e) {
  if (!e.exact64) return encode_block(w, e.s, e.r_hi, e.r_lo);
  return encode_block_exact(w, e.s);
}

// Table of ScaleEntry for every code byte of one s_g, filled by the CTA's
// 256 threads (one each; codes above 0x7E follow the same formula).
__device__ __forceinline__ void fill_scale_table(ScaleEntry *tab, float sg) {
  static_assert(kThreads == 256, "one table entry per thread");
  tab[threadIdx.x] = make_scale_entry(__fmul_rn(sg, e4m3_value(threadIdx.x)));
  __syncthreads();
}

// E4M3 code of amax / (k s_g) (k = 6: the max rule; k = 4: the second
// candidate of Four Over Six), exact (nearest even, saturating at 448), from
// D = k s_g (exact in fp64) and R = 1/D split as r_hi + r_lo: t = amax R, the
// residual amax - t D is exact in one fp64 fma, and the same odd-code rule
// picks between the two e4m3x2 conversions.  Where R passes 2^100 (s_g below
// about 2^-102, tensor maxima below about 2^-91; R itself can pass the fp32
// range) R 2^-64 is split instead and amax enters as amax 2^64 (exact: amax
// is at most about 2688 s_g there).
struct MaxRule {
  double D;
  float r_hi, r_lo, pre;
};
__device__ __forceinline__ MaxRule make_max_rule(float s_g, double k = 6.0) {
  MaxRule m;
  m.D = k * (double)s_g;
  double R = 1.0 / m.D;
  m.pre = 1.0f;
  if (R > 0x1p100) {
    R *= 0x1p-64;
    m.pre = 0x1p64f;
  }
  m.r_hi = (float)R;
  m.r_lo = (float)(R - (double)m.r_hi);
  return m;
}
__device__ __forceinline__ uint32_t max_rule_code_fast(float amax, const MaxRule &m) {
  const float as = amax * m.pre;
  const float t = fmaf(as, m.r_hi, as * m.r_lo);
  const double rho = fma(-(double)t, m.D, (double)amax);
  const float ta = __int_as_float(__float_as_int(t) + (rho > 0.0 ? 1 : (rho < 0.0 ? -1 : 0)));
  unsigned short pair;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(ta), "f"(t));
  const uint32_t ct = pair & 0xFFu, ca = pair >> 8;
  return (ct & 1u) ? ct : ca;  // equal, or the odd one of two neighbours
}

// The same code with the fp64 residual only near a midpoint.  t as above is
// within 2^-23.9 of q; fl(t (1 + 2^-22)) and fl(t (1 - 2^-22)) lie at least
// 2^-22.4 t from t (the product's rounding takes at most 2^-24), so they
// bracket q.  Where both round to the same code no E4M3 rounding midpoint lies
// between them (nearest-even rounding is monotone, and a midpoint on an end
// goes to that end's side, as q does), and that code is q's (saturation above
// 448 included); otherwise, for a quotient within about 2^-22 of a midpoint,
// the residual decides.
__device__ __forceinline__ uint32_t max_rule_code_margin(float amax, const MaxRule &m) {
  const float as = amax * m.pre;
  const float t = fmaf(as, m.r_hi, as * m.r_lo);
  const float2 b = __fmul2_rn(make_float2(t, t), make_float2(1.0f + 0x1p-22f, 1.0f - 0x1p-22f));
  unsigned short pair;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(b.x), "f"(b.y));
  const uint32_t cu = pair >> 8, cd = pair & 0xFFu;
  return cu == cd ? cu : max_rule_code_fast(amax, m);
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
  chained_entry(w);
  const int64_t b = blockIdx.y;
  const MaxRule mr = make_max_rule(s_g[b]);
  w += b * nblk * kBlock;
  codes += b * nblk;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nblk;
       i += (int64_t)gridDim.x * kThreads) {
    uint32_t v[8];
    load_block(w + i * kBlock, v);
    const float amax = __uint_as_float(amax_bits8(v) << 16);
    codes[i] = (uint8_t)max_rule_code_margin(amax, mr);
  }
}

// Signed E2M1 value of code i of a packed block (fp32, exact).
__device__ __forceinline__ float e2m1_code_value(uint2 q, int i) {
  const uint32_t code = ((i < 8 ? q.x : q.y) >> (4 * (i & 7))) & 0xFu;
  const uint32_t k = code & 7u;
  const float mag = k < 2 ? 0.5f * k : (1.0f + 0.5f * (float)(k & 1u)) * (float)(1 << ((k >> 1) - 1));
  return (code & 8u) ? -mag : mag;
}

// Block MSE at scale s in fp32 (a screen: every d_i is rounded once and the
// 16 non-negative terms are summed with one rounding each, so the error
// stays below 2^-20 relative plus, where terms or partial sums fall into the
// subnormal range (tensor scales near 1e-20 and below), 2^-145 absolute).
// Codes back to values by the hardware e2m1x2 -> f16x2 conversion (exact).
__device__ __forceinline__ float block_mse32(const uint32_t w[8], uint2 q, float s) {
  float e = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t byte = ((j < 4 ? q.x : q.y) >> (8 * (j & 3))) & 0xFFu;
    const uint32_t h2 = cvt_f16x2_from_e2m1x2(byte);
    const float d0 = fmaf(-f16_lo_to_float(h2), s, bf16_lo(w[j]));
    const float d1 = fmaf(-f16_hi_to_float(h2), s, bf16_hi(w[j]));
    e = fmaf(d0, d0, e);
    e = fmaf(d1, d1, e);
  }
  return e;
}

// The fp32 block MSE at a table entry's scale, straight from the values:
// t = fl(x r_hi) (r_hi = 1/s rounded down: |t - q| <= 2^-23 |q| for the exact
// quotient q), each pair rounded from t (one conversion) and its byte decoded
// by the hardware e2m1x2 -> f16x2 conversion in the same asm block, then d_i =
// x_i - v_i s and the d_i^2 summed by fma in two partial sums (even and odd
// elements, each in element order), added at the end.  The codes are those of
// t, not always of q: where a rounding midpoint M lies between q and t, t
// takes the other neighbour, and |d_i| (about half a grid step times s either
// way) moves by at most 2 |q - M| s <= 2^-22 |q| s, at most 2^-19.7 of itself
// (the worst case M = 5 with a step of 2); d_i^2 then moves by at most
// 2^-18.7, and with the roundings of the sums the screen stays within 2^-18.4
// of the definition -- inside its 2^-16 threshold.  The exact comparison
// below uses exact codes.
__device__ __forceinline__ uint32_t e2m1x2_round_decode(float hi, float lo) {
  uint32_t h2;
  asm("{\n\t.reg .b8 q;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q, %1, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, q;\n\t}"
      : "=r"(h2)
      : "f"(hi), "f"(lo));
  return h2;
}
__device__ __forceinline__ float block_mse32_entry(const uint32_t w[8], const ScaleEntry &e) {
  if (e.exact64) return block_mse32(w, encode_block_exact(w, e.s), e.s);
  // paired fp32 arithmetic on each value pair (each lane rounded as its
  // scalar form): even elements accumulate in .x, odd ones in .y
  const float2 rh = make_float2(e.r_hi, e.r_hi), ns = make_float2(-e.s, -e.s);
  float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 x = make_float2(bf16_lo(w[j]), bf16_hi(w[j]));
    const float2 t = __fmul2_rn(x, rh);
    const uint32_t h2 = e2m1x2_round_decode(t.y, t.x);
    const float2 d = __ffma2_rn(make_float2(f16_lo_to_float(h2), f16_hi_to_float(h2)), ns, x);
    acc = __ffma2_rn(d, d, acc);
  }
  return acc.x + acc.y;
}

// Both candidates' fp32 block MSEs in one pass over the values (each pair
// unpacked once), each with exactly block_mse32_entry's arithmetic.
__device__ __forceinline__ void block_mse32_two(const uint32_t w[8], const ScaleEntry &ea,
                                                const ScaleEntry &eb, float &fa, float &fb) {
  if (ea.exact64 || eb.exact64) {
    fa = block_mse32_entry(w, ea);
    fb = block_mse32_entry(w, eb);
    return;
  }
  const float2 rha = make_float2(ea.r_hi, ea.r_hi), nsa = make_float2(-ea.s, -ea.s);
  const float2 rhb = make_float2(eb.r_hi, eb.r_hi), nsb = make_float2(-eb.s, -eb.s);
  float2 acca = make_float2(0.0f, 0.0f), accb = acca;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 x = make_float2(bf16_lo(w[j]), bf16_hi(w[j]));
    const float2 ta = __fmul2_rn(x, rha), tb = __fmul2_rn(x, rhb);
    const uint32_t ha = e2m1x2_round_decode(ta.y, ta.x), hb = e2m1x2_round_decode(tb.y, tb.x);
    const float2 da = __ffma2_rn(make_float2(f16_lo_to_float(ha), f16_hi_to_float(ha)), nsa, x);
    const float2 db = __ffma2_rn(make_float2(f16_lo_to_float(hb), f16_hi_to_float(hb)), nsb, x);
    acca = __ffma2_rn(da, da, acca);
    accb = __ffma2_rn(db, db, accb);
  }
  fa = acca.x + acca.y;
  fb = accb.x + accb.y;
}

// Block MSE at the table entry's scale in fp64, with the operations of the
// definition in its order: d_i = w_i - v_i s, e += d_i^2, i = 0..15, each
// product and sum rounded on its own (no fused multiply-add), so that two
// candidates compare exactly as in the definition.
__device__ __noinline__ double block_mse64(const uint32_t w[8], uint2 q, float sf) {
  const double s = (double)sf;
  double e = 0.0;
#pragma unroll 1
  for (int i = 0; i < 16; ++i) {
    const double v = (double)e2m1_code_value(q, i);
    const double x = (double)((i & 1) ? bf16_hi(w[i >> 1]) : bf16_lo(w[i >> 1]));
    const double d = __dsub_rn(x, __dmul_rn(v, s));
    e = __dadd_rn(e, __dmul_rn(d, d));
  }
  return e;
}

// Per-CTA constants of Four Over Six: the two max rules (k = 6, 4).
struct FourSixConsts {
  MaxRule m6, m4;
};

// The exact fp64 comparison of Four Over Six's two candidates (codes lo <
// hi) for a block whose fp32 screen could not separate them; the block by
// value, so that the caller keeps nothing in memory for this rare path.
__device__ __noinline__ uint32_t four_over_six_exact(uint4 w0, uint4 w1, ScaleEntry el,
                                                     ScaleEntry eh, uint32_t lo, uint32_t hi) {
  const uint32_t v[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
  const uint2 ql = encode_block_entry(v, el), qh = encode_block_entry(v, eh);
  return block_mse64(v, qh, eh.s) < block_mse64(v, ql, el.s) ? hi : lo;
}

// One block's Four Over Six code (see four_over_six_kernel).  plain: neither
// max rule pre-scales its quotient (so amax enters as it is).
__device__ __forceinline__ uint32_t four_over_six_code(const uint32_t v[8],
                                                       const ScaleEntry *tab,
                                                       const FourSixConsts &cs, bool plain,
                                                       float2 r_hi, float2 r_lo) {
  const float amax = __uint_as_float(amax_bits8(v) << 16);
  // max_rule_code_margin for both codes at once: the quotients paired (each
  // lane rounded as the scalar t), the brackets of both in two conversions
  // (c4 in the upper byte), the residuals where either code is in doubt or a
  // max rule pre-scales.
  const float2 a = make_float2(amax, amax);
  const float2 t = __ffma2_rn(a, r_hi, __fmul2_rn(a, r_lo));
  const float2 tu = __fmul2_rn(t, make_float2(1.0f + 0x1p-22f, 1.0f + 0x1p-22f));
  const float2 td = __fmul2_rn(t, make_float2(1.0f - 0x1p-22f, 1.0f - 0x1p-22f));
  unsigned short pu, pd;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pu) : "f"(tu.y), "f"(tu.x));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pd) : "f"(td.y), "f"(td.x));
  uint32_t c6 = pu & 0xFFu, c4 = pu >> 8;
  if (!plain) {
    c6 = max_rule_code_fast(amax, cs.m6);
    c4 = max_rule_code_fast(amax, cs.m4);
  } else if (pu != pd) {
    // max_rule_code_fast's residual step on the quotients already formed
    const double A = (double)amax;
    const double r6 = fma(-(double)t.x, cs.m6.D, A), r4 = fma(-(double)t.y, cs.m4.D, A);
    const float a6 = __int_as_float(__float_as_int(t.x) + (r6 > 0.0 ? 1 : (r6 < 0.0 ? -1 : 0)));
    const float a4 = __int_as_float(__float_as_int(t.y) + (r4 > 0.0 ? 1 : (r4 < 0.0 ? -1 : 0)));
    unsigned short pt, pa;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pt) : "f"(t.y), "f"(t.x));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pa) : "f"(a4), "f"(a6));
    const uint32_t t6 = pt & 0xFFu, t4 = pt >> 8;
    c6 = (t6 & 1u) ? t6 : (pa & 0xFFu);  // equal, or the odd one of two neighbours
    c4 = (t4 & 1u) ? t4 : (uint32_t)(pa >> 8);
  }
  const uint32_t lo = min(c4, c6), hi = max(c4, c6);
  uint32_t code = lo;
  if (amax > 0.0f && hi != lo) {
    // fp32 screen; the exact fp64 comparison only when the two are close
    // (relative 2^-16, or absolute 2^-130 for subnormal sums)
    const ScaleEntry el = tab[lo], eh = tab[hi];
    float fl, fh;
    block_mse32_two(v, el, eh, fl, fh);
    if (fabsf(fh - fl) > fmaf(0x1p-16f, fmaxf(fh, fl), 0x1p-130f)) {
      code = fh < fl ? hi : lo;
    } else {
      code = four_over_six_exact(make_uint4(v[0], v[1], v[2], v[3]),
                                 make_uint4(v[4], v[5], v[6], v[7]), el, eh, lo, hi);
    }
  }
  return amax > 0.0f ? code : 0u;
}

// Four Over Six (the Local-Hessian write-up, "The NVFP4 structure": one of
// two candidate scales per block): the max-rule code and the code of
// amax / (4 s_g), whichever block MSE is smaller, the smaller code on a tie;
// an all-zero block gets code 0.
__global__ void __launch_bounds__(kThreads, 3)
    four_over_six_kernel(const uint16_t *__restrict__ w, int64_t nblk,
                         const float *__restrict__ s_g, uint8_t *__restrict__ codes) {
  chained_entry(w);
  const int64_t b = blockIdx.y;
  w += b * nblk * kBlock;
  codes += b * nblk;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  uint32_t v[8];
  if (i < nblk) load_block(w + i * kBlock, v);
  // the max rules (by the first lane of each of two warps; the others read
  // them) and the table are formed while the first block is in flight
  const float sg = s_g[b];
  __shared__ FourSixConsts cs;
  __shared__ ScaleEntry tab[256];
  if (threadIdx.x == 0) cs.m6 = make_max_rule(sg, 6.0);
  if (threadIdx.x == 32) cs.m4 = make_max_rule(sg, 4.0);
  fill_scale_table(tab, sg);
  const bool plain = cs.m6.pre == 1.0f && cs.m4.pre == 1.0f;
  const float2 r_hi = make_float2(cs.m6.r_hi, cs.m4.r_hi);
  const float2 r_lo = make_float2(cs.m6.r_lo, cs.m4.r_lo);
  for (; i < nblk; i += stride) {
    // issue the next block's loads before this block's arithmetic
    uint32_t nv[8];
    const int64_t n = i + stride;
    if (n < nblk) load_block(w + n * kBlock, nv);
    codes[i] = (uint8_t)four_over_six_code(v, tab, cs, plain, r_hi, r_lo);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = nv[j];
  }
}

__global__ void __launch_bounds__(kThreads) pack_kernel(const uint16_t *__restrict__ w,
                                                        int64_t nblk,
                                                        const float *__restrict__ s_g,
                                                        const uint8_t *__restrict__ codes,
                                                        uint8_t *__restrict__ packed) {
  chained_entry(w);
  const int64_t b = blockIdx.y;
  w += b * nblk * kBlock;
  codes += b * nblk;
  packed += b * nblk * (kBlock / 2);
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  uint32_t v[8];
  uint32_t code = 0;
  if (i < nblk) {
    load_block(w + i * kBlock, v);
    code = codes[i];
  }
  // the table is built while the first block is in flight
  __shared__ ScaleEntry tab[256];
  fill_scale_table(tab, s_g[b]);
  for (; i < nblk; i += stride) {
    // issue the next block's loads before this block's arithmetic
    uint32_t nv[8];
    uint32_t ncode = 0;
    const int64_t n = i + stride;
    if (n < nblk) {
      load_block(w + n * kBlock, nv);
      ncode = codes[n];
    }
    st_stream_v2(packed + i * 8, encode_block_entry(v, tab[code]));
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = nv[j];
    code = ncode;
  }
}

__global__ void __launch_bounds__(kThreads) dequant_kernel(const uint8_t *__restrict__ packed,
                                                           const uint8_t *__restrict__ codes,
                                                           const float *__restrict__ s_g,
                                                           int64_t nblk,
                                                           uint16_t *__restrict__ out) {
  chained_entry(packed);
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
  chained_entry(x);
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  uint32_t v[8];
  if (i < nblk) load_block(x + i * kBlock, v);
  // the table is built while the first block is in flight
  const float sg = *s_g;
  const MaxRule mr = make_max_rule(sg);
  __shared__ ScaleEntry tab[256];
  fill_scale_table(tab, sg);
  for (; i < nblk; i += stride) {
    // issue the next block's loads before this block's arithmetic
    uint32_t nv[8];
    const int64_t n = i + stride;
    if (n < nblk) load_block(x + n * kBlock, nv);
    const float amax = __uint_as_float(amax_bits8(v) << 16);
    const uint32_t code = max_rule_code_fast(amax, mr);
    const ScaleEntry se = tab[code];
    const float s = se.s;
    const uint2 q = encode_block_entry(v, se);
    const uint32_t bytes[8] = {q.x & 0xFFu, (q.x >> 8) & 0xFFu, (q.x >> 16) & 0xFFu, q.x >> 24,
                               q.y & 0xFFu, (q.y >> 8) & 0xFFu, (q.y >> 16) & 0xFFu, q.y >> 24};
    store_dequant(out + i * kBlock, bytes, s);
    if (packed) st_stream_v2(packed + i * 8, q);
    if (codes) codes[i] = (uint8_t)code;
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = nv[j];
  }
}

// Sum of (x - y)^2 over a tensor for its bf16 fake-quant output y at the
// given tensor scale (the static-range fake-quant without its writes), in
// fp64; one partial per CTA, in a fixed order within the CTA.
__global__ void __launch_bounds__(kThreads) quant_error_kernel(const uint16_t *__restrict__ x,
                                                               int64_t nblk,
                                                               const float *__restrict__ s_g,
                                                               double *__restrict__ partial) {
  chained_entry(x);
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  uint32_t v[8];
  if (i < nblk) load_block(x + i * kBlock, v);
  const float sg = *s_g;
  const MaxRule mr = make_max_rule(sg);
  __shared__ ScaleEntry tab[256];
  fill_scale_table(tab, sg);
  double acc = 0.0;
  for (; i < nblk; i += stride) {
    uint32_t nv[8];
    const int64_t n = i + stride;
    if (n < nblk) load_block(x + n * kBlock, nv);
    const float amax = __uint_as_float(amax_bits8(v) << 16);
    const ScaleEntry se = tab[max_rule_code_fast(amax, mr)];
    const uint2 q = encode_block_entry(v, se);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t y = dequant_byte(((j < 4 ? q.x : q.y) >> (8 * (j & 3))) & 0xFFu, se.s);
      const double d0 = (double)bf16_lo(v[j]) - (double)bf16_lo(y);
      const double d1 = (double)bf16_hi(v[j]) - (double)bf16_hi(y);
      acc += d0 * d0 + d1 * d1;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = nv[j];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  __shared__ double warp_sum[kThreads / 32];
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) t += warp_sum[w];
    partial[blockIdx.x] = t;
  }
}

__global__ void error_reduce_kernel(const double *__restrict__ partial, int n,
                                    double *__restrict__ out) {
  chained_entry();
  double t = 0.0;
  for (int i = 0; i < n; ++i) t += partial[i];
  *out = t;
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

// CTAs per batch element for a kernel whose CTAs pay a set-up (a scale
// table, fp64 reciprocals) before their blocks: up to eight blocks per
// thread, so that the set-up is amortised, but never fewer than four waves
// of resident CTAs (`resident` per SM) across the whole batch, which keeps
// the tail short.
int amortised_grid(int64_t batch, int64_t nblk, int resident) {
  const int64_t need = (nblk + kThreads - 1) / kThreads;  // one block per thread
  const int64_t by_work = (batch * nblk + 8 * kThreads - 1) / (8 * kThreads);
  const int64_t by_waves = std::min(batch * need, (int64_t)sm_count() * resident * 4);
  const int64_t total = std::max(by_work, by_waves);
  return (int)std::min(std::min(need, (total + batch - 1) / batch), (int64_t)1 << 30);
}

cudaError_t launch_global_scale(const uint16_t *x, int64_t batch, int64_t n_per_batch,
                                float *s_g, cudaStream_t st) {
  // the maxima are accumulated by atomicMax from zero (a kernel rather than a
  // memset, so that the launches stay chained)
  cudaError_t e = launch_first(zero_words_kernel, dim3((unsigned)((batch + 127) / 128)),
                                 dim3(128), 0, st, reinterpret_cast<uint32_t *>(s_g), batch);
  if (e != cudaSuccess) return e;
  if (n_per_batch > 0) {
    const int64_t nv = n_per_batch / 8;
    int gx = grid_for(nv / 4 + 1, 8);
    const int64_t per_batch_cap = ((int64_t)sm_count() * 8 + batch - 1) / batch;
    if (gx > per_batch_cap) gx = (int)(per_batch_cap > 0 ? per_batch_cap : 1);
    e = launch_chained(amax_kernel, dim3(gx, (unsigned)batch), dim3(kThreads), 0, st, x,
                       n_per_batch, reinterpret_cast<uint32_t *>(s_g));
    if (e != cudaSuccess) return e;
  }
  return launch_chained(global_scale_finish_kernel, dim3((unsigned)((batch + 127) / 128)),
                        dim3(128), 0, st, s_g, batch);
}

cudaError_t launch_scale_max(const uint16_t *w, int64_t batch, int64_t nblk, const float *s_g,
                             uint8_t *codes, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  int gx = grid_for(nblk, 16);
  return launch_first(max_rule_kernel, dim3(gx, (unsigned)batch), dim3(kThreads), 0, st, w,
                        nblk, s_g, codes);
}

cudaError_t launch_four_over_six(const uint16_t *w, int64_t batch, int64_t nblk,
                                 const float *s_g, uint8_t *codes, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  const int gx = amortised_grid(batch, nblk, 3);  // 78 registers: three CTAs per SM
  return launch_first(four_over_six_kernel, dim3(gx, (unsigned)batch), dim3(kThreads), 0, st,
                        w, nblk, s_g, codes);
}

cudaError_t launch_pack(const uint16_t *w, int64_t batch, int64_t nblk, const float *s_g,
                        const uint8_t *codes, uint8_t *packed, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  const int gx = amortised_grid(batch, nblk, 5);
  return launch_first(pack_kernel, dim3(gx, (unsigned)batch), dim3(kThreads), 0, st, w, nblk,
                        s_g, codes, packed);
}

cudaError_t launch_dequant(const uint8_t *packed, const uint8_t *codes, const float *s_g,
                           int64_t batch, int64_t nblk, uint16_t *out, cudaStream_t st) {
  if (nblk == 0) return cudaSuccess;
  int gx = grid_for(nblk, 16);
  return launch_first(dequant_kernel, dim3(gx, (unsigned)batch), dim3(kThreads), 0, st, packed,
                        codes, s_g, nblk, out);
}

cudaError_t launch_fake_quant(const uint16_t *x, int64_t rows, int64_t C, uint16_t *out,
                              uint8_t *packed, uint8_t *codes, float *s_g, cudaStream_t st) {
  const int64_t n = rows * C;
  cudaError_t e = launch_global_scale(x, 1, n, s_g, st);
  if (e != cudaSuccess || n == 0) return e;
  const int64_t nblk = n / kBlock;
  int gx = grid_for(nblk, 16);
  return launch_chained(fake_quant_kernel, dim3(gx), dim3(kThreads), 0, st, x, nblk,
                        static_cast<const float *>(s_g), out, packed, codes);
}

cudaError_t launch_fake_quant_static(const uint16_t *x, int64_t rows, int64_t C, const float *s_g,
                                     uint16_t *out, uint8_t *packed, uint8_t *codes,
                                     cudaStream_t st) {
  const int64_t nblk = rows * C / kBlock;
  if (nblk == 0) return cudaSuccess;
  const int gx = grid_for(nblk, 16);
  return launch_first(fake_quant_kernel, dim3(gx), dim3(kThreads), 0, st, x, nblk, s_g, out,
                        packed, codes);
}

cudaError_t launch_quant_error(const uint16_t *x, int64_t rows, int64_t C, const float *s_g,
                               double *err, cudaStream_t st) {
  const int64_t nblk = rows * C / kBlock;
  if (nblk == 0) return cudaMemsetAsync(err, 0, sizeof(double), st);
  const int gx = grid_for(nblk, 8);
  double *partial = nullptr;
  cudaError_t e = scratch_alloc(reinterpret_cast<void **>(&partial), sizeof(double) * gx, st);
  if (e != cudaSuccess) return e;
  e = launch_first(quant_error_kernel, dim3(gx), dim3(kThreads), 0, st, x, nblk, s_g, partial);
  if (e == cudaSuccess)
    e = launch_chained(error_reduce_kernel, dim3(1), dim3(1), 0, st,
                       static_cast<const double *>(partial), gx, err);
  const cudaError_t ef = scratch_free(partial, st);
  return e != cudaSuccess ? e : ef;
}

cudaError_t read_and_clear_device_status(cudaStream_t st, int *out) {
  int zero = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(out, g_device_status, sizeof(int));
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return e;
  // the Gram kernels keep their own flag (a timed-out wait), the
  // calibration kernels theirs (a quantile on a non-finite value), the GPTQ
  // kernels theirs (a Hessian that is not positive definite)
  int gram = 0, calib = 0, gptq = 0;
  e = read_and_clear_gram_status(st, &gram);
  if (e == cudaSuccess) e = read_and_clear_calib_status(st, &calib);
  if (e == cudaSuccess) e = read_and_clear_gptq_status(st, &gptq);
  if (*out == 0) *out = gram ? gram : (calib ? calib : gptq);
  return e;
}

}  // namespace nvfp4
