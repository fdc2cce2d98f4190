// Device helpers shared by the NVFP4 kernels: format conversions and the
// exact E2M1 / E4M3 rounding decisions.
//
// Formats ([BT] = Baseten, "What makes high-quality NVFP4", section "Why do
// we need scales?"; [LH] = the Local-Hessian write-up, section "The NVFP4
// structure"):
//   E2M1: sign<<3 | k, magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}[k].
//   E4M3 (FN): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, subnormals
//   m * 2^-9, largest finite 448 (code 0x7E).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace nvfp4 {

constexpr int kBlock = 16;        // values per block
constexpr int kCandidates = 126;  // positive finite non-zero E4M3 codes 0x01..0x7E

// ------------------------------------------------------------- bf16 / fp32
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// E4M3 code -> fp32 value (exact).  Codes 0x01..0x07 are subnormal.
__device__ __forceinline__ float e4m3_to_float(uint32_t c) {
  c &= 0x7Fu;
  if (c < 8u) return (float)c * 0.001953125f;  // m * 2^-9, exact
  // normal: exponent field e = c >> 3, value (8 + m) * 2^(e - 10); fp32 bits:
  // biased exponent e + 120, mantissa m << 20  ==  (c << 20) + (120 << 23)
  return __uint_as_float((c << 20) + (120u << 23));
}

// ---------------------------------------------------------- hardware cvt
// One byte of two E2M1 codes -> f16x2 (low nibble in the low half).
__device__ __forceinline__ uint32_t cvt_f16x2_from_e2m1x2(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "mov.b32 {q0, q1, q2, q3}, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, q0;\n\t}"
      : "=r"(r) : "r"(byte));
  return r;
}

__device__ __forceinline__ float f16_lo_to_float(uint32_t h2) {
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}
__device__ __forceinline__ float f16_hi_to_float(uint32_t h2) {
  return __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}

// ------------------------------------------------------ exact E2M1 encode
// Magnitude index k of |x| / s on the exact real line (s > 0), by the sign of
// |x| - mu * s computed in fp64 (exact: |x| has 24 bits at most, mu * s 27).
// Ties go to the even index: up across midpoint i on "greater" when i is
// even, on "greater or equal" when i is odd.
__device__ __forceinline__ uint32_t e2m1_mag_exact(float a, float s) {
  if (!(s > 0.0f)) return 0u;
  const double da = (double)a, ds = (double)s;
  uint32_t k = 0;
  k += (da > 0.25 * ds);
  k += (da >= 0.75 * ds);
  k += (da > 1.25 * ds);
  k += (da >= 1.75 * ds);
  k += (da > 2.5 * ds);
  k += (da >= 3.5 * ds);
  k += (da > 5.0 * ds);
  return k;
}

// Certificate that plain rounding of a quotient is exact.  For s >= 2^-100
// finite and every bf16 value x, t = fl(x (r_hi + r_lo)) with r_hi + r_lo =
// 1/s to about 2^-46 lies within one float of q = x / s.  Hardware
// round-to-nearest-even of t can then differ from that of q only if an E2M1
// rounding midpoint (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5: at most three
// significant bits), times a power of two, lies within one float of q.  x
// has at most 8 significant bits, so q = x / s sits within relative 2^-21 of
// m 2^k (m = 1, 3, 5, 7) only if m s sits within relative 2^-21 of a number
// with 8 significant bits.  Returns true when that holds for no m: no value
// at scale s comes near a midpoint.  m s is exact in fp64; its significand
// bits below the eighth must stay more than 2^-20 (in units of the leading
// bit, i.e. 2^32 units of 2^-52) away from 0 and from 1.
__device__ __forceinline__ bool quotients_far_from_midpoints(float s) {
  bool far = true;
#pragma unroll
  for (int m = 1; m <= 7; m += 2) {
    const double p = (double)s * (double)m;
    const unsigned long long rem =
        (unsigned long long)__double_as_longlong(p) & ((1ull << 45) - 1ull);
    far = far && rem > (1ull << 32) && rem < (1ull << 45) - (1ull << 32);
  }
  return far;
}

__device__ __forceinline__ float effective_scale(float s_g, uint32_t code) {
  return __fmul_rn(s_g, e4m3_to_float(code));
}

// Largest |x| of 8 packed bf16 pairs (sign bits masked, bf16 magnitudes order
// like unsigned integers).
__device__ __forceinline__ uint32_t amax_bits8(const uint32_t w[8]) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = __vmaxu2(m, w[i] & 0x7FFF7FFFu);
  return max(m & 0xFFFFu, m >> 16);
}

}  // namespace nvfp4

namespace nvfp4 {
// Streaming 128-bit global accesses: inputs are read once (no L1 allocation),
// outputs are written once (evict-first).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ void st_stream_v4(void *p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};"
               :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ void st_stream_v2(void *p, uint2 v) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" :: "l"(p), "r"(v.x), "r"(v.y) : "memory");
}
}  // namespace nvfp4
