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
// Two fp32 -> two E2M1 codes in one byte (round to nearest even, saturating
// at +-6).  `hi` lands in bits 7..4, `lo` in bits 3..0.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %1, %2;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r & 0xFFu;
}

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

// Reciprocal bracket of a scale: r_lo <= 1/s <= r_hi.
struct ScaleRecip {
  float s, r_lo, r_hi;
};

__device__ __forceinline__ ScaleRecip make_recip(float s) {
  ScaleRecip r;
  r.s = s;
  r.r_lo = __frcp_rd(s);
  r.r_hi = __frcp_ru(s);
  return r;
}

// Packed magnitude codes of 2 elements (a0 -> low nibble, a1 -> high) from
// the reciprocal bracket: t_lo <= |x|/s <= t_hi elementwise, rounding is
// monotone, so equal codes at both ends are the exact answer.  `mismatch`
// accumulates any disagreement (then the caller redoes the block exactly).
__device__ __forceinline__ uint32_t e2m1_pair_bracket(float a0, float a1, const ScaleRecip &r,
                                                      uint32_t &mismatch) {
  uint32_t lo = cvt_e2m1x2(__fmul_rd(a1, r.r_lo), __fmul_rd(a0, r.r_lo));
  uint32_t hi = cvt_e2m1x2(__fmul_ru(a1, r.r_hi), __fmul_ru(a0, r.r_hi));
  mismatch |= lo ^ hi;
  return lo;
}

// ------------------------------------------------------ exact E4M3 round
// E4M3 code (0..126) of num / den rounded to nearest even, saturating at 448,
// for num >= 0, den > 0 given as fp64 values whose exact quotient is at
// least 2^-32 (relative) away from every E4M3 midpoint unless equal to it
// (true for num a bf16 value and den = 6 * s_g, s_g an fp32 value).  The
// fp64 quotient then sits on the same side of every midpoint as the exact
// one, and the rounding below is exact arithmetic on it.
__device__ __forceinline__ uint32_t e4m3_round_quotient(double num, double den) {
  double q = __ddiv_rn(num, den);
  if (!(q < 448.0)) return 0x7Eu;            // saturate (also catches +inf)
  if (q < 0.015625) {                        // below 2^-6: subnormal grid m * 2^-9
    return (uint32_t)rint(q * 512.0);        // 0..8; 8 is the first normal code
  }
  int e;
  double m = frexp(q, &e);                   // q = m * 2^e, m in [0.5, 1)
  // q = (1 + f/8) * 2^(e-1) with f = (2m - 1) * 8 in [0, 8); round f to even
  double f = rint((2.0 * m - 1.0) * 8.0);    // 0..8, 8 carries into the exponent
  uint32_t code = (uint32_t)(((e - 1 + 7) << 3) + (int)f);
  return code > 0x7Eu ? 0x7Eu : code;
}

// Max rule: code of block amax a_max given s_g (exact decision).
__device__ __forceinline__ uint32_t max_rule_code(float a_max, float s_g) {
  if (a_max == 0.0f) return 0u;
  return e4m3_round_quotient((double)a_max, 6.0 * (double)s_g);
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
