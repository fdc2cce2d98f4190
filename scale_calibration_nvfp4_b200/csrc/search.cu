// Exhaustive block-scale search over the 126 positive finite non-zero E4M3
// codes: MSE objective and Local-Hessian objective.
//
// Method: the Local-Hessian write-up "4 比特量化到底让模型笨了多少？" (of NVIDIA
// Model Optimizer's "Improving NVFP4 Accuracy with Local-Hessian Weight
// Scales"): section "The NVFP4 structure" (MSE tries all 126 scales and keeps
// the smallest weight error) and section "A different objective" (E(s) =
// ||delta X||^2 = tr(delta X X^T delta^T); the block-diagonal approximation
// solves each 16-value block alone against its 16x16 H_b, still trying all
// 126 candidates).  MSE is the same search with H_b = I.
//
// Work mapping.  A CTA owns one column block b of one batch element and a run
// of rows; a warp takes 16 rows at a time, laid out like the A operand of a
// 16x8x16 tensor-core MMA: lane (g, t) holds elements {2t, 2t+1, 2t+8, 2t+9}
// of rows g and g+8.
//
// Per candidate scale s the objective is rewritten with H_b = L L^T (fp64
// Cholesky once per column block, in factor_kernel; semidefinite pivots
// dropped):
//     E = ||L^T delta||^2,  delta = w - s v,   so   L^T delta = p - s u,
// with p = L^T w fixed per row and u = L^T v.  The signed E2M1 values v are
// exact in f16, so u comes from two f16 MMAs per 8 outputs against L split
// into an f16 high and low part (22 significant bits), accumulated in fp32;
// for MSE the B operand is the identity and u = v exactly.  The CUDA cores
// only form z = p - s u and sum z^2.
//
// Exact E2M1 codes without a fallback branch.  Candidate values are o * 2^p
// with odd o in {1, 3, ..., 15}, and s(c) = fl(s_g o) 2^p exactly, so for each
// element and each odd part o the signed quotient q = w / fl(s_g o) is formed
// once, as t from a double-float reciprocal: t is one of the two floats
// around q.  Candidates of class o scale t by 2^-p exactly.  Every rounding
// midpoint of E2M1 is a float with at most 3 significant bits, so a t with
// more bits is no midpoint at any scale of the class, and its hardware
// round-to-nearest-even gives q's code.  A t with at most 3 significant bits
// moves once per class towards q by one fma, t + rho 16 / fl(s_g o) with the
// exact residual rho = w - t fl(s_g o): a non-zero residual of such a t puts
// the moved value between one float and 2^-19 |q| from t on q's side, off
// the midpoint and short of any other decision; a zero residual (of either
// sign) leaves t.  Classes whose S passes quotients_far_from_midpoints (no
// bf16 value comes near a midpoint) skip that step.
//
// Winner: fp32 screen keeping the best three objectives; the candidates that
// the screen's error bound cannot separate are re-scored in fp64 straight
// from the definition (delta H_b delta^T with exact E2M1 codes, one element
// per lane, two candidates per warp pass) and the first minimum in ascending
// code order wins.
//
// Screen error (Local-Hessian; all quantities in the screen's units, each row
// scaled by its 2^kw and L by sigma).  The screen forms z = p - s u from two
// tensor-core products whose errors do not shrink with z: with
// a_j = sum_i |W_i| |sigma L_ij| and A = ||a||_2,
//   - the f16 high/low split of sigma L errs by 2^-22 |sigma L| + 2^-25 per
//     entry, the fp32 rounding of the fp64 factor by 2^-24 |L|;
//   - one m16n8k16 MMA with fp32 accumulation errs by at most
//     kappa (sum |a_k b_k| + |c|), kappa = 2^-18 (products exact, addends
//     aligned to the largest with 24 bits kept, truncated or rounded: at
//     most 17 ulps of the largest, 2^-18.9; the assumption is checked on the
//     device by the test suite);
//   - |s v_i| <= 2 |W_i| (E2M1 rounds a quotient up by at most a factor 2)
//     and |delta_i| <= 3 |W_i|.
// So every z_j is off by at most (6.006 kappa + 2^-20) a_j + 2^-4, and with
// D = ||that||_2 <= kAccErr A + kAbsErr and F the dropped-pivot part
// (||H - L L^T||_inf ||delta||^2), the screen objective b and the exact E
// satisfy |b - E| <= 2 Q sqrt(b) + 6 Q^2 + 2^-17 b, Q = D + sqrt(F).  A
// block is re-scored when its best two are within kTieBand b2 + 4 Q
// sqrt(b2) + 12 Q^2 (both errors), and with all 126 candidates when the
// third is too; the pruning bounds keep 2 kTieBand b1 + 4102 Q^2 to spare
// (2 Q sqrt(b1) <= 2^12 Q^2 + 2^-12 b1).  For MSE, u = v and p = W exactly
// and only the relative error of the sums is left (Q = 0).
#include <cuda_fp16.h>

#include "chained.cuh"
#include "common.cuh"
#include "internal.h"

namespace nvfp4 {

// Statistics of the work the searches do since the last reset; nothing reads
// them on the device.  [0] MSE and [1] Local-Hessian (block, candidate)
// objective evaluations of the fp32 screen; rows re-scored in fp64 over their
// best two candidates ([2] MSE, [4] Local-Hessian) and over all 126 ([3] MSE,
// [5] Local-Hessian).
__device__ unsigned long long g_search_evals[6];

namespace {

constexpr int kThreads = 128;  // 4 warps
constexpr int kWarps = kThreads / 32;
constexpr int kTileRows = 16;
// Rows per CTA: 256 (four 16-row tiles per warp), or 128 when a problem has
// few CTAs (the tail of the last wave then costs less).
constexpr int kRowsLarge = kWarps * kTileRows * 4, kRowsSmall = kWarps * kTileRows * 2;
constexpr float kTieBand = 1.0f / 4096.0f;
// Absolute part of the band and of the pruning margins: where terms or
// partial sums fall into the fp32 subnormal range (elements far below their
// row's largest; every row itself is scaled into [2^14, 2^15)), each
// operation errs by up to 2^-150 and a key moves by up to 127 * 2^-149, far
// below this; elsewhere it changes nothing.
constexpr float kAbsBand = 0x1p-130f;
constexpr float kZeroFloor = 0x1p-40f;  // relative to ||p||^2
// Absolute screen error per row (Local-Hessian): D <= kAccErr A + kAbsErr,
// A from the product of |W| with the high part of |sigma L| (positive terms:
// the 2^-9 inflation covers its own accumulation and the low part).
constexpr float kAccErr = 0x1.ap-16f * (1.0f + 0x1p-9f);  // 6.5 kappa, kappa = 2^-18
constexpr float kAbsErr = 0.5f;  // the split's 2^-25 floor, at most 0.25 in these units
constexpr int kMaxClasses = kCandidates;

// Candidate classes by odd part o of the E4M3 value o * 2^p (p >= -9):
// start of each class (o = 1, 3, ..., 15) in candidate order.
__constant__ int kClassBegin[9] = {0, 18, 35, 51, 67, 82, 97, 112, 126};

struct ClassInfo {
  float S, r_hi, r_lo;  // S = fl(s_g o), 1/S = r_hi + r_lo
  int end;              // one past its last candidate
  int certified;        // no quotient |w| / S comes near a rounding midpoint
};
struct CandInfo {
  float f;      // 2^-p, scales the class quotient to this candidate
  float pad;
  float s;      // effective scale fl(s_g e4m3(c))
  int c;        // E4M3 code
};

// ----------------------------------------------------------------- helpers
__device__ __forceinline__ void mma_f16_16816(float d[4], const uint32_t a[4], uint32_t b0,
                                              uint32_t b1, const float c[4]) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
        "f"(c[2]), "f"(c[3]));
}

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// The factor kernel works on two 16x16 blocks per warp: the lanes of each
// half (16 lanes) own one row each of their block, and every shuffle and
// reduction below stays inside the half.
constexpr unsigned kFull = 0xFFFFFFFFu;

// Cooperative Cholesky of the 16x16 block in Hs (fp32, row-major) by one
// half-warp, lane r owning row r.  A pivot at or below 1e-12 of the largest
// diagonal (or non-finite) drops its column, which keeps a positive
// semidefinite H usable.  Writes the full lower-triangular factor (zeros above
// the diagonal) to Lf (fp32) and Ld (fp64).
__device__ void cholesky16(const float *Hs, float *Lf, double *Ld) {
  const int r = threadIdx.x & 15;
  double a[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) a[j] = (double)Hs[r * 16 + j];
  double diag = 0.0;
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (j == r) diag = a[j];
  double maxdiag = diag;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) maxdiag = fmax(maxdiag, __shfl_xor_sync(kFull, maxdiag, o));
  const double tol = 1e-12 * maxdiag;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const double akk = __shfl_sync(kFull, a[k], k, 16);
    const bool ok = (akk > tol) && (akk < 1e300);
    const double piv = ok ? sqrt(akk) : 0.0;
    double lik = 0.0;
    if (r == k) lik = piv;
    else if (r > k && ok) lik = a[k] / piv;
    Lf[r * 16 + k] = (float)lik;  // zero above the diagonal
    Ld[r * 16 + k] = lik;
#pragma unroll
    for (int j = k + 1; j < 16; ++j) {
      const double ljk = __shfl_sync(kFull, lik, j, 16);
      a[j] = fma(-lik, ljk, a[j]);
    }
  }
}

// Lower bound of the smallest eigenvalue of L L^T, computed by one half-warp
// and returned to each of its lanes: 0.98 / ||(L L^T)^-1||_1.  For a
// symmetric matrix the column-sum norm bounds the 2-norm from above, so this
// bounds lambda_min from below (with 2% to spare for rounding).  Lane r forms
// column r of the inverse by a forward and a backward triangular solve in
// fp64.  A dropped pivot (zero diagonal in L) makes the matrix singular: the
// bound is 0 (no pruning).  So it is too when max diag(L L^T)
// ||(L L^T)^-1||_1 exceeds 10^4: L L^T differs from H by at most 2^-23
// trace(H) <= 2^-19 max diag(H) (fp32 rounding of the factor), which then
// stays below 2% of lambda_min.  The same sweeps give the diagonal of the
// inverse: cdiag[r] = 0.97 / ((L L^T)^-1)_rr (0 where lambda is), a lower
// bound of min { x^T H x : x_r = 1 } = 1 / (H^-1)_rr under the same
// condition (the diagonal entry moves by at most 1.9% relative).
__device__ __forceinline__ float lambda_lower_bound(const float *Lf, double *inv_d,
                                                   float *cdiag) {
  const int lane = threadIdx.x & 31, r = lane & 15;
  // 1 / L_kk and the largest diagonal entry of L L^T (lane r: row r)
  double maxdiag = 0.0;
  const double d = (double)Lf[r * 16 + r];
  inv_d[r] = 1.0 / d;
#pragma unroll
  for (int m = 0; m < 16; ++m) maxdiag = fma((double)Lf[r * 16 + m], (double)Lf[r * 16 + m], maxdiag);
  const bool singular = (__ballot_sync(kFull, d == 0.0) >> (lane & 16)) & 0xFFFFu;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) maxdiag = fmax(maxdiag, __shfl_xor_sync(kFull, maxdiag, o));
  __syncwarp();
  double colsum = 0.0, dinv = 0.0;
  if (!singular) {
    // column sweeps: acc = e_r, then L y = acc, then L^T z = y (in place;
    // fully unrolled, so acc stays in registers; the factor is read through a
    // volatile pointer so its loads stay in program order and are not all
    // hoisted into registers)
    const volatile float *Lv = Lf;
    double acc[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) acc[m] = (m == r) ? 1.0 : 0.0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      acc[k] *= inv_d[k];
#pragma unroll
      for (int m = k + 1; m < 16; ++m) acc[m] = fma(-(double)Lv[m * 16 + k], acc[k], acc[m]);
    }
#pragma unroll
    for (int k = 15; k >= 0; --k) {
      acc[k] *= inv_d[k];
      colsum += fabs(acc[k]);
#pragma unroll
      for (int m = 0; m < k; ++m) acc[m] = fma(-(double)Lv[k * 16 + m], acc[k], acc[m]);
    }
#pragma unroll
    for (int m = 0; m < 16; ++m)
      if (m == r) dinv = acc[m];  // ((L L^T)^-1)_rr
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) colsum = fmax(colsum, __shfl_xor_sync(kFull, colsum, o));
  const bool valid = !singular && colsum > 0.0 && colsum < 1e300 && maxdiag * colsum <= 1e4;
  cdiag[r] = valid && dinv > 0.0 ? (float)(0.97 / dinv) : 0.0f;
  return valid ? (float)(0.98 / colsum) : 0.0f;
}

// fp64 objective of one candidate from the definition, computed by a
// half-warp: lane l holds element j = l & 15 of the block (value x) and the
// lanes of each half score their own candidate c.  Exact E2M1 codes,
// delta_j = x_j - v_j s, row_j = sum_k H_jk delta_k, E = sum_j delta_j row_j
// (MSE: H = I); every lane of the half returns the same E.
__device__ __noinline__ double objective64_half(float x, float s_g, int c, const float *Hs) {
  const int lane = threadIdx.x & 31, j = lane & 15, half = lane & 16;
  const float s = effective_scale(s_g, (uint32_t)c);
  const uint32_t k = e2m1_mag_exact(fabsf(x), s);
  const double v = k < 2 ? 0.5 * k : (1.0 + 0.5 * (double)(k & 1)) * (double)(1 << ((k >> 1) - 1));
  const double d = (double)x - copysign(v, (double)x) * (double)s;
  double row = d;
  if (Hs) {
    row = 0.0;
#pragma unroll 4
    for (int m = 0; m < 16; ++m)
      row = fma((double)Hs[j * 16 + m], __shfl_sync(0xFFFFFFFFu, d, half | m), row);
  }
  double e = d * row;
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) e += __shfl_xor_sync(0xFFFFFFFFu, e, o);
  return e;
}

// Near-tie resolution for one block by the whole warp: fp64 scores of
// {c1, c2}, or of every candidate (two per pass) when more than two may lie
// in the band; the first minimum in ascending code order wins.  Every lane
// returns the result.
__device__ __noinline__ int refine_block(const uint16_t *wrow, float s_g, const float *Hs,
                                         int c1, int c2, bool full, float *obj) {
  const int lane = threadIdx.x & 31;
  // the work statistic: one more row re-scored (over the best two or over
  // every candidate), for this rule
  if (lane == 0) atomicAdd(&g_search_evals[(Hs ? 4 : 2) + (full ? 1 : 0)], 1ull);
  const float x = __uint_as_float((uint32_t)wrow[lane & 15] << 16);
  double best = __longlong_as_double(0x7FF0000000000000LL);
  int best_c = 1;
  if (full) {
#pragma unroll 1
    for (int c = 1; c < kCandidates; c += 2) {
      const double e = objective64_half(x, s_g, c + (lane >> 4), Hs);
      const double ea = __shfl_sync(0xFFFFFFFFu, e, 0), eb = __shfl_sync(0xFFFFFFFFu, e, 16);
      if (ea < best) {
        best = ea;
        best_c = c;
      }
      if (eb < best) {
        best = eb;
        best_c = c + 1;
      }
    }
  } else {
    const int lo = min(c1, c2), hi = max(c1, c2);
    const double e = objective64_half(x, s_g, lane < 16 ? lo : hi, Hs);
    const double el = __shfl_sync(0xFFFFFFFFu, e, 0), eh = __shfl_sync(0xFFFFFFFFu, e, 16);
    best = el;
    best_c = lo;
    if (eh < el) {
      best = eh;
      best_c = hi;
    }
  }
  *obj = (float)best;
  return best_c;
}

// An upper bound of sqrt(x) for x >= 0 from the hardware approximation
// (relative error far below 2^-16, so the 2^-16 inflation keeps it above the
// exact root; only bounds are formed with it).
__device__ __forceinline__ float sqrt_up(float x) {
  float r;
  asm("sqrt.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r * (1.0f + 0x1p-16f);
}

// Objective and code in one sortable value: a non-negative float whose seven
// lowest mantissa bits are replaced by the code (relative change below
// 2^-16, far inside the re-score band); equal objectives order by code.
__device__ __forceinline__ float key_of(float e, int c) {
  return __int_as_float((__float_as_int(e) & ~0x7F) | c);
}
__device__ __forceinline__ int code_of(float key) { return __float_as_int(key) & 0x7F; }

// Keep the three smallest keys.
__device__ __forceinline__ void track3(float key, float &b1, float &b2, float &b3) {
  b3 = fminf(b3, fmaxf(b2, key));
  b2 = fminf(b2, fmaxf(b1, key));
  b1 = fminf(b1, key);
}

// Four signed pairs rounded to E2M1 (nearest even, saturating; a negative
// value that rounds to zero gives -0) and decoded to f16x2 in one asm block:
// A[i] holds (lo_i, hi_i), the MMA's A fragment, with no packing of the codes
// in between.
__device__ __forceinline__ void round_decode4(float h0, float l0, float h1, float l1, float h2,
                                              float l2, float h3, float l3, uint32_t A[4]) {
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %4, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %6, %7;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %8, %9;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %10, %11;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, q0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, q1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, q2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, q3;\n\t}"
      : "=r"(A[0]), "=r"(A[1]), "=r"(A[2]), "=r"(A[3])
      : "f"(h0), "f"(l0), "f"(h1), "f"(l1), "f"(h2), "f"(l2), "f"(h3), "f"(l3));
}

// Select word t (0..3) of four without local memory.
__device__ __forceinline__ uint32_t pick4(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                          int t) {
  return t == 0 ? w0 : (t == 1 ? w1 : (t == 2 ? w2 : w3));
}

// One candidate: codes, the tensor-core product u, z = p - s u, and the row
// objective after a quad reduce-scatter (lanes t < 2: row g, t >= 2: row
// g + 8).  tq holds the signed class quotients (moved off a possible
// midpoint where one could occur), f scales them to this candidate exactly;
// sm0 and sm1 multiply u in rows g and g + 8 (accumulator elements 0, 1 and
// 2, 3 of both n-tiles), each row carrying its own power-of-two scale.
template <bool kLH>
__device__ __forceinline__ float candidate_objective(const float tq[8], float f, float sm0,
                                                     float sm1, const uint32_t bh[2][2],
                                                     const uint32_t bl[2][2],
                                                     const float pz[2][4], bool upper) {
  const float zero4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  // paired fp32 arithmetic (two independent lanes per instruction, each
  // rounded as its scalar form)
  const float2 ff = make_float2(f, f);
  const float2 q0 = __fmul2_rn(make_float2(tq[0], tq[1]), ff);
  const float2 q1 = __fmul2_rn(make_float2(tq[2], tq[3]), ff);
  const float2 q2 = __fmul2_rn(make_float2(tq[4], tq[5]), ff);
  const float2 q3 = __fmul2_rn(make_float2(tq[6], tq[7]), ff);
  uint32_t A[4];
  round_decode4(q0.y, q0.x, q1.y, q1.x, q2.y, q2.x, q3.y, q3.x, A);
  float u0[4], u1[4];
  mma_f16_16816(u0, A, bh[0][0], bh[0][1], zero4);
  mma_f16_16816(u1, A, bh[1][0], bh[1][1], zero4);
  if (kLH) {
    mma_f16_16816(u0, A, bl[0][0], bl[0][1], u0);
    mma_f16_16816(u1, A, bl[1][0], bl[1][1], u1);
  }
  // z = p - s u: row g in accumulator elements 0, 1, row g + 8 in 2, 3
  const float2 n0 = make_float2(-sm0, -sm0), n1 = make_float2(-sm1, -sm1);
  const float2 za = __ffma2_rn(make_float2(u0[0], u0[1]), n0, make_float2(pz[0][0], pz[0][1]));
  const float2 zb = __ffma2_rn(make_float2(u0[2], u0[3]), n1, make_float2(pz[0][2], pz[0][3]));
  const float2 zc = __ffma2_rn(make_float2(u1[0], u1[1]), n0, make_float2(pz[1][0], pz[1][1]));
  const float2 zd = __ffma2_rn(make_float2(u1[2], u1[3]), n1, make_float2(pz[1][2], pz[1][3]));
  const float2 ea = __ffma2_rn(zc, zc, __fmul2_rn(za, za));  // row g
  const float2 eb = __ffma2_rn(zd, zd, __fmul2_rn(zb, zb));  // row g + 8
  const float e0 = ea.x + ea.y, e1 = eb.x + eb.y;
  // the same sums in the same order on both lanes of a pair
  float mine = upper ? e1 : e0;
  const float other = upper ? e0 : e1;
  mine += __shfl_xor_sync(0xFFFFFFFFu, other, 2);
  mine += __shfl_xor_sync(0xFFFFFFFFu, mine, 1);
  return mine;
}

// Per column block (and batch element) of H, from factor_kernel: the f16
// high/low B-operand fragments of sigma L for every lane, sigma, the pruning
// bounds' factors, the dropped-pivot residual and the zero-H flag.
struct Factor {
  float sigma;   // power of two putting max |L| in [2^14, 2^15)
  float sl2;     // sigma^2 lambda, lambda a lower bound of lambda_min(L L^T) (0 when unknown)
  int zero;      // H_b == 0 (every candidate scores 0)
  float rsq;     // 12 sqrt(sigma^2 ||H - L L^T||_inf), rounded up; inf if unknown
  float cs[16];  // sigma^2 times lower bounds of 1 / (H^-1)_rr (0 where lambda is 0)
};

// A bound of ||H - Ld Ld^T||_inf by one half-warp, returned to each lane of
// the half: 2^-40 max diag(H) covers the rounding of the fp64 factor (its
// backward error is below 16 * 17 * 2^-53 max diag(H)) and of this sum;
// where a pivot was dropped (`dropped`: the half's factor has a zero on the
// diagonal) the residual itself is added, lane r summing row r.
__device__ __forceinline__ double factor_residual(const float *Hs, const double *Ld,
                                                  bool dropped) {
  const int r = threadIdx.x & 15;
  double rs = 0.0, dg = (double)Hs[r * 16 + r];
  if (dropped) {
#pragma unroll 1
    for (int j = 0; j < 16; ++j) {
      double x = (double)Hs[r * 16 + j];
#pragma unroll
      for (int k = 0; k < 16; ++k) x = fma(-Ld[r * 16 + k], Ld[j * 16 + k], x);
      rs += fabs(x);
    }
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {
    rs = fmax(rs, __shfl_xor_sync(kFull, rs, o));
    dg = fmax(dg, __shfl_xor_sync(kFull, dg, o));
  }
  return rs + 0x1p-40 * dg;
}

// Two column blocks of H per warp (half h of the lanes takes block 2 x + h of
// batch element y; an odd last block leaves half 1 with zeros and nothing to
// write).
__global__ void __launch_bounds__(32)
    factor_kernel(const float *__restrict__ H, int64_t nb, uint4 *__restrict__ frag,
                  Factor *__restrict__ fac) {
  chained_entry();
  __shared__ float Hs[2][256];
  __shared__ float Lf[2][256];
  __shared__ double Ld[2][256];
  __shared__ double inv_d[2][16];
  __shared__ float cdiag[2][16];
  const int lane = threadIdx.x, h = lane >> 4, r = lane & 15;
  const int64_t j0 = (int64_t)blockIdx.x * 2;
  const int64_t base = (int64_t)blockIdx.y * nb;  // first block of this batch element
  const bool live = j0 + h < nb;
  const float *Hb = H + (base + j0 + h) * 256;
  for (int i = r; i < 256; i += 16) Hs[h][i] = live ? Hb[i] : 0.0f;
  __syncwarp();
  cholesky16(Hs[h], Lf[h], Ld[h]);
  __syncwarp();
  const bool dropped = (__ballot_sync(kFull, Lf[h][r * 16 + r] == 0.0f) >> (lane & 16)) & 0xFFFFu;
  const double resid = factor_residual(Hs[h], Ld[h], dropped);
  float m = 0.0f;
  for (int i = r; i < 256; i += 16) m = fmaxf(m, fabsf(Lf[h][i]));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
  const float lam = lambda_lower_bound(Lf[h], inv_d[h], cdiag[h]);
  __syncwarp();  // cdiag written by every lane of the half
  int e = 0;
  frexpf(m, &e);  // m < 2^e
  const float sigma = m > 0.0f ? ldexpf(1.0f, 15 - e) : 1.0f;
  if (live && r == 0) {
    // the search's factors in its units (sigma^2 lambda and sigma^2 cdiag
    // stay below 16 * 2^30: lambda, cdiag <= max diag(L L^T) <= 16 max |L|^2)
    Factor f;
    const double s2 = (double)sigma * (double)sigma;
    f.sigma = sigma;
    f.sl2 = __double2float_rd(s2 * (double)lam);
    f.zero = !(m > 0.0f);
    const double rsq = 12.0 * sqrt(resid * s2) * (1.0 + 0x1p-40);  // rounded up below
    f.rsq = rsq < 3.0e38 ? __double2float_ru(rsq) : __int_as_float(0x7F800000);  // NaN too
#pragma unroll
    for (int i = 0; i < 16; ++i) f.cs[i] = __double2float_rd(s2 * (double)cdiag[h][i]);
    fac[base + j0 + h] = f;
  }
  // every lane's fragments of both blocks: B[k][n] = sigma L[k][n], n = 8 nt
  // + g, k = 2t + 8 half + {0, 1}
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int hb = 0; hb < 2; ++hb) {
    const float sg = __shfl_sync(kFull, sigma, 16 * hb);
    if (j0 + hb >= nb) break;
    const float *L = Lf[hb];
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int n = nt * 8 + g;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int k0 = 2 * t + 8 * half;
        const float x0 = L[k0 * 16 + n] * sg, x1 = L[(k0 + 1) * 16 + n] * sg;
        const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
        const __half l0 = __float2half_rn(x0 - __half2float(h0));
        const __half l1 = __float2half_rn(x1 - __half2float(h1));
        hi[nt * 2 + half] = pack_half2(h0, h1);
        lo[nt * 2 + half] = pack_half2(l0, l1);
      }
    }
    const int64_t blk = base + j0 + hb;
    frag[(blk * 32 + lane) * 2] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    frag[(blk * 32 + lane) * 2 + 1] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// Resident CTAs per SM.  Local-Hessian eight (64 registers, 8 bytes of
// spill; measured 1.9% faster on the MoE experts and 1.3% on the dense layer
// than 66 registers at seven); MSE nine (53 registers).
constexpr int kLhCtasPerSm = 8, kMseCtasPerSm = 9;

template <bool kLH, int kRowsPerCta>
__global__ void __launch_bounds__(kThreads, kLH ? kLhCtasPerSm : kMseCtasPerSm)
    search_kernel(const uint16_t *__restrict__ w, int64_t R, int64_t C,
                  const float *__restrict__ s_g_arr, const float *__restrict__ H,
                  const uint4 *__restrict__ frag, const Factor *__restrict__ fac,
                  uint8_t *__restrict__ codes, float *__restrict__ best_obj) {
  static_assert((kRowsPerCta & (kRowsPerCta - 1)) == 0 && kRowsPerCta <= 4096 &&
                    kRowsPerCta % (kWarps * kTileRows) == 0,
                "the row sort needs a power-of-two row count up to 2^12");
  const int64_t nb = C / kBlock;
  const int64_t b = blockIdx.y;
  const int64_t batch = blockIdx.z;
  const int64_t row_base = (int64_t)blockIdx.x * kRowsPerCta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const bool upper = t >= 2;  // which of the lane's two rows it finishes

  __shared__ ClassInfo cls[kMaxClasses];
  __shared__ CandInfo cand[kCandidates];
  __shared__ float cdiag_sh[16];  // bounds of 1 / (H^-1)_rr of this column block
  __shared__ int ncls_sh;
  __shared__ uint4 Ws[kRowsPerCta][2];     // the CTA's 16-element row segments
  __shared__ uint32_t keys[kRowsPerCta];  // amax << 16 | local row, sorted

  // MSE: the call's first kernel (its wait returns at once).  Local-Hessian:
  // chained to this call's factor kernel, which started after all earlier
  // work on the stream had completed and neither reads nor writes W, s_g,
  // codes or best_obj: the rows are loaded and sorted while it finishes, and
  // the wait comes before the first read of its output.
  if constexpr (!kLH) chained_entry(w);
  const float s_g = s_g_arr[batch];
  const uint16_t *wb = w + batch * R * C + b * kBlock;
  uint8_t *cb = codes + batch * R * nb + b;
  float *ob = best_obj ? best_obj + batch * R * nb + b : nullptr;

  // ---- the product's B operand: B = I for MSE here; the Local-Hessian factor
  // of H_b (from factor_kernel) and its zero-H shortcut come after the sort
  const int64_t blk = batch * nb + b;
  const float *Hb = nullptr;  // H_b, the definition, for re-scoring (Local-Hessian)
  float sigma = 1.0f, sl2 = 1.0f;  // MSE: H = I
  float rsq = 0.0f;                // 12 sqrt(sigma^2 ||H - L L^T||_inf) (Local-Hessian)
  uint32_t bh[2][2], bl[2][2];
  if (!kLH) {
    if (threadIdx.x < 16) cdiag_sh[threadIdx.x] = 1.0f;  // H = I
    // B = I: u = v exactly
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int n = nt * 8 + g, k0 = 2 * t + 8 * half;
        bh[nt][half] = pack_half2(__float2half_rn(k0 == n ? 1.0f : 0.0f),
                                  __float2half_rn(k0 + 1 == n ? 1.0f : 0.0f));
        bl[nt][half] = 0u;
      }
  }

  // ---- candidate tables (per CTA, from this batch element's s_g)
  const bool by_class = s_g >= 0x1p-100f && s_g < 0x1p100f;
  if (threadIdx.x < kCandidates) {
    const int c = threadIdx.x + 1;
    const int M = c < 8 ? c : 8 + (c & 7);
    const int E = c < 8 ? -9 : (c >> 3) - 10;
    const int tz = __ffs(M) - 1;
    const int o = M >> tz, p = E + tz;
    const int k = (o - 1) >> 1;
    const float s = effective_scale(s_g, (uint32_t)c);
    const int pos = by_class ? kClassBegin[k] + (p + 9) : c - 1;
    CandInfo ci;
    ci.pad = 0.0f;
    ci.f = by_class ? ldexpf(1.0f, -p) : 1.0f;
    ci.s = s;
    ci.c = c;
    cand[pos] = ci;
    const int ncls = by_class ? 8 : kCandidates;
    if (threadIdx.x < ncls) {
      const float S = by_class ? __fmul_rn(s_g, (float)(2 * threadIdx.x + 1)) : s;
      const double rr = 1.0 / (double)S;
      ClassInfo k2;
      k2.S = S;
      k2.r_hi = (float)rr;
      k2.r_lo = (float)(rr - (double)k2.r_hi);
      k2.end = by_class ? kClassBegin[threadIdx.x + 1] : (int)threadIdx.x + 1;
      k2.certified = S >= 0x1p-100f && S < 0x1p100f && quotients_far_from_midpoints(S);
      cls[threadIdx.x] = k2;
    }
    if (threadIdx.x == 0) ncls_sh = ncls;
  }
  __syncthreads();
  const int ncls = ncls_sh;

  // ---- the CTA's rows, staged in shared memory and ordered by amax so that
  // every warp tile holds rows of similar magnitude: the pruning bounds below
  // then stop the candidate walk at nearly the same point for all 16 rows.
  // Sort key: amax (bf16 magnitude bits, bits 16..31), the position of the
  // row's largest element (bits 12..15) and the local row index (bits
  // 0..11); rows past the end get magnitude 0xFFFF (zero data) and sort last.
  for (int i = threadIdx.x; i < kRowsPerCta; i += kThreads) {
    const int64_t r = row_base + i;
    uint4 a0 = make_uint4(0u, 0u, 0u, 0u), a1 = a0;
    uint32_t key = 0xFFFF0000u | (uint32_t)i;
    if (r < R) {
      const uint4 *q = reinterpret_cast<const uint4 *>(wb + r * C);
      a0 = ld_stream_v4(q);
      a1 = ld_stream_v4(q + 1);
      const uint32_t w8[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      // amax bits, then the position of an element that reaches it (for the
      // row's saturation bound), then the local row
      const uint32_t am = amax_bits8(w8);
      uint32_t pos = 0;  // (the MSE rule's saturation factor is 1 for every position)
      if constexpr (kLH) {
#pragma unroll
        for (int e = 15; e >= 0; --e) {
          const uint32_t mag = ((e & 1) ? (w8[e >> 1] >> 16) : w8[e >> 1]) & 0x7FFFu;
          pos = mag == am ? (uint32_t)e : pos;
        }
      }
      key = (am << 16) | (pos << 12) | (uint32_t)i;
    }
    Ws[i][0] = a0;
    Ws[i][1] = a1;
    keys[i] = key;
  }
  __syncthreads();
  // bitonic sort of the keys, ascending; pair p of a step compares keys i
  // and i + stride with i = 2p - (p mod stride), p < kRowsPerCta / 2
  for (int size = 2; size <= kRowsPerCta; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int p = threadIdx.x; p < kRowsPerCta / 2; p += kThreads) {
        const int i = 2 * p - (p & (stride - 1));
        const int j = i + stride;
        const uint32_t ki = keys[i], kj = keys[j];
        if ((ki > kj) == ((i & size) == 0)) {
          keys[i] = kj;
          keys[j] = ki;
        }
      }
      __syncthreads();
    }
  }

  if constexpr (kLH) {
    chained_entry();
    Hb = H + blk * 256;
    const Factor f = fac[blk];
    if (f.zero) {  // every candidate scores 0: the smallest code wins
      const int64_t r_end = min(R, row_base + kRowsPerCta);
      for (int64_t r = row_base + threadIdx.x; r < r_end; r += kThreads) {
        cb[r * nb] = 1;
        if (ob) ob[r * nb] = 0.0f;
      }
      return;
    }
    sigma = f.sigma;
    sl2 = f.sl2;
    rsq = f.rsq;
    if (threadIdx.x < 16) cdiag_sh[threadIdx.x] = fac[blk].cs[threadIdx.x];
    const uint4 h = frag[(blk * 32 + lane) * 2], l = frag[(blk * 32 + lane) * 2 + 1];
    bh[0][0] = h.x; bh[0][1] = h.y; bh[1][0] = h.z; bh[1][1] = h.w;
    bl[0][0] = l.x; bl[0][1] = l.y; bl[1][0] = l.z; bl[1][1] = l.w;
    __syncthreads();  // cdiag_sh
  }

  uint32_t evals = 0;  // (at most 16 tiles x 126 candidates x 16 rows per warp)
  for (int tile = warp; tile < kRowsPerCta / kTileRows; tile += kWarps) {
    const uint32_t kg = keys[tile * kTileRows + g], kg8 = keys[tile * kTileRows + g + 8];
    const bool v0 = (kg >> 16) != 0xFFFFu, v1 = (kg8 >> 16) != 0xFFFFu;
    if (!__any_sync(0xFFFFFFFFu, v0 || v1)) break;  // only padding from here on
    const int i0 = (int)(kg & 0xFFFu), i1 = (int)(kg8 & 0xFFFu);
    uint32_t W0[8], W1[8];
    {
      const uint4 a0 = Ws[i0][0], a1 = Ws[i0][1], c0 = Ws[i1][0], c1 = Ws[i1][1];
      W0[0] = a0.x; W0[1] = a0.y; W0[2] = a0.z; W0[3] = a0.w;
      W0[4] = a1.x; W0[5] = a1.y; W0[6] = a1.z; W0[7] = a1.w;
      W1[0] = c0.x; W1[1] = c0.y; W1[2] = c0.z; W1[3] = c0.w;
      W1[4] = c1.x; W1[5] = c1.y; W1[6] = c1.z; W1[7] = c1.w;
    }
    // rows of the tile that are not padding (each row sits in four lanes)
    const uint32_t nvalid =
        (__popc(__ballot_sync(0xFFFFFFFFu, v0)) + __popc(__ballot_sync(0xFFFFFFFFu, v1))) >> 2;
    uint32_t ncand = 0;  // candidates evaluated for the tile
    // row amax (bf16 magnitude bits; 0 for padding) and the tile's largest
    const uint32_t am0 = v0 ? kg >> 16 : 0u, am1 = v1 ? kg8 >> 16 : 0u;
    const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, max(am0, am1));
    // this lane's four pairs in MMA order: (g,2t) (g+8,2t) (g,2t+8) (g+8,2t+8)
    const uint32_t pw[4] = {pick4(W0[0], W0[1], W0[2], W0[3], t),
                            pick4(W1[0], W1[1], W1[2], W1[3], t),
                            pick4(W0[4], W0[5], W0[6], W0[7], t),
                            pick4(W1[4], W1[5], W1[6], W1[7], t)};
    // element k of the lane in C order: 2i, 2i+1 = low, high half of pair i
    // (row g: elements 0, 1, 4, 5; row g + 8: 2, 3, 6, 7)
    float xs[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      xs[2 * i] = bf16_lo(pw[i]);
      xs[2 * i + 1] = bf16_hi(pw[i]);
    }
    // p = L^T w at the C positions: pz[nt][0..1] row g, n = 8nt + 2t + {0,1};
    // pz[nt][2..3] row g+8, same n.  Local-Hessian: from the tensor cores
    // with each row's w scaled by its own 2^kw (exact; the row's largest |w|
    // lands in [2^14, 2^15) in f16, so every row keeps f16's full precision
    // whatever the other rows of the tile hold), so pz and every z below
    // carry the factor sigma_L 2^kw of their row, removed from the reported
    // objective at the end.  MSE: p = 2^kw w.
    float pz[2][4];
    // Both rules scale each row this way: objectives and bounds then stay in
    // the normal fp32 range for tiny and for huge weights alike (2^kw at most
    // 2^127: a row whose largest |w| is below 2^-113 lands lower, its bf16
    // values still exact in f16).  Objectives carry zscale^2 = (sigma 2^kw)^2
    // of the lane's row, kept as its exponent: zscale itself can pass the
    // fp32 range (sigma <= 2^90 for an fp32 H), and nothing below multiplies
    // by it.  Padding and all-zero rows take 2^0.
    const int kw0 = am0 ? min(14 - ((int)(am0 >> 7) - 127), 127) : 0;
    const int kw1 = am1 ? min(14 - ((int)(am1 >> 7) - 127), 127) : 0;
    const float wsc0 = ldexpf(1.0f, kw0), wsc1 = ldexpf(1.0f, kw1);
    const float wsc = upper ? wsc1 : wsc0;  // the lane's own row
    int zexp = upper ? kw1 : kw0;
    // Q of the lane's row: the absolute part of the screen's error bound
    // (see the file header); 0 for MSE, whose screen is exact up to the
    // relative rounding of its sums
    float qerr = 0.0f;
    if (kLH) {
      zexp += (int)((__float_as_uint(sigma) >> 23) & 0xFFu) - 127;
      uint32_t Aw[4];  // pairs 0, 2: row g; 1, 3: row g + 8
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float ws = (i & 1) ? wsc1 : wsc0;
        Aw[i] = pack_half2(__float2half_rn(xs[2 * i] * ws), __float2half_rn(xs[2 * i + 1] * ws));
      }
      const float zero4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      mma_f16_16816(pz[0], Aw, bh[0][0], bh[0][1], zero4);
      mma_f16_16816(pz[1], Aw, bh[1][0], bh[1][1], zero4);
      mma_f16_16816(pz[0], Aw, bl[0][0], bl[0][1], pz[0]);
      mma_f16_16816(pz[1], Aw, bl[1][0], bl[1][1], pz[1]);
      // a = |W| |sigma L_hi| (sign bits cleared), A = ||a||_2 per row
      constexpr uint32_t kAbs = 0x7FFF7FFFu;
      uint32_t Wa[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) Wa[i] = Aw[i] & kAbs;
      float a0[4], a1[4];
      mma_f16_16816(a0, Wa, bh[0][0] & kAbs, bh[0][1] & kAbs, zero4);
      mma_f16_16816(a1, Wa, bh[1][0] & kAbs, bh[1][1] & kAbs, zero4);
      // rows g (elements 0, 1) and g + 8 (2, 3): the quad reduce-scatter of
      // the objective, lanes t < 2 keep row g
      const float aa0 = fmaf(a0[0], a0[0], fmaf(a0[1], a0[1], fmaf(a1[0], a1[0], a1[1] * a1[1])));
      const float aa1 = fmaf(a0[2], a0[2], fmaf(a0[3], a0[3], fmaf(a1[2], a1[2], a1[3] * a1[3])));
      float aa = upper ? aa1 : aa0;
      aa += __shfl_xor_sync(0xFFFFFFFFu, upper ? aa0 : aa1, 2);
      aa += __shfl_xor_sync(0xFFFFFFFFu, aa, 1);
      // dropped pivots: sqrt(F) <= 12 sqrt(rho) max|W| of the row
      const float wmax = __uint_as_float((upper ? am1 : am0) << 16) * wsc;
      qerr = fmaf(kAccErr, sqrt_up(aa), kAbsErr) + rsq * wmax;
    } else {
      pz[0][0] = xs[0] * wsc0; pz[0][1] = xs[1] * wsc0; pz[0][2] = xs[2] * wsc1;
      pz[0][3] = xs[3] * wsc1; pz[1][0] = xs[4] * wsc0; pz[1][1] = xs[5] * wsc0;
      pz[1][2] = xs[6] * wsc1; pz[1][3] = xs[7] * wsc1;
    }
    // multiplier of u in z: s 2^kw of the row (for Local-Hessian u carries
    // sigma_L), passed per candidate as s * wsc0 and s * wsc1
    float pp0 = pz[0][0] * pz[0][0] + pz[0][1] * pz[0][1] + pz[1][0] * pz[1][0] +
                pz[1][1] * pz[1][1];
    float pp1 = pz[0][2] * pz[0][2] + pz[0][3] * pz[0][3] + pz[1][2] * pz[1][2] +
                pz[1][3] * pz[1][3];
    pp0 += __shfl_xor_sync(0xFFFFFFFFu, pp0, 1);
    pp0 += __shfl_xor_sync(0xFFFFFFFFu, pp0, 2);
    pp1 += __shfl_xor_sync(0xFFFFFFFFu, pp1, 1);
    pp1 += __shfl_xor_sync(0xFFFFFFFFu, pp1, 2);
    const float inf = __int_as_float(0x7F800000);
    float b1 = inf, b2 = inf, b3 = inf;
    // Pruning, with lambda a lower bound of the smallest eigenvalue of H_b
    // (1 for MSE); both bounds are in the objective's units (zscale^2 lambda
    // = sl^2 2^2kw, with sl = sigma sqrt(lambda) <= 2^17 and the values scaled
    // by 2^kw before squaring) and a candidate is skipped only when its bound
    // exceeds the best objective beyond the tie band, for every row of the
    // warp.
    //  - small scales: for s < amax_row / 6 the row's largest value
    //    saturates, |delta| >= amax_row - 6 s, so E >= lambda (amax_row -
    //    6 s)^2, growing as s falls;
    //  - large scales: every |w_i| <= s / 4 encodes to 0 (the tie at 1/4 goes
    //    to the even code), so E >= lambda sum of those w_i^2, growing as s
    //    rises.
    // Each class is walked from its first scale at or above the tile's
    // largest amax / 6 downwards, then from there upwards.  Rows past the end
    // and all-zero rows never hold the warp back.
    const float amax_row = __uint_as_float((upper ? am1 : am0) << 16);

    // saturation bound of the lane's row: its largest element (position i,
    // from the row's sort key; any one of equal maxima) alone forces
    // E >= |delta_i|^2 / (H^-1)_ii
    const float ss2 = kLH ? cdiag_sh[((upper ? kg8 : kg) >> 12) & 0xFu] : 1.0f;
    const float amax_w = amax_row * wsc, m6w = -6.0f * wsc;
    const float row_floor = kZeroFloor * (upper ? pp1 : pp0);
    // what the tile's epilogue needs, formed here so that nothing else stays
    // live across the candidate walk: the lane's row, whether it finishes
    // it, and whether a tile value lies above 2^100 s_g
    const int my_row = upper ? i1 : i0;
    const bool owner = (t & 1) == 0 && (upper ? v1 : v0);
    const bool tile_over = __uint_as_float(m << 16) > 0x1p100f * s_g;
    // a candidate is skipped when its lower bound, less the bound's own
    // rounding, exceeds what the best so far can be: b1 (1 + 2 kTieBand) +
    // 4102 Q^2 + the floors
    // (rows past the end and all-zero rows take -inf, so that they never
    // hold the warp back: every check runs after at least one evaluation,
    // so b1 is finite there)
    const float prune_pad =
        amax_row == 0.0f ? -__int_as_float(0x7F800000)
                         : fmaf(4102.0f * qerr, qerr, row_floor + kAbsBand);
    // the bounds' factors with their rounding allowance
    const float ss2t = ss2 * (1.0f - 2.0f * kTieBand), sl2t = sl2 * (1.0f - 2.0f * kTieBand);
    const float smax = __uint_as_float(m << 16) * (1.0f / 6.0f);

    int jbegin = 0;
    for (int k = 0; k < ncls; ++k) {
      const ClassInfo ci = cls[k];
      // class quotient t per element (within one float of q)
      float tq[8];
      if constexpr (kLH) {
        const float2 rhi = make_float2(ci.r_hi, ci.r_hi), rlo = make_float2(ci.r_lo, ci.r_lo);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const float2 x2 = make_float2(xs[e], xs[e + 1]);
          const float2 t2 = __ffma2_rn(x2, rhi, __fmul2_rn(x2, rlo));
          tq[e] = t2.x;
          tq[e + 1] = t2.y;
        }
      } else {  // unpaired: the paired form spilled at nine MSE CTAs per SM
#pragma unroll
        for (int e = 0; e < 8; ++e) tq[e] = fmaf(xs[e], ci.r_hi, xs[e] * ci.r_lo);
      }
      // uncertified classes: a quotient with at most 3 significant bits
      // (every rounding midpoint is one, and so is every power-of-two
      // multiple) moves towards q = w / S: v = t + rho (16 / S), rounded
      // once, with the exact residual rho = w - t S.  For such a t a non-zero
      // residual lies between 2^-27 |q| S and one float of q times S (w has 8
      // significant bits, t S at most 27), so v lands at least one float and
      // at most 2^-19 |q| from t on q's side: off the midpoint, and short of
      // any other rounding decision (at least 4% away).  A zero residual of
      // either sign leaves t.  Every other t is not a midpoint at any scale
      // of the class and rounds like q.
      if (!ci.certified) {
        const float2 nS = make_float2(-ci.S, -ci.S);
        const float2 r16 = make_float2(16.0f * ci.r_hi, 16.0f * ci.r_hi);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const float2 t2 = make_float2(tq[e], tq[e + 1]);
          const float2 rho = __ffma2_rn(t2, nS, make_float2(xs[e], xs[e + 1]));
          const float2 v2 = __ffma2_rn(rho, r16, t2);
          tq[e] = (__float_as_uint(t2.x) & 0x1FFFFFu) == 0u ? v2.x : t2.x;
          tq[e + 1] = (__float_as_uint(t2.y) & 0x1FFFFFu) == 0u ? v2.y : t2.y;
        }
      }
      // first candidate of the class at or above smax (scales ascend within a
      // class; a class has at most 18 candidates)
      const int jl = jbegin + lane;
      const uint32_t ge = __ballot_sync(0xFFFFFFFFu, jl < ci.end && cand[jl].s >= smax);
      const int js = ge ? jbegin + __ffs(ge) - 1 : ci.end - 1;
      // downwards from js (scales halve at every step of a class)
      for (int j = js; j >= jbegin; --j) {
        const CandInfo c0 = cand[j];
        if (j < js) {
          // saturation bound at this scale (every later one is smaller)
          // (amax_row - 6 s) 2^kw where the row's largest value saturates,
          // else 0 (no bound: the threshold is positive for real rows)
          const float d = fmaxf(fmaf(m6w, c0.s, amax_w), 0.0f);
          const bool done = ss2t * d * d > fmaf(b1, 1.0f + 2.0f * kTieBand, prune_pad);
          if (__all_sync(0xFFFFFFFFu, done)) break;
        }
        const float e0 = candidate_objective<kLH>(tq, c0.f, c0.s * wsc0, c0.s * wsc1, bh,
                                                  bl, pz, upper);
        track3(key_of(e0, c0.c), b1, b2, b3);
        ++ncand;
      }
      // upwards from js + 1
      for (int j = js + 1; j < ci.end; ++j) {
        const CandInfo c0 = cand[j];
        // zero-code bound at this scale (every later one is larger)
        const float q4 = 0.25f * c0.s;
        // pairs (e, e + 1) lie in one row: e = 0, 4 in row g, e = 2, 6 in g + 8
        float2 ugp = make_float2(0.0f, 0.0f), ug8p = ugp;
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const float2 x2 = make_float2(fabsf(xs[e]) <= q4 ? xs[e] : 0.0f,
                                        fabsf(xs[e + 1]) <= q4 ? xs[e + 1] : 0.0f);
          const float ws = (e & 2) ? wsc1 : wsc0;
          const float2 v2 = __fmul2_rn(x2, make_float2(ws, ws));
          if ((e & 2) == 0) ugp = __ffma2_rn(v2, v2, ugp);
          else ug8p = __ffma2_rn(v2, v2, ug8p);
        }
        const float ug = ugp.x + ugp.y, ug8 = ug8p.x + ug8p.y;
        // the same quad reduce-scatter as the objective: lanes t < 2 keep row g
        float zero_sum = upper ? ug8 : ug;
        zero_sum += __shfl_xor_sync(0xFFFFFFFFu, upper ? ug : ug8, 2);
        zero_sum += __shfl_xor_sync(0xFFFFFFFFu, zero_sum, 1);
        const bool done = sl2t * zero_sum > fmaf(b1, 1.0f + 2.0f * kTieBand, prune_pad);
        if (__all_sync(0xFFFFFFFFu, done)) break;
        const float e0 = candidate_objective<kLH>(tq, c0.f, c0.s * wsc0, c0.s * wsc1, bh,
                                                  bl, pz, upper);
        track3(key_of(e0, c0.c), b1, b2, b3);
        ++ncand;
      }
      jbegin = ci.end;
    }

    evals += ncand * nvalid;

    // lane t = 0 finishes row g, lane t = 2 row g + 8; near ties are
    // re-scored by the whole warp, one row at a time
    const int64_t r = row_base + my_row;
    int code = code_of(b1);
    float obj = ldexpf(b1, -2 * zexp);
    int need = 0;  // 1: re-score the best two, 2: re-score every candidate
    if (owner) {
      const float fl = row_floor;
      if (amax_w == 0.0f) {  // all-zero row: every candidate scores exactly 0
        code = 1;
        obj = 0.0f;
      } else if (!by_class || tile_over) {
        // s_g outside [2^-100, 2^100): the per-candidate fp32 reciprocals can
        // leave the normal range; or a tile value above 2^100 s_g (a tensor
        // scale far below the weights' own, amax / 2688): the class
        // quotients w / S can overflow fp32.  The screen then only orders,
        // and every candidate is re-scored in fp64.
        need = 2;
      } else if (kLH) {
        // both candidates' screen errors: kTieBand b + 2 Q sqrt(b) + 6 Q^2
        // each (b3 may be infinite when pruning left two: then all 126)
        const float q4 = 4.0f * qerr, q12 = fmaf(12.0f * qerr, qerr, kAbsBand);
        const float big = 3.0e38f;
        if (b2 - b1 <= fmaf(kTieBand, b2, fmaf(q4, sqrt_up(fminf(b2, big)), q12)) ||
            b1 <= fmaf(16.0f * qerr, qerr, fl))
          need = (b3 - b1 > fmaf(kTieBand, b3, fmaf(q4, sqrt_up(fminf(b3, big)), q12 + fl))) ? 1
                                                                                          : 2;
      } else if (b2 - b1 <= kTieBand * b2 + kAbsBand || b1 <= fl) {
        // MSE: u = v and p = W exactly, Q = 0
        need = (b3 - b1 > kTieBand * b3 + fl + kAbsBand) ? 1 : 2;
      }
    }
    for (uint32_t pend = __ballot_sync(0xFFFFFFFFu, need != 0); pend; pend &= pend - 1) {
      const int src = __ffs(pend) - 1;
      const int64_t rr = __shfl_sync(0xFFFFFFFFu, (long long)r, src);
      const int n = __shfl_sync(0xFFFFFFFFu, need, src);
      const int k1 = __shfl_sync(0xFFFFFFFFu, code_of(b1), src);
      const int k2 = __shfl_sync(0xFFFFFFFFu, code_of(b2), src);
      float o;
      const int c = refine_block(wb + rr * C, s_g, Hb, k1, k2, n == 2, &o);
      if (lane == src) {
        code = c;
        obj = o;
      }
    }
    if (owner) {
      cb[r * nb] = (uint8_t)code;
      if (ob) ob[r * nb] = obj;
    }
  }
  if (lane == 0) {
    if (evals) atomicAdd(&g_search_evals[kLH ? 1 : 0], (unsigned long long)evals);
  }
}

// Diagnostic of the screen's error model: tile i of a [n][16][16] (f16,
// row-major, m x k), b [n][16][8] (f16, k x n) and c [n][16][8] (fp32)
// through one mma_f16_16816 call, the instruction the screen uses, with
// d [n][16][8] written.  One warp per tile.
__global__ void mma_probe_kernel(const uint16_t *__restrict__ a, const uint16_t *__restrict__ b,
                                 const float *__restrict__ c, float *__restrict__ d, int64_t n) {
  const int64_t tile = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (tile >= n) return;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const uint16_t *A = a + tile * 256, *B = b + tile * 128;
  const float *Cm = c + tile * 128;
  float *D = d + tile * 128;
  auto pair = [](uint16_t lo, uint16_t hi) { return (uint32_t)lo | ((uint32_t)hi << 16); };
  const uint32_t af[4] = {pair(A[g * 16 + 2 * t], A[g * 16 + 2 * t + 1]),
                          pair(A[(g + 8) * 16 + 2 * t], A[(g + 8) * 16 + 2 * t + 1]),
                          pair(A[g * 16 + 2 * t + 8], A[g * 16 + 2 * t + 9]),
                          pair(A[(g + 8) * 16 + 2 * t + 8], A[(g + 8) * 16 + 2 * t + 9])};
  const uint32_t b0 = pair(B[(2 * t) * 8 + g], B[(2 * t + 1) * 8 + g]);
  const uint32_t b1 = pair(B[(2 * t + 8) * 8 + g], B[(2 * t + 9) * 8 + g]);
  const float cf[4] = {Cm[g * 8 + 2 * t], Cm[g * 8 + 2 * t + 1], Cm[(g + 8) * 8 + 2 * t],
                       Cm[(g + 8) * 8 + 2 * t + 1]};
  float df[4];
  mma_f16_16816(df, af, b0, b1, cf);
  D[g * 8 + 2 * t] = df[0];
  D[g * 8 + 2 * t + 1] = df[1];
  D[(g + 8) * 8 + 2 * t] = df[2];
  D[(g + 8) * 8 + 2 * t + 1] = df[3];
}

}  // namespace

cudaError_t launch_mma_probe(const uint16_t *a, const uint16_t *b, const float *c, float *d,
                             int64_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  mma_probe_kernel<<<(unsigned)((n + 3) / 4), 128, 0, st>>>(a, b, c, d, n);
  return cudaGetLastError();
}

cudaError_t read_search_evaluations(cudaStream_t st, unsigned long long out[6], bool reset) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_search_evals, sizeof(g_search_evals), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess && reset) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_search_evals);
    if (e == cudaSuccess) e = cudaMemsetAsync(p, 0, sizeof(g_search_evals), st);
  }
  const cudaError_t es = cudaStreamSynchronize(st);
  return e != cudaSuccess ? e : es;
}

cudaError_t launch_scale_search(const uint16_t *w, int64_t batch, int64_t R, int64_t C,
                                const float *s_g, const float *H, uint8_t *codes,
                                float *best_obj, int local_hessian, cudaStream_t st) {
  if (R == 0 || C == 0) return cudaSuccess;
  // Local-Hessian: 128-row CTAs when 256-row ones would fill fewer than six
  // waves of the resident CTAs (dense 4096 x 4096: 4096 CTAs of 256 rows,
  // about four waves; measured 2% faster there, 3.5% slower on the 128 MoE
  // experts, which have 47 waves).  The MSE search measured slower with the
  // smaller groups of rows sorted together and keeps 256.
  const int64_t ctas_large = (R + kRowsLarge - 1) / kRowsLarge * (C / kBlock) * batch;
  const bool small = local_hessian && ctas_large < (int64_t)sm_count() * kLhCtasPerSm * 6;
  const int rows = small ? kRowsSmall : kRowsLarge;
  dim3 grid((unsigned)((R + rows - 1) / rows), (unsigned)(C / kBlock), (unsigned)batch);
  if (!local_hessian) {
    return launch_first(small ? search_kernel<false, kRowsSmall>
                                : search_kernel<false, kRowsLarge>,
                          grid, dim3(kThreads), 0, st, w, R, C, s_g, nullptr, nullptr, nullptr,
                          codes, best_obj);
  }
  // factors of every H_b first (stream-ordered scratch, freed after the search)
  const int64_t nblocks = batch * (C / kBlock);
  const size_t frag_bytes = (size_t)nblocks * 32 * 2 * sizeof(uint4);
  void *scratch = nullptr;
  cudaError_t e = scratch_alloc(&scratch, frag_bytes + (size_t)nblocks * sizeof(Factor), st);
  if (e != cudaSuccess) return e;
  uint4 *frag = static_cast<uint4 *>(scratch);
  Factor *fac = reinterpret_cast<Factor *>(static_cast<char *>(scratch) + frag_bytes);
  const int64_t nb = C / kBlock;
  // the search kernel reads W and s_g before waiting for the factor kernel
  // (see its prologue): nothing may come between the two launches, and the
  // factor kernel starts after all earlier work
  e = launch_first(factor_kernel, dim3((unsigned)((nb + 1) / 2), (unsigned)batch), dim3(32), 0,
                     st, H, nb, frag, fac);
  if (e == cudaSuccess)
    e = launch_chained(small ? search_kernel<true, kRowsSmall> : search_kernel<true, kRowsLarge>,
                       grid, dim3(kThreads), 0, st, w, R, C, s_g, H,
                       static_cast<const uint4 *>(frag), static_cast<const Factor *>(fac), codes,
                       best_obj);
  const cudaError_t ef = scratch_free(scratch, st);
  return e != cudaSuccess ? e : ef;
}

}  // namespace nvfp4
