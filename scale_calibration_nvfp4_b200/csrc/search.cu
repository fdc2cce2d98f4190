// Exhaustive block-scale search over the 126 positive finite non-zero E4M3
// codes: MSE objective and Local-Hessian objective.
//
// Method: the Local-Hessian write-up "4 比特量化到底让模型笨了多少？" (of NVIDIA
// Model Optimizer's "Improving NVFP4 Accuracy with Local-Hessian Weight
// Scales"): section "The NVFP4 structure" (MSE tries all 126 scales and keeps
// the smallest weight error) and section "A different objective" (E(s) =
// ||delta X||^2 = tr(delta X X^T delta^T); the block-diagonal approximation
// solves each 16-value block alone against its 16x16 H_b, still trying all
// 126 candidates).
//
// Mapping: one CTA owns one column block b of one batch element and a run
// of rows; one thread owns one row's block.  All threads of a CTA share H_b,
// so its factor L (H_b = L L^T, fp64 Cholesky by one warp, semidefinite
// pivots dropped) lives in every thread's registers as warp-uniform values
// and E = ||L^T delta||^2 costs 136 + 16 FMA per candidate instead of 272.
// Candidate scales and their reciprocal bracket sit in shared memory
// (broadcast reads).  Each candidate's E2M1 codes come from the hardware
// fp32 -> e2m1x2 conversion at both ends of the bracket t_lo <= |w|/s <= t_hi;
// a disagreement (|w|/s within ~2^-23 of a rounding midpoint) falls back to
// the exact fp64 midpoint test.
//
// Exactness of the winner: the fp32 screen tracks the best two objectives.
// If they are within 2^-12 relative, the row's block is re-scored in a second
// pass: candidates whose fp32 objective lies inside that band are evaluated
// in fp64 straight from H_b (delta H_b delta^T), and the first minimum in
// ascending code order wins, as in the plain definition.
#include "common.cuh"
#include "internal.h"

namespace nvfp4 {
namespace {

constexpr int kSearchThreads = 128;
constexpr int kRowIters = 4;
constexpr float kTieBand = 1.0f / 4096.0f;
constexpr int kTriangle = 136;  // 16 * 17 / 2

// Offset of column k in the packed lower triangle (column-major, rows j >= k).
__host__ __device__ constexpr int tri_col(int k) { return 16 * k - (k * (k - 1)) / 2; }

// Cooperative Cholesky of the 16x16 block in Hs (fp32, row-major) by warp 0,
// lanes 0..15 owning one row each.  A pivot at or below 1e-12 of the largest
// diagonal (or non-finite) drops its column, which keeps a positive
// semidefinite H usable.  Writes the packed factor to Ls.
__device__ void cholesky16(const float *Hs, float *Ls) {
  const int lane = threadIdx.x & 31;
  const bool own = lane < 16;
  double a[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) a[j] = own ? (double)Hs[lane * 16 + j] : 0.0;
  double diag = 0.0;
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (j == lane) diag = a[j];
  double maxdiag = diag;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) maxdiag = fmax(maxdiag, __shfl_xor_sync(0xFFFFFFFFu, maxdiag, o));
  const double tol = 1e-12 * maxdiag;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const double akk = __shfl_sync(0xFFFFFFFFu, a[k], k);
    const bool ok = (akk > tol) && (akk < 1e300);
    const double piv = ok ? sqrt(akk) : 0.0;
    double lik = 0.0;
    if (lane == k) lik = piv;
    else if (own && lane > k && ok) lik = a[k] / piv;
    if (own && lane >= k) Ls[tri_col(k) + (lane - k)] = (float)lik;
#pragma unroll
    for (int j = k + 1; j < 16; ++j) {
      const double ljk = __shfl_sync(0xFFFFFFFFu, lik, j);
      a[j] = fma(-lik, ljk, a[j]);
    }
  }
}

// fp32 objective of candidate c for one block, and the signed E2M1 values
// v[] it uses.  `Lf` is the packed factor (registers in the screen, shared
// memory in the re-score: both hold the same fp32 values and the arithmetic
// below is a fixed sequence of fmaf, so both paths give identical results).
template <bool kLH, typename LT>
__device__ __forceinline__ float candidate_objective(const float x[16], const uint32_t sgn[8],
                                                     const float4 t, const LT &Lf,
                                                     float v[16]) {
  const ScaleRecip rr = {t.x, t.y, t.z};
  uint32_t bytes[8], mismatch = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    bytes[j] = e2m1_pair_bracket(fabsf(x[2 * j]), fabsf(x[2 * j + 1]), rr, mismatch);
  if (mismatch) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      bytes[j] = e2m1_mag_exact(fabsf(x[2 * j]), t.x) |
                 (e2m1_mag_exact(fabsf(x[2 * j + 1]), t.x) << 4);
  }
  float d[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t h2 = cvt_f16x2_from_e2m1x2(bytes[j] | sgn[j]);
    v[2 * j] = f16_lo_to_float(h2);
    v[2 * j + 1] = f16_hi_to_float(h2);
    d[2 * j] = fmaf(-v[2 * j], t.x, x[2 * j]);
    d[2 * j + 1] = fmaf(-v[2 * j + 1], t.x, x[2 * j + 1]);
  }
  float e = 0.0f;
  if (kLH) {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float z = 0.0f;
#pragma unroll
      for (int j = k; j < 16; ++j) z = fmaf(Lf[tri_col(k) + (j - k)], d[j], z);
      e = fmaf(z, z, e);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) e = fmaf(d[j], d[j], e);
  }
  return e;
}

__device__ __forceinline__ void unpack_block(const uint32_t wv[8], float x[16], uint32_t sgn[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    x[2 * j] = bf16_lo(wv[j]);
    x[2 * j + 1] = bf16_hi(wv[j]);
    sgn[j] = ((wv[j] >> 12) & 0x8u) | ((wv[j] >> 24) & 0x80u);
  }
}

// Packed factor from shared memory with non-hoistable loads, so the compiler
// keeps it out of registers outside the candidate loop that uses it.
__device__ __forceinline__ void load_factor(const float *Ls, float L[kTriangle]) {
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(Ls);
#pragma unroll
  for (int i = 0; i < kTriangle; i += 4) {
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(L[i]), "=f"(L[i + 1]), "=f"(L[i + 2]), "=f"(L[i + 3])
                 : "r"(base + 4 * i));
  }
}

// Near-tie re-score of one block: every candidate whose fp32 objective is
// within `band` is evaluated in fp64 from the definition (delta H delta^T, or
// delta delta^T for MSE); the first minimum in ascending code order wins.
template <bool kLH>
__device__ __noinline__ int rescore_block(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                          uint32_t w4, uint32_t w5, uint32_t w6, uint32_t w7,
                                          const float4 *tab, const float *Ls, const float *Hs,
                                          float band, double *best_out) {
  const uint32_t wv[8] = {w0, w1, w2, w3, w4, w5, w6, w7};
  float x[16];
  uint32_t sgn[8];
  unpack_block(wv, x, sgn);
  double best = __longlong_as_double(0x7FF0000000000000LL);
  int best_c = 1;
  for (int c = 1; c <= kCandidates; ++c) {
    const float4 t = tab[c - 1];
    float v[16];
    float L[kLH ? kTriangle : 4];
    if (kLH) load_factor(Ls, L);
    const float e = candidate_objective<kLH>(x, sgn, t, L, v);
    if (!(e <= band)) continue;
    double dd[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) dd[j] = (double)x[j] - (double)v[j] * (double)t.x;
    double e64 = 0.0;
    if (kLH) {
      for (int j = 0; j < 16; ++j) {
        double row = 0.0;
        for (int k = 0; k < 16; ++k) row = fma((double)Hs[j * 16 + k], dd[k], row);
        e64 = fma(dd[j], row, e64);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) e64 = fma(dd[j], dd[j], e64);
    }
    if (e64 < best) {
      best = e64;
      best_c = c;
    }
  }
  *best_out = best;
  return best_c;
}

template <bool kLH>
__global__ void __launch_bounds__(kSearchThreads)
    search_kernel(const uint16_t *__restrict__ w, int64_t R, int64_t C,
                  const float *__restrict__ s_g, const float *__restrict__ H,
                  uint8_t *__restrict__ codes, float *__restrict__ best_obj) {
  const int64_t nb = C / kBlock;
  const int64_t b = blockIdx.y;
  const int64_t batch = blockIdx.z;
  const int64_t row0 = (int64_t)blockIdx.x * kSearchThreads * kRowIters;

  __shared__ float4 tab[kCandidates];
  __shared__ float Hs[kLH ? 256 : 1];
  __shared__ __align__(16) float Ls[kLH ? kTriangle : 4];

  const float sg = s_g[batch];
  for (int c = threadIdx.x; c < kCandidates; c += kSearchThreads) {
    const float s = effective_scale(sg, (uint32_t)(c + 1));
    const ScaleRecip r = make_recip(s);
    tab[c] = make_float4(s, r.r_lo, r.r_hi, 0.0f);
  }
  if (kLH) {
    const float *Hb = H + (batch * nb + b) * 256;
    for (int i = threadIdx.x; i < 256; i += kSearchThreads) Hs[i] = Hb[i];
    __syncthreads();
    if (threadIdx.x < 32) cholesky16(Hs, Ls);
  }
  __syncthreads();

  const uint16_t *wb = w + batch * R * C + b * kBlock;
  uint8_t *cb = codes + batch * R * nb + b;
  float *ob = best_obj ? best_obj + batch * R * nb + b : nullptr;

  for (int it = 0; it < kRowIters; ++it) {
    const int64_t r = row0 + it * kSearchThreads + threadIdx.x;
    if (r >= R) break;
    uint32_t wv[8];
    {
      const uint4 *q = reinterpret_cast<const uint4 *>(wb + r * C);
      const uint4 v0 = ld_stream_v4(q), v1 = ld_stream_v4(q + 1);
      wv[0] = v0.x; wv[1] = v0.y; wv[2] = v0.z; wv[3] = v0.w;
      wv[4] = v1.x; wv[5] = v1.y; wv[6] = v1.z; wv[7] = v1.w;
    }
    float x[16];
    uint32_t sgn[8];
    unpack_block(wv, x, sgn);
    // the factor is reloaded per row so that it is not live across the
    // (rare) re-score call
    float L[kLH ? kTriangle : 4];
    if (kLH) load_factor(Ls, L);

    float best1 = __int_as_float(0x7F800000), best2 = __int_as_float(0x7F800000);
    int c1 = 1;
    for (int c = 1; c <= kCandidates; ++c) {
      float v[16];
      const float e = candidate_objective<kLH>(x, sgn, tab[c - 1], L, v);
      if (e < best1) {
        best2 = best1;
        best1 = e;
        c1 = c;
      } else {
        best2 = fminf(best2, e);
      }
    }
    float obj = best1;
    if (best2 - best1 <= kTieBand * best2) {
      double e64;
      c1 = rescore_block<kLH>(wv[0], wv[1], wv[2], wv[3], wv[4], wv[5], wv[6], wv[7], tab, Ls,
                              Hs, best1 + kTieBand * best2, &e64);
      obj = (float)e64;
    }
    cb[r * nb] = (uint8_t)c1;
    if (ob) ob[r * nb] = obj;
  }
}

}  // namespace

cudaError_t launch_scale_search(const uint16_t *w, int64_t batch, int64_t R, int64_t C,
                                const float *s_g, const float *H, uint8_t *codes,
                                float *best_obj, int local_hessian, cudaStream_t st) {
  if (R == 0 || C == 0) return cudaSuccess;
  const int64_t rows_per_cta = (int64_t)kSearchThreads * kRowIters;
  dim3 grid((unsigned)((R + rows_per_cta - 1) / rows_per_cta), (unsigned)(C / kBlock),
            (unsigned)batch);
  if (local_hessian)
    search_kernel<true><<<grid, kSearchThreads, 0, st>>>(w, R, C, s_g, H, codes, best_obj);
  else
    search_kernel<false><<<grid, kSearchThreads, 0, st>>>(w, R, C, s_g, nullptr, codes,
                                                          best_obj);
  return cudaGetLastError();
}

}  // namespace nvfp4
