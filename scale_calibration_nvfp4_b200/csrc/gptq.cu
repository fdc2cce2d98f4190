// GPTQ rounding of NVFP4 weights at given block scales (the Local-Hessian
// write-up, "Trying it": Local-Hessian picks the scales, GPTQ changes the
// rounding, and the two combine; GPTQ is Frantar et al., "GPTQ: Accurate
// Post-Training Quantization for Generative Pre-trained Transformers",
// dampening and the Cholesky reformulation of its column loop).
//
// GPTQ rounds the columns of W in order and moves every column not yet
// rounded so that the output error ||(W - Q) X||^2 stays least, through the
// upper Cholesky factor U of the inverse of the dampened Hessian
// H + lambda I (lambda = damp * mean(diag H)).  With H = T T^T, T upper
// triangular (the Cholesky factor of H taken from the last index down),
// U = T^-1, and the value column k holds when it is rounded is
//
//   w'_k = w_k + (1 / T_kk) sum_{j<k} (w_j - q_j) T_jk
//
// (from W - Q = E U with E the scaled errors of the column loop), so no
// inverse is formed: one Cholesky factor and one running product.  All of it
// is fp64.
//
//  - gptq_lambda_kernel / gptq_prepare_kernel: lambda per Hessian, then
//    Hd = J (H + lambda I) J in fp64 (J reverses the index order), whose
//    lower Cholesky factor L gives T = J L J;
//  - chol_diag_kernel, chol_panel_kernel and the fp64 GEMM: blocked
//    right-looking Cholesky of Hd in place, 32-column panels (the diagonal
//    block by one warp, the rows below it by triangular solves, the trailing
//    matrix by a rank-32 update);
//  - gptq_block_kernel: 32 columns at a time, one thread per row, the
//    in-block part of the sum above from registers and the block of T from
//    shared memory; rounding by the exact fp64 midpoint test; the errors
//    w_j - q_j replace the consumed sums;
//  - the fp64 GEMM again: the block's errors times the next rows of T, added
//    to the running sums of every later column (lazy batch updates).
#include <cmath>

#include "common.cuh"
#include "internal.h"
#include "../../include/nvfp4.h"

namespace nvfp4 {

// Sticky status of the GPTQ kernels (a Hessian that is not positive
// definite after dampening), read with the library status.
__device__ int g_gptq_status = 0;

namespace {

constexpr int kPanel = 32;  // columns per Cholesky panel and per GPTQ block

// ----------------------------------------------------------------- fp64 GEMM
// C[m][n] += alpha sum_k A[m][k] B[k][n] for m < M, n < N, with arbitrary
// (also negative) element strides and a batch index in blockIdx.z.  `lower`:
// tiles lying wholly above the diagonal (every n > every m) are skipped.
struct GemmF64 {
  int64_t M, N, K;
  double alpha;
  const double *A;
  int64_t sAm, sAk, bsA;
  const double *B;
  int64_t sBk, sBn, bsB;
  double *C;
  int64_t sCm, sCn, bsC;
  int lower;
};

constexpr int kGM = 64, kGN = 64, kGK = 16, kGThreads = 256;

__global__ void __launch_bounds__(kGThreads) gemm_f64_kernel(const GemmF64 g) {
  const int64_t m0 = (int64_t)blockIdx.y * kGM, n0 = (int64_t)blockIdx.x * kGN;
  if (g.lower && n0 > m0 + kGM - 1) return;
  const int64_t z = blockIdx.z;
  const double *A = g.A + z * g.bsA;
  const double *B = g.B + z * g.bsB;
  double *Cz = g.C + z * g.bsC;
  __shared__ __align__(16) double As[kGK][kGM];
  __shared__ __align__(16) double Bs[kGK][kGN];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  // unit-stride dimension first in the tile loads (coalesced)
  const bool a_k_fast = g.sAk == 1 || g.sAk == -1;
  const bool b_n_fast = g.sBn == 1 || g.sBn == -1;
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  for (int64_t k0 = 0; k0 < g.K; k0 += kGK) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = tid + kGThreads * e;  // 0..1023
      const int am = a_k_fast ? idx >> 4 : idx & 63, ak = a_k_fast ? idx & 15 : idx >> 6;
      const int64_t gm = m0 + am, gk = k0 + ak;
      As[ak][am] = (gm < g.M && gk < g.K) ? A[gm * g.sAm + gk * g.sAk] : 0.0;
      const int bn = b_n_fast ? idx & 63 : idx >> 4, bk = b_n_fast ? idx >> 6 : idx & 15;
      const int64_t gn = n0 + bn, gk2 = k0 + bk;
      Bs[bk][bn] = (gn < g.N && gk2 < g.K) ? B[gk2 * g.sBk + gn * g.sBn] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      const double2 a01 = *reinterpret_cast<const double2 *>(&As[kk][ty * 4]);
      const double2 a23 = *reinterpret_cast<const double2 *>(&As[kk][ty * 4 + 2]);
      const double2 b01 = *reinterpret_cast<const double2 *>(&Bs[kk][tx * 4]);
      const double2 b23 = *reinterpret_cast<const double2 *>(&Bs[kk][tx * 4 + 2]);
      const double a[4] = {a01.x, a01.y, a23.x, a23.y};
      const double b[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 4 + j;
      if (n < g.N) {
        double *c = Cz + m * g.sCm + n * g.sCn;
        *c = fma(g.alpha, acc[i][j], *c);
      }
    }
  }
}

cudaError_t gemm_f64(const GemmF64 &g, int64_t batch, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return cudaSuccess;
  const dim3 grid((unsigned)((g.N + kGN - 1) / kGN), (unsigned)((g.M + kGM - 1) / kGM),
                  (unsigned)batch);
  gemm_f64_kernel<<<grid, kGThreads, 0, st>>>(g);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ Cholesky
// The nw x nw diagonal block at (p0, p0) of every batch element's matrix,
// factored in place by one warp (lane i holds row i; column k is finished at
// step k and its rank-1 update applied to the later columns).  A pivot that
// is not positive (or not finite) sets the status and makes the factor NaN.
__global__ void __launch_bounds__(32) chol_diag_kernel(double *A, int64_t C, int64_t p0, int nw) {
  const int lane = threadIdx.x;
  double *Ab = A + (int64_t)blockIdx.x * C * C + p0 * C + p0;
  double a[kPanel];
#pragma unroll
  for (int j = 0; j < kPanel; ++j)
    a[j] = (lane < nw && j <= lane) ? Ab[(int64_t)lane * C + j] : 0.0;
#pragma unroll
  for (int k = 0; k < kPanel; ++k) {
    if (k < nw) {
      const double piv = __shfl_sync(0xFFFFFFFFu, a[k], k);
      const bool ok = piv > 0.0 && piv < INFINITY;
      if (!ok && lane == 0) atomicExch(&g_gptq_status, (int)NVFP4_ERR_NOT_POSITIVE_DEFINITE);
      const double lkk = ok ? sqrt(piv) : __longlong_as_double(0x7FF8000000000000LL);
      const double l = lane == k ? lkk : (lane > k ? a[k] / lkk : 0.0);
      a[k] = l;
#pragma unroll
      for (int j = k + 1; j < kPanel; ++j) {
        const double ljk = __shfl_sync(0xFFFFFFFFu, l, j);
        if (lane >= j) a[j] = fma(-l, ljk, a[j]);
      }
    }
  }
  if (lane < nw)
#pragma unroll
    for (int j = 0; j < kPanel; ++j)
      if (j <= lane) Ab[(int64_t)lane * C + j] = a[j];
}

// Rows p0 + nw .. C-1 of the panel: x L_pp^T = a by forward substitution,
// one thread per row, the factored diagonal block in shared memory.
constexpr int kRowThreads = 128;

__global__ void __launch_bounds__(kRowThreads)
    chol_panel_kernel(double *A, int64_t C, int64_t p0, int nw) {
  __shared__ double L[kPanel][kPanel + 1];
  double *Ab = A + (int64_t)blockIdx.y * C * C;
  for (int idx = threadIdx.x; idx < kPanel * kPanel; idx += kRowThreads) {
    const int r = idx / kPanel, c = idx % kPanel;
    L[r][c] = (r < nw && c <= r) ? Ab[(p0 + r) * C + p0 + c] : 0.0;
  }
  __syncthreads();
  const int64_t i = p0 + nw + (int64_t)blockIdx.x * kRowThreads + threadIdx.x;
  if (i >= C) return;
  double *row = Ab + i * C + p0;
  double x[kPanel];
#pragma unroll
  for (int k = 0; k < kPanel; ++k) {
    if (k < nw) {
      double v = row[k];
#pragma unroll
      for (int m = 0; m < k; ++m) v = fma(-x[m], L[k][m], v);
      x[k] = v / L[k][k];
      row[k] = x[k];
    } else {
      x[k] = 0.0;
    }
  }
}

cudaError_t cholesky_in_place(double *A, int64_t C, int64_t batch, cudaStream_t st) {
  for (int64_t p0 = 0; p0 < C; p0 += kPanel) {
    const int nw = (int)(C - p0 < kPanel ? C - p0 : kPanel);
    chol_diag_kernel<<<(unsigned)batch, 32, 0, st>>>(A, C, p0, nw);
    const int64_t rest = C - p0 - nw;
    if (rest > 0) {
      const dim3 grid((unsigned)((rest + kRowThreads - 1) / kRowThreads), (unsigned)batch);
      chol_panel_kernel<<<grid, kRowThreads, 0, st>>>(A, C, p0, nw);
      // trailing block -= panel panel^T (lower triangle)
      GemmF64 g;
      g.M = rest; g.N = rest; g.K = nw; g.alpha = -1.0;
      g.A = A + (p0 + nw) * C + p0; g.sAm = C; g.sAk = 1; g.bsA = C * C;
      g.B = g.A; g.sBk = 1; g.sBn = C; g.bsB = C * C;
      g.C = A + (p0 + nw) * C + p0 + nw; g.sCm = C; g.sCn = 1; g.bsC = C * C;
      g.lower = 1;
      cudaError_t e = gemm_f64(g, batch, st);
      if (e != cudaSuccess) return e;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ---------------------------------------------------------------------- GPTQ
// lambda = damp * mean(diag H), the diagonal summed in a fixed order.
__global__ void __launch_bounds__(32)
    gptq_lambda_kernel(const float *H, int64_t C, double damp, double *lam) {
  const float *Hb = H + (int64_t)blockIdx.x * C * C;
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < C; i += 32) s += (double)Hb[i * C + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if (threadIdx.x == 0) lam[blockIdx.x] = damp * (s / (double)C);
}

// Hd[i][j] = H[C-1-i][C-1-j] + lambda [i == j], in fp64 (lower triangle).
__global__ void __launch_bounds__(256)
    gptq_prepare_kernel(const float *H, int64_t C, const double *lam, double *Hd) {
  const int64_t b = blockIdx.y;
  const float *Hb = H + b * C * C;
  double *Db = Hd + b * C * C;
  const double l = lam[b];
  const int64_t n = C * C;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = idx / C, j = idx - i * C;
    if (j > i) continue;
    double v = (double)Hb[(C - 1 - i) * C + (C - 1 - j)];
    if (i == j) v += l;
    Db[idx] = v;
  }
}

// E2M1 magnitude index of |x| / s for an fp64 x: the count of midpoints
// mu_i s below |x| (ties to the even index), exact since mu_i s is exact in
// fp64; 0 when s is not positive.
__device__ __forceinline__ int e2m1_index64(double a, double s) {
  if (!(s > 0.0)) return 0;
  return (a > 0.25 * s) + (a >= 0.75 * s) + (a > 1.25 * s) + (a >= 1.75 * s) + (a > 2.5 * s) +
         (a >= 3.5 * s) + (a > 5.0 * s);
}

__device__ __forceinline__ double e2m1_magnitude(int k) {
  return k < 2 ? 0.5 * k : (1.0 + 0.5 * (double)(k & 1)) * (double)(1 << ((k >> 1) - 1));
}

// Columns c0 .. c0+nw-1 of every row: the value at rounding, its code, and
// the error w - q written over the consumed running sum.  L is the lower
// Cholesky factor of the reversed Hessian: T[i][j] = L[C-1-i][C-1-j].
__global__ void __launch_bounds__(kRowThreads)
    gptq_block_kernel(const uint16_t *__restrict__ w, int64_t R, int64_t C,
                      const float *__restrict__ s_g, const uint8_t *__restrict__ codes,
                      const double *__restrict__ L, double *__restrict__ SD,
                      uint8_t *__restrict__ packed, int64_t c0, int nw) {
  const int64_t b = blockIdx.y;
  __shared__ double T[kPanel][kPanel + 1];  // T[c0 + j][c0 + k], j <= k
  const double *Lb = L + b * C * C;
  for (int idx = threadIdx.x; idx < kPanel * kPanel; idx += kRowThreads) {
    const int j = idx / kPanel, k = idx % kPanel;
    T[j][k] = (j <= k && k < nw) ? Lb[(C - 1 - c0 - j) * C + (C - 1 - c0 - k)] : 0.0;
  }
  __syncthreads();
  const int64_t r = (int64_t)blockIdx.x * kRowThreads + threadIdx.x;
  if (r >= R) return;
  const float sg = s_g[b];
  const int64_t row = b * R + r;
  const uint16_t *wr = w + row * C;
  double *sd = SD + row * C;
  const uint8_t *cr = codes + row * (C / kBlock);
  uint8_t *pr = packed + row * (C / 2);
  double d[kPanel];
  uint32_t lo = 0;
#pragma unroll
  for (int k = 0; k < kPanel; ++k) {
    if (k < nw) {
      const int64_t col = c0 + k;
      double acc = sd[col];
#pragma unroll
      for (int j = 0; j < k; ++j) acc = fma(d[j], T[j][k], acc);
      const double wk = (double)__uint_as_float((uint32_t)wr[col] << 16);
      const double x = wk + acc / T[k][k];
      const double s = (double)effective_scale(sg, cr[col / kBlock]);
      const int kq = e2m1_index64(fabs(x), s);
      const double q = e2m1_magnitude(kq) * s;
      const bool neg = signbit(x);
      d[k] = wk - (neg ? -q : q);
      sd[col] = d[k];
      const uint32_t code = (uint32_t)kq | (neg ? 8u : 0u);
      if (k & 1) pr[col >> 1] = (uint8_t)(lo | (code << 4));
      else lo = code;
    } else {
      d[k] = 0.0;
    }
  }
}

}  // namespace

cudaError_t launch_gptq(const uint16_t *w, int64_t batch, int64_t R, int64_t C, const float *s_g,
                        const uint8_t *codes, const float *H, double damp, uint8_t *packed,
                        cudaStream_t st) {
  if (R == 0 || C == 0) return cudaSuccess;
  // scratch: lambda | Hd (-> its factor) | running sums / errors
  const size_t lam_bytes = ((size_t)batch * sizeof(double) + 255) / 256 * 256;
  const size_t hd_bytes = (size_t)batch * (size_t)C * (size_t)C * sizeof(double);
  const size_t sd_bytes = (size_t)batch * (size_t)R * (size_t)C * sizeof(double);
  unsigned char *scratch = nullptr;
  cudaError_t e = scratch_alloc(reinterpret_cast<void **>(&scratch), lam_bytes + hd_bytes + sd_bytes,
                                st);
  if (e != cudaSuccess) return e;
  double *lam = reinterpret_cast<double *>(scratch);
  double *Hd = reinterpret_cast<double *>(scratch + lam_bytes);
  double *SD = reinterpret_cast<double *>(scratch + lam_bytes + hd_bytes);
  e = cudaMemsetAsync(SD, 0, sd_bytes, st);
  if (e == cudaSuccess) {
    gptq_lambda_kernel<<<(unsigned)batch, 32, 0, st>>>(H, C, damp, lam);
    const int64_t n = C * C;
    int64_t gx = (n + 255) / 256;
    if (gx > (int64_t)sm_count() * 8) gx = (int64_t)sm_count() * 8;
    gptq_prepare_kernel<<<dim3((unsigned)gx, (unsigned)batch), 256, 0, st>>>(H, C, lam, Hd);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cholesky_in_place(Hd, C, batch, st);
  for (int64_t c0 = 0; e == cudaSuccess && c0 < C; c0 += kPanel) {
    const int nw = (int)(C - c0 < kPanel ? C - c0 : kPanel);
    const dim3 grid((unsigned)((R + kRowThreads - 1) / kRowThreads), (unsigned)batch);
    gptq_block_kernel<<<grid, kRowThreads, 0, st>>>(w, R, C, s_g, codes, Hd, SD, packed, c0, nw);
    e = cudaGetLastError();
    const int64_t c1 = c0 + nw;
    if (e == cudaSuccess && c1 < C) {
      // running sums of columns c1.. += errors of this block x rows c0.. of T
      GemmF64 g;
      g.M = R; g.N = C - c1; g.K = nw; g.alpha = 1.0;
      g.A = SD + c0; g.sAm = C; g.sAk = 1; g.bsA = R * C;
      g.B = Hd + (C - 1 - c0) * C + (C - 1 - c1); g.sBk = -C; g.sBn = -1; g.bsB = C * C;
      g.C = SD + c1; g.sCm = C; g.sCn = 1; g.bsC = R * C;
      g.lower = 0;
      e = gemm_f64(g, batch, st);
    }
  }
  const cudaError_t ef = scratch_free(scratch, st);
  return e != cudaSuccess ? e : ef;
}

cudaError_t read_and_clear_gptq_status(cudaStream_t st, int *out) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_gptq_status, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && *out != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_gptq_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  }
  return e;
}

}  // namespace nvfp4
