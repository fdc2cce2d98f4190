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
//  - chol_block_kernel and the fp64 GEMM: blocked right-looking Cholesky of
//    Hd in place, 128-column panels (the diagonal block factored and
//    inverted by one CTA, the rows below it solved by a GEMM with that
//    inverse, the trailing matrix by a rank-128 update split so that most of
//    it overlaps the next panel on a second stream);
//  - gptq_block_kernel: 128 columns at a time, sixteen lanes per row each
//    holding 8 columns' running sums in registers; each column is rounded
//    by its owner lane (exact fp64 midpoint test), its error shuffled to the
//    row's lanes and added times T to the later columns' sums; the errors
//    w_j - q_j replace the consumed sums;
//  - the fp64 GEMM (fp64 tensor-core MMA) again: each block's errors times
//    the next rows of T, added to the running sums of every later column
//    (lazy batch updates, rank 128).
#include <cmath>
#include <mutex>

#include "chained.cuh"
#include "common.cuh"
#include "internal.h"
#include "../../include/nvfp4.h"

namespace nvfp4 {

// Sticky status of the GPTQ kernels (a Hessian that is not positive
// definite after dampening), read with the library status.
__device__ int g_gptq_status = 0;

namespace {

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
  int lower;      // skip tiles wholly above the diagonal
  int overwrite;  // C = alpha A B (C is not read)
};

// BM x BN output tile per CTA (128 x 64 for out-of-place products, 64 x 128
// for the in-place panel solve, which must be one CTA column) on the fp64
// tensor-core instruction (mma.sync m8n8k4 f64; tcgen05 has no f64 kind):
// eight warps, each a grid of 8 x 8 accumulator tiles (32 x 32 per warp, two
// CTAs per SM).  k-slabs of 16 are
// staged in shared memory by a three-stage cp.async pipeline (8-byte copies,
// so any stride works; the unit-stride dimension is copied fastest), both
// operands stored [row][k] with a row stride of 20 doubles, which keeps the
// fragment reads (8 rows x 4 consecutive k) free of bank conflicts.
constexpr int kGK = 16, kGThreads = 256, kGStages = 3;
constexpr int kGRow = kGK + 4;  // shared-memory row stride (doubles)
template <int BM, int BN>
constexpr int gemm_smem() { return kGStages * (BM + BN) * kGRow * (int)sizeof(double); }

__device__ __forceinline__ void cp_async8(double *smem, const double *gmem, bool pred) {
  const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
  const int n = pred ? 8 : 0;  // 0: fill with zeros, read nothing
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(sa), "l"(gmem), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_1() {
  asm volatile("cp.async.wait_group 1;\n" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

// D (8x8) += A (8x4, row) B (4x8, col).  Lane l holds A[l/4][l%4],
// B[l%4][l/4] and D[l/4][2(l%4)], D[l/4][2(l%4)+1].
__device__ __forceinline__ void dmma_8x8x4(double d[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

template <int BM, int BN>
__global__ void __launch_bounds__(kGThreads, BM * BN <= 8192 ? 2 : 1)
    gemm_f64_kernel(const GemmF64 g) {
  constexpr int kGM = BM, kGN = BN;
  constexpr int kWarpsN = BN / 32, kWarpsM = 8 / kWarpsN;
  constexpr int kTm = kGM / kWarpsM / 8, kTn = 4;  // 8x8 tiles per warp
  constexpr int kACopies = kGM * kGK / kGThreads, kBCopies = kGN * kGK / kGThreads;
  const int64_t m0 = (int64_t)blockIdx.y * kGM, n0 = (int64_t)blockIdx.x * kGN;
  if (g.lower && n0 > m0 + kGM - 1) return;
  // operands arrive by cp.async (volatile asm, kept after the wait) and
  // ordinary loads
  chained_entry();
  const int64_t z = blockIdx.z;
  const double *A = g.A + z * g.bsA;
  const double *B = g.B + z * g.bsB;
  double *Cz = g.C + z * g.bsC;
  extern __shared__ __align__(16) double gsm[];
  double *As = gsm;                            // [stage][m][k]
  double *Bs = gsm + kGStages * kGM * kGRow;   // [stage][n][k]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = (warp / kWarpsN) * (kTm * 8), wn = (warp % kWarpsN) * 32;  // warp tile origin
  const int gr = lane >> 2, gc = lane & 3;
  // This thread's eight copies per operand and slab lie on one line: element
  // e sits at (row0 + e drow, k0 + kk0 + e dk) with one of drow, dk zero
  // (16 rows apart when k is the unit-stride dimension, else 2 k apart), so
  // their addresses and bounds come from a base, two steps and a row mask.
  const bool a_k_fast = g.sAk == 1 || g.sAk == -1;
  const bool b_k_fast = g.sBk == 1 || g.sBk == -1;
  const int a_r0 = a_k_fast ? tid >> 4 : tid & (kGM - 1), a_k0 = a_k_fast ? tid & 15 : tid / kGM;
  const int a_dr = a_k_fast ? 16 : 0, a_dk = a_k_fast ? 0 : kGThreads / kGM;
  const int b_r0 = b_k_fast ? tid >> 4 : tid & (kGN - 1), b_k0 = b_k_fast ? tid & 15 : tid / kGN;
  const int b_dr = b_k_fast ? 16 : 0, b_dk = b_k_fast ? 0 : kGThreads / kGN;
  const double *a_base = A + (m0 + a_r0) * g.sAm + a_k0 * g.sAk;
  const double *b_base = B + (n0 + b_r0) * g.sBn + b_k0 * g.sBk;
  const int64_t a_step = a_dr * g.sAm + a_dk * g.sAk, b_step = b_dr * g.sBn + b_dk * g.sBk;
  const int64_t a_slab = kGK * g.sAk, b_slab = kGK * g.sBk;
  const int a_soff = a_r0 * kGRow + a_k0, a_sstep = a_dr * kGRow + a_dk;
  const int b_soff = b_r0 * kGRow + b_k0, b_sstep = b_dr * kGRow + b_dk;
  uint32_t a_rows = 0, b_rows = 0;  // bit e: row of copy e in range
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    if (e < kACopies) a_rows |= (uint32_t)(m0 + a_r0 + e * a_dr < g.M) << e;
    if (e < kBCopies) b_rows |= (uint32_t)(n0 + b_r0 + e * b_dr < g.N) << e;
  }
  const int64_t nslab = (g.K + kGK - 1) / kGK;

  auto issue = [&](int64_t t) {
    if (t < nslab) {
      const int st = (int)(t % kGStages);
      const int64_t k0 = t * kGK;
      double *as = As + st * kGM * kGRow + a_soff, *bs = Bs + st * kGN * kGRow + b_soff;
      const double *pa = a_base + t * a_slab, *pb = b_base + t * b_slab;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (e < kACopies) {
          const bool oka = ((a_rows >> e) & 1u) && k0 + a_k0 + e * a_dk < g.K;
          cp_async8(as + e * a_sstep, oka ? pa + e * a_step : A, oka);
        }
        if (e < kBCopies) {
          const bool okb = ((b_rows >> e) & 1u) && k0 + b_k0 + e * b_dk < g.K;
          cp_async8(bs + e * b_sstep, okb ? pb + e * b_step : B, okb);
        }
      }
    }
    cp_async_commit();  // possibly empty: keeps the group count uniform
  };

  double acc[kTm][kTn][2];
#pragma unroll
  for (int i = 0; i < kTm; ++i)
#pragma unroll
    for (int j = 0; j < kTn; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
  issue(0);
  issue(1);
  for (int64_t t = 0; t < nslab; ++t) {
    cp_async_wait_1();  // slab t has landed (only slab t + 1 may be in flight)
    __syncthreads();
    issue(t + 2);  // into the stage read at step t - 1, finished by every thread
    const int st = (int)(t % kGStages);
    const double *as = As + st * kGM * kGRow + (wm + gr) * kGRow + gc;
    const double *bs = Bs + st * kGN * kGRow + (wn + gr) * kGRow + gc;
#pragma unroll
    for (int k4 = 0; k4 < kGK; k4 += 4) {
      double a[kTm], b[kTn];
#pragma unroll
      for (int i = 0; i < kTm; ++i) a[i] = as[i * 8 * kGRow + k4];
#pragma unroll
      for (int j = 0; j < kTn; ++j) b[j] = bs[j * 8 * kGRow + k4];
#pragma unroll
      for (int i = 0; i < kTm; ++i)
#pragma unroll
        for (int j = 0; j < kTn; ++j) dmma_8x8x4(acc[i][j], a[i], b[j]);
    }
  }
  // C += alpha acc, one accumulator row (8 values) at a time: the loads of a
  // row are issued before its stores (the compiler cannot tell that the
  // addresses differ, so a load never passes an earlier store)
#pragma unroll
  for (int i = 0; i < kTm; ++i) {
    const int64_t m = m0 + wm + i * 8 + gr;
    double cv[kTn][2];
#pragma unroll
    for (int j = 0; j < kTn; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t n = n0 + wn + j * 8 + gc * 2 + h;
        cv[j][h] = (m < g.M && n < g.N && !g.overwrite) ? Cz[m * g.sCm + n * g.sCn] : 0.0;
      }
#pragma unroll
    for (int j = 0; j < kTn; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t n = n0 + wn + j * 8 + gc * 2 + h;
        if (m < g.M && n < g.N) Cz[m * g.sCm + n * g.sCn] = fma(g.alpha, acc[i][j][h], cv[j][h]);
      }
  }
}

std::mutex g_gemm_attr_mu;
bool g_gemm_attr[64] = {};

template <int BM, int BN>
cudaError_t gemm_launch(const GemmF64 &g, int64_t batch, cudaStream_t st) {
  const dim3 grid((unsigned)((g.N + BN - 1) / BN), (unsigned)((g.M + BM - 1) / BM),
                  (unsigned)batch);
  return launch_chained(gemm_f64_kernel<BM, BN>, grid, dim3(kGThreads), gemm_smem<BM, BN>(), st,
                        g);
}

// An in-place product (C aliasing A, `overwrite`) must run as one CTA column
// (N <= 128, 128-wide tiles): every CTA reads all of its rows' A before
// writing them, and no other CTA touches those rows.  Its tiles are 64 rows
// high, so that the panel's rows spread over twice as many SMs.
cudaError_t gemm_f64(const GemmF64 &g, int64_t batch, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return cudaSuccess;
  if (g.overwrite && g.N > 128) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lk(g_gemm_attr_mu);
    if (!g_gemm_attr[dev]) {
      e = cudaFuncSetAttribute(gemm_f64_kernel<64, 128>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem<64, 128>());
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gemm_f64_kernel<128, 64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem<128, 64>());
      if (e != cudaSuccess) return e;
      g_gemm_attr[dev] = true;
    }
  }
  // 128 x 64 tiles, two CTAs per SM, hide one tile's prologue and epilogue
  // behind the other's products (measured 8% faster on the dense layer's
  // GPTQ than 128 x 128 tiles, one CTA per SM)
  if (g.overwrite) return gemm_launch<64, 128>(g, batch, st);
  return gemm_launch<128, 64>(g, batch, st);
}

// ------------------------------------------------------------------ Cholesky
// Blocked right-looking Cholesky of every batch element's matrix, in place
// (lower triangle), 128-column panels:
//  - chol_block_kernel: one CTA per batch element factors the panel's
//    diagonal block, writes the factor L_pp back and its inverse L_pp^-1 to
//    a scratch block;
//  - the rows below the block: X = A_panel L_pp^-T, one fp64 GEMM, in place;
//  - the trailing matrix: -= X X^T, one fp64 GEMM on the lower triangle.
// A pivot that is not positive (or not finite) sets the status and makes
// the factor NaN.
//
// In chol_block_kernel each of the 256 threads keeps an 8 x 8 tile of the
// block in registers: rows ty + 16 i, columns tx + 16 j (tx, ty = thread
// index mod / div 16).  Factor step k: the owners of column k publish it to
// a shared vector (double-buffered, one barrier per step), every thread
// takes the pivot p = A_kk and applies A_rc -= A_rk A_ck / p to its entries
// with k < c <= r (64 independent updates); column k is scaled by p^-1/2
// at the end.  The inverse X = L^-1 is the same pattern on the identity:
// step k finishes row k of X (scaled by 1 / L_kk) from the row's owners and
// removes it from the later rows, X_rc -= L_rk X_kc.
constexpr int kBig = 128;  // columns per Cholesky panel and per GPTQ block
constexpr int kCholThreads = 256;
constexpr int kSRow = kBig + 1;  // shared-memory row stride (doubles)
constexpr int kCholSmem = (kBig * kSRow + 4 * kBig) * (int)sizeof(double);  // 136,192 B

__global__ void __launch_bounds__(kCholThreads, 1)
    chol_block_kernel(double *A, int64_t C, int64_t P0, int nw, double *Linv) {
  chained_entry();
  extern __shared__ double csm[];
  double *Lsm = csm;                 // [kBig][kSRow], the factor
  double *vec = Lsm + kBig * kSRow;  // [2][kBig] column (factor) / row (inverse) of step k
  double *inv = vec + 2 * kBig;      // p_k^-1/2
  double *dinv = inv + kBig;         // 1 / L_kk
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  double *Ab = A + (int64_t)blockIdx.x * C * C + P0 * C + P0;
  double *Lb = Linv + (int64_t)blockIdx.x * kBig * kBig;
  double a[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = ty + 16 * i, c = tx + 16 * j;
      a[i][j] = (r < nw && c <= r) ? Ab[(int64_t)r * C + c] : 0.0;
    }
  // ---- factor.  At step k = 16 j0 + kk only rows and columns above k
  // change: tile rows and columns i, j >= j0 (j0 is a compile-time constant
  // of each unrolled copy), and within them the zeroed multipliers of rows
  // and columns <= k leave entries as they are.  Entries above the diagonal
  // take products too and are never read.
#pragma unroll
  for (int j0 = 0; j0 < 8; ++j0) {
    for (int kk = 0; kk < 16; ++kk) {
      const int k = 16 * j0 + kk;
      if (k >= nw) break;
      double *col = vec + (k & 1) * kBig;
      if (tx == kk) {
#pragma unroll
        for (int i = j0; i < 8; ++i) {
          const int r = ty + 16 * i;
          if (r >= k) col[r] = a[i][j0];
        }
      }
      __syncthreads();
      const double p = col[k];
      const bool ok = p > 0.0 && p < INFINITY;
      const double iv = ok ? rsqrt(p) : __longlong_as_double(0x7FF8000000000000LL);
      if (tid == 0) {
        inv[k] = iv;
        if (!ok) atomicExch(&g_gptq_status, (int)NVFP4_ERR_NOT_POSITIVE_DEFINITE);
      }
      const double iv2 = iv * iv;
      double cr[8], cc[8];
#pragma unroll
      for (int i = j0; i < 8; ++i) {
        const int r = ty + 16 * i, c = tx + 16 * i;
        cr[i] = r > k && r < nw ? col[r] * iv2 : 0.0;
        cc[i] = c > k && c < nw ? col[c] : 0.0;
      }
#pragma unroll
      for (int i = j0; i < 8; ++i)
#pragma unroll
        for (int j = j0; j < 8; ++j) a[i][j] = fma(-cr[i], cc[j], a[i][j]);
    }
  }
  __syncthreads();
  // scale the columns, write the factor back and keep it in shared memory
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = ty + 16 * i, c = tx + 16 * j;
      if (r < nw && c <= r) {
        const double l = a[i][j] * inv[c];
        Lsm[r * kSRow + c] = l;
        Ab[(int64_t)r * C + c] = l;
      }
    }
  __syncthreads();
  for (int k = tid; k < nw; k += kCholThreads) dinv[k] = 1.0 / Lsm[k * kSRow + k];
  // ---- inverse: identity in the registers, rows finished in order
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) a[i][j] = (ty + 16 * i == tx + 16 * j) ? 1.0 : 0.0;
  __syncthreads();
  // At step k = 16 i0 + kk only rows below k (tile rows i >= i0) take
  // X_rc -= L_rk X_kc, and only in columns c <= k (tile columns j <= i0).
#pragma unroll
  for (int i0 = 0; i0 < 8; ++i0) {
    for (int kk = 0; kk < 16; ++kk) {
      const int k = 16 * i0 + kk;
      if (k >= nw) break;
      double *row = vec + (k & 1) * kBig;
      if (ty == kk) {
        const double d = dinv[k];
#pragma unroll
        for (int j = 0; j <= i0; ++j) {
          const int c = tx + 16 * j;
          if (c <= k) {
            a[i0][j] *= d;
            row[c] = a[i0][j];
          }
        }
      }
      __syncthreads();
      double xr[8], lr[8];
#pragma unroll
      for (int j = 0; j <= i0; ++j) {
        const int c = tx + 16 * j;
        xr[j] = c <= k ? row[c] : 0.0;
      }
#pragma unroll
      for (int i = i0; i < 8; ++i) {
        const int r = ty + 16 * i;
        lr[i] = r > k && r < nw ? Lsm[r * kSRow + k] : 0.0;
      }
#pragma unroll
      for (int i = i0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j <= i0; ++j) a[i][j] = fma(-lr[i], xr[j], a[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = ty + 16 * i, c = tx + 16 * j;
      Lb[r * kBig + c] = (r < nw && c <= r) ? a[i][j] : 0.0;
    }
}

std::mutex g_chol_attr_mu;
bool g_chol_attr[64] = {};

template <class K>
cudaError_t ensure_smem_attr(K kernel, int bytes, std::mutex &mu, bool *flags) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (!flags[dev]) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    flags[dev] = true;
  }
  return cudaSuccess;
}

// Linv: scratch [batch][128][128].
// Look-ahead: each panel's trailing update is split into the next panel's
// 128 columns, on the caller's stream, and the columns beyond, on a second
// stream, where it overlaps the next panel's factor and solve.  The next
// panel's own split update waits for it (both write the columns after the
// next panel); everything else they touch is disjoint.
cudaError_t cholesky_in_place(double *A, int64_t C, int64_t batch, double *Linv,
                              cudaStream_t st) {
  cudaError_t e = ensure_smem_attr(chol_block_kernel, kCholSmem, g_chol_attr_mu, g_chol_attr);
  if (e != cudaSuccess) return e;
  const int64_t CC = C * C;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_main = nullptr, ev_side = nullptr;
  e = cudaStreamCreateWithFlags(&side, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_main, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_side, cudaEventDisableTiming);
  bool side_used = false;
  // A[r0.., r0 .. r0+ncols) -= X X^T on the lower triangle, X = the panel's
  // rows r0.. in its columns P0 .. P0+nw
  auto trailing = [&](int64_t P0, int nw, int64_t r0, int64_t ncols, cudaStream_t s) {
    GemmF64 g{};
    g.M = C - r0; g.N = ncols; g.K = nw; g.alpha = -1.0;
    g.A = A + r0 * C + P0; g.sAm = C; g.sAk = 1; g.bsA = CC;
    g.B = g.A; g.sBk = 1; g.sBn = C; g.bsB = CC;
    g.C = A + r0 * C + r0; g.sCm = C; g.sCn = 1; g.bsC = CC;
    g.lower = 1;
    return gemm_f64(g, batch, s);
  };
  for (int64_t P0 = 0; e == cudaSuccess && P0 < C; P0 += kBig) {
    const int nw = (int)(C - P0 < kBig ? C - P0 : kBig);
    e = launch_chained(chol_block_kernel, dim3((unsigned)batch), dim3(kCholThreads), kCholSmem, st,
                       A, C, P0, nw, Linv);
    const int64_t P1 = P0 + nw, rest = C - P1;
    if (e != cudaSuccess || rest <= 0) break;
    {
      // rows below the block: X = A_panel L_pp^-T (in place: one CTA column)
      GemmF64 g{};
      g.M = rest; g.N = nw; g.K = nw; g.alpha = 1.0;
      g.A = A + P1 * C + P0; g.sAm = C; g.sAk = 1; g.bsA = CC;
      g.B = Linv; g.sBk = 1; g.sBn = kBig; g.bsB = (int64_t)kBig * kBig;
      g.C = A + P1 * C + P0; g.sCm = C; g.sCn = 1; g.bsC = CC;
      g.overwrite = 1;
      e = gemm_f64(g, batch, st);
    }
    // the next panel's columns, after the earlier panels' updates beyond them
    if (e == cudaSuccess && side_used) e = cudaStreamWaitEvent(st, ev_side, 0);
    const int64_t nw2 = rest < kBig ? rest : kBig, P2 = P1 + nw2;
    if (e == cudaSuccess) e = trailing(P0, nw, P1, nw2, st);
    if (e == cudaSuccess && C - P2 > 0) {
      e = cudaEventRecord(ev_main, st);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(side, ev_main, 0);
      if (e == cudaSuccess) e = trailing(P0, nw, P2, C - P2, side);
      if (e == cudaSuccess) e = cudaEventRecord(ev_side, side);
      side_used = side_used || e == cudaSuccess;
    }
  }
  // join the second stream before anything reads the factor
  if (side_used) {
    const cudaError_t ej = cudaStreamWaitEvent(st, ev_side, 0);
    if (e == cudaSuccess) e = ej;
  }
  if (ev_main) cudaEventDestroy(ev_main);
  if (ev_side) cudaEventDestroy(ev_side);
  if (side) cudaStreamDestroy(side);
  return e;
}

// ---------------------------------------------------------------------- GPTQ
// lambda = damp * mean(diag H), the diagonal summed in a fixed order.
__global__ void __launch_bounds__(32)
    gptq_lambda_kernel(const float *H, int64_t C, double damp, double *lam) {
  chained_entry();
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
  chained_entry();
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

// Columns c0 .. c0+nw-1 (nw <= 128) of every row: the value at rounding,
// its code, and the error w - q written over the consumed running sum.  L is
// the lower Cholesky factor of the reversed Hessian: T[i][j] = L[C-1-i][C-1-j].
// kLanes lanes take one row, lane q the columns kCols q .. kCols q + kCols - 1
// of the block (kCols = 128 / kLanes) with their running sums in registers.
// Column k = kCols q0 + kk is rounded by its owner lane, whose error goes to
// the row's lanes by a shuffle; then every lane adds error x T[k][m] to the
// running sums of its columns m > k (independent updates: the dependent chain
// per column is one fma and the rounding).  The block of T (upper triangle)
// sits in shared memory, one copy per CTA of kRowsPerCta rows, each lane's
// chunk of a row followed by one double of padding: at every step the lanes
// of a row read one element of each chunk, kCols + 1 doubles apart, which
// puts them in distinct banks (kCols apart they all shared one).
constexpr int kRowsPerCta = 32;
template <int kLanes>
__host__ __device__ constexpr int block_row_stride() { return kBig + kLanes; }  // doubles
template <int kLanes>
constexpr int block_smem() {
  return (kBig * block_row_stride<kLanes>() + kBig) * (int)sizeof(double);
}

template <int kLanes>
__global__ void __launch_bounds__(kLanes * kRowsPerCta)
    gptq_block_kernel(const uint16_t *__restrict__ w, int64_t R, int64_t C,
                      const float *__restrict__ s_g, const uint8_t *__restrict__ codes,
                      const double *__restrict__ L, double *__restrict__ SD,
                      uint8_t *__restrict__ packed, int64_t c0, int nw) {
  constexpr int kThreadsB = kLanes * kRowsPerCta;
  constexpr int kCols = kBig / kLanes;  // columns per lane
  constexpr int kTS = block_row_stride<kLanes>();
  static_assert(kCols % 8 == 0, "a lane's columns are whole packed words");
  chained_entry();
  extern __shared__ double bsm[];
  double *T = bsm;                // [j][k + k / kCols], j <= k
  double *Tinv = T + kBig * kTS;  // 1 / T[k][k]
  const int64_t b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, q = lane & (kLanes - 1);
  const double *Lb = L + b * C * C;
  // stage T (upper triangle, zeros elsewhere) with asynchronous copies
  for (int idx = tid; idx < kBig * kBig; idx += kThreadsB) {
    const int j = idx / kBig, k = idx - j * kBig;
    const bool in = j <= k && k < nw;
    cp_async8(T + j * kTS + k + k / kCols, in ? Lb + (C - 1 - c0 - j) * C + (C - 1 - c0 - k) : Lb,
              in);
  }
  cp_async_commit();
  const int64_t r = (int64_t)blockIdx.x * kRowsPerCta + tid / kLanes;
  const bool live = r < R;
  const int64_t row = b * R + (live ? r : 0);
  const int cq = kCols * q;               // first column of this lane
  const int ncols = nw - cq;              // columns of this lane inside the block
  double *sd = SD + row * C + c0 + cq;
  const uint16_t *wr = w + row * C + c0 + cq;
  double S[kCols];
  uint32_t wv[kCols / 2];  // the lane's bf16 weights, two per word
#pragma unroll
  for (int m = 0; m < kCols; ++m) S[m] = (live && m < ncols) ? sd[m] : 0.0;
#pragma unroll
  for (int m = 0; m < kCols / 2; ++m)
    wv[m] = (live && 2 * m < ncols) ? *reinterpret_cast<const uint32_t *>(wr + 2 * m) : 0u;
  const float sg = s_g[b];
  const uint8_t *cr = codes + row * (C / kBlock) + (c0 + cq) / kBlock;
  // the scales of the lane's columns (one per 16; one for kCols <= 16) and,
  // per scale, the E2M1 rounding thresholds and grid values times it (exact
  // in fp64), so that a column's rounding is seven compares and a select
  // chain (the dependent chain from one column to the next is its fp64
  // fmas, one compare, one subtraction and the shuffle)
  constexpr int kScales = (kCols + kBlock - 1) / kBlock;
  double thr[kScales][7], val[kScales][8];
#pragma unroll
  for (int i = 0; i < kScales; ++i) {
    const double sc = (live && ncols > kBlock * i) ? (double)effective_scale(sg, cr[i]) : 0.0;
    const double tf[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
    const double vf[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    // no scale (s = 0, or not a number): every test fails, index 0
    const double nan = __longlong_as_double(0x7FF8000000000000LL);
#pragma unroll
    for (int j = 0; j < 7; ++j) thr[i][j] = sc > 0.0 ? tf[j] * sc : nan;
#pragma unroll
    for (int j = 0; j < 8; ++j) val[i][j] = vf[j] * sc;
  }
  cp_async_wait_all();
  __syncthreads();
  for (int k = tid; k < kBig; k += kThreadsB)
    Tinv[k] = k < nw ? 1.0 / T[k * kTS + k + k / kCols] : 0.0;
  __syncthreads();
  uint32_t pk[kCols / 8];  // the lane's codes
#pragma unroll
  for (int i = 0; i < kCols / 8; ++i) pk[i] = 0u;
  const int src = lane & ~(kLanes - 1);
  for (int q0 = 0; q0 < kLanes; ++q0) {
    if (kCols * q0 >= nw) break;
#pragma unroll
    for (int kk = 0; kk < kCols; ++kk) {
      const int k = kCols * q0 + kk;
      const bool valid = k < nw;
      // the owner lane rounds column k (every lane computes; only q == q0 keeps it)
      const double wk = (double)__uint_as_float(
          (kk & 1) ? (wv[kk >> 1] & 0xFFFF0000u) : (wv[kk >> 1] << 16));
      const double x = fma(S[kk], valid ? Tinv[k] : 0.0, wk);
      // nearest-even E2M1 magnitude index of |x| / s (ties: 0.25, 1.25, 2.5
      // and 5 go down, 0.75, 1.75 and 3.5 up; 0 where s = 0) and its value
      const double a = fabs(x);
      const double *th = thr[kk / kBlock], *vs = val[kk / kBlock];
      const bool p0 = a > th[0], p1 = a >= th[1], p2 = a > th[2], p3 = a >= th[3];
      const bool p4 = a > th[4], p5 = a >= th[5], p6 = a > th[6];
      double qv = p0 ? vs[1] : vs[0];
      qv = p1 ? vs[2] : qv;
      qv = p2 ? vs[3] : qv;
      qv = p3 ? vs[4] : qv;
      qv = p4 ? vs[5] : qv;
      qv = p5 ? vs[6] : qv;
      qv = p6 ? vs[7] : qv;
      const int kq = (int)p0 + (int)p1 + (int)p2 + (int)p3 + (int)p4 + (int)p5 + (int)p6;
      const bool neg = signbit(x);
      const double d = wk - (neg ? -qv : qv);
      if (q == q0) {
        S[kk] = d;
        pk[kk >> 3] |= ((uint32_t)kq | (neg ? 8u : 0u)) << (4 * (kk & 7));
      }
      const double e = valid ? __shfl_sync(0xFFFFFFFFu, d, src | q0) : 0.0;
      // running sums of the later columns of the row
      const double *Tk = T + k * kTS + cq + q;
#pragma unroll
      for (int m = 0; m < kCols; ++m) {
        const bool later = q > q0 || (q == q0 && m > kk);
        if (later) S[m] = fma(e, Tk[m], S[m]);
      }
    }
  }
  if (!live) return;
#pragma unroll
  for (int m = 0; m < kCols; ++m)
    if (m < ncols) sd[m] = S[m];
  // byte stores: a row of packed codes starts on any 8-byte boundary
  uint8_t *pr = packed + row * (C / 2) + (c0 + cq) / 2;
#pragma unroll
  for (int i = 0; i < kCols / 2; ++i)
    if (2 * i < ncols) pr[i] = (uint8_t)(pk[i >> 2] >> (8 * (i & 3)));
}

// lanes per row of the column-block kernel: sixteen (eight columns each, 16
// warps per SM) measured 4% faster on the dense layer's GPTQ than four (32
// columns each, 4 warps per SM, latency-bound on each column's chain) and
// eight, with the padded T rows; without the padding the lanes' reads of T
// shared one bank and more lanes were slower
constexpr int kBlockLanes = 16;

std::mutex g_block_attr_mu;
bool g_block_attr[64] = {};

}  // namespace

cudaError_t launch_gptq(const uint16_t *w, int64_t batch, int64_t R, int64_t C, const float *s_g,
                        const uint8_t *codes, const float *H, double damp, uint8_t *packed,
                        cudaStream_t st) {
  if (R == 0 || C == 0) return cudaSuccess;
  // scratch: lambda | Hd (-> its factor) | running sums / errors | the
  // inverse of the current 128-column diagonal block
  const size_t lam_bytes = ((size_t)batch * sizeof(double) + 255) / 256 * 256;
  const size_t hd_bytes = (size_t)batch * (size_t)C * (size_t)C * sizeof(double);
  const size_t sd_bytes = (size_t)batch * (size_t)R * (size_t)C * sizeof(double);
  const size_t li_bytes = (size_t)batch * kBig * kBig * sizeof(double);
  unsigned char *scratch = nullptr;
  cudaError_t e = scratch_alloc(reinterpret_cast<void **>(&scratch),
                                lam_bytes + hd_bytes + sd_bytes + li_bytes, st);
  if (e != cudaSuccess) return e;
  double *lam = reinterpret_cast<double *>(scratch);
  double *Hd = reinterpret_cast<double *>(scratch + lam_bytes);
  double *SD = reinterpret_cast<double *>(scratch + lam_bytes + hd_bytes);
  double *Linv = reinterpret_cast<double *>(scratch + lam_bytes + hd_bytes + sd_bytes);
  e = cudaMemsetAsync(SD, 0, sd_bytes, st);
  if (e == cudaSuccess) {
    e = launch_first(gptq_lambda_kernel, dim3((unsigned)batch), dim3(32), 0, st, H, C, damp, lam);
    const int64_t n = C * C;
    int64_t gx = (n + 255) / 256;
    if (gx > (int64_t)sm_count() * 8) gx = (int64_t)sm_count() * 8;
    if (e == cudaSuccess)
      e = launch_chained(gptq_prepare_kernel, dim3((unsigned)gx, (unsigned)batch), dim3(256), 0,
                         st, H, C, static_cast<const double *>(lam), Hd);
  }
  if (e == cudaSuccess) e = cholesky_in_place(Hd, C, batch, Linv, st);
  // columns in blocks of 128: each row of a block on kBlockLanes lanes, then the
  // block's errors added to the running sums of every later column (rank-128)
  if (e == cudaSuccess)
    e = ensure_smem_attr(gptq_block_kernel<kBlockLanes>, block_smem<kBlockLanes>(),
                         g_block_attr_mu, g_block_attr);
  const int64_t RC = R * C, CC = C * C;
  for (int64_t c0 = 0; e == cudaSuccess && c0 < C; c0 += kBig) {
    const int nw = (int)(C - c0 < kBig ? C - c0 : kBig);
    const dim3 grid((unsigned)((R + kRowsPerCta - 1) / kRowsPerCta), (unsigned)batch);
    e = launch_chained(gptq_block_kernel<kBlockLanes>, grid, dim3(kBlockLanes * kRowsPerCta),
                       block_smem<kBlockLanes>(), st, w, R, C, s_g, codes,
                       static_cast<const double *>(Hd), SD,
                       packed, c0, nw);
    const int64_t c1 = c0 + nw;
    if (e == cudaSuccess && c1 < C) {
      // SD[:, c1:] += SD[:, c0:c1] T[c0:c1, c1:], T[i][j] = Hd[C-1-i][C-1-j]
      GemmF64 g{};
      g.M = R; g.N = C - c1; g.K = nw; g.alpha = 1.0;
      g.A = SD + c0; g.sAm = C; g.sAk = 1; g.bsA = RC;
      g.B = Hd + (C - 1 - c0) * C + (C - 1 - c1); g.sBk = -C; g.sBn = -1; g.bsB = CC;
      g.C = SD + c1; g.sCm = C; g.sCn = 1; g.bsC = RC;
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
