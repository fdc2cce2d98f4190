// NVFP4 x NVFP4 matrix product on the fifth-generation tensor cores: the
// consumer of the packed codes, block codes and tensor scales this library
// produces (the W4A4 serving write-up: weights and activations both NVFP4;
// Baseten, "What makes high-quality NVFP4", "Block scaling": a value is its
// E2M1 code times its block scale times the tensor scale).
//
//   Y[m][n] = s_ga s_gb sum_k (v(a_mk) e4m3(ca_m,k/16)) (v(b_nk) e4m3(cb_n,k/16))
//
// A [M, K] and B [N, K] are row-major with K contiguous (activations times
// weights^T).  The product runs as a CUTLASS/CuTe sm100 block-scaled GEMM
// (tcgen05.mma with E2M1 operands and one UE4M3 scale per 16 values along K,
// fp32 accumulation in tensor memory, TMA loads, 128x256x256 tiles on one
// SM, no cluster multicast); the scale codes are first moved from the
// library's row-major [rows][K/16] layout into the interleaved layout the
// MMA reads scales in (128-row x 4-scale atoms), and s_ga s_gb is applied in
// the epilogue before the bf16 store.
#include <cute/tensor.hpp>
#include <cutlass/cutlass.h>
#include <cutlass/detail/sm100_blockscaled_layout.hpp>
#include <cutlass/epilogue/collective/collective_builder.hpp>
#include <cutlass/gemm/collective/collective_builder.hpp>
#include <cutlass/gemm/device/gemm_universal_adapter.h>
#include <cutlass/gemm/kernel/gemm_universal.hpp>
#include <cutlass/util/packed_stride.hpp>

#include "chained.cuh"
#include "internal.h"

namespace nvfp4 {
namespace {

using namespace cute;

using ElementA = cutlass::nv_float4_t<cutlass::float_e2m1_t>;
using ElementB = cutlass::nv_float4_t<cutlass::float_e2m1_t>;
using LayoutATag = cutlass::layout::RowMajor;     // A [M, K], K contiguous
using LayoutBTag = cutlass::layout::ColumnMajor;  // B as K x N with K contiguous: [N, K]
using ElementD = cutlass::bfloat16_t;
using LayoutDTag = cutlass::layout::RowMajor;
constexpr int kAlignAB = 32;  // E2M1 values per 16 bytes
constexpr int kAlignD = 128 / cutlass::sizeof_bits<ElementD>::value;
using ElementAccumulator = float;
using MmaTileShape = Shape<_128, _256, _256>;
using ClusterShape = Shape<_1, _1, _1>;

using CollectiveEpilogue = typename cutlass::epilogue::collective::CollectiveBuilder<
    cutlass::arch::Sm100, cutlass::arch::OpClassBlockScaledTensorOp, MmaTileShape, ClusterShape,
    cutlass::epilogue::collective::EpilogueTileAuto, ElementAccumulator, ElementAccumulator,
    void, LayoutDTag, kAlignD, ElementD, LayoutDTag, kAlignD,
    cutlass::epilogue::collective::EpilogueScheduleAuto>::CollectiveOp;

using CollectiveMainloop = typename cutlass::gemm::collective::CollectiveBuilder<
    cutlass::arch::Sm100, cutlass::arch::OpClassBlockScaledTensorOp, ElementA, LayoutATag,
    kAlignAB, ElementB, LayoutBTag, kAlignAB, ElementAccumulator, MmaTileShape, ClusterShape,
    cutlass::gemm::collective::StageCountAutoCarveout<static_cast<int>(
        sizeof(typename CollectiveEpilogue::SharedStorage))>,
    cutlass::gemm::collective::KernelScheduleAuto>::CollectiveOp;

using GemmKernel = cutlass::gemm::kernel::GemmUniversal<Shape<int, int, int, int>,
                                                        CollectiveMainloop, CollectiveEpilogue,
                                                        void>;
using Gemm = cutlass::gemm::device::GemmUniversalAdapter<GemmKernel>;

using StrideA = typename GemmKernel::StrideA;
using StrideB = typename GemmKernel::StrideB;
using StrideC = typename GemmKernel::StrideC;
using StrideD = typename GemmKernel::StrideD;
using LayoutSFA = typename CollectiveMainloop::LayoutSFA;
using LayoutSFB = typename CollectiveMainloop::LayoutSFB;
using ScaleConfig = typename CollectiveMainloop::Sm1xxBlkScaledConfig;

// Block codes [rows][K/16] (row-major) -> the MMA's scale layout.  `layout`
// maps (row, k, batch) to the scale of element k of the row.
template <class Layout>
__global__ void scale_layout_kernel(const uint8_t *__restrict__ src, int64_t rows, int64_t kb,
                                    Layout layout, uint8_t *__restrict__ dst) {
  chained_entry();
  const int64_t n = rows * kb;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / kb, b = i - r * kb;
    dst[layout((int)r, (int)(b * 16), 0)] = src[i];
  }
}

__global__ void product_kernel(const float *a, const float *b, float *out) {
  chained_entry();
  *out = *a * *b;
}

int grid_for_elems(int64_t n) {
  const int64_t cap = (int64_t)sm_count() * 8;
  const int64_t need = (n + 255) / 256;
  return (int)(need < 1 ? 1 : (need < cap ? need : cap));
}

}  // namespace

cudaError_t launch_gemm_fp4(const uint8_t *a_packed, const uint8_t *a_codes, const float *a_sg,
                            const uint8_t *b_packed, const uint8_t *b_codes, const float *b_sg,
                            int64_t M, int64_t N, int64_t K, uint16_t *out, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  const auto problem = make_shape((int)M, (int)N, (int)K, 1);
  const LayoutSFA lsfa = ScaleConfig::tile_atom_to_shape_SFA(problem);
  const LayoutSFB lsfb = ScaleConfig::tile_atom_to_shape_SFB(problem);
  const size_t nsfa = (size_t)size(filter_zeros(lsfa));
  const size_t nsfb = (size_t)size(filter_zeros(lsfb));
  const StrideA sa = cutlass::make_cute_packed_stride(StrideA{}, {(int)M, (int)K, 1});
  const StrideB sb = cutlass::make_cute_packed_stride(StrideB{}, {(int)N, (int)K, 1});
  const StrideC sc = cutlass::make_cute_packed_stride(StrideC{}, {(int)M, (int)N, 1});
  const StrideD sd = cutlass::make_cute_packed_stride(StrideD{}, {(int)M, (int)N, 1});

  auto round256 = [](size_t x) { return (x + 255) / 256 * 256; };
  typename Gemm::Arguments args{
      cutlass::gemm::GemmUniversalMode::kGemm,
      {(int)M, (int)N, (int)K, 1},
      {reinterpret_cast<typename ElementA::DataType const *>(a_packed), sa,
       reinterpret_cast<typename ElementB::DataType const *>(b_packed), sb, nullptr, lsfa,
       nullptr, lsfb},
      {{1.0f, 0.0f}, nullptr, sc, reinterpret_cast<ElementD *>(out), sd}};
  const size_t ws_bytes = Gemm::get_workspace_size(args);
  // scratch: alpha | scales of A | scales of B | GEMM workspace
  const size_t off_sfa = 256, off_sfb = off_sfa + round256(nsfa);
  const size_t off_ws = off_sfb + round256(nsfb);
  unsigned char *scratch = nullptr;
  cudaError_t e = scratch_alloc(reinterpret_cast<void **>(&scratch), off_ws + ws_bytes + 256, st);
  if (e != cudaSuccess) return e;
  float *alpha = reinterpret_cast<float *>(scratch);
  uint8_t *sfa = scratch + off_sfa;
  uint8_t *sfb = scratch + off_sfb;
  // padding of the scale atoms must hold zero scales (never NaN codes)
  e = cudaMemsetAsync(sfa, 0, off_ws - off_sfa, st);
  if (e == cudaSuccess) {
    // (the CUTLASS GEMM below is launched plainly: its own grid-dependency
    // wait is compiled only where CUTLASS enables it)
    e = launch_first(scale_layout_kernel<LayoutSFA>, dim3(grid_for_elems(M * (K / 16))),
                       dim3(256), 0, st, a_codes, M, K / 16, lsfa, sfa);
    if (e == cudaSuccess)
      e = launch_chained(scale_layout_kernel<LayoutSFB>, dim3(grid_for_elems(N * (K / 16))),
                         dim3(256), 0, st, b_codes, N, K / 16, lsfb, sfb);
    if (e == cudaSuccess)
      e = launch_chained(product_kernel, dim3(1), dim3(1), 0, st, a_sg, b_sg, alpha);
  }
  if (e == cudaSuccess) {
    args.mainloop.ptr_SFA = reinterpret_cast<typename ElementA::ScaleFactorType const *>(sfa);
    args.mainloop.ptr_SFB = reinterpret_cast<typename ElementB::ScaleFactorType const *>(sfb);
    args.epilogue.thread.alpha_ptr = alpha;
    Gemm gemm;
    if (gemm.can_implement(args) != cutlass::Status::kSuccess) e = cudaErrorNotSupported;
    else if (gemm.initialize(args, scratch + off_ws, st) != cutlass::Status::kSuccess)
      e = cudaErrorLaunchFailure;
    else if (gemm.run(st) != cutlass::Status::kSuccess)
      e = cudaErrorLaunchFailure;
    if (e == cudaSuccess) e = cudaGetLastError();
  }
  const cudaError_t ef = scratch_free(scratch, st);
  return e != cudaSuccess ? e : ef;
}

}  // namespace nvfp4
