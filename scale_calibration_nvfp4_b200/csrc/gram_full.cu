// Full Gram accumulation H += X^T X over all C channels (the Local-Hessian
// write-up, "A different objective": the output-error Hessian is X X^T with
// X channels-by-tokens; "Trying it": GPTQ, which that page combines with
// Local-Hessian scales, needs the whole matrix, not only its 16x16 diagonal
// blocks).
//
// X is tokens-by-channels [N, C] row-major bf16, so X^T X is a dense
// contraction over the N tokens: it runs on the fifth-generation tensor
// cores as a CUTLASS/CuTe sm100 GEMM (tcgen05.mma with bf16 operands staged
// by TMA, fp32 accumulation in tensor memory, 128x256x64 tiles on one SM, no
// cluster multicast).  Both operands are X itself: A = X^T is C x N with the
// channel index contiguous (column-major), B = X is N x C with the channel
// index contiguous (row-major).  The epilogue adds the product to H in fp32
// (D = A B + H, in place).
#include <cute/tensor.hpp>
#include <cutlass/cutlass.h>
#include <cutlass/epilogue/collective/collective_builder.hpp>
#include <cutlass/gemm/collective/collective_builder.hpp>
#include <cutlass/gemm/device/gemm_universal_adapter.h>
#include <cutlass/gemm/kernel/gemm_universal.hpp>
#include <cutlass/util/packed_stride.hpp>

#include "internal.h"

namespace nvfp4 {
namespace {

using namespace cute;

using ElementAB = cutlass::bfloat16_t;
using LayoutATag = cutlass::layout::ColumnMajor;  // X^T: element (c, t) at t * C + c
using LayoutBTag = cutlass::layout::RowMajor;     // X:   element (t, c) at t * C + c
using ElementCD = float;
using LayoutCDTag = cutlass::layout::RowMajor;
constexpr int kAlignAB = 8;  // bf16 values per 16 bytes
constexpr int kAlignCD = 4;
using ElementAccumulator = float;
using MmaTileShape = Shape<_128, _256, _64>;
using ClusterShape = Shape<_1, _1, _1>;

using CollectiveEpilogue = typename cutlass::epilogue::collective::CollectiveBuilder<
    cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, MmaTileShape, ClusterShape,
    cutlass::epilogue::collective::EpilogueTileAuto, ElementAccumulator, ElementAccumulator,
    ElementCD, LayoutCDTag, kAlignCD, ElementCD, LayoutCDTag, kAlignCD,
    cutlass::epilogue::collective::EpilogueScheduleAuto>::CollectiveOp;

using CollectiveMainloop = typename cutlass::gemm::collective::CollectiveBuilder<
    cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, ElementAB, LayoutATag, kAlignAB,
    ElementAB, LayoutBTag, kAlignAB, ElementAccumulator, MmaTileShape, ClusterShape,
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

}  // namespace

cudaError_t launch_gram_full(const uint16_t *x, int64_t n_tok, int64_t C, float *H,
                             cudaStream_t st) {
  if (n_tok == 0 || C == 0) return cudaSuccess;
  const int M = (int)C, N = (int)C, K = (int)n_tok;
  const StrideA sa = cutlass::make_cute_packed_stride(StrideA{}, {M, K, 1});
  const StrideB sb = cutlass::make_cute_packed_stride(StrideB{}, {N, K, 1});
  const StrideC sc = cutlass::make_cute_packed_stride(StrideC{}, {M, N, 1});
  const StrideD sd = cutlass::make_cute_packed_stride(StrideD{}, {M, N, 1});
  const auto *xp = reinterpret_cast<const ElementAB *>(x);
  typename Gemm::Arguments args{cutlass::gemm::GemmUniversalMode::kGemm,
                                {M, N, K, 1},
                                {xp, sa, xp, sb},
                                {{1.0f, 1.0f}, H, sc, H, sd}};
  const size_t ws_bytes = Gemm::get_workspace_size(args);
  void *ws = nullptr;
  cudaError_t e = cudaSuccess;
  if (ws_bytes) {
    e = scratch_alloc(&ws, ws_bytes, st);
    if (e != cudaSuccess) return e;
  }
  Gemm gemm;
  if (gemm.can_implement(args) != cutlass::Status::kSuccess) e = cudaErrorNotSupported;
  else if (gemm.initialize(args, ws, st) != cutlass::Status::kSuccess) e = cudaErrorLaunchFailure;
  else if (gemm.run(st) != cutlass::Status::kSuccess) e = cudaErrorLaunchFailure;
  if (e == cudaSuccess) e = cudaGetLastError();
  const cudaError_t ef = ws ? scratch_free(ws, st) : cudaSuccess;
  return e != cudaSuccess ? e : ef;
}

}  // namespace nvfp4
