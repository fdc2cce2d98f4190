// Chained launches (programmatic dependent launch).
//
// Within an API call, every kernel after the first is launched with
// programmatic stream serialisation: its CTAs may be scheduled while the
// kernel before it is still running (once every CTA of that kernel has
// released its dependents), so its launch and the distribution of its CTAs
// overlap the previous kernel's tail instead of following it.  In exchange
// each kernel waits, in `chained_entry`, for the previous kernel to complete
// and its writes to be visible before it touches global memory that earlier
// work on the stream may write or read, and releases its dependents only
// after that wait, so the chain never runs ahead of stream order.
//
// The first kernel of a call is launched plainly (`launch_first`): it starts
// after all earlier work on the stream, its wait returns at once, and its
// release lets the call's second kernel be scheduled early.
//
// A kernel that reads, before its wait, inputs the previous kernel neither
// writes nor reads (the Local-Hessian search, whose predecessor is always
// the factor kernel of the same call) says so where it does it.
#pragma once
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

namespace nvfp4 {

// Keeps a pointer's loads after the wait.  Ordinary loads and stores, and
// volatile asm (TMA, cp.async), stay after it by its memory clobber; a
// non-volatile inline-asm load (the streaming loads, __ldcs) declares no
// memory dependence, so the pointer it reads through is passed through a
// volatile empty asm placed after the wait.
template <typename P>
__device__ __forceinline__ void after_wait(P &p) {
  uint64_t u = reinterpret_cast<uint64_t>(p);
  asm volatile("" : "+l"(u));
  p = reinterpret_cast<P>(u);
}

// Waits for the previous kernel on the stream, then lets the next one be
// scheduled; `p` are the pointers the kernel reads through non-volatile asm.
template <typename... P>
__device__ __forceinline__ void chained_entry(P &...p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  (after_wait(p), ...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_with(bool chained, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                        size_t smem, cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = chained ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// A kernel after another kernel of the same call: launched with programmatic
// stream serialisation on `st`.
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t st, Args &&...args) {
  return launch_with(true, kernel, grid, block, smem, st, std::forward<Args>(args)...);
}

// The first kernel of a call: an ordinary launch, after all earlier work on
// the stream.  (Chaining it to the caller's previous kernel let its CTAs
// take SM slots while that kernel's last wave still ran: measured slower
// across the calls of a calibration step than the chain within each call.)
template <typename... KArgs, typename... Args>
cudaError_t launch_first(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                         cudaStream_t st, Args &&...args) {
  return launch_with(false, kernel, grid, block, smem, st, std::forward<Args>(args)...);
}

}  // namespace nvfp4
