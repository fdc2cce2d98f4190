// Block-diagonal Gram accumulation H[j] += X_j^T X_j over calibration tokens
// (the Local-Hessian write-up "4 比特量化到底让模型笨了多少？", section "A
// different objective": H = X X^T is the (half) Hessian of the output error;
// the block-diagonal approximation keeps only its 16x16 diagonal blocks).
//
// Data path: a CTA owns a group of up to 8 column blocks (128 channels) and a
// range of tokens.  Token tiles [64 tokens x 128 channels] of bf16 stream from
// HBM into shared memory by the tensor-memory accelerator: one thread issues
// two 2-D tile copies (64 x 64 bf16 each, 128-byte swizzle) per stage into a
// 4-stage ring, completion is tracked by one mbarrier per stage, and no other
// thread computes an address.  Warp w owns column block w of the group: per
// 16 tokens one ldmatrix.x4.trans (through the swizzle, bank-conflict free)
// yields X_j^T as the A fragment of a 16x8x16 bf16 MMA, and the same four
// registers are the B fragments of the two 8-channel halves, so the 16x16
// block comes from two MMAs with no wasted product (bf16 x bf16 products are
// exact in fp32, sums are fp32).  Each CTA writes its fp32 partial block to a
// scratch buffer; a second kernel adds the partials of a group to H in a
// fixed order, so the result does not depend on scheduling.
//
// Every wait on an mbarrier is bounded (one second of %globaltimer): on
// expiry the CTA records NVFP4_ERR_DEVICE_TIMEOUT in this file's device
// status, waits (bounded again, ten seconds in all) for its own copies still
// in flight, writes nothing and returns.  The reduce kernel adds nothing to H
// while that status is set, so a Gram call whose CTA gave up leaves H as it
// was, and so do later Gram calls until the status is read and cleared.  If
// the copies in flight do not land within the second bound either, the CTA
// returns anyway and records NVFP4_ERR_DEVICE_UNDRAINED: shared memory of its
// SM may then still receive those copies.
#include <algorithm>
#include <mutex>

#include <cuda.h>

#include "chained.cuh"
#include "common.cuh"
#include "internal.h"
#include "../../include/nvfp4.h"

namespace nvfp4 {

// Sticky device status of the Gram kernels (NVFP4_OK,
// NVFP4_ERR_DEVICE_TIMEOUT or NVFP4_ERR_DEVICE_UNDRAINED, the larger code
// kept), read and cleared with the library status.
__device__ int g_gram_status = 0;

namespace {

constexpr int kGramThreads = 256;             // 8 warps
constexpr int kGroupBlocks = 8;               // column blocks per CTA
constexpr int kTileTok = 64;                  // tokens per pipeline stage
constexpr int kStages = 4;
constexpr int kBoxCols = 64;                  // channels per tile copy (128 bytes)
constexpr int kBoxBytes = kTileTok * kBoxCols * 2;  // 8 KiB
constexpr int kStageBytes = 2 * kBoxBytes;          // 16 KiB
constexpr int kGramSmem = kStages * kStageBytes + 1024;  // + alignment slack
constexpr int64_t kGroupedItemTokens = 2048;  // tokens per work item, grouped form
constexpr int64_t kMaxTokensPerLaunch = (int64_t)1 << 30;  // tile row coordinates fit int32
constexpr unsigned long long kWaitLimitNs = 1000000000ull;
constexpr unsigned long long kDrainLimitNs = 10000000000ull;  // after a timeout, for all stages

struct ItemRange {
  int64_t group, t_begin, t_end;
};

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for phase `parity` of an mbarrier, for at most kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_test(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (!mbar_test(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// One 64 x 64 bf16 tile (channels x0.., tokens y0..) into shared memory,
// completing on `bar`.  Rows past the tensor's end arrive as zeros.
__device__ __forceinline__ void tma_load_tile(uint32_t dst, const CUtensorMap *tmap, int x0,
                                              int y0, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x0), "r"(y0), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t r[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16 pair of tokens (tok, tok + 1) kept only where the token is below n.
__device__ __forceinline__ uint32_t keep_tokens(uint32_t pair, int tok, int n) {
  return pair & ((tok < n ? 0x0000FFFFu : 0u) | (tok + 1 < n ? 0xFFFF0000u : 0u));
}

// Work item -> (group, token range).  Uniform split of one group when
// `items` == nullptr, else the device table built by build_items_kernel.
__device__ __forceinline__ bool item_range(int64_t item, const ItemRange *items,
                                           const int64_t *n_items_dev, int64_t n_tok,
                                           int64_t per_item, ItemRange &out) {
  if (items) {
    if (item >= *n_items_dev) return false;
    out = items[item];
    return true;
  }
  out.group = 0;
  out.t_begin = item * per_item;
  out.t_end = min(n_tok, out.t_begin + per_item);
  return out.t_begin < out.t_end;
}

// `tmap`: X as a 2-D bf16 tensor [n_tok rows, C columns], 64 x 64 boxes,
// 128-byte swizzle, zero fill past the end.
__global__ void __launch_bounds__(kGramThreads)
    gram_partial_kernel(const __grid_constant__ CUtensorMap tmap, int64_t C,
                        const ItemRange *items, const int64_t *n_items_dev, int64_t n_tok,
                        int64_t per_item, float *__restrict__ partial) {
  chained_entry();
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[kStages];
  const int64_t nb = C / kBlock;
  const int64_t item = blockIdx.x;
  const int64_t cg = blockIdx.y;
  ItemRange ir;
  if (!item_range(item, items, n_items_dev, n_tok, per_item, ir)) return;
  const int width = (int)min((int64_t)kGroupBlocks, nb - cg * kGroupBlocks);  // column blocks
  const int ntiles = (int)((ir.t_end - ir.t_begin + kTileTok - 1) / kTileTok);
  // 1024-byte aligned ring (the swizzle pattern repeats every 1024 bytes)
  const uint32_t sraw = (uint32_t)__cvta_generic_to_shared(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  const uint32_t bar0 = (uint32_t)__cvta_generic_to_shared(&full[0]);
  const int x0 = (int)(cg * kGroupBlocks * kBlock);

  auto issue = [&](int tile, int stage) {
    const uint32_t bar = bar0 + 8u * stage;
    const int y0 = (int)(ir.t_begin + (int64_t)tile * kTileTok);
    mbar_expect_tx(bar, kStageBytes);
    tma_load_tile(sbase + stage * kStageBytes, &tmap, x0, y0, bar);
    tma_load_tile(sbase + stage * kStageBytes + kBoxBytes, &tmap, x0 + kBoxCols, y0, bar);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(bar0 + 8u * s, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0)
    for (int s = 0; s < kStages && s < ntiles; ++s) issue(s, s);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = lane & 3;
  float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
  // ldmatrix rows of this lane inside a 16-token step, and its 16-byte chunk
  // of the 128-byte row (channel block warp & 3 of box warp >> 2), swizzled
  const int lrow = (lane & 7) + ((lane >> 4) & 1) * 8;
  const uint32_t chunk = (uint32_t)(((warp & 3) * 2 + ((lane >> 3) & 1)) ^ (lane & 7));
  const uint32_t lane_off = (uint32_t)(warp >> 2) * kBoxBytes + (uint32_t)lrow * 128u + chunk * 16u;

  bool timed_out = false;
  int tile = 0;
  for (; tile < ntiles; ++tile) {
    const int stage = tile % kStages;
    const bool ok = mbar_wait_bounded(bar0 + 8u * stage, (uint32_t)(tile / kStages) & 1u);
    if (ok && warp < width) {
      const uint32_t st = sbase + (uint32_t)stage * kStageBytes + lane_off;
      // tokens of this tile that belong to the item (the last tile of a
      // grouped item may run into the next group)
      const int nvalid = (int)min((int64_t)kTileTok, ir.t_end - ir.t_begin - (int64_t)tile * kTileTok);
#pragma unroll
      for (int k = 0; k < kTileTok / 16; ++k) {
        uint32_t a[4];
        ldmatrix_x4_trans(st + k * 16 * 128, a);
        if (nvalid < kTileTok) {
          a[0] = keep_tokens(a[0], k * 16 + 2 * t, nvalid);
          a[1] = keep_tokens(a[1], k * 16 + 2 * t, nvalid);
          a[2] = keep_tokens(a[2], k * 16 + 8 + 2 * t, nvalid);
          a[3] = keep_tokens(a[3], k * 16 + 8 + 2 * t, nvalid);
        }
        mma_bf16_16816(d0, a, a[0], a[2]);
        mma_bf16_16816(d1, a, a[1], a[3]);
      }
    }
    // every thread is done with the stage (and agrees on a timeout) before
    // it is refilled
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      break;
    }
    if (threadIdx.x == 0 && tile + kStages < ntiles) issue(tile + kStages, stage);
  }

  if (timed_out) {
    if (threadIdx.x == 0) atomicMax(&g_gram_status, (int)NVFP4_ERR_DEVICE_TIMEOUT);
    // copies still in flight land in this CTA's shared memory: wait for them
    // before leaving, under one deadline for all stages
    if (threadIdx.x == 0) {
      const unsigned long long t0 = global_ns();
      bool drained = true;
      for (int u = tile; u < ntiles && u < tile + kStages && drained; ++u) {
        const uint32_t bar = bar0 + 8u * (u % kStages), par = (uint32_t)(u / kStages) & 1u;
        while (!mbar_test(bar, par)) {
          if (global_ns() - t0 > kDrainLimitNs) {
            drained = false;
            break;
          }
        }
      }
      if (!drained) atomicMax(&g_gram_status, (int)NVFP4_ERR_DEVICE_UNDRAINED);
    }
    __syncthreads();
    return;
  }

  if (warp < width) {
    const int64_t j = cg * kGroupBlocks + warp;
    float *P = partial + (item * nb + j) * 256;
    const int g = lane >> 2;
    P[g * 16 + 2 * t] = d0[0];
    P[g * 16 + 2 * t + 1] = d0[1];
    P[(g + 8) * 16 + 2 * t] = d0[2];
    P[(g + 8) * 16 + 2 * t + 1] = d0[3];
    P[g * 16 + 8 + 2 * t] = d1[0];
    P[g * 16 + 8 + 2 * t + 1] = d1[1];
    P[(g + 8) * 16 + 8 + 2 * t] = d1[2];
    P[(g + 8) * 16 + 8 + 2 * t + 1] = d1[3];
  }
}

// Diagnostic: one warp waits on an mbarrier that nothing arrives on, so the
// bounded wait runs out after kWaitLimitNs and the timeout status is set (no
// copy is in flight).  Exercises the same wait and status path as
// gram_partial_kernel.
__global__ void wait_timeout_probe_kernel() {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = (uint32_t)__cvta_generic_to_shared(&bar);
  if (threadIdx.x == 0) mbar_init(b, 1);
  __syncwarp();
  const bool ok = mbar_wait_bounded(b, 0);
  if (!ok && threadIdx.x == 0) atomicMax(&g_gram_status, (int)NVFP4_ERR_DEVICE_TIMEOUT);
}

// H[g][e] += sum of the partials of group g's items, in item order, four
// consecutive entries per thread (16-byte loads of the partials; the
// partials are library scratch, 256-byte aligned, and a group is a multiple
// of 256 floats), group g = blockIdx.y (grid-stride beyond 65,535 groups).
// Nothing is added while a timed-out wait is on record (a partial of this
// call may then be missing, and its slot holds stale data).
__global__ void gram_reduce_kernel(const float *__restrict__ partial, int64_t per_group,
                                   int64_t G, const int64_t *__restrict__ item_start,
                                   int64_t n_items_uniform, float *__restrict__ H) {
  chained_entry();
  // the status once per CTA (a load of the one word by every thread queued
  // millions of requests on one L2 slice)
  __shared__ int status;
  if (threadIdx.x == 0) status = *(volatile const int *)&g_gram_status;
  __syncthreads();
  if (status != 0) return;
  const int64_t e = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (e >= per_group) return;
  const int64_t stride4 = per_group / 4;
  for (int64_t g = blockIdx.y; g < G; g += gridDim.y) {
    int64_t i0 = 0, i1 = n_items_uniform;
    if (item_start) {
      i0 = item_start[g];
      i1 = item_start[g + 1];
    }
    const float4 *p4 = reinterpret_cast<const float4 *>(partial + e);
    // eight loads in flight, then their sum in item order (the largest group
    // of a routed batch can hold tens of items)
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    int64_t i = i0;
    for (; i + 8 <= i1; i += 8) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = p4[(i + u) * stride4];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        acc.x += v[u].x;
        acc.y += v[u].y;
        acc.z += v[u].z;
        acc.w += v[u].w;
      }
    }
    for (; i < i1; ++i) {
      const float4 v = p4[i * stride4];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    float *h = H + g * per_group + e;  // 4-byte aligned: scalar updates
    h[0] += acc.x;
    h[1] += acc.y;
    h[2] += acc.z;
    h[3] += acc.w;
  }
}

__global__ void build_items_kernel(const int64_t *__restrict__ offsets, int64_t G, int64_t n_tok,
                                   int64_t per_item, int64_t max_items,
                                   int64_t *__restrict__ item_start, ItemRange *__restrict__ items,
                                   int64_t *__restrict__ n_items) {
  chained_entry();
  __shared__ int64_t warp_sums[32];
  __shared__ int64_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  auto clamp_off = [&](int64_t g) {
    int64_t o = offsets[g];
    return o < 0 ? (int64_t)0 : (o > n_tok ? n_tok : o);
  };
  for (int64_t base = 0; base < G; base += blockDim.x) {
    const int64_t g = base + threadIdx.x;
    int64_t cnt = 0, lo = 0, hi = 0;
    if (g < G) {
      lo = clamp_off(g);
      hi = clamp_off(g + 1);
      if (hi < lo) hi = lo;
      cnt = (hi - lo + per_item - 1) / per_item;
    }
    // block-wide inclusive scan of cnt
    int64_t v = cnt;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t n = __shfl_up_sync(0xFFFFFFFFu, v, o);
      if (lane >= o) v += n;
    }
    if (lane == 31) warp_sums[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int64_t s = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int64_t n = __shfl_up_sync(0xFFFFFFFFu, s, o);
        if (lane >= o) s += n;
      }
      warp_sums[lane] = s;
    }
    __syncthreads();
    const int64_t excl = carry + (warp ? warp_sums[warp - 1] : 0) + v - cnt;
    if (g < G) {
      item_start[g] = excl;
      for (int64_t c = 0; c < cnt && excl + c < max_items; ++c) {
        ItemRange r;
        r.group = g;
        r.t_begin = lo + c * per_item;
        r.t_end = min(hi, r.t_begin + per_item);
        items[excl + c] = r;
      }
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = excl + cnt;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    item_start[G] = carry;
    *n_items = carry < max_items ? carry : max_items;
  }
}

constexpr int kMaxDevices = 64;
bool g_smem_attr_set[kMaxDevices] = {};

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (no link-time dependency on the driver library).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

// X [n_rows, C] bf16 (row stride C elements) as 64 x 64 tiles, 128-byte
// swizzle, zeros past the end.  The caller has checked that x is 16-byte
// aligned and C a multiple of 16 (so the row stride is a multiple of 32 bytes).
cudaError_t make_x_tensor_map(const uint16_t *x, int64_t n_rows, int64_t C, CUtensorMap *out) {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  if (!g_encode) return cudaErrorNotSupported;
  const cuuint64_t gdim[2] = {(cuuint64_t)C, (cuuint64_t)n_rows};
  const cuuint64_t gstride[1] = {(cuuint64_t)C * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBoxCols, (cuuint32_t)kTileTok};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = g_encode(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                             const_cast<uint16_t *>(x), gdim, gstride, box, estride,
                             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t ensure_smem_attr() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!g_smem_attr_set[dev]) {
    e = cudaFuncSetAttribute(gram_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGramSmem);
    if (e != cudaSuccess) return e;
    g_smem_attr_set[dev] = true;
  }
  return cudaSuccess;
}

// Token items of the uniform split: enough CTAs for a few waves of 3 resident
// CTAs per SM, at least 4 tiles per item, at most `cap` items.
void uniform_items(int64_t n_tok, int64_t ngroups, int64_t cap, int64_t *items_out,
                   int64_t *per_item_out) {
  const int64_t target = (int64_t)sm_count() * 3 * 2;
  int64_t items = (target + ngroups - 1) / ngroups;
  const int64_t max_items = (n_tok + 4 * kTileTok - 1) / (4 * kTileTok);
  if (items > max_items) items = max_items;
  if (items > cap) items = cap;
  if (items < 1) items = 1;
  int64_t per_item = (n_tok + items - 1) / items;
  per_item = (per_item + kTileTok - 1) / kTileTok * kTileTok;
  *items_out = (n_tok + per_item - 1) / per_item;
  *per_item_out = per_item;
}

// One uniform split over n_tok tokens (fewer than 2^30): `items` partials of
// `per_item` tokens into `partial`, then their fixed-order sum into H.
cudaError_t gram_uniform(const uint16_t *x, int64_t n_tok, int64_t C, float *H, float *partial,
                         int64_t items, int64_t per_item, cudaStream_t st) {
  const int64_t nb = C / kBlock;
  const int64_t ngroups = (nb + kGroupBlocks - 1) / kGroupBlocks;
  const int64_t per_group = nb * 256;
  CUtensorMap tmap;
  cudaError_t e = make_x_tensor_map(x, n_tok, C, &tmap);
  if (e != cudaSuccess) return e;
  e = launch_first(gram_partial_kernel, dim3((unsigned)items, (unsigned)ngroups),
                     dim3(kGramThreads), kGramSmem, st, tmap, C, nullptr, nullptr, n_tok, per_item,
                     partial);
  if (e != cudaSuccess) return e;
  return launch_chained(gram_reduce_kernel, dim3((unsigned)((per_group / 4 + 255) / 256)),
                        dim3(256), 0, st, static_cast<const float *>(partial), per_group,
                        (int64_t)1, nullptr, items, H);
}

}  // namespace

cudaError_t launch_gram(const uint16_t *x, const int64_t *offsets, int64_t G, int64_t n_tok,
                        int64_t C, float *H, cudaStream_t st) {
  if (n_tok == 0 || C == 0 || G == 0) return cudaSuccess;
  cudaError_t e = ensure_smem_attr();
  if (e != cudaSuccess) return e;
  const int64_t nb = C / kBlock;
  const int64_t ngroups = (nb + kGroupBlocks - 1) / kGroupBlocks;
  const int64_t per_group = nb * 256;

  if (!offsets) {
    // token chunks of at most 2^30 (tile row coordinates are 32-bit)
    for (int64_t t0 = 0; t0 < n_tok; t0 += kMaxTokensPerLaunch) {
      const int64_t n = std::min(kMaxTokensPerLaunch, n_tok - t0);
      int64_t items, per_item;
      uniform_items(n, ngroups, INT64_MAX, &items, &per_item);
      float *partial = nullptr;
      e = scratch_alloc((void **)&partial, sizeof(float) * items * per_group, st);
      if (e != cudaSuccess) return e;
      e = gram_uniform(x + t0 * C, n, C, H, partial, items, per_item, st);
      const cudaError_t e2 = scratch_free(partial, st);
      if (e == cudaSuccess) e = e2;
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }

  if (n_tok > kMaxTokensPerLaunch) return cudaErrorInvalidValue;
  CUtensorMap tmap;
  e = make_x_tensor_map(x, n_tok, C, &tmap);
  if (e != cudaSuccess) return e;
  const int64_t per_item = kGroupedItemTokens;
  const int64_t max_items = n_tok / per_item + G;
  // scratch layout: item_start [G+1] | n_items [1] | items [max_items] | partials
  const size_t off_items = (sizeof(int64_t) * (G + 2) + 255) / 256 * 256;
  const size_t off_part = (off_items + sizeof(ItemRange) * max_items + 255) / 256 * 256;
  const size_t bytes = off_part + sizeof(float) * max_items * per_group;
  unsigned char *ws = nullptr;
  e = scratch_alloc((void **)&ws, bytes, st);
  if (e != cudaSuccess) return e;
  int64_t *item_start = reinterpret_cast<int64_t *>(ws);
  int64_t *n_items = item_start + G + 1;
  ItemRange *items = reinterpret_cast<ItemRange *>(ws + off_items);
  float *partial = reinterpret_cast<float *>(ws + off_part);
  e = launch_first(build_items_kernel, dim3(1), dim3(1024), 0, st, offsets, G, n_tok, per_item,
                     max_items, item_start, items, n_items);
  if (e == cudaSuccess)
    e = launch_chained(gram_partial_kernel, dim3((unsigned)max_items, (unsigned)ngroups),
                       dim3(kGramThreads), kGramSmem, st, tmap, C,
                       static_cast<const ItemRange *>(items), static_cast<const int64_t *>(n_items),
                       n_tok, per_item, partial);
  if (e == cudaSuccess)
    e = launch_chained(gram_reduce_kernel,
                       dim3((unsigned)((per_group / 4 + 255) / 256),
                            (unsigned)std::min<int64_t>(G, 65535)),
                       dim3(256), 0, st, static_cast<const float *>(partial), per_group, G,
                       static_cast<const int64_t *>(item_start), (int64_t)0, H);
  cudaError_t e2 = scratch_free(ws, st);
  return e != cudaSuccess ? e : e2;
}

cudaError_t launch_wait_timeout_probe(cudaStream_t st) {
  wait_timeout_probe_kernel<<<1, 32, 0, st>>>();
  return cudaGetLastError();
}

cudaError_t read_and_clear_gram_status(cudaStream_t st, int *out) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_gram_status, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  if (*out != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_gram_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  }
  return e;
}

// ---------------------------------------------------------------------------
// Gram accumulation without any allocation.
//
// The per-item partial sums of this entry point live in one fixed array of
// this file, so the call never allocates.  It exists for callers that may not
// allocate device memory themselves: code that hands all of HBM to its own
// allocator or runs under a fixed memory budget (a library-side allocation
// could fail there or take memory the caller has planned for something else),
// and code that cannot afford an allocation's latency or implicit device
// synchronisation in the middle of a calibration loop.
//
// The array is 16 MiB (kNoAllocPartialFloats floats) and is held by every
// device that loads the library until the process exits.  A call needs
// C/16 * 1 KiB per token range, so C is limited to 262,144 channels; fewer
// token ranges are used when C is large.  All calls on a device share the
// array: calls that overlap on the GPU (different streams, or graphs replayed
// concurrently) race on it and must be serialised by the caller.  Every
// partial a call reads it has written first, so nothing needs clearing
// between calls; the one exception is a call whose CTA gave up waiting for
// its tile copies, and there the reduce adds nothing to H (see the timeout
// handling above).  The first call on each device looks up the array's device address
// (cudaGetSymbolAddress, with that device current) and caches it; make that
// first call before any stream capture.
constexpr size_t kNoAllocPartialFloats = (size_t)4 << 20;  // 16 MiB
static __device__ __align__(256) float g_noalloc_partials[kNoAllocPartialFloats];

namespace {
std::mutex g_noalloc_mu;
float *g_noalloc_ptr[kMaxDevices] = {};

cudaError_t noalloc_partials(float **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_partials);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = static_cast<float *>(p);
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}
}  // namespace

int64_t gram_noalloc_max_channels() {
  return (int64_t)(kNoAllocPartialFloats / 256) * kBlock;
}

cudaError_t launch_gram_noalloc(const uint16_t *x, int64_t n_tok, int64_t C, float *H,
                                cudaStream_t st) {
  if (n_tok == 0 || C == 0) return cudaSuccess;
  const int64_t nb = C / kBlock;
  const int64_t per_group = nb * 256;
  const int64_t cap = (int64_t)(kNoAllocPartialFloats / (size_t)per_group);
  if (cap < 1) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr();
  if (e != cudaSuccess) return e;
  float *partial = nullptr;
  e = noalloc_partials(&partial);
  if (e != cudaSuccess) return e;
  const int64_t ngroups = (nb + kGroupBlocks - 1) / kGroupBlocks;
  for (int64_t t0 = 0; t0 < n_tok; t0 += kMaxTokensPerLaunch) {
    const int64_t n = std::min(kMaxTokensPerLaunch, n_tok - t0);
    int64_t items, per_item;
    uniform_items(n, ngroups, cap, &items, &per_item);
    e = gram_uniform(x + t0 * C, n, C, H, partial, items, per_item, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace nvfp4
