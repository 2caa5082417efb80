// Per-query TopK over the indexer scores:  S_t = TopK_{j<=t}(I_tj, k)
// ("DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section "Lightning Indexer", TopK
// formula; when the prefix holds no more than k positions all of them are taken, the handbook's
// k = min(L, TOPK) in "MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与 DSA").
//
// One CTA of 1024 threads per query row. Scores become order-preserving uint32 keys; a radix
// select over 11 + 11 + 10 bits finds the exact k-th largest key with shared-memory histograms.
// A last, ordered pass (warp ballots plus a block scan per 1024 positions) emits every position
// above the threshold and the first `remaining` positions equal to it, in increasing position
// order, so the result is deterministic: among equal scores the smaller position wins.
// Rows up to kCacheCap scores are kept in shared memory after the first read; longer rows are
// re-read from L2 on each pass.
#include <cuda_runtime.h>

#include <cmath>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kCacheCap = 24576;  // 96 KB of keys in shared memory

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;  // -0 ranks as +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Block-wide inclusive scan of one value per thread; `scratch` holds kWarps ints.
__device__ __forceinline__ int block_inclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = scratch[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    scratch[lane] = s;
  }
  __syncthreads();
  const int r = x + (wid > 0 ? scratch[wid - 1] : 0);
  *total = scratch[kWarps - 1];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThreads) topk_kernel(const int32_t* __restrict__ row_pos,
                                                        const float* __restrict__ scores, int64_t ld, int k,
                                                        int32_t* __restrict__ S, int use_cache) {
  extern __shared__ uint32_t tk_smem[];
  uint32_t* hist = tk_smem;                // [kBins]
  uint32_t* cache = tk_smem + kBins;       // [kCacheCap] when use_cache
  __shared__ int scan_scratch[kWarps];
  __shared__ uint32_t sh_prefix, sh_remaining;

  const int t = blockIdx.x;
  const int L = __ldg(row_pos + t) + 1;
  const float* row = scores + static_cast<int64_t>(t) * ld;
  int32_t* out = S + static_cast<int64_t>(t) * k;

  if (L <= k) {
    for (int j = threadIdx.x; j < k; j += kThreads) out[j] = (j < L) ? j : -1;
    return;
  }
  const bool cached = use_cache && L <= kCacheCap;

  uint32_t prefix = 0, mask = 0, remaining = static_cast<uint32_t>(k);
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const uint32_t nb = 1u << widths[pass];
    const uint32_t bmask = nb - 1u;
    for (uint32_t i = threadIdx.x; i < kBins; i += kThreads) hist[i] = 0u;
    __syncthreads();
    if (pass == 0) {
      for (int j = threadIdx.x; j < L; j += kThreads) {
        const uint32_t u = order_key(__ldg(row + j));
        if (cached) cache[j] = u;
        atomicAdd(&hist[u >> shift], 1u);
      }
    } else {
      for (int j = threadIdx.x; j < L; j += kThreads) {
        const uint32_t u = cached ? cache[j] : order_key(__ldg(row + j));
        if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & bmask], 1u);
      }
    }
    __syncthreads();
    // counts from the top bin down: thread i owns descending bins 2i, 2i+1
    const int d0 = 2 * threadIdx.x, d1 = d0 + 1;
    const uint32_t c0 = (static_cast<uint32_t>(d0) < nb) ? hist[nb - 1 - d0] : 0u;
    const uint32_t c1 = (static_cast<uint32_t>(d1) < nb) ? hist[nb - 1 - d1] : 0u;
    int total;
    const int incl = block_inclusive_scan(static_cast<int>(c0 + c1), scan_scratch, &total);
    const uint32_t before = static_cast<uint32_t>(incl) - c0 - c1;  // count in bins above d0
    if (before < remaining && remaining <= before + c0) {
      sh_prefix = prefix | ((nb - 1 - d0) << shift);
      sh_remaining = remaining - before;
    } else if (before + c0 < remaining && remaining <= before + c0 + c1) {
      sh_prefix = prefix | ((nb - 1 - d1) << shift);
      sh_remaining = remaining - before - c0;
    }
    __syncthreads();
    prefix = sh_prefix;
    remaining = sh_remaining;
    mask |= bmask << shift;
    __syncthreads();
  }

  // ordered emission: keys above the threshold, then the first `remaining` keys equal to it
  int out_pos = 0;
  uint32_t ties_seen = 0;
  const int lane = threadIdx.x & 31;
  for (int base = 0; base < L; base += kThreads) {
    const int j = base + threadIdx.x;
    uint32_t u = 0;
    if (j < L) u = cached ? cache[j] : order_key(__ldg(row + j));
    const bool gt = j < L && u > prefix;
    const bool tie = j < L && u == prefix;
    int tie_total;
    const int tie_incl = block_inclusive_scan(tie ? 1 : 0, scan_scratch, &tie_total);
    const bool sel = gt || (tie && ties_seen + static_cast<uint32_t>(tie_incl - 1) < remaining);
    int sel_total;
    const int sel_incl = block_inclusive_scan(sel ? 1 : 0, scan_scratch, &sel_total);
    if (sel) {
      const int slot = out_pos + sel_incl - 1;
      if (slot < k) out[slot] = j;
    }
    out_pos += sel_total;
    ties_seen += static_cast<uint32_t>(tie_total);
    (void)lane;
  }
  for (int s = out_pos + static_cast<int>(threadIdx.x); s < k; s += kThreads) out[s] = -1;
}

}  // namespace

int launch_topk(const BatchDev& b, const void* plan, const float* scores, int64_t ld, int k, int32_t* S,
                void* stream) {
  if (b.T == 0) return 0;
  PlanView pv = plan_view(const_cast<void*>(plan), b.B, b.T);
  const int use_cache = 1;
  const int cap = b.max_seq_len < kCacheCap ? b.max_seq_len : kCacheCap;
  const size_t smem = sizeof(uint32_t) * (kBins + static_cast<size_t>(cap));
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sizeof(uint32_t) * (kBins + kCacheCap)));
  if (e != cudaSuccess) return static_cast<int>(e);
  topk_kernel<<<b.T, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(pv.row_pos, scores, ld, k, S,
                                                                          use_cache && cap >= 1);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace dsa
