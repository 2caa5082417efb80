// Per-query TopK over the indexer scores:  S_t = TopK_{j<=t}(I_tj, k)
// ("DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section "Lightning Indexer", TopK
// formula; when the prefix holds no more than k positions all of them are taken, the handbook's
// k = min(L, TOPK) in "MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与 DSA").
//
// One CTA of 1024 threads per query row. Scores become order-preserving uint32 keys; a radix
// select over 11 + 11 + 10 bits finds the exact k-th largest key with shared-memory histograms
// (warp-aggregated atomics: scores crowd into a few exponent bins). A last pass over contiguous
// per-warp segments (ballot-ordered, two block scans) emits every position above the threshold and
// the first `remaining` positions equal to it, in increasing position order, so the result is
// deterministic: among equal scores the smaller position wins.
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

// hist[bin] += 1 for every lane, one atomic per distinct bin in the warp (scores cluster in a
// few exponent bins, so plain per-lane atomics would serialise on them).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(act, bin);
  if ((threadIdx.x & 31) == static_cast<uint32_t>(__ffs(peers) - 1)) atomicAdd(&hist[bin], __popc(peers));
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
    const int L_pad = (L + 31) & ~31;  // whole warps take part in the aggregated atomics
    if (pass == 0) {
      for (int j = threadIdx.x; j < L_pad; j += kThreads) {
        uint32_t u = 0;
        if (j < L) {
          u = order_key(__ldg(row + j));
          if (cached) cache[j] = u;
        }
        hist_add(hist, u >> shift, j < L);
      }
    } else {
      for (int j = threadIdx.x; j < L_pad; j += kThreads) {
        uint32_t u = 0;
        if (j < L) u = cached ? cache[j] : order_key(__ldg(row + j));
        hist_add(hist, (u >> shift) & bmask, j < L && (u & mask) == prefix);
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

  // Ordered emission. Warp w owns the contiguous positions [w*SEG, (w+1)*SEG), visited 32
  // consecutive positions at a time (conflict-free, ballot-ordered). Two block scans over the
  // per-warp counts rank the ties (the first `remaining` in position order are taken) and give
  // each warp its output offset.
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int SEG = 32 * ((L + kThreads - 1) / kThreads);
  const int wj0 = min(L, wid * SEG), wj1 = min(L, wj0 + SEG);
  int w_gt = 0, w_tie = 0;
  for (int base = wj0; base < wj1; base += 32) {
    const int j = base + lane;
    const uint32_t u = (j < wj1) ? (cached ? cache[j] : order_key(__ldg(row + j))) : 0u;
    w_gt += __popc(__ballot_sync(0xffffffffu, j < wj1 && u > prefix));
    w_tie += __popc(__ballot_sync(0xffffffffu, j < wj1 && u == prefix));
  }
  int total;
  const int tie_incl = __shfl_sync(0xffffffffu, block_inclusive_scan(lane == 0 ? w_tie : 0, scan_scratch, &total), 0);
  const int tie_take = max(0, min(w_tie, static_cast<int>(remaining) - (tie_incl - w_tie)));
  const int sel = w_gt + tie_take;
  const int sel_incl = __shfl_sync(0xffffffffu, block_inclusive_scan(lane == 0 ? sel : 0, scan_scratch, &total), 0);
  int slot = sel_incl - sel, ties_left = tie_take;
  for (int base = wj0; base < wj1; base += 32) {
    const int j = base + lane;
    const uint32_t u = (j < wj1) ? (cached ? cache[j] : order_key(__ldg(row + j))) : 0u;
    const bool gt = j < wj1 && u > prefix;
    const bool tie = j < wj1 && u == prefix;
    const uint32_t tie_mask = __ballot_sync(0xffffffffu, tie);
    const bool take = gt || (tie && __popc(tie_mask & lt_mask) < ties_left);
    const uint32_t take_mask = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int o = slot + __popc(take_mask & lt_mask);
      if (o < k) out[o] = j;
    }
    slot += __popc(take_mask);
    ties_left -= min(__popc(tie_mask), ties_left);
  }
  for (int s2 = total + static_cast<int>(threadIdx.x); s2 < k; s2 += kThreads) out[s2] = -1;
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
