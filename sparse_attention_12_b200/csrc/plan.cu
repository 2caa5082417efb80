// Batch plan: request/position of every query row and the indexer's work list.
//
// Query i of request b sits at position n_b - m_b + i (the cache length counts the request's own
// query tokens) and sees positions [0, p]: the causal set C_t of "DeepSeek Sparse Attention：从 SWA
// 到稀疏 Attention 计算", section "SWA：让固定窗口沿序列移动", in 0-based form.
//
// The indexer groups up to 256/nhI consecutive queries of one request so that one FP8 MMA covers
// 256 query-head columns; a group's work is its key tiles of 128 positions up to its last
// query's position. One CTA of 1024 threads builds everything (a few microseconds).
#include <cuda_runtime.h>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

namespace dsa {
namespace {

constexpr int kPlanThreads = 1024;

// Block-wide exclusive scan of `n` int32 values in place (src may alias dst); returns the total.
__device__ int32_t block_exclusive_scan(int32_t* data, int n, int32_t* warp_sums) {
  int32_t carry = 0;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int base = 0; base < n; base += kPlanThreads) {
    const int i = base + threadIdx.x;
    int32_t v = (i < n) ? data[i] : 0;
    int32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int32_t s = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int32_t y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      warp_sums[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int32_t before = (wid > 0 ? warp_sums[wid - 1] : 0) + carry;
    if (i < n) data[i] = before + x - v;
    const int32_t chunk_total = warp_sums[31];
    __syncthreads();
    carry += chunk_total;
  }
  return carry;
}

constexpr int kPlanSmemMaxB = 3968;  // (3 B + 2) int32 stay under the 48 KB default

// Last index i in [0, n) with a[i] <= key (a non-decreasing); -1 if none.
__device__ __forceinline__ int upper_index(const int32_t* a, int n, int32_t key) {
  int lo = 0, hi = n;  // answer in [lo-1, hi-1]
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] <= key)  // plain load: `a` may have been written earlier in this kernel
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo - 1;
}

// With B <= kPlanSmemMaxB the per-request arrays (cu_q, seq_lens, group offsets) are staged in
// shared memory, so the per-row and per-group binary searches run there instead of through L2.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(BatchDev bd, int nhI, void* plan_base, int staged) {
  __shared__ int32_t warp_sums[32];
  extern __shared__ int32_t plan_smem[];  // [B+1] cu_q, [B] seq_lens, [B+1] group offsets when staged
  PlanView pv = plan_view(plan_base, bd.B, bd.T);
  const int B = bd.B, T = bd.T;
  const int qpg = kIdxCols / nhI;
  uint32_t* status = &pv.hdr->status;
  pdl_trigger();
  pdl_wait();  // the plan may still be read by the kernels of the previous call
  const int32_t* cuq = bd.cu_q;
  const int32_t* sl = bd.seq_lens;
  int32_t* goff = pv.req_goff;
  if (staged) {
    int32_t* s_cuq = plan_smem;
    int32_t* s_sl = plan_smem + (B + 1);
    for (int i = threadIdx.x; i <= B; i += kPlanThreads) s_cuq[i] = __ldg(bd.cu_q + i);
    for (int i = threadIdx.x; i < B; i += kPlanThreads) s_sl[i] = __ldg(bd.seq_lens + i);
    cuq = s_cuq;
    sl = s_sl;
    goff = plan_smem + (2 * B + 1);
  }
  if (threadIdx.x == 0) *status = 0u;
  __syncthreads();

  // groups per request, then their offsets
  for (int b = threadIdx.x; b < B; b += kPlanThreads) {
    const int m = cuq[b + 1] - cuq[b];
    const int n = sl[b];
    if (m < 0 || n < m || n > bd.max_seq_len || (n > 0 && (n + kPage - 1) / kPage > bd.max_pages) ||
        (m > 0 && n < 1))
      report_error(status, kDevErrIndex);
    goff[b] = m > 0 ? (m + qpg - 1) / qpg : 0;
  }
  if (threadIdx.x == 0) goff[B] = 0;
  __syncthreads();
  const int G = block_exclusive_scan(goff, B + 1, warp_sums);
  // goff[B] now holds the total; rows and groups next
  if (staged)
    for (int i = threadIdx.x; i <= B; i += kPlanThreads) pv.req_goff[i] = goff[i];
  for (int t = threadIdx.x; t < T; t += kPlanThreads) {
    const int b = upper_index(cuq, B + 1, t);
    if (b < 0 || b >= B) {
      report_error(status, kDevErrIndex);
      pv.row_req[t] = 0;
      pv.row_pos[t] = 0;
      continue;
    }
    const int c0 = cuq[b], m = cuq[b + 1] - c0;
    const int n = sl[b];
    pv.row_req[t] = b;
    pv.row_pos[t] = n - m + (t - c0);
  }
  for (int g = threadIdx.x; g < G; g += kPlanThreads) {
    const int b = upper_index(goff, B, g);
    const int li = g - goff[b];
    const int c0 = cuq[b], m = cuq[b + 1] - c0;
    const int n = sl[b];
    const int nq = min(qpg, m - li * qpg);
    const int pos0 = n - m + li * qpg;
    const int p_last = pos0 + nq - 1;
    pv.grp_row0[g] = c0 + li * qpg;
    pv.grp_nq[g] = nq;
    pv.grp_req[g] = b;
    pv.grp_pos0[g] = pos0;
    pv.grp_tile0[g] = (p_last + kIdxTileKeys) / kIdxTileKeys;
  }
  if (threadIdx.x == 0) pv.grp_tile0[G] = 0;
  __syncthreads();
  const int total = block_exclusive_scan(pv.grp_tile0, G + 1, warp_sums);
  if (threadIdx.x == 0) {
    pv.hdr->total_tiles = total;
    pv.hdr->num_groups = G;
    pv.hdr->nhI = nhI;
    pv.hdr->qpg = qpg;
    pv.hdr->T = T;
    pv.hdr->B = B;
  }
}

}  // namespace

int launch_plan(const BatchDev& b, int nhI, void* plan, void* stream) {
  const int staged = b.B <= kPlanSmemMaxB ? 1 : 0;
  const size_t smem = staged ? sizeof(int32_t) * (3 * static_cast<size_t>(b.B) + 2) : 0;
  const cudaError_t e = launch_pdl(plan_kernel, dim3(1), dim3(kPlanThreads), smem, stream, b, nhI, plan, staged);
  if (e != cudaSuccess) return static_cast<int>(e);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace dsa
