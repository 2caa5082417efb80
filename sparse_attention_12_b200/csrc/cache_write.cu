// Writing new positions into the two caches: the step just before the indexer scores.
//
// Every query row t (request b, position p) is a new token. Its indexer key and its latent row go
// to slot p % 64 of page block_table[b][p / 64]:
//   s = max_d |k_d| / 448 (1 for an all-zero key), codes_d = e4m3(k_d / s), both divisions in fp32;
//   kI_cache[page][slot] = codes, kI_scale[page][slot] = s, kv_cache[page][slot] = c (576 bf16).
// ("MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与 DSA": per token the latent vector in bf16
// and the indexer key as FP8 plus a 4-byte scale, both caches paged; "DeepSeek Sparse Attention：从
// SWA 到稀疏 Attention 计算", Lightning Indexer section: one indexer key per position, shared by the
// indexer heads, kept in its own key cache.) e4m3 is OCP E4M3 with round-to-nearest-even and
// saturation at +-448 (the hardware conversion with satfinite).
//
// One warp per row: each lane converts 4 key values (one coalesced 128-byte store per warp) and
// copies 2-3 16-byte chunks of the latent row. HBM-bound: 512 + 1152 bytes read, 132 + 1152 written
// per row.
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

namespace dsa {
namespace {

constexpr int kRowsPerBlock = 8;  // one warp per row

__global__ void __launch_bounds__(32 * kRowsPerBlock)
    cache_write_kernel(BatchDev bd, const int32_t* __restrict__ row_req, const int32_t* __restrict__ row_pos,
                       const float* __restrict__ k_new, const uint16_t* __restrict__ c_new,
                       uint8_t* __restrict__ kI_cache, float* __restrict__ kI_scale, uint16_t* __restrict__ kv_cache,
                       uint32_t* status) {
  pdl_trigger();
  pdl_wait();  // the plan (row -> request, position) and the caches the previous kernels read
  const int t = blockIdx.x * kRowsPerBlock + static_cast<int>(threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= bd.T) return;
  const int b = __ldg(row_req + t), p = __ldg(row_pos + t);
  const int pg = __ldg(bd.block_table + static_cast<int64_t>(b) * bd.max_pages + p / kPage);
  if (pg < 0 || pg >= bd.num_pages) {
    if (lane == 0) report_error(status, kDevErrIndex);
    return;
  }
  const int64_t slot = static_cast<int64_t>(pg) * kPage + p % kPage;

  // indexer key: lane l holds elements 4l .. 4l+3
  const float4 x = __ldg(reinterpret_cast<const float4*>(k_new + static_cast<int64_t>(t) * kDIdx) + lane);
  // a non-finite key has no FP8 encoding (it would store NaN codes): the row is not written
  const bool finite = isfinite(x.x) && isfinite(x.y) && isfinite(x.z) && isfinite(x.w);
  if (!__all_sync(0xffffffffu, finite)) {
    if (lane == 0) report_error(status, kDevErrValue);
    return;
  }
  const float m = fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w)));
  // non-negative floats order like their bit patterns
  const float amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
  const float s = amax > 0.f ? amax / 448.0f : 1.0f;
  const uint32_t q0 = __nv_cvt_float_to_fp8(x.x / s, __NV_SATFINITE, __NV_E4M3);
  const uint32_t q1 = __nv_cvt_float_to_fp8(x.y / s, __NV_SATFINITE, __NV_E4M3);
  const uint32_t q2 = __nv_cvt_float_to_fp8(x.z / s, __NV_SATFINITE, __NV_E4M3);
  const uint32_t q3 = __nv_cvt_float_to_fp8(x.w / s, __NV_SATFINITE, __NV_E4M3);
  reinterpret_cast<uint32_t*>(kI_cache + slot * kDIdx)[lane] = q0 | (q1 << 8) | (q2 << 16) | (q3 << 24);
  if (lane == 0) kI_scale[slot] = s;

  // latent row: 72 chunks of 16 bytes
  const uint4* src = reinterpret_cast<const uint4*>(c_new + static_cast<int64_t>(t) * kDLat);
  uint4* dst = reinterpret_cast<uint4*>(kv_cache + slot * kDLat);
  for (int i = lane; i < kDLat * 2 / 16; i += 32) dst[i] = __ldg(src + i);
}

}  // namespace

int launch_cache_write(const BatchDev& b, const void* plan, const float* k_new, const void* c_new, uint8_t* kI_cache,
                       float* kI_scale, void* kv_cache, void* stream) {
  if (b.T == 0) return 0;
  PlanView pv = plan_view(const_cast<void*>(plan), b.B, b.T);
  const int blocks = (b.T + kRowsPerBlock - 1) / kRowsPerBlock;
  return static_cast<int>(launch_pdl(cache_write_kernel, dim3(blocks), dim3(32 * kRowsPerBlock), 0, stream, b,
                                     static_cast<const int32_t*>(pv.row_req), static_cast<const int32_t*>(pv.row_pos),
                                     k_new, static_cast<const uint16_t*>(c_new), kI_cache, kI_scale,
                                     static_cast<uint16_t*>(kv_cache), &pv.hdr->status));
}

}  // namespace dsa
