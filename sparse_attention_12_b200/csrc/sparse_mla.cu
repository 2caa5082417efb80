// Sparse MLA on the selected positions (sm_100a).
//
// For query row t with index set S_t and every head h:
//   z_hj = scale * q_th . c_j  (576 dims),   o_th = sum_{j in S_t} softmax_j(z_hj) * c_j[0:512]
// ("DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section "Sparse Attention", the masked
// softmax with M = 0 on S_t, computed by reading only the selected rows; absorbed MLA with a
// 576-wide latent shared by all heads per "MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与
// DSA". S_t is shared by all heads.)
//
// One CTA per (query row, half of the 512 value dims, split of S_t); one CTA per SM.
//   * Q (128 heads x 576, bf16): dims 0..319 sit in TMEM and feed the S = Q C^T MMAs as the A
//     operand; dims 320..575 sit in shared memory (TMA, 128-byte swizzle).
//   * Latent rows c_j are gathered 32 at a time through the block table with TMA tile::gather4
//     (4 rows x 64 dims per copy, 72 copies per tile) into a 4-stage ring; the tensor map's 128-byte
//     swizzle follows the shared-memory address, so 4-row copies at 512-byte steps build the
//     canonical K-major UMMA layout (9 blocks of 64 dims, 8-row atoms).
//   * S tile [128 heads x 32 keys] accumulates in TMEM (double-buffered), the softmax warps turn it
//     into P (bf16) in TMEM, and O[:, half] (128 x 256 fp32) accumulates in TMEM from P x V with
//     V read from the same shared-memory stage in its MN-major view.
//   * Online softmax with lazy rescaling: the reference maximum only moves when a tile's maximum
//     exceeds it by more than 2^8, so O is rarely touched outside the MMAs.
// TMEM columns: O 0..255 | S 256..319 (2 x 32) | P 320..351 (2 x 16) | Q 352..511 (160).
// Warps: 0 gather producer (TMA), 1 MMA issuer (+ TMEM allocator), 2-5 softmax and epilogue.
//
// Splits (several CTAs over one S_t) write normalised partial outputs and their log-sum-exp to the
// workspace; a combine kernel merges them: o = sum_s exp(lse_s - lse) o_s.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

namespace dsa {

int make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* ptr, uint64_t inner,
                 uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows);

namespace {

constexpr int kTileKeys = 32;
constexpr int kStages = 4;
constexpr int kBlkBytes = kTileKeys * 128;           // one 64-dim block of a tile: 4 KB
constexpr int kStageBytes = 9 * kBlkBytes;           // 36 KB
constexpr int kQTmemDims = 320;                      // Q dims held in TMEM
constexpr int kQSmemBlocks = (kDLat - kQTmemDims) / 64;  // 4 blocks in shared memory
constexpr int kQBlkBytes = 128 * 128;                // 16 KB
constexpr int kMaxKeysPerCta = 2048;
constexpr int kThreads = 192;
constexpr float kRescaleThreshold = 8.0f;            // log2 units

constexpr uint32_t kColO = 0, kColS = 256, kColP = 320, kColQ = 352;

struct MlaSmem {
  static constexpr int kQ = 0;
  static constexpr int kStage0 = kQ + kQSmemBlocks * kQBlkBytes;      // 64 KB
  static constexpr int kRows = kStage0 + kStages * kStageBytes;        // 208 KB
  static constexpr int kBars = kRows + kMaxKeysPerCta * 4;             // 216 KB
  static constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 2 + 1 + 1;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kTotal = kTmemSlot + 16;
  static constexpr int kDynamic = kTotal + 1024;
};
static_assert(MlaSmem::kDynamic <= 232448, "sparse MLA shared memory exceeds the 227 KB limit");

struct MlaParams {
  BatchDev bd;
  const int32_t* row_req;
  const int32_t* row_pos;
  const uint16_t* q;
  const uint16_t* kv;
  const int32_t* S;
  int k;
  int H;
  int nsplit;
  int chunk;          // S_t entries per split (multiple of 32)
  float scale_log2;   // softmax scale * log2(e)
  uint16_t* out;
  float* lse;
  float* part_o;      // [T, nsplit, H, 512] when nsplit > 1
  float* part_lse;    // [T, nsplit, H]
  uint32_t* status;
};

__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kvmap,
                      const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  int32_t* rows = reinterpret_cast<int32_t*>(base + MlaSmem::kRows);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + MlaSmem::kBars);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + kStages;
  uint64_t* s_full = bars + 2 * kStages;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* p_free = p_full + 2;
  uint64_t* o_full = p_free + 2;
  uint64_t* q_full = o_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + MlaSmem::kTmemSlot);

  const int warp = warp_id(), lane = lane_id();
  const int t = blockIdx.x, v = blockIdx.y, split = blockIdx.z;
  const int H = p.H;
  const int b = __ldg(p.row_req + t);
  const int pos = __ldg(p.row_pos + t);
  const int nvis = min(p.k, pos + 1);                 // entries of S_t that can be valid
  const int e0 = split * p.chunk;
  const int nkeys = max(0, min(nvis - e0, p.chunk));  // entries this CTA reads
  const int ntiles = (nkeys + kTileKeys - 1) / kTileKeys;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(q_full, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- set-up: physical rows of this CTA's entries, Q into shared memory and TMEM ----------
  const int32_t* S_row = p.S + static_cast<int64_t>(t) * p.k + e0;
  const int32_t* bt_row = p.bd.block_table + static_cast<int64_t>(b) * p.bd.max_pages;
  const int n_b = __ldg(p.bd.seq_lens + b);
  for (int e = threadIdx.x; e < nkeys; e += kThreads) {
    const int j = __ldg(S_row + e);
    int r = -1;
    if (j >= 0) {
      if (j > pos || j >= n_b) {
        report_error(p.status, kDevErrIndex);
      } else {
        const int pg = __ldg(bt_row + j / kPage);
        if (pg < 0 || pg >= p.bd.num_pages)
          report_error(p.status, kDevErrIndex);
        else
          r = pg * kPage + (j % kPage);
      }
    }
    rows[e] = r;
  }
  if (threadIdx.x == 0 && ntiles > 0) {
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kvmap);
    mbar_arrive_expect_tx(q_full, kQSmemBlocks * kQBlkBytes);
    for (int i = 0; i < kQSmemBlocks; ++i)
      tma_load_2d(base + MlaSmem::kQ + i * kQBlkBytes, &qmap, kQTmemDims + 64 * i, t * H, q_full);
  }
  const int quad = warp & 3;
  const int h = quad * 32 + lane;  // head = TMEM lane owned by this softmax thread
  const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
  if (warp >= 2 && ntiles > 0) {
    const uint4* src = reinterpret_cast<const uint4*>(p.q + (static_cast<int64_t>(t) * H + h) * kDLat);
#pragma unroll 1
    for (int c = 0; c < kQTmemDims / 64; ++c) {  // 5 chunks of 64 dims = 32 TMEM columns
      uint32_t r[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint4 x = make_uint4(0, 0, 0, 0);
        if (h < H) x = __ldg(src + c * 8 + i);
        r[4 * i + 0] = x.x;
        r[4 * i + 1] = x.y;
        r[4 * i + 2] = x.z;
        r[4 * i + 3] = x.w;
      }
      tmem_st32(tmem + lane_base + kColQ + 32 * c, r);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // ---------------- gather producer (TMA gather4; lanes 0..8 own one 64-dim block each) ----------
    bool ok = true;
    for (int it = 0; it < ntiles && ok; ++it) {
      const int s = it % kStages;
      if (lane == 0) {
        ok = mbar_wait(&kv_empty[s], ((it / kStages) & 1) ^ 1, p.status, kDevErrTimeout);
        if (ok) mbar_arrive_expect_tx(&kv_full[s], kTileKeys * kDLat * 2);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane < kDLat / 64) {
        uint8_t* dst = base + MlaSmem::kStage0 + s * kStageBytes + lane * kBlkBytes;
#pragma unroll
        for (int g = 0; g < kTileKeys / 4; ++g) {
          int r[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int e = it * kTileKeys + 4 * g + i;
            r[i] = (e < nkeys) ? rows[e] : -1;
            if (r[i] < 0) r[i] = 0;  // masked in the softmax; any readable row will do
          }
          tma_gather4(dst + g * 512, &kvmap, lane * 64, r[0], r[1], r[2], r[3], &kv_full[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && ntiles > 0) {
      bool ok = mbar_wait(q_full, 0, p.status, kDevErrTimeout);
      const uint32_t idesc_s = umma_idesc(128, kTileKeys, 1, 0, 0);  // bf16, K-major A and B
      const uint32_t idesc_o = umma_idesc(128, 256, 1, 0, 1);        // bf16, B MN-major
      // Descriptors are built once; a K step only moves the 14-bit start-address field, so it is a
      // plain add of a compile-time constant (addresses stay below 256 KB: no carry out of the field).
      const uint64_t q_desc0 = umma_desc_sw128(smem_u32(base + MlaSmem::kQ), 16, 1024);
      const uint64_t k_desc0 = umma_desc_sw128(smem_u32(base + MlaSmem::kStage0), 16, 1024);
      const uint64_t v_desc0 = umma_desc_sw128(smem_u32(base + MlaSmem::kStage0) + 4 * v * kBlkBytes, kBlkBytes, 1024);
      for (int it = 0; it <= ntiles && ok; ++it) {
        if (it < ntiles) {
          const int s = it % kStages, sb = it & 1;
          ok = mbar_wait(&kv_full[s], (it / kStages) & 1, p.status, kDevErrTimeout) &&
               mbar_wait(&s_free[sb], ((it >> 1) & 1) ^ 1, p.status, kDevErrTimeout);
          if (!ok) break;
          tc_fence_after();
          const uint64_t kd = k_desc0 + static_cast<uint64_t>((s * kStageBytes) >> 4);
          const uint32_t d = tmem + kColS + 32 * sb;
#pragma unroll
          for (int ks = 0; ks < kDLat / 16; ++ks) {
            const uint64_t bdesc = kd + static_cast<uint64_t>(((ks >> 2) * kBlkBytes + (ks & 3) * 32) >> 4);
            if (ks < kQTmemDims / 16) {
              mma_bf16_ts(d, tmem + kColQ + 8 * ks, bdesc, idesc_s, ks > 0 ? 1u : 0u);
            } else {
              const int qs = ks - kQTmemDims / 16;
              const uint64_t adesc = q_desc0 + static_cast<uint64_t>(((qs >> 2) * kQBlkBytes + (qs & 3) * 32) >> 4);
              mma_bf16_ss(d, adesc, bdesc, idesc_s, 1u);
            }
          }
          mma_commit(&s_full[sb]);
        }
        if (it >= 1) {
          const int i = it - 1, pb = i & 1, s = i % kStages;
          ok = mbar_wait(&p_full[pb], (i >> 1) & 1, p.status, kDevErrTimeout);
          if (!ok) break;
          tc_fence_after();
          const uint64_t vd = v_desc0 + static_cast<uint64_t>((s * kStageBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kTileKeys / 16; ++kk) {
            mma_bf16_ts(tmem + kColO, tmem + kColP + 16 * pb + 8 * kk, vd + static_cast<uint64_t>((kk * 2048) >> 4),
                        idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&p_free[pb]);
          mma_commit(&kv_empty[s]);
          if (i == ntiles - 1) mma_commit(o_full);
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax + epilogue (warps 2..5, one head per thread) ----------------
    // l: sum of the fp32 weights (for the log-sum-exp); lr: sum of the bf16-rounded weights the
    // P x V MMA actually uses (normalises O, so the output weights sum to one).
    float m_ref = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    for (int it = 0; it < ntiles && ok; ++it) {
      const int sb = it & 1;
      ok = mbar_wait(&s_full[sb], (it >> 1) & 1, p.status, kDevErrTimeout);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t sv[32];
      tmem_ld32(tmem + lane_base + kColS + 32 * sb, sv);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      float x[32];
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int e = it * kTileKeys + c;
        const bool valid = e < nkeys && rows[e] >= 0;
        x[c] = valid ? __uint_as_float(sv[c]) * p.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, x[c]);
      }
      // Lazy rescale, decided per head but executed by the whole warp (TMEM loads/stores are
      // warp-collective): lanes that keep their reference use alpha = 1.
      const bool need = tmax > m_ref + kRescaleThreshold;
      const float alpha = need ? exp2f(m_ref - tmax) : 1.f;  // 0 when m_ref is -inf
      if (__any_sync(0xffffffffu, need && it >= 1 && m_ref > -INFINITY)) {
        ok = mbar_wait(&p_free[(it - 1) & 1], ((it - 1) >> 1) & 1, p.status, kDevErrTimeout);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + kColO + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem + lane_base + kColO + 32 * c, o);
        }
        tmem_wait_st();
      }
      if (need) {
        l *= alpha;
        lr *= alpha;
        m_ref = tmax;
      }
      if (it >= 2) {
        ok = mbar_wait(&p_free[sb], ((it - 2) >> 1) & 1, p.status, kDevErrTimeout);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
      }
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float p0 = (m_ref > -INFINITY) ? exp2f(x[2 * c] - m_ref) : 0.f;
        const float p1 = (m_ref > -INFINITY) ? exp2f(x[2 * c + 1] - m_ref) : 0.f;
        const __nv_bfloat162 bp = __floats2bfloat162_rn(p0, p1);
        l += p0 + p1;
        lr += __low2float(bp) + __high2float(bp);
        pk[c] = *reinterpret_cast<const uint32_t*>(&bp);
      }
      tmem_st16(tmem + lane_base + kColP + 16 * sb, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok && ntiles > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(o_full, 0, p.status, kDevErrTimeout));
      tc_fence_after();
    }
    const float inv = (lr > 0.f) ? 1.f / lr : 0.f;
    const float lse_nat = (l > 0.f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
    const bool have_o = ok && ntiles > 0;
    if (p.nsplit == 1) {
      uint16_t* dst = p.out + (static_cast<int64_t>(t) * H + h) * kDV + v * 256;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(tmem + lane_base + kColO + 32 * c, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        if (h < H) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
            d4[i] = w;
          }
        }
      }
      if (v == 0 && h < H && p.lse) p.lse[static_cast<int64_t>(t) * H + h] = lse_nat;
    } else {
      const int64_t prow = (static_cast<int64_t>(t) * p.nsplit + split) * H + h;
      float* dst = p.part_o + prow * kDV + v * 256;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(tmem + lane_base + kColO + 32 * c, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        if (h < H) {
          float4* d4 = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
        }
      }
      if (v == 0 && h < H) p.part_lse[prow] = lse_nat;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One warp per (row, head): o = sum_s exp(lse_s - lse) o_s, lse = log sum_s exp(lse_s).
__global__ void __launch_bounds__(256) mla_combine_kernel(const float* __restrict__ part_o,
                                                          const float* __restrict__ part_lse, int T, int H,
                                                          int nsplit, uint16_t* __restrict__ out,
                                                          float* __restrict__ lse) {
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= T * H) return;
  const int t = gw / H, h = gw % H;
  float mx = -INFINITY;
  for (int s = 0; s < nsplit; ++s) mx = fmaxf(mx, __ldg(part_lse + (static_cast<int64_t>(t) * nsplit + s) * H + h));
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (mx > -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const int64_t prow = (static_cast<int64_t>(t) * nsplit + s) * H + h;
      const float w = expf(__ldg(part_lse + prow) - mx);
      wsum += w;
      const float4* src = reinterpret_cast<const float4*>(part_o + prow * kDV) + lane * 4;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 x = __ldg(src + i);
        acc[4 * i + 0] = fmaf(w, x.x, acc[4 * i + 0]);
        acc[4 * i + 1] = fmaf(w, x.y, acc[4 * i + 1]);
        acc[4 * i + 2] = fmaf(w, x.z, acc[4 * i + 2]);
        acc[4 * i + 3] = fmaf(w, x.w, acc[4 * i + 3]);
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<int64_t>(t) * H + h) * kDV) + lane * 2;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    uint4 w;
    w.x = pack_bf16x2(acc[8 * i + 0] * inv, acc[8 * i + 1] * inv);
    w.y = pack_bf16x2(acc[8 * i + 2] * inv, acc[8 * i + 3] * inv);
    w.z = pack_bf16x2(acc[8 * i + 4] * inv, acc[8 * i + 5] * inv);
    w.w = pack_bf16x2(acc[8 * i + 6] * inv, acc[8 * i + 7] * inv);
    dst[i] = w;
  }
  if (lane == 0 && lse) lse[static_cast<int64_t>(t) * H + h] = (wsum > 0.f) ? mx + logf(wsum) : -INFINITY;
}

}  // namespace

int sparse_mla_splits(int T, int k) {
  const int min_splits = (k + kMaxKeysPerCta - 1) / kMaxKeysPerCta;
  const int ctas = 2 * T;
  int n = 1;
  if (ctas > 0 && ctas < 111) n = (148 + ctas - 1) / ctas;
  const int max_by_tiles = (k + kTileKeys - 1) / kTileKeys;
  if (n > 16) n = 16;
  if (n > max_by_tiles) n = max_by_tiles;
  if (n < min_splits) n = min_splits;
  return n;
}

size_t sparse_mla_ws_bytes(int T, int H, int k) {
  const int n = sparse_mla_splits(T, k);
  if (n <= 1) return 0;
  return align16(sizeof(float) * static_cast<size_t>(T) * n * H * kDV) +
         align16(sizeof(float) * static_cast<size_t>(T) * n * H);
}

int launch_sparse_mla(const BatchDev& b, const void* plan, const void* q, int H, const void* kv_cache,
                      const int32_t* S, int k, float softmax_scale, void* out, float* lse, void* ws, void* stream) {
  if (b.T == 0) return 0;
  PlanView pv = plan_view(const_cast<void*>(plan), b.B, b.T);
  MlaParams prm{};
  prm.bd = b;
  prm.row_req = pv.row_req;
  prm.row_pos = pv.row_pos;
  prm.q = static_cast<const uint16_t*>(q);
  prm.kv = static_cast<const uint16_t*>(kv_cache);
  prm.S = S;
  prm.k = k;
  prm.H = H;
  prm.nsplit = sparse_mla_splits(b.T, k);
  const int per = (k + prm.nsplit - 1) / prm.nsplit;
  prm.chunk = (per + kTileKeys - 1) / kTileKeys * kTileKeys;
  prm.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634);
  prm.out = static_cast<uint16_t*>(out);
  prm.lse = lse;
  if (prm.nsplit > 1) {
    prm.part_o = static_cast<float*>(ws);
    prm.part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                            align16(sizeof(float) * static_cast<size_t>(b.T) * prm.nsplit * H * kDV));
  }
  prm.status = &pv.hdr->status;

  CUtensorMap qmap, kvmap;
  int e = make_tmap_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, kDLat, static_cast<uint64_t>(b.T) * H,
                       kDLat * 2, 64, 128);
  if (e) return e;
  e = make_tmap_2d(&kvmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kv_cache, kDLat,
                   static_cast<uint64_t>(b.num_pages) * kPage, kDLat * 2, 64, 1);
  if (e) return e;
  cudaError_t ce =
      cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, MlaSmem::kDynamic);
  if (ce != cudaSuccess) return static_cast<int>(ce);
  dim3 grid(b.T, 2, prm.nsplit);
  sparse_mla_kernel<<<grid, kThreads, MlaSmem::kDynamic, static_cast<cudaStream_t>(stream)>>>(qmap, kvmap, prm);
  ce = cudaGetLastError();
  if (ce != cudaSuccess) return static_cast<int>(ce);
  if (prm.nsplit > 1) {
    const int warps = b.T * H;
    mla_combine_kernel<<<(warps + 7) / 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        prm.part_o, prm.part_lse, b.T, H, prm.nsplit, prm.out, lse);
    ce = cudaGetLastError();
  }
  return static_cast<int>(ce);
}

}  // namespace dsa
