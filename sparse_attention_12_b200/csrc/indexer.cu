// Lightning-Indexer scores on sm_100a.
//
//   I_tj = s^q_t * s^k_j * sum_r w_tr * ReLU(q_tr . k_j),   j <= p_t
//
// ("DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section "Lightning Indexer", formula
// for I_tj; FP8 with 64 heads of width 128 per "MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：
// NSA 与 DSA", which names this kernel an FP8 small GEMM + ReLU + weighted sum.) The per-token
// scales are positive, so they factor out of the ReLU and are applied once per score.
//
// GEMM view: M = 128 keys (two 64-position pages of the paged key cache), N = queries x heads of one
// "group" (<= 256 columns), K = 128 FP8 bytes. One tcgen05 kind::f8f6f4 MMA chain of 4 x K32 per
// tile accumulates fp32 in TMEM: TMEM lane i holds key i, column q*nhI + r holds head r of query q.
// The epilogue thread that owns lane i reads its row, applies ReLU, w and the head sum in
// registers and writes one fp32 score per query; the per-head products never leave the SM.
//
// Persistent CTAs (one per SM) walk a contiguous slice of the plan's tile list. Warp roles:
//   warp 0      TMA producer: key pages (via the block table) into a ring of 9..12 stages, the
//               tile's s^k into its own ring (cp.async), query tiles and the group's w / s^q into
//               a 2-deep buffer
//   warp 1      TMEM allocator and single-thread MMA issuer
//   warps 2..9  epilogue (two warps per TMEM lane quadrant; the (tile, query) items alternate
//               between the two, so a single-query decode group keeps both busy)
// Decode tiles are HBM-bound (16 KB of keys per 128x64x128 MMA chain); prefill tiles are
// tensor-bound with the 8 epilogue warps keeping pace with the MMA.
#include <cuda.h>
#include <cuda_runtime.h>

#include <type_traits>

#include <cmath>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

#ifdef DSA_TEST_FAULTS
// Test-only build (never the product library): a switch that makes every indexer CTA leave the
// keys of its first tile unloaded, so that the MMA issuer's bounded wait runs out and the kernel
// must record DSA_ERR_TIMEOUT, let its other copies land, free TMEM and return.
__device__ int g_test_fault = 0;
extern "C" int dsa_test_set_fault(int code) {
  return static_cast<int>(cudaMemcpyToSymbol(g_test_fault, &code, sizeof(code)));
}
#endif

namespace dsa {
namespace {

constexpr int kMaxStages = 14;  // key stages: as many as shared memory holds next to the query buffers
constexpr int kScaleSlots = 16;  // s^k of a tile (512 B) in its own ring: key stages free at MMA completion
constexpr int kStageBytes = kIdxTileKeys * kDIdx;  // 16 KB
constexpr int kMaxAcc = 8;
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;

struct __align__(16) GroupMeta {
  int32_t row0, nq, pos0, req;
};

// Shared memory: the fixed part first, then two query buffers of qbytes (the group's query box,
// 8 KB for one query of 64 heads, up to 32 KB) and as many 16 KB key stages as fit; the host
// computes qbytes and the stage count (12 stages for decode, 9 for 256-row prefill groups).
struct IdxSmem {
  // byte offsets relative to the 1024-aligned base
  static constexpr int kW = 0;                                     // float [2][256]
  static constexpr int kScale = kW + 2 * kIdxCols * 4;            // float [kScaleSlots][128]: s^k of a tile
  static constexpr int kSq = kScale + kScaleSlots * kIdxTileKeys * 4;  // float [2][16]
  static constexpr int kMeta = kSq + 2 * 16 * 4;                  // GroupMeta [2]
  static constexpr int kBars = kMeta + 2 * 16;                    // uint64 barriers
  static constexpr int kNumBars = 2 * kMaxStages + 4 + 2 * kMaxAcc + 2 * kScaleSlots + 1;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kFixed = (kTmemSlot + 16 + 1023) / 1024 * 1024;  // query buffers start here
  static constexpr int kLimit = 232448 - 1024;  // 227 KB less the slack for the 1024-byte alignment
};

struct IdxParams {
  BatchDev bd;
  const PlanHeader* hdr;
  const int32_t* grp_row0;
  const int32_t* grp_nq;
  const int32_t* grp_req;
  const int32_t* grp_pos0;
  const int32_t* grp_tile0;
  const float* qI_scale;
  const float* wI;
  const float* kI_scale;
  float* scores;
  int64_t ld;
  int ncols;      // TMEM columns per accumulator buffer (power of two >= 32)
  int nacc;       // accumulator buffers
  int qbox_rows;  // query rows per TMA box
  int qbytes;     // bytes per query buffer (multiple of 1024)
  int nstages;    // key stages
  uint32_t* status;
};

// Last group g in [0, G) with tile0[g] <= u (tile0 strictly increasing, tile0[0] = 0 <= u),
// searched by a whole warp with 32 probes per round: about log32(G) dependent loads.
__device__ __forceinline__ int find_group_warp(const int32_t* tile0, int G, int u) {
  const int lane = threadIdx.x & 31;
  int lo = 0, hi = G - 1;  // the answer lies in [lo, hi]
  while (hi > lo) {
    const int span = hi - lo;
    const int pos = lo + static_cast<int>((static_cast<int64_t>(lane + 1) * span + 31) / 32);  // in (lo, hi]
    const bool le = __ldg(tile0 + pos) <= u;  // true on a prefix of the lanes
    const uint32_t m = __ballot_sync(0xffffffffu, le);
    const int l = m ? 31 - __clz(m) : -1;
    const int p0 = __shfl_sync(0xffffffffu, pos, 0);
    const int pl = __shfl_sync(0xffffffffu, pos, l < 0 ? 0 : l);
    const int pn = __shfl_sync(0xffffffffu, pos, l < 31 ? l + 1 : 31);
    if (l < 0) {
      hi = p0 - 1;
    } else {
      lo = pl;
      if (l < 31) hi = pn - 1;
    }
  }
  return lo;
}

template <int NHI>
__global__ void __launch_bounds__(kThreads, 1)
    index_scores_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                        const IdxParams p) {
  constexpr int QPG = kIdxCols / NHI;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float* g_w = reinterpret_cast<float*>(base + IdxSmem::kW);
  float* g_sq = reinterpret_cast<float*>(base + IdxSmem::kSq);
  float* g_scale = reinterpret_cast<float*>(base + IdxSmem::kScale);
  GroupMeta* g_meta = reinterpret_cast<GroupMeta*>(base + IdxSmem::kMeta);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + IdxSmem::kBars);
  uint64_t* kfull = bars;
  uint64_t* kempty = bars + kMaxStages;
  uint64_t* qfull = bars + 2 * kMaxStages;
  uint64_t* qempty = qfull + 2;
  uint64_t* tfull = qempty + 2;
  uint64_t* tempty = tfull + kMaxAcc;
  uint64_t* sfull = tempty + kMaxAcc;
  uint64_t* sempty = sfull + kScaleSlots;
  uint64_t* mdone = sempty + kScaleSlots;  // the MMA issuer's last commit (drained before TMEM is freed)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + IdxSmem::kTmemSlot);

  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nstages; ++s) {
      mbar_init(&kfull[s], 1);  // TMA bytes of the keys
      mbar_init(&kempty[s], 1);  // MMA done with the keys
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&qfull[b], 1);
      mbar_init(&qempty[b], 1 + kEpiWarps);
    }
    for (int c = 0; c < kScaleSlots; ++c) {
      mbar_init(&sfull[c], 32);          // one cp.async arrival per producer lane
      mbar_init(&sempty[c], kEpiWarps);  // epilogue read the scales
    }
    for (int a = 0; a < kMaxAcc; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);
    }
    mbar_init(mdone, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&qmap);
  }
  pdl_trigger();
  pdl_wait();  // the plan, written by the previous kernel
  const int G = p.hdr->num_groups;
  const int U = p.hdr->total_tiles;
  const int u0 = static_cast<int>((static_cast<int64_t>(U) * blockIdx.x) / gridDim.x);
  const int u1 = static_cast<int>((static_cast<int64_t>(U) * (blockIdx.x + 1)) / gridDim.x);
  const int g_first = (u0 < u1) ? find_group_warp(p.grp_tile0, G, u0) : 0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (u0 < u1) {
    if (warp == 0) {
      // ---------------- producer ----------------
      int g = g_first;
      int gstart = __ldg(p.grp_tile0 + g), gend = __ldg(p.grp_tile0 + g + 1);
      GroupMeta gm{};
      int qcount = 0;
      int pg_base = -1;  // first logical page held in `pg_cache`
      int pg_cache = 0, pg_next = 0;  // this window's page ids and the next window's (prefetched)
      bool ok = true;
      int s = 0, s_par = 1, c = 0, c_par = 1;  // ring positions of tile it and the parity to wait for
      int issued = 0, q_issued = 0;            // key tiles and query boxes whose loads went out
      int skipped = -1;                        // a key tile left unloaded by the test-only fault switch
      for (int u = u0, it = 0; u < u1 && ok; ++u, ++it) {
        const bool newg = (u == u0) || (u == gend);
        if (u == gend) {
          ++g;
          gstart = gend;
          gend = __ldg(p.grp_tile0 + g + 1);
        }
        if (newg) {
          const int qb = qcount & 1;
          if (lane == 0) ok = mbar_wait(&qempty[qb], ((qcount >> 1) & 1) ^ 1, p.status, kDevErrTimeout);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          gm.row0 = __ldg(p.grp_row0 + g);
          gm.nq = __ldg(p.grp_nq + g);
          gm.pos0 = __ldg(p.grp_pos0 + g);
          gm.req = __ldg(p.grp_req + g);
          for (int idx = lane; idx < QPG * NHI; idx += 32) {
            const int q = idx / NHI;
            g_w[qb * kIdxCols + idx] = (q < gm.nq) ? __ldg(p.wI + static_cast<int64_t>(gm.row0 + q) * NHI + (idx % NHI)) : 0.f;
          }
          if (lane < QPG) g_sq[qb * 16 + lane] = (lane < gm.nq) ? __ldg(p.qI_scale + gm.row0 + lane) : 0.f;
          if (lane == 0) g_meta[qb] = gm;
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_expect_tx(&qfull[qb], static_cast<uint32_t>(p.qbox_rows * kDIdx));
            tma_load_2d(base + IdxSmem::kFixed + qb * p.qbytes, &qmap, 0, gm.row0 * NHI, &qfull[qb]);
          }
          ++qcount;
          q_issued = qcount;
          pg_base = -1;
        }
        const int kt = u - gstart;
        const int lp0 = 2 * kt;
        // block-table window of 32 logical pages, refreshed every 16 tiles; the next window is
        // loaded one window ahead so the refresh does not wait on memory
        if (pg_base < 0 || lp0 >= pg_base + 32) {
          const int npages = (gm.pos0 + gm.nq - 1) / kPage + 1;
          const int32_t* bt = p.bd.block_table + static_cast<int64_t>(gm.req) * p.bd.max_pages;
          if (pg_base >= 0 && lp0 == pg_base + 32) {
            pg_cache = pg_next;
          } else {
            pg_cache = (lp0 + lane < npages) ? __ldg(bt + lp0 + lane) : 0;
          }
          pg_base = lp0;
          pg_next = (pg_base + 32 + lane < npages) ? __ldg(bt + pg_base + 32 + lane) : 0;
        }
        const int pg0 = __shfl_sync(0xffffffffu, pg_cache, lp0 - pg_base);
        const int pg1 = __shfl_sync(0xffffffffu, pg_cache, lp0 + 1 - pg_base);
        // every lane tests the two slots itself (no broadcast on the per-tile path)
        ok = mbar_wait(&kempty[s], s_par, p.status, kDevErrTimeout) &&
             mbar_wait(&sempty[c], c_par, p.status, kDevErrTimeout);
        if (!__all_sync(0xffffffffu, ok)) break;
        const int p_last = gm.pos0 + gm.nq - 1;
        const bool v1 = (lp0 + 1) * kPage <= p_last;
        const int q0 = min(max(pg0, 0), p.bd.num_pages - 1), q1 = min(max(pg1, 0), p.bd.num_pages - 1);
#ifdef DSA_TEST_FAULTS
        const bool skip = g_test_fault == 1 && it == 0;  // this tile's keys never arrive
#else
        constexpr bool skip = false;
#endif
        if (skip) skipped = it;
        if (lane == 0 && !skip) {
          if (pg0 < 0 || pg0 >= p.bd.num_pages || (v1 && (pg1 < 0 || pg1 >= p.bd.num_pages)))
            report_error(p.status, kDevErrIndex);
          uint8_t* dst = base + IdxSmem::kFixed + 2 * p.qbytes + s * kStageBytes;
          mbar_arrive_expect_tx(&kfull[s], static_cast<uint32_t>((v1 ? 2 : 1) * kPage * kDIdx));
          tma_load_2d(dst, &kmap, 0, q0 * kPage, &kfull[s]);
          if (v1) tma_load_2d(dst + kPage * kDIdx, &kmap, 0, q1 * kPage, &kfull[s]);
        }
        issued = it + 1;
        // s^k of the tile's 128 keys: 16 bytes per lane (lanes 0..15 page 0, 16..31 page 1)
        cp_async_16(smem_u32(g_scale + c * kIdxTileKeys + 4 * lane),
                    p.kI_scale + static_cast<int64_t>(lane < 16 ? q0 : q1) * kPage + 4 * (lane & 15));
        cp_async_mbar_arrive_noinc(&sfull[c]);
        if (++s == p.nstages) s = 0, s_par ^= 1;
        if (++c == kScaleSlots) c = 0, c_par ^= 1;
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
      // no copy may still be landing when the CTA exits, also after an error: the last loads of
      // every key stage and query buffer (already complete in a run without errors)
      if (lane == 0) {
        for (int j = max(0, issued - p.nstages); j < issued; ++j)
          if (j != skipped) mbar_drain(&kfull[j % p.nstages], (j / p.nstages) & 1, p.status);
        for (int j = max(0, q_issued - 2); j < q_issued; ++j) mbar_drain(&qfull[j & 1], (j >> 1) & 1, p.status);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ---------------- MMA issuer ----------------
      if (lane == 0) {
        // the group bounds and sizes come one group ahead, so a group switch waits on no load
        int g = g_first;
        int gend = __ldg(p.grp_tile0 + g + 1);
        int nq = __ldg(p.grp_nq + g);
        int g_last = (g + 1 < G) ? g + 1 : g;
        int gend_next = __ldg(p.grp_tile0 + g_last + 1), nq_next = __ldg(p.grp_nq + g_last);
        int qcount = 0, qb = 0;
        int s = 0, s_par = 0, a = 0, a_par = 1;  // key stage and accumulator of tile it, parities to wait for
        bool ok = true;
        for (int u = u0, it = 0; u < u1 && ok; ++u, ++it) {
          const bool newg = (u == u0) || (u == gend);
          if (u == gend) {
            ++g;
            gend = gend_next;
            nq = nq_next;
            g_last = (g + 1 < G) ? g + 1 : g;
            gend_next = __ldg(p.grp_tile0 + g_last + 1);
            nq_next = __ldg(p.grp_nq + g_last);
          }
          if (newg) {
            qb = qcount & 1;
            ok = mbar_wait(&qfull[qb], (qcount >> 1) & 1, p.status, kDevErrTimeout);
            if (!ok) break;
            ++qcount;
          }
          ok = mbar_wait(&kfull[s], s_par, p.status, kDevErrTimeout) &&
               mbar_wait(&tempty[a], a_par, p.status, kDevErrTimeout);
          if (!ok) break;
          tc_fence_after();
          const uint32_t idesc = umma_idesc(128, static_cast<uint32_t>(nq * NHI), 0, 0, 0);
          const uint64_t ad =
              umma_desc_sw128(smem_u32(base + IdxSmem::kFixed + 2 * p.qbytes + s * kStageBytes), 16, 1024);
          const uint64_t bd = umma_desc_sw128(smem_u32(base + IdxSmem::kFixed + qb * p.qbytes), 16, 1024);
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * p.ncols);
#pragma unroll
          for (int k = 0; k < kDIdx / 32; ++k)  // K step of 32 bytes = +2 in the start-address field
            mma_f8_ss(d_tmem, ad + 2 * k, bd + 2 * k, idesc, k > 0 ? 1u : 0u);
          mma_commit(&kempty[s]);
          mma_commit(&tfull[a]);
          if (u + 1 == gend || u + 1 == u1) mma_commit(&qempty[qb]);
          if (++s == p.nstages) s = 0, s_par ^= 1;
          if (++a == p.nacc) a = 0, a_par ^= 1;
        }
        // every MMA this thread issued has completed before TMEM is freed (also after an error)
        mma_commit(mdone);
        mbar_drain(mdone, 0, p.status);
      }
      __syncwarp();
    } else {
      // ---------------- epilogue ----------------
      const int ew = warp - 2;
      const int quad = warp & 3;
      const int half = ew >> 2;
      const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
      int g = g_first;
      int gstart = __ldg(p.grp_tile0 + g), gend = __ldg(p.grp_tile0 + g + 1);
      int gend_next = __ldg(p.grp_tile0 + min(g + 1, G - 1) + 1);  // one group ahead
      int qcount = 0, qb = 0;
      int a = 0, a_par = 0;  // accumulator of tile it and the parity to wait for
      GroupMeta gm{};
      bool ok = true;
      for (int u = u0, it = 0; u < u1 && ok; ++u, ++it) {
        const bool newg = (u == u0) || (u == gend);
        if (u == gend) {
          ++g;
          gstart = gend;
          gend = gend_next;
          gend_next = __ldg(p.grp_tile0 + min(g + 1, G - 1) + 1);
        }
        if (newg) {
          qb = qcount & 1;
          ok = __all_sync(0xffffffffu, mbar_wait(&qfull[qb], (qcount >> 1) & 1, p.status, kDevErrTimeout));
          if (!ok) break;
          gm = g_meta[qb];
          ++qcount;
        }
        const int kt = u - gstart;
        const int j = kt * kIdxTileKeys + quad * 32 + lane;
        const int p_last = gm.pos0 + gm.nq - 1;
        const int c = it % kScaleSlots;
        // (not kfull: key stages recycle at MMA completion and may run a whole ring ahead of here)
        ok = __all_sync(0xffffffffu, mbar_wait(&sfull[c], (it / kScaleSlots) & 1, p.status, kDevErrTimeout) &&
                                         mbar_wait(&tfull[a], a_par, p.status, kDevErrTimeout));
        if (!ok) break;
        const float sk = (j <= p_last) ? g_scale[c * kIdxTileKeys + quad * 32 + lane] : 0.f;
        tc_fence_after();
        const uint32_t t_row = tmem_base + lane_base + static_cast<uint32_t>(a * p.ncols);
        // items (tile it, query q) alternate between the quadrant's two warps; a warp takes its
        // items two at a time (q and q + 2) when it has two, so that eight independent chains hide
        // the latency of the head sum. Per item the arithmetic and its order are the same.
        auto items = [&](auto two_tag, int qa) {
          constexpr bool kTwo = decltype(two_tag)::value;
          const int qz = kTwo ? qa + 2 : qa;
          const float4* wa = reinterpret_cast<const float4*>(g_w + qb * kIdxCols + qa * NHI);
          const float4* wz = reinterpret_cast<const float4*>(g_w + qb * kIdxCols + qz * NHI);
          // chains (a0, a1) and (a2, a3) of each item advance in pairs: one instruction per two heads
          float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);
          float2 z01 = make_float2(0.f, 0.f), z23 = make_float2(0.f, 0.f);
          auto accumulate = [&](const uint32_t* v, const float4* w4, int nv, int w0, float2& x01, float2& x23) {
#pragma unroll
            for (int i = 0; i < nv / 4; ++i) {
              const float4 ww = w4[w0 / 4 + i];
              x01 = fma_f32x2(make_float2(fmaxf(__uint_as_float(v[4 * i + 0]), 0.f), fmaxf(__uint_as_float(v[4 * i + 1]), 0.f)),
                              make_float2(ww.x, ww.y), x01);
              x23 = fma_f32x2(make_float2(fmaxf(__uint_as_float(v[4 * i + 2]), 0.f), fmaxf(__uint_as_float(v[4 * i + 3]), 0.f)),
                              make_float2(ww.z, ww.w), x23);
            }
          };
          if constexpr (NHI % 32 == 0) {
#pragma unroll
            for (int cc = 0; cc < NHI / 32; ++cc) {
              uint32_t va[32], vz[32];
              tmem_ld32(t_row + static_cast<uint32_t>(qa * NHI + cc * 32), va);
              if constexpr (kTwo) tmem_ld32(t_row + static_cast<uint32_t>(qz * NHI + cc * 32), vz);
              tmem_wait_ld();
              accumulate(va, wa, 32, cc * 32, a01, a23);
              if constexpr (kTwo) accumulate(vz, wz, 32, cc * 32, z01, z23);
            }
          } else {
            uint32_t va[16], vz[16];
            tmem_ld16(t_row + static_cast<uint32_t>(qa * NHI), va);
            if constexpr (kTwo) tmem_ld16(t_row + static_cast<uint32_t>(qz * NHI), vz);
            tmem_wait_ld();
            accumulate(va, wa, 16, 0, a01, a23);
            if constexpr (kTwo) accumulate(vz, wz, 16, 0, z01, z23);
          }
          auto store = [&](int q, float2 x01, float2 x23) {
            const float acc = (x01.x + x01.y) + (x23.x + x23.y);
            float score = acc * g_sq[qb * 16 + q] * sk;
            if (j > gm.pos0 + q) score = -INFINITY;
            if (j < p.ld) p.scores[static_cast<int64_t>(gm.row0 + q) * p.ld + j] = score;
          };
          store(qa, a01, a23);
          if constexpr (kTwo) store(qz, z01, z23);
        };
        for (int q = (half + it * gm.nq) & 1; q < gm.nq; q += 4) {
          if (q + 2 < gm.nq)
            items(std::true_type{}, q);
          else
            items(std::false_type{}, q);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sempty[c]);
          mbar_arrive(&tempty[a]);
          if (u + 1 == gend || u + 1 == u1) mbar_arrive(&qempty[qb]);
        }
        if (++a == p.nacc) a = 0, a_par ^= 1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

}  // namespace

int make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* ptr, uint64_t inner,
                 uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return static_cast<int>(cudaErrorNotSupported);
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  (void)elem_bytes;
  CUresult r = fn(map, dtype, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : static_cast<int>(cudaErrorInvalidValue);
}

// 3D tiled map (x innermost): dims {d0, d1, d2}, byte strides of dims 1 and 2, box {b0, b1, b2}.
int make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return static_cast<int>(cudaErrorNotSupported);
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, dtype, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : static_cast<int>(cudaErrorInvalidValue);
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
  }
  return n;
}

template <int NHI>
static int launch_index_scores_t(const BatchDev& b, const void* plan, const uint8_t* qI, const float* qI_scale,
                                 const float* wI, const uint8_t* kI_cache, const float* kI_scale, float* scores,
                                 int64_t ld, void* stream) {
  constexpr int QPG = kIdxCols / NHI;
  PlanView pv = plan_view(const_cast<void*>(plan), b.B, b.T);
  IdxParams prm{};
  prm.bd = b;
  prm.hdr = pv.hdr;
  prm.grp_row0 = pv.grp_row0;
  prm.grp_nq = pv.grp_nq;
  prm.grp_req = pv.grp_req;
  prm.grp_pos0 = pv.grp_pos0;
  prm.grp_tile0 = pv.grp_tile0;
  prm.qI_scale = qI_scale;
  prm.wI = wI;
  prm.kI_scale = kI_scale;
  prm.scores = scores;
  prm.ld = ld;
  const int qmax = b.max_q < QPG ? b.max_q : QPG;
  int ncols = 32;
  while (ncols < qmax * NHI) ncols <<= 1;
  prm.ncols = ncols;
  prm.nacc = (512 / ncols) < kMaxAcc ? (512 / ncols) : kMaxAcc;
  prm.qbox_rows = qmax * NHI;
  prm.status = &pv.hdr->status;

  CUtensorMap kmap, qmap;
  int e = make_tmap_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kI_cache, kDIdx,
                       static_cast<uint64_t>(b.num_pages) * kPage, kDIdx, kDIdx, kPage);
  if (e) return e;
  e = make_tmap_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, qI, kDIdx, static_cast<uint64_t>(b.T) * NHI, kDIdx,
                   kDIdx, static_cast<uint32_t>(prm.qbox_rows));
  if (e) return e;
  auto kern = index_scores_kernel<NHI>;
  prm.qbytes = (prm.qbox_rows * kDIdx + 1023) / 1024 * 1024;
  prm.nstages = (IdxSmem::kLimit - IdxSmem::kFixed - 2 * prm.qbytes) / kStageBytes;
  if (prm.nstages > kMaxStages) prm.nstages = kMaxStages;
  if (prm.nstages < 2) return static_cast<int>(cudaErrorInvalidValue);
  const int smem = IdxSmem::kFixed + 2 * prm.qbytes + prm.nstages * kStageBytes + 1024;
  cudaError_t ce = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (ce != cudaSuccess) return static_cast<int>(ce);
  return static_cast<int>(
      launch_pdl(kern, dim3(num_sms()), dim3(kThreads), static_cast<size_t>(smem), stream, kmap, qmap, prm));
}

int launch_index_scores(const BatchDev& b, const void* plan, const uint8_t* qI, const float* qI_scale,
                        const float* wI, int nhI, const uint8_t* kI_cache, const float* kI_scale, float* scores,
                        int64_t ld, void* stream) {
  switch (nhI) {
    case 16:
      return launch_index_scores_t<16>(b, plan, qI, qI_scale, wI, kI_cache, kI_scale, scores, ld, stream);
    case 32:
      return launch_index_scores_t<32>(b, plan, qI, qI_scale, wI, kI_cache, kI_scale, scores, ld, stream);
    case 64:
      return launch_index_scores_t<64>(b, plan, qI, qI_scale, wI, kI_cache, kI_scale, scores, ld, stream);
    case 128:
      return launch_index_scores_t<128>(b, plan, qI, qI_scale, wI, kI_cache, kI_scale, scores, ld, stream);
    default:
      return static_cast<int>(cudaErrorInvalidValue);
  }
}

}  // namespace dsa
