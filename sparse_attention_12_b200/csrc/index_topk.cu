// Fused Lightning-Indexer scores and TopK for decode batches (sm_100a): the score rows never leave
// the SMs.
//
//   I_tj = s^q_t * s^k_j * sum_r w_tr * ReLU(q_tr . k_j),   S_t = TopK_{j<=t}(I_tj, k)
//
// ("DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section "Lightning Indexer", formulas
// for I_tj and S_t; the page "MTP 与稀疏注意力：NSA 与 DSA", section "对推理引擎的新要求", names the
// FP8 scoring and the per-query top-k as the kernels DSA asks of an engine.)
//
// One cluster of C CTAs per request (all of its m_b <= 256/nhI queries form one MMA group). CTA r
// scores its contiguous slice of the request's 128-key tiles exactly as the indexer kernel does --
// TMA of the paged FP8 keys into a ring, one tcgen05 kind::f8f6f4 chain per tile into TMEM (keys on
// M, query-heads on N), an epilogue that applies ReLU, w, the head sum and the scales -- but writes
// each score as an order-preserving key into its own shared memory instead of a score row in HBM.
// When its slice is scored, the CTA's 16 warps run the exact cluster selection of
// select_cluster.cuh for every query of the request (the CTAs exchange their histograms,
// candidates and counts through distributed shared memory) and write S_t, positions in increasing
// order, ties to the smaller position: the same S_t that dsa_index_scores followed by dsa_topk
// gives for the same scores.
//
// Warp roles during the scoring: warp 0 TMA/cp.async producer, warp 1 TMEM allocator and MMA
// issuer, warps 2..9 epilogue (two per TMEM lane quadrant), warps 10..15 wait. The host picks C
// (1, 2, 4 or 8) and the key-ring depth so that the scores (queries x slice x 4 B), the ring, the
// query box and the histograms fill one SM's shared memory: one CTA per SM, so the 512-column TMEM
// allocation never waits for another CTA.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"
#include "select_cluster.cuh"

namespace dsa {

int make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* ptr, uint64_t inner,
                 uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows);

namespace {

constexpr int kThreads = 512;
constexpr int kEpiWarps = 8;
constexpr int kMaxStages = 12;
constexpr int kMinStages = 3;
constexpr int kScaleSlots = 16;
constexpr int kStageBytes = kIdxTileKeys * kDIdx;  // 16 KB: two pages of keys
constexpr int kMaxAcc = 8;
constexpr int kMaxCluster = sel::kMaxCluster;
constexpr int kMaxSliceKeys = 4 * kThreads * sel::kMaxChunks;  // 32768 keys per CTA and query
constexpr int kSmemLimit = 232448 - 1024;                         // 227 KB less the alignment slack

struct FusedSmem {
  static constexpr int kW = 0;                                           // float [256]
  static constexpr int kSq = kW + kIdxCols * 4;                          // float [16]
  static constexpr int kScale = kSq + 16 * 4;                            // float [kScaleSlots][128]
  static constexpr int kBars = kScale + kScaleSlots * kIdxTileKeys * 4;  // uint64 barriers
  static constexpr int kNumBars = 2 * kMaxStages + 1 + 2 * kMaxAcc + 2 * kScaleSlots + 1;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kFixed = (kTmemSlot + 16 + 1023) / 1024 * 1024;  // the query box starts here
};

struct FusedParams {
  BatchDev bd;
  const float* qI_scale;
  const float* wI;
  const float* kI_scale;
  int32_t* S;
  int k;
  int qbytes;      // bytes of the query box buffer (multiple of 1024)
  int qbox_rows;   // query rows per TMA box
  int ncols;       // TMEM columns per accumulator (power of two >= 32)
  int nacc;        // accumulator buffers
  int nstages;     // key stages
  int slice_cap;   // keys per query the score cache holds (multiple of 128)
  int ring_off;    // byte offsets of the key ring, the score cache and the histograms
  int cache_off;
  int hist_off;
  uint32_t* status;
};

template <int NHI>
__global__ void __launch_bounds__(kThreads, 1)
    index_topk_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                      const FusedParams p) {
  constexpr int QPG = kIdxCols / NHI;
  extern __shared__ uint8_t smem_raw[];
  __shared__ sel::Shared<kThreads> sh;
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float* g_w = reinterpret_cast<float*>(base + FusedSmem::kW);
  float* g_sq = reinterpret_cast<float*>(base + FusedSmem::kSq);
  float* g_scale = reinterpret_cast<float*>(base + FusedSmem::kScale);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + FusedSmem::kBars);
  uint64_t* kfull = bars;
  uint64_t* kempty = bars + kMaxStages;
  uint64_t* qfull = bars + 2 * kMaxStages;
  uint64_t* tfull = qfull + 1;
  uint64_t* tempty = tfull + kMaxAcc;
  uint64_t* sfull = tempty + kMaxAcc;
  uint64_t* sempty = sfull + kScaleSlots;
  uint64_t* mdone = sempty + kScaleSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + FusedSmem::kTmemSlot);
  uint8_t* qbuf = base + FusedSmem::kFixed;
  uint8_t* ring = base + p.ring_off;
  uint32_t* cache = reinterpret_cast<uint32_t*>(base + p.cache_off);  // [max_q][slice_cap] order keys
  uint32_t* hist = reinterpret_cast<uint32_t*>(base + p.hist_off);
  const uint32_t C = cluster_nctarank(), rank = cluster_ctarank();
  const int b = static_cast<int>(blockIdx.x / C);
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nstages; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
    }
    mbar_init(qfull, 1);
    for (int c = 0; c < kScaleSlots; ++c) {
      mbar_init(&sfull[c], 32);  // one cp.async arrival per producer lane
      mbar_init(&sempty[c], kEpiWarps);
    }
    for (int a = 0; a < kMaxAcc; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);
    }
    mbar_init(mdone, 1);
    fence_barrier_init();
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&qmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  sel::clear_state<kThreads>(sh, hist, C);
  sel::cluster_arrive();  // matched by the first selection's wait (or the no-op one below)
  pdl_trigger();
  pdl_wait();  // the caches and S may be written or read by the previous kernels
  const int row0 = __ldg(p.bd.cu_q + b);
  const int m = __ldg(p.bd.cu_q + b + 1) - row0;
  const int n_b = __ldg(p.bd.seq_lens + b);
  const int ntiles = (n_b + kIdxTileKeys - 1) / kIdxTileKeys;
  const int tpc = (ntiles + static_cast<int>(C) - 1) / static_cast<int>(C);
  const int t0 = min(ntiles, static_cast<int>(rank) * tpc);
  const int nt = (m > 0) ? min(ntiles, t0 + tpc) - t0 : 0;  // this CTA's tiles t0 .. t0 + nt - 1
  const int kbase = t0 * kIdxTileKeys;                       // its first position
  const int kend = min(n_b, (t0 + nt) * kIdxTileKeys);      // one past its last position
  const int p_last = n_b - 1;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (nt > 0) {
    if (warp == 0) {
      // ---------------- producer: the queries once, then the keys of tiles t0 .. t0 + nt - 1 ----------------
      for (int idx = lane; idx < QPG * NHI; idx += 32) {
        const int q = idx / NHI;
        g_w[idx] = (q < m) ? __ldg(p.wI + static_cast<int64_t>(row0 + q) * NHI + (idx % NHI)) : 0.f;
      }
      if (lane < QPG) g_sq[lane] = (lane < m) ? __ldg(p.qI_scale + row0 + lane) : 0.f;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(qfull, static_cast<uint32_t>(p.qbox_rows * kDIdx));
        tma_load_2d(qbuf, &qmap, 0, row0 * NHI, qfull);
      }
      const int32_t* bt = p.bd.block_table + static_cast<int64_t>(b) * p.bd.max_pages;
      const int npages = p_last / kPage + 1;
      int pg_base = -1, pg_cache = 0, pg_next = 0;  // a 32-page window of the block table, the next one prefetched
      bool ok = true;
      int issued = 0, skipped = -1;
      int s = 0, s_par = 1, c = 0, c_par = 1;
      for (int it = 0; it < nt && ok; ++it) {
        const int lp0 = 2 * (t0 + it);
        if (pg_base < 0 || lp0 >= pg_base + 32) {
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
        ok = mbar_wait(&kempty[s], s_par, p.status, kDevErrTimeout) &&
             mbar_wait(&sempty[c], c_par, p.status, kDevErrTimeout);
        if (!__all_sync(0xffffffffu, ok)) break;
        const bool v1 = (lp0 + 1) * kPage <= p_last;
        const int q0 = min(max(pg0, 0), p.bd.num_pages - 1), q1 = min(max(pg1, 0), p.bd.num_pages - 1);
        if (lane == 0) {
          if (pg0 < 0 || pg0 >= p.bd.num_pages || (v1 && (pg1 < 0 || pg1 >= p.bd.num_pages)))
            report_error(p.status, kDevErrIndex);
          uint8_t* dst = ring + s * kStageBytes;
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
      // no copy may still be landing when the CTA moves on, also after an error
      if (lane == 0) {
        for (int j = max(0, issued - p.nstages); j < issued; ++j)
          if (j != skipped) mbar_drain(&kfull[j % p.nstages], (j / p.nstages) & 1, p.status);
        mbar_drain(qfull, 0, p.status);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ---------------- MMA issuer ----------------
      if (lane == 0) {
        bool ok = mbar_wait(qfull, 0, p.status, kDevErrTimeout);
        const uint32_t idesc = umma_idesc(128, static_cast<uint32_t>(m * NHI), 0, 0, 0);
        const uint64_t bd = umma_desc_sw128(smem_u32(qbuf), 16, 1024);
        int s = 0, s_par = 0, a = 0, a_par = 1;  // key stage and accumulator of tile it, parities to wait for
        for (int it = 0; it < nt && ok; ++it) {
          ok = mbar_wait(&kfull[s], s_par, p.status, kDevErrTimeout) &&
               mbar_wait(&tempty[a], a_par, p.status, kDevErrTimeout);
          if (!ok) break;
          tc_fence_after();
          const uint64_t ad = umma_desc_sw128(smem_u32(ring + s * kStageBytes), 16, 1024);
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * p.ncols);
#pragma unroll
          for (int kk = 0; kk < kDIdx / 32; ++kk)  // K step of 32 bytes = +2 in the start-address field
            mma_f8_ss(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, kk > 0 ? 1u : 0u);
          mma_commit(&kempty[s]);
          mma_commit(&tfull[a]);
          if (++s == p.nstages) s = 0, s_par ^= 1;
          if (++a == p.nacc) a = 0, a_par ^= 1;
        }
        // every MMA this thread issued has completed before TMEM is freed (also after an error)
        mma_commit(mdone);
        mbar_drain(mdone, 0, p.status);
      }
      __syncwarp();
    } else if (warp < 2 + kEpiWarps) {
      // ---------------- epilogue: scores -> order keys in shared memory ----------------
      const int ew = warp - 2;
      const int quad = warp & 3;
      const int half = ew >> 2;
      const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
      bool ok = true;
      int a = 0, a_par = 0;  // accumulator of tile it and the parity to wait for
      for (int it = 0; it < nt && ok; ++it, (++a == p.nacc) ? (a = 0, a_par ^= 1) : 0) {
        const int c = it % kScaleSlots;
        ok = __all_sync(0xffffffffu, mbar_wait(&sfull[c], (it / kScaleSlots) & 1, p.status, kDevErrTimeout) &&
                                         mbar_wait(&tfull[a], a_par, p.status, kDevErrTimeout));
        if (!ok) break;
        const int jl = it * kIdxTileKeys + quad * 32 + lane;  // key index within this CTA's slice
        const float sk = (kbase + jl <= p_last) ? g_scale[c * kIdxTileKeys + quad * 32 + lane] : 0.f;
        tc_fence_after();
        const uint32_t t_row = tmem_base + lane_base + static_cast<uint32_t>(a * p.ncols);
        for (int q = (half + it * m) & 1; q < m; q += 2) {  // (tile, query) items alternate between the two warps
          const float4* w4 = reinterpret_cast<const float4*>(g_w + q * NHI);
          float2 a01 = make_float2(0.f, 0.f), a23 = make_float2(0.f, 0.f);  // four chains: the head sum is latency-bound
          auto accumulate = [&](const uint32_t* v, int nv, int w0) {
#pragma unroll
            for (int i = 0; i < nv / 4; ++i) {
              const float4 ww = w4[w0 / 4 + i];
              // chains (a0, a1) and (a2, a3) advance in pairs: one instruction per two heads
              a01 = fma_f32x2(make_float2(fmaxf(__uint_as_float(v[4 * i + 0]), 0.f), fmaxf(__uint_as_float(v[4 * i + 1]), 0.f)),
                              make_float2(ww.x, ww.y), a01);
              a23 = fma_f32x2(make_float2(fmaxf(__uint_as_float(v[4 * i + 2]), 0.f), fmaxf(__uint_as_float(v[4 * i + 3]), 0.f)),
                              make_float2(ww.z, ww.w), a23);
            }
          };
          if constexpr (NHI % 32 == 0) {
#pragma unroll
            for (int cc = 0; cc < NHI / 32; ++cc) {
              uint32_t v[32];
              tmem_ld32(t_row + static_cast<uint32_t>(q * NHI + cc * 32), v);
              tmem_wait_ld();
              accumulate(v, 32, cc * 32);
            }
          } else {
            uint32_t v[16];
            tmem_ld16(t_row + static_cast<uint32_t>(q * NHI), v);
            tmem_wait_ld();
            accumulate(v, 16, 0);
          }
          const float score = ((a01.x + a01.y) + (a23.x + a23.y)) * g_sq[q] * sk;
          cache[q * p.slice_cap + jl] = sel::order_key(score);  // positions past the query are never read
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sempty[c]);
          mbar_arrive(&tempty[a]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();  // every score of this CTA's slice is in shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }

  // ---------------- selection, one query of the request after the other ----------------
  for (int q = 0; q < m; ++q) {
    const int L = n_b - m + q + 1;  // query q sits at position n_b - m + q
    int32_t* out = p.S + static_cast<int64_t>(row0 + q) * p.k;
    if (L <= p.k) {  // every visible position, then padding (the same branch in every CTA)
      sel::cluster_wait();
      const int per = (p.k + static_cast<int>(C) - 1) / static_cast<int>(C);
      const int j1 = min(p.k, static_cast<int>(rank + 1) * per);
      for (int j = static_cast<int>(rank) * per + threadIdx.x; j < j1; j += kThreads) out[j] = j < L ? j : -1;
      sel::cluster_arrive();
      continue;
    }
    const int nq = max(0, min(kend, L) - kbase);  // this CTA's keys visible to query q
    sel::select_topk<kThreads>(cache + q * p.slice_cap, nq, kbase, p.k, out, sh, hist, C, rank);
  }
  sel::cluster_wait();  // no CTA leaves while a peer may still address its shared memory
}

// Shared-memory plan of the fused kernel for a cluster size: ok = false when it does not fit with at
// least kMinStages key stages.
struct FusedPlan {
  bool ok;
  int C, slice_cap, qbytes, qbox_rows, nstages, ring_off, cache_off, hist_off, smem;
};

FusedPlan fused_plan(int max_q, int max_seq_len, int nhI, int C) {
  FusedPlan f{};
  f.C = C;
  const int ntiles = (max_seq_len + kIdxTileKeys - 1) / kIdxTileKeys;
  const int tpc = (ntiles + C - 1) / C;
  f.slice_cap = tpc * kIdxTileKeys;
  f.qbox_rows = max_q * nhI;
  f.qbytes = (f.qbox_rows * kDIdx + 1023) / 1024 * 1024;
  const int qpg = kIdxCols / nhI;
  const size_t cache = sizeof(uint32_t) * static_cast<size_t>(max_q) * f.slice_cap;
  const size_t hist = sizeof(uint32_t) * static_cast<size_t>(sel::hist_words(C));
  const size_t statics = sizeof(sel::Shared<kThreads>);
  f.ring_off = FusedSmem::kFixed + f.qbytes;
  const long rest = static_cast<long>(kSmemLimit) - static_cast<long>(statics) - f.ring_off -
                    static_cast<long>(cache) - static_cast<long>(hist);
  f.nstages = static_cast<int>(std::min<long>(kMaxStages, rest / kStageBytes));
  f.cache_off = f.ring_off + f.nstages * kStageBytes;
  f.hist_off = f.cache_off + static_cast<int>(cache);
  f.smem = f.hist_off + static_cast<int>(hist) + 1024;
  f.ok = f.slice_cap <= kMaxSliceKeys && f.nstages >= kMinStages && max_q <= qpg;
  return f;
}

}  // namespace

// Cluster size for the fused kernel, or 0 when this batch does not take it: every request's queries
// form one MMA group (max_q <= 256 / nhI), and a slice's scores fit one SM's shared memory. Among
// the sizes that fit, the smallest with about 16384 positions per CTA or fewer (so that the longest
// request does not hold the GPU), and no smaller than what fills the SMs once.
int index_topk_cluster_size(int B, int max_q, int max_seq_len, int nhI) {
  if (B <= 0 || max_q < 1 || max_q > kIdxCols / nhI || max_seq_len > kMaxTopKRow) return 0;
  int want = 1;
  while (want < kMaxCluster && B * want * 2 <= 148) want <<= 1;
  while (want < kMaxCluster && (max_seq_len + want - 1) / want > 16384) want <<= 1;
  for (int C = want; C <= kMaxCluster; C <<= 1)
    if (fused_plan(max_q, max_seq_len, nhI, C).ok) return C;
  return 0;
}

template <int NHI>
static int launch_index_topk_t(const BatchDev& b, const void* plan, const uint8_t* qI, const float* qI_scale,
                               const float* wI, const uint8_t* kI_cache, const float* kI_scale, int k, int32_t* S,
                               int C, void* stream) {
  PlanView pv = plan_view(const_cast<void*>(plan), b.B, b.T);
  const FusedPlan f = fused_plan(b.max_q, b.max_seq_len, NHI, C);
  if (!f.ok) return static_cast<int>(cudaErrorInvalidValue);
  FusedParams prm{};
  prm.bd = b;
  prm.qI_scale = qI_scale;
  prm.wI = wI;
  prm.kI_scale = kI_scale;
  prm.S = S;
  prm.k = k;
  prm.qbytes = f.qbytes;
  prm.qbox_rows = f.qbox_rows;
  int ncols = 32;
  while (ncols < b.max_q * NHI) ncols <<= 1;
  prm.ncols = ncols;
  prm.nacc = std::min(kMaxAcc, 512 / ncols);
  prm.nstages = f.nstages;
  prm.slice_cap = f.slice_cap;
  prm.ring_off = f.ring_off;
  prm.cache_off = f.cache_off;
  prm.hist_off = f.hist_off;
  prm.status = &pv.hdr->status;
  CUtensorMap kmap, qmap;
  int e = make_tmap_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kI_cache, kDIdx,
                       static_cast<uint64_t>(b.num_pages) * kPage, kDIdx, kDIdx, kPage);
  if (e) return e;
  e = make_tmap_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, qI, kDIdx, static_cast<uint64_t>(b.T) * NHI, kDIdx, kDIdx,
                   static_cast<uint32_t>(f.qbox_rows));
  if (e) return e;
  auto kern = index_topk_kernel<NHI>;
  cudaError_t ce = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, f.smem);
  if (ce != cudaSuccess) return static_cast<int>(ce);
  return static_cast<int>(launch_pdl_cluster(kern, dim3(b.B * C), dim3(kThreads), static_cast<size_t>(f.smem), stream,
                                             static_cast<unsigned>(C), kmap, qmap, prm));
}

int launch_index_topk(const BatchDev& b, const void* plan, const uint8_t* qI, const float* qI_scale, const float* wI,
                      int nhI, const uint8_t* kI_cache, const float* kI_scale, int k, int32_t* S, void* stream) {
  if (b.T == 0) return 0;
  const int C = index_topk_cluster_size(b.B, b.max_q, b.max_seq_len, nhI);
  if (C == 0) return static_cast<int>(cudaErrorInvalidValue);
  switch (nhI) {
    case 16:
      return launch_index_topk_t<16>(b, plan, qI, qI_scale, wI, kI_cache, kI_scale, k, S, C, stream);
    case 32:
      return launch_index_topk_t<32>(b, plan, qI, qI_scale, wI, kI_cache, kI_scale, k, S, C, stream);
    case 64:
      return launch_index_topk_t<64>(b, plan, qI, qI_scale, wI, kI_cache, kI_scale, k, S, C, stream);
    case 128:
      return launch_index_topk_t<128>(b, plan, qI, qI_scale, wI, kI_cache, kI_scale, k, S, C, stream);
    default:
      return static_cast<int>(cudaErrorInvalidValue);
  }
}

}  // namespace dsa
