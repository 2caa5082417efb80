// Sparse MLA on the selected positions (sm_100a).
//
// For query row t with index set S_t and every head h:
//   z_hj = scale * q_th . c_j  (576 dims),   o_th = sum_{j in S_t} softmax_j(z_hj) * c_j[0:512]
// ("DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section "Sparse Attention", the masked
// softmax with M = 0 on S_t, computed by reading only the selected rows; absorbed MLA with a
// 576-wide latent shared by all heads per "MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与
// DSA". S_t is shared by all heads.)
//
// One cluster of two CTAs (on two SMs) per (query row, split of S_t):
//
//   S-CTA (rank 0): S = Q C^T and the softmax.
//     * Q (128 heads x 576 bf16): dims 0..511 in TMEM as the A operand (256 columns), the 64 rope
//       dims in shared memory (one 128-byte-swizzled block).
//     * 8 producer warps gather latent dims 0..511 of the selected rows with 16-byte cp.async (8
//       lanes per 128-byte row segment, XOR-swizzled on the way into the canonical 128-byte-swizzled
//       K-major UMMA layout) into an 8-slot ring (slot = 64-dim block of the current tile); a ninth
//       warp fetches the rope dims 512..575 with TMA gather4 (4 rows per copy) into a 2-slot ring.
//       Random 1152-byte rows need hundreds of loads in flight per SM; the TMA engine runs beside
//       the load/store unit and adds to the rate one SM reaches with cp.async alone.
//     * Each tile of 128 keys costs 36 tcgen05.mma (M=128 heads, N=128 keys, K=16), which run at
//       the full bf16 rate; S tiles are double-buffered in TMEM (2 x 128 columns).
//     * Eight softmax warps (two per TMEM lane quadrant, 64 keys each) read S twice (maximum, then
//       exponentials), keep an online softmax whose reference maximum only moves when a tile's
//       maximum exceeds it by more than 2^8, and write bf16 P, the per-head rescale factors and
//       per-quadrant rescale flags straight into the O-CTA's shared memory with st.async, whose
//       bytes complete the O-CTA's barrier for that P buffer (two buffers, alternating by tile).
//   O-CTA (rank 1): O = P V.
//     * O (128 heads x 512 fp32) fills its whole TMEM. V = c[0:512] of the same rows (mostly L2
//       hits: the S-CTA fetched them) is gathered by 8 producer warps in units of 128 keys x 128
//       dims (4 per tile).
//     * Per tile: 32 tcgen05.mma (M=128, N=128 dims, K=16 keys), A = P (shared memory, K-major),
//       B = V (MN-major). Completion is multicast back to the S-CTA to free the P buffer.
//     * Eight correction warps rescale O rows in TMEM when a quadrant is flagged (rare), and at
//       the end normalise O; the bf16 rows are staged in shared memory and leave with TMA stores.
//
// Splits (several clusters over one S_t) write normalised partial outputs and their log-sum-exp
// to the workspace; a combine kernel merges them: o = sum_s exp(lse_s - lse) o_s.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

namespace dsa {

int make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* ptr, uint64_t inner,
                 uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows);
int make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2);

namespace {

constexpr int kRowBytes = kDLat * 2;         // 1152
constexpr int kTile = 128;                   // keys per tile (MMA N for S, K-extent for P V)
constexpr int kMaxKeysPerCta = 2048;         // S_t entries one cluster handles
constexpr int kMaxTiles = kMaxKeysPerCta / kTile;
constexpr int kBlk = kTile * 128;            // 128 keys x 64 dims bf16 = 16 KB
constexpr int kKSlots = 8;                   // S-CTA cp.async ring: latent blocks 0..7 of a tile, slot = block
constexpr int kRSlots = 2;                   // S-CTA TMA ring: the rope block (dims 512..575) of a tile
constexpr int kVSlots = 4;                   // O-CTA ring slots (two 64-dim blocks of one tile each)
constexpr int kProdWarps = 8;                // warps 0..7: cp.async gather producers
// A producer group fills one ring unit at a time; each ring slot belongs to exactly one group
// (slot % groups == group), so a group never runs two uses ahead of the consumer on a slot's
// barrier, which a parity wait could not tell from one use ahead.
constexpr int kSGroupWarps = 2, kSGroups = kProdWarps / kSGroupWarps;  // S-CTA: 4 groups, 8 slots
constexpr int kOGroupWarps = 2, kOGroups = kProdWarps / kOGroupWarps;  // O-CTA: 4 groups, 4 slots
constexpr int kMmaWarp = kProdWarps;         // warp 8: TMEM allocator and MMA issuer
constexpr int kSoftWarp0 = kProdWarps + 1;   // warps 9..16: softmax (S-CTA) / correction (O-CTA),
constexpr int kSoftWarps = 8;                //   two per TMEM lane quadrant
constexpr int kSubs = kSoftWarps / 4;        // column halves per quadrant
constexpr int kRopeWarp = kSoftWarp0 + kSoftWarps;  // warp 17: rope blocks by TMA gather4 (S-CTA only)
constexpr int kThreads = 32 * (kRopeWarp + 1);
constexpr int kRowIters = (kMaxKeysPerCta + kThreads - 1) / kThreads;
constexpr float kRescaleThreshold = 8.0f;    // log2 units

// TMEM columns
constexpr uint32_t kColS = 0;      // S-CTA: S tiles at 0 and 128
constexpr uint32_t kColQ = 256;    // S-CTA: Q dims 0..511
constexpr uint32_t kColO = 0;      // O-CTA: O, 512 columns

// A P block as shipped from the S-CTA to the O-CTA: P (two 64-key blocks of [128 heads][128 B],
// swizzled), alpha[128] floats, flags[4] words.
constexpr int kPBytes = 2 * kBlk;
constexpr int kPAlpha = kPBytes;
constexpr int kPFlags = kPAlpha + 128 * 4;
constexpr int kPShip = kPFlags + 4 * 4;      // 33296 bytes, a multiple of 16
constexpr int kPStride = 33 * 1024;          // keeps every P block 1024-byte aligned

struct Smem {
  // S-CTA
  static constexpr int kQRope = 0;                               // 16 KB
  static constexpr int kKRing = kQRope + kBlk;                   // 8 x 16 KB (Q dims 0..511 at start)
  static constexpr int kRRing = kKRing + kKSlots * kBlk;         // 2 x 16 KB
  static constexpr int kRed = kRRing + kRSlots * kBlk;           // float [2][kSubs][128]: tile maxima
  static constexpr int kRedL = kRed + 2 * kSubs * 128 * 4;       // float [2][kSubs][128]: l, lr
  static constexpr int kSEnd = kRedL + 2 * kSubs * 128 * 4;
  // O-CTA
  static constexpr int kP = 0;                                   // 2 P blocks, kPStride apart
  static constexpr int kVRing = kP + 2 * kPStride;               // 4 x 32 KB; output staging at the end
  static constexpr int kStats = kVRing + kVSlots * 2 * kBlk;     // float [3][128]: m, l, lr
  static constexpr int kOEnd = kStats + 3 * 128 * 4;
  // both
  static constexpr int kCommon = (kSEnd > kOEnd ? kSEnd : kOEnd);
  static constexpr int kRows = kCommon;                          // int32 [2048] physical rows
  static constexpr int kMasks = kRows + kMaxKeysPerCta * 4;      // u32 [16][4] validity bits
  static constexpr int kBars = kMasks + kMaxTiles * 4 * 4;
  static constexpr int kNumBars = 64;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kTotal = kTmemSlot + 16;
  static constexpr int kDynamic = kTotal + 1024;
};
static_assert(Smem::kDynamic <= 232448, "sparse MLA shared memory exceeds the 227 KB limit");
static_assert(kPShip <= kPStride && kPShip % 16 == 0, "P block");
static_assert(kKSlots % kSGroups == 0 && kVSlots % kOGroups == 0, "every ring slot needs a single owner group");
static_assert(kKSlots == 8, "one cp.async slot per latent block of a tile");
static_assert(kTile == 32 * 2 * kSubs, "softmax warps cover a tile");

// barrier indices (same offsets in both CTAs; each CTA initialises the ones it owns)
enum : int {
  // S-CTA
  B_KFULL = 0,                      // [8]  cp.async arrivals of one producer group
  B_KEMPTY = B_KFULL + kKSlots,     // [8]  MMA commit
  B_RFULL = B_KEMPTY + kKSlots,     // [2]  TMA bytes of a rope block
  B_REMPTY = B_RFULL + kRSlots,     // [2]  MMA commit
  B_QROPE = B_REMPTY + kRSlots,     // 1    TMA of Q
  B_QCONS = B_QROPE + 1,            // 1    softmax warps moved Q out of the ring (8 warps)
  B_QRED = B_QCONS + 1,             // [2][4] partial maxima of one quadrant written (kSubs warps)
  B_QEND = B_QRED + 8,              // [4]  partial sums of one quadrant written (kSubs warps)
  B_SFULL = B_QEND + 4,             // [2]  MMA -> softmax
  B_SFREE = B_SFULL + 2,            // [2]  softmax -> MMA (8 warps)
  B_PFREE = B_SFREE + 2,            // [2]  O-CTA MMA -> S-CTA (multicast commit): P buffer consumed
  // O-CTA
  B_VFULL = B_PFREE + 2,            // [4]  cp.async arrivals of one producer group
  B_VEMPTY = B_VFULL + kVSlots,     // [4]  MMA commit
  B_PFULL = B_VEMPTY + kVSlots,     // [2]  one remote arrival + the P block's bytes (st.async)
  B_OREADY = B_PFULL + 2,           // [2]  correction warps -> MMA (8 warps)
  B_ODONE = B_OREADY + 2,           // 1    MMA -> correction warps (once per tile)
  B_OFINAL = B_ODONE + 1,           // 1    MMA -> epilogue (once, after the last tile)
  B_STATS = B_OFINAL + 1,           // 1    S-CTA softmax -> O-CTA epilogue (128 remote arrivals)
  // both
  B_MDONE = B_STATS + 1,            // 1    the MMA issuer's last commit (drained before TMEM is freed)
  B_COUNT = B_MDONE + 1
};
static_assert(B_COUNT <= Smem::kNumBars, "barrier space");

struct MlaParams {
  BatchDev bd;
  const int32_t* row_req;
  const int32_t* row_pos;
  const uint16_t* q;
  const uint8_t* kv;  // latent cache, rows of 1152 bytes
  const int32_t* S;
  int k;
  int H;
  int nsplit;
  int chunk;          // S_t entries per split (multiple of kTile)
  float scale_log2;   // softmax scale * log2(e)
  uint16_t* out;
  float* lse;
  float* part_o;      // [T, nsplit, H, 512] when nsplit > 1
  float* part_lse;    // [T, nsplit, H]
  uint32_t* status;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kvmap,
                      const __grid_constant__ CUtensorMap omap, const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  int32_t* rows = reinterpret_cast<int32_t*>(base + Smem::kRows);
  uint32_t* masks = reinterpret_cast<uint32_t*>(base + Smem::kMasks);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + Smem::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + Smem::kTmemSlot);

  const uint32_t rank = cluster_ctarank();
  const bool is_s = rank == 0;
  const int warp = warp_id(), lane = lane_id();
  const int unit = blockIdx.x >> 1;
  const int t = unit / p.nsplit, split = unit % p.nsplit;
  const int H = p.H;

  if (threadIdx.x == 0) {
    if (is_s) {
      for (int i = 0; i < kKSlots; ++i) {
        mbar_init(&bar[B_KFULL + i], 32 * kSGroupWarps);  // one cp.async arrival per producer lane
        mbar_init(&bar[B_KEMPTY + i], 1);
      }
      for (int i = 0; i < kRSlots; ++i) {
        mbar_init(&bar[B_RFULL + i], 1);
        mbar_init(&bar[B_REMPTY + i], 1);
      }
      mbar_init(&bar[B_QROPE], 1);
      mbar_init(&bar[B_QCONS], kSoftWarps);
      for (int i = 0; i < 8; ++i) mbar_init(&bar[B_QRED + i], kSubs);
      for (int i = 0; i < 4; ++i) mbar_init(&bar[B_QEND + i], kSubs);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&bar[B_SFULL + i], 1);
        mbar_init(&bar[B_SFREE + i], kSoftWarps);
        mbar_init(&bar[B_PFREE + i], 1);
      }
    } else {
      for (int i = 0; i < kVSlots; ++i) {
        mbar_init(&bar[B_VFULL + i], 32 * kOGroupWarps);
        mbar_init(&bar[B_VEMPTY + i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&bar[B_PFULL + i], 1);
        mbar_init(&bar[B_OREADY + i], kSoftWarps);
      }
      mbar_init(&bar[B_ODONE], 1);
      mbar_init(&bar[B_OFINAL], 1);
      mbar_init(&bar[B_STATS], 128);
    }
    mbar_init(&bar[B_MDONE], 1);
    fence_barrier_init();
    tma_prefetch_desc(&qmap);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  // everything above stays inside this CTA; from here on the kernel reads the plan and S_t
  pdl_trigger();
  pdl_wait();
  const int b = __ldg(p.row_req + t);
  const int pos = __ldg(p.row_pos + t);
  const int nvis = min(p.k, pos + 1);
  const int e0 = split * p.chunk;
  const int nkeys = max(0, min(nvis - e0, p.chunk));
  const int ntiles = (nkeys + kTile - 1) / kTile;
  if (threadIdx.x == 0 && is_s && ntiles > 0) {  // Q: 9 boxes of 128 heads x 64 dims; dims 0..511 -> ring
    mbar_arrive_expect_tx(&bar[B_QROPE], 9 * kBlk);
    for (int blk = 0; blk < 8; ++blk) tma_load_2d(base + Smem::kKRing + blk * kBlk, &qmap, 64 * blk, t * H, &bar[B_QROPE]);
    tma_load_2d(base + Smem::kQRope, &qmap, 512, t * H, &bar[B_QROPE]);
  }

  // physical rows of this cluster's entries (both CTAs); -1 marks an entry to skip
  const int32_t* S_row = p.S + static_cast<int64_t>(t) * p.k + e0;
  const int32_t* bt_row = p.bd.block_table + static_cast<int64_t>(b) * p.bd.max_pages;
  const int n_b = __ldg(p.bd.seq_lens + b);
  {
    // all index loads first, then all page lookups: two dependent round trips to memory in total
    int jv[kRowIters], pg[kRowIters];
#pragma unroll
    for (int it = 0; it < kRowIters; ++it) {
      const int e = threadIdx.x + it * kThreads;
      jv[it] = (e < nkeys) ? __ldg(S_row + e) : -1;
    }
#pragma unroll
    for (int it = 0; it < kRowIters; ++it) {
      const int j = jv[it];
      const bool in_range = j >= 0 && j <= pos && j < n_b;
      if (j >= 0 && !in_range) report_error(p.status, kDevErrIndex);
      pg[it] = in_range ? __ldg(bt_row + j / kPage) : -1;
      if (!in_range) jv[it] = -1;
    }
#pragma unroll
    for (int it = 0; it < kRowIters; ++it) {
      const int e = threadIdx.x + it * kThreads;
      if (e < ntiles * kTile) {
        int r = -1;
        if (jv[it] >= 0) {
          if (pg[it] < 0 || pg[it] >= p.bd.num_pages)
            report_error(p.status, kDevErrIndex);
          else
            r = pg[it] * kPage + (jv[it] % kPage);
        }
        rows[e] = r;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int quad = warp & 3;
  const int sub = (warp - kSoftWarp0) >> 2;  // softmax / correction warps: which column half
  const int h = quad * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;

  if (is_s) {
    if (static_cast<int>(threadIdx.x) < ntiles * 4) {  // mask word w of tile i covers keys 32w..32w+31
      const int i = threadIdx.x >> 2, w = threadIdx.x & 3;
      uint32_t m = 0;
      for (int c = 0; c < 32; ++c) m |= (rows[i * kTile + 32 * w + c] >= 0 ? 1u : 0u) << c;
      masks[threadIdx.x] = m;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrival
  tc_fence_after();

  if (is_s) {
    if (warp < kProdWarps) {
      // ---------- S-CTA producers: latent blocks 0..7; group g fills blocks g and g + 4 of every tile ----------
      // lane l of warp wg copies 16-byte chunk (l & 7) of rows r_lo + 4j + (l >> 3) of its fifth of the unit
      const int g = warp / kSGroupWarps, wg = warp % kSGroupWarps;
      const int r_lo = (wg * kTile) / kSGroupWarps, r_hi = ((wg + 1) * kTile) / kSGroupWarps;
      bool ok = ntiles == 0 || mbar_wait(&bar[B_QCONS], 0, p.status, kDevErrTimeout);
      for (int u = g; u < ntiles * kKSlots && ok; u += kSGroups) {
        const int i = u / kKSlots, blk = u % kKSlots;  // the slot is the block
        ok = mbar_wait(&bar[B_KEMPTY + blk], (i & 1) ^ 1, p.status, kDevErrTimeout);
        if (!ok) break;
        const uint32_t sbase = smem_u32(base + Smem::kKRing + blk * kBlk);
        const int c = lane & 7;
#pragma unroll 4
        for (int r = r_lo + (lane >> 3); r < r_hi; r += 4) {
          const int prow = max(rows[i * kTile + r], 0);
          cp_async_16(sbase + r * 128 + ((c ^ (r & 7)) << 4), p.kv + static_cast<int64_t>(prow) * kRowBytes + blk * 128 + c * 16);
        }
        cp_async_mbar_arrive_noinc(&bar[B_KFULL + blk]);
      }
      if (!ok) asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == kMmaWarp) {
      // ---------- S-CTA MMA issuer: S[h, key] = Q . C^T over 9 blocks of 64 dims ----------
      if (lane == 0 && ntiles > 0) {
        // Q rope in shared memory (TMA) and Q dims 0..511 in TMEM (softmax warps) before the first MMA
        bool ok = mbar_wait(&bar[B_QROPE], 0, p.status, kDevErrTimeout) &&
                  mbar_wait(&bar[B_QCONS], 0, p.status, kDevErrTimeout);
        tc_fence_after();
        const uint32_t idesc = umma_idesc(128, kTile, 1, 0, 0);
        const uint64_t kdesc0 = umma_desc_sw128(smem_u32(base + Smem::kKRing), 16, 1024);
        const uint64_t rrdesc0 = umma_desc_sw128(smem_u32(base + Smem::kRRing), 16, 1024);
        const uint64_t rdesc = umma_desc_sw128(smem_u32(base + Smem::kQRope), 16, 1024);
        for (int i = 0; i < ntiles && ok; ++i) {
          const int sb = i & 1;
          ok = mbar_wait(&bar[B_SFREE + sb], ((i >> 1) & 1) ^ 1, p.status, kDevErrTimeout);
          if (!ok) break;
          const uint32_t d = tmem + kColS + kTile * sb;
          for (int blk = 0; blk < kKSlots && ok; ++blk) {  // latent dims 0..511: A = Q from TMEM
            ok = mbar_wait(&bar[B_KFULL + blk], i & 1, p.status, kDevErrTimeout);
            if (!ok) break;
            fence_proxy_async_smem();  // cp.async (generic proxy) writes -> tensor-core reads
            tc_fence_after();
            const uint64_t bd = kdesc0 + static_cast<uint64_t>((blk * kBlk) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ts(d, tmem + kColQ + 32 * blk + 8 * kk, bd + 2 * kk, idesc, (blk | kk) ? 1u : 0u);
            mma_commit(&bar[B_KEMPTY + blk]);
          }
          if (!ok) break;
          {  // rope dims 512..575: A = Q rope from shared memory
            const int rs = i % kRSlots;
            ok = mbar_wait(&bar[B_RFULL + rs], (i / kRSlots) & 1, p.status, kDevErrTimeout);
            if (!ok) break;
            tc_fence_after();
            const uint64_t bd = rrdesc0 + static_cast<uint64_t>((rs * kBlk) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(d, rdesc + 2 * kk, bd + 2 * kk, idesc, 1u);
            mma_commit(&bar[B_REMPTY + rs]);
          }
          if (!ok) break;
          mma_commit(&bar[B_SFULL + sb]);
        }
        // every MMA this thread issued has completed before TMEM is freed (also after an error)
        mma_commit(&bar[B_MDONE]);
        mbar_drain(&bar[B_MDONE], 0, p.status);
      }
      __syncwarp();
    } else if (warp == kRopeWarp) {
      // ---------- S-CTA rope producer: dims 512..575 of a tile's 128 rows, 32 TMA gathers of 4 rows ----------
      // (the TMA engine runs beside the cp.async path and adds to the gather rate of this SM)
      bool ok = true;
      int issued = 0;  // tiles whose gathers went out
      if (lane == 0 && ntiles > 0) tma_prefetch_desc(&kvmap);
      for (int i = 0; i < ntiles && ok; ++i) {
        const int rs = i % kRSlots;
        bool w = true;
        if (lane == 0) {
          w = mbar_wait(&bar[B_REMPTY + rs], ((i / kRSlots) & 1) ^ 1, p.status, kDevErrTimeout);
          if (w) mbar_arrive_expect_tx(&bar[B_RFULL + rs], kBlk);
        }
        ok = __shfl_sync(0xffffffffu, w, 0);
        if (!ok) break;
        const int32_t* rr = rows + i * kTile + 4 * lane;
        tma_gather4(base + Smem::kRRing + rs * kBlk + lane * 512, &kvmap, 512, max(rr[0], 0), max(rr[1], 0),
                    max(rr[2], 0), max(rr[3], 0), &bar[B_RFULL + rs]);
        issued = i + 1;
      }
      // no gather may still be landing when the CTA exits, also after an error (the MMA normally
      // consumed them all)
      if (lane == 0)
        for (int i = max(0, issued - kRSlots); i < issued; ++i)
          mbar_drain(&bar[B_RFULL + i % kRSlots], (i / kRSlots) & 1, p.status);
      __syncwarp();
    } else {
      // ---------- S-CTA softmax (warps 9..16: thread = head h, keys 64*sub .. 64*sub+63) ----------
      float* red = reinterpret_cast<float*>(base + Smem::kRed);    // [2][kSubs][128]
      float* redl = reinterpret_cast<float*>(base + Smem::kRedL);  // [2][kSubs][128]: l, lr
      const uint32_t peer_p = peer_addr(smem_u32(base + Smem::kP), 1);
      const uint32_t peer_pfull = peer_addr(smem_u32(&bar[B_PFULL]), 1);
      float m_ref = -INFINITY, l = 0.f, lr = 0.f;
      bool ok = true;
      if (ntiles > 0) {
        // Q dims 0..511: blocks 4*sub .. 4*sub+3 (ring slots) -> TMEM columns (lane = head)
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_QROPE], 0, p.status, kDevErrTimeout));
        if (ok) {
          for (int blk = 4 * sub; blk < 4 * sub + 4; ++blk) {
            const uint8_t* rowp = base + Smem::kKRing + blk * kBlk + h * 128;
            uint32_t r[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 x = (h < H) ? *reinterpret_cast<const uint4*>(rowp + ((c ^ (h & 7)) << 4)) : make_uint4(0, 0, 0, 0);
              r[4 * c + 0] = x.x;
              r[4 * c + 1] = x.y;
              r[4 * c + 2] = x.z;
              r[4 * c + 3] = x.w;
            }
            tmem_st32(tmem + lane_base + kColQ + 32 * blk, r);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_QCONS]);  // ring slots may be refilled
      }
      for (int i = 0; i < ntiles && ok; ++i) {
        const int sb = i & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_SFULL + sb], (i >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        tc_fence_after();
        const uint32_t srow = tmem + lane_base + kColS + kTile * sb + 64 * sub;
        // pass 1: maximum over this warp's 64 keys (scaled, log2 units)
        float pmax = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32_sync(srow + 32 * c, v);
          const uint32_t m = masks[4 * i + 2 * sub + c];
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if ((m >> j) & 1u) pmax = fmaxf(pmax, __uint_as_float(v[j]) * p.scale_log2);
        }
        // tile maximum of head h across this quadrant's warps (shared memory + mbarrier)
        red[(sb * kSubs + sub) * 128 + h] = pmax;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_QRED + sb * 4 + quad]);
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_QRED + sb * 4 + quad], (i >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        float tmax = -INFINITY;
#pragma unroll
        for (int s2 = 0; s2 < kSubs; ++s2) tmax = fmaxf(tmax, red[(sb * kSubs + s2) * 128 + h]);
        const bool need = tmax > m_ref + kRescaleThreshold;
        const float alpha = need ? exp2f(m_ref - tmax) : 1.f;  // 0 when m_ref is -inf
        if (need) {
          l *= alpha;
          lr *= alpha;
          m_ref = tmax;
        }
        const bool quad_rescale = __any_sync(0xffffffffu, need && i > 0);
        // the O-CTA's product of tile i - 2 must have released its P buffer sb
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_PFREE + sb], ((i >> 1) & 1) ^ 1, p.status, kDevErrTimeout));
        if (!ok) break;
        const uint32_t pbuf = peer_p + static_cast<uint32_t>(sb * kPStride);
        const uint32_t pbar = peer_pfull + static_cast<uint32_t>(sb * 8);
        // the one arrival of the peer's PFULL[sb] phase, with the bytes the st.async below deliver
        if (warp == kSoftWarp0 && lane == 0) mbar_arrive_expect_tx_remote(pbar, kPShip);
        // pass 2: P[h, 64*sub .. +63] (bf16) straight into the peer's K-major swizzled P buffer:
        // block sub (64 keys), chunks of 8 keys XOR-swizzled by head
        const float m_use = (m_ref > -INFINITY) ? m_ref : 0.f;  // m_ref = -inf: every key so far masked
        const uint32_t prow = pbuf + static_cast<uint32_t>(sub * kBlk + h * 128);
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32_sync(srow + 32 * c, v);
          const uint32_t m = masks[4 * i + 2 * sub + c];
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {  // 8 keys = one 16-byte chunk
            uint32_t w[4];
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
              const int j0 = 8 * q8 + 2 * q2;
              const float p0 = ((m >> j0) & 1u) ? fast_exp2(fmaf(__uint_as_float(v[j0]), p.scale_log2, -m_use)) : 0.f;
              const float p1 = ((m >> (j0 + 1)) & 1u) ? fast_exp2(fmaf(__uint_as_float(v[j0 + 1]), p.scale_log2, -m_use)) : 0.f;
              const __nv_bfloat162 bp = __floats2bfloat162_rn(p0, p1);
              l += p0 + p1;
              lr += __low2float(bp) + __high2float(bp);
              w[q2] = *reinterpret_cast<const uint32_t*>(&bp);
            }
            const int chunk = 4 * c + q8;  // chunk 0..7 within block `sub`
            st_async_v4(prow + static_cast<uint32_t>((chunk ^ (h & 7)) << 4), w[0], w[1], w[2], w[3], pbar);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_SFREE + sb]);
        if (sub == 0) {
          st_async_b32(pbuf + static_cast<uint32_t>(kPAlpha + h * 4), __float_as_uint(alpha), pbar);
          if (lane == 0) st_async_b32(pbuf + static_cast<uint32_t>(kPFlags + quad * 4), quad_rescale ? 1u : 0u, pbar);
        }
      }
      // per-head sums over the quadrant's warps, then the final statistics (always sent, so the
      // O-CTA never waits in vain)
      redl[(0 * kSubs + sub) * 128 + h] = l;
      redl[(1 * kSubs + sub) * 128 + h] = lr;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_QEND + quad]);
      const bool sums_ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_QEND + quad], 0, p.status, kDevErrTimeout));
      if (sub == 0) {
        float lt = 0.f, lrt = 0.f;
        if (sums_ok) {
          for (int s2 = 0; s2 < kSubs; ++s2) {
            lt += redl[(0 * kSubs + s2) * 128 + h];
            lrt += redl[(1 * kSubs + s2) * 128 + h];
          }
        }
        const uint32_t peer_stats = peer_addr(smem_u32(base + Smem::kStats), 1);
        st_cluster_f32(peer_stats + static_cast<uint32_t>(h * 4), m_ref);
        st_cluster_f32(peer_stats + static_cast<uint32_t>((128 + h) * 4), lt);
        st_cluster_f32(peer_stats + static_cast<uint32_t>((256 + h) * 4), lrt);
        mbar_arrive_remote(peer_addr(smem_u32(&bar[B_STATS]), 1));
      }
      // the O-CTA's last multicast commits land in this CTA's barriers: wait for them before exit
      if (ok && ntiles > 0 && warp == kSoftWarp0 && lane == 0) {
        const int i1 = ntiles - 1;
        mbar_wait(&bar[B_PFREE + (i1 & 1)], (i1 >> 1) & 1, p.status, kDevErrTimeout);
        if (ntiles > 1) mbar_wait(&bar[B_PFREE + ((i1 - 1) & 1)], ((i1 - 1) >> 1) & 1, p.status, kDevErrTimeout);
      }
      __syncwarp();
    }
  } else {
    if (warp < kProdWarps) {
      // ---------- O-CTA producers: V in units of 128 keys x 128 dims (2 blocks), one unit per group ----
      // lane l copies 16-byte chunk (l & 15) of rows r_lo + 2j + (l >> 4) of its warp's share of the unit
      const int g = warp / kOGroupWarps, wg = warp % kOGroupWarps;
      const int r_lo = (wg * kTile) / kOGroupWarps, r_hi = ((wg + 1) * kTile) / kOGroupWarps;
      bool ok = true;
      for (int u = g; u < ntiles * 4 && ok; u += kOGroups) {
        const int i = u / 4, qd = u % 4, slot = u % kVSlots;
        ok = mbar_wait(&bar[B_VEMPTY + slot], ((u / kVSlots) & 1) ^ 1, p.status, kDevErrTimeout);
        if (!ok) break;
        const uint32_t sbase = smem_u32(base + Smem::kVRing + slot * 2 * kBlk);
        const int c = lane & 15;
#pragma unroll 4
        for (int r = r_lo + (lane >> 4); r < r_hi; r += 2) {  // 16 lanes per 256-byte row segment
          const int prow = max(rows[i * kTile + r], 0);
          cp_async_16(sbase + (c >> 3) * kBlk + r * 128 + (((c & 7) ^ (r & 7)) << 4),
                      p.kv + static_cast<int64_t>(prow) * kRowBytes + qd * 256 + c * 16);
        }
        cp_async_mbar_arrive_noinc(&bar[B_VFULL + slot]);
      }
      if (!ok) asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == kMmaWarp) {
      // ---------- O-CTA MMA issuer: O[:, 128qd..] += P . V[:, 128qd..] ----------
      if (lane == 0 && ntiles > 0) {
        const uint32_t idesc = umma_idesc(128, 128, 1, 0, 1);  // bf16, A K-major, B MN-major
        const uint64_t pdesc0 = umma_desc_sw128(smem_u32(base + Smem::kP), 16, 1024);
        const uint64_t vdesc0 = umma_desc_sw128(smem_u32(base + Smem::kVRing), kBlk, 1024);
        bool ok = true;
        for (int i = 0; i < ntiles && ok; ++i) {
          const int pb = i & 1;
          ok = mbar_wait(&bar[B_OREADY + pb], (i >> 1) & 1, p.status, kDevErrTimeout) &&
               mbar_wait_cluster(&bar[B_PFULL + pb], (i >> 1) & 1, p.status, kDevErrTimeout);
          if (!ok) break;
          fence_proxy_async_smem();  // P arrived by st.async -> tensor-core reads
          tc_fence_after();
          const uint64_t pd = pdesc0 + static_cast<uint64_t>((pb * kPStride) >> 4);
          for (int qd = 0; qd < 4; ++qd) {
            const int u = i * 4 + qd, slot = u % kVSlots;
            ok = mbar_wait(&bar[B_VFULL + slot], (u / kVSlots) & 1, p.status, kDevErrTimeout);
            if (!ok) break;
            fence_proxy_async_smem();
            tc_fence_after();
            const uint64_t vd = vdesc0 + static_cast<uint64_t>((slot * 2 * kBlk) >> 4);
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint64_t ad = pd + static_cast<uint64_t>(((kk >> 2) * kBlk + (kk & 3) * 32) >> 4);
              mma_bf16_ss(tmem + kColO + 128 * qd, ad, vd + static_cast<uint64_t>((kk * 2048) >> 4), idesc,
                          (i > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&bar[B_VEMPTY + slot]);
          }
          if (!ok) break;
          mma_commit(&bar[B_ODONE]);
          if (i == ntiles - 1) mma_commit(&bar[B_OFINAL]);
          mma_commit_multicast(&bar[B_PFREE + pb], 1);  // to the S-CTA (rank 0)
        }
        // every MMA this thread issued has completed before TMEM is freed (also after an error)
        mma_commit(&bar[B_MDONE]);
        mbar_drain(&bar[B_MDONE], 0, p.status);
      }
      __syncwarp();
    } else if (warp < kSoftWarp0 + kSoftWarps) {
      // ---------- O-CTA correction + epilogue (warps 9..16: head h, O columns 256*sub .. +255) ------
      const volatile float* stats = reinterpret_cast<const volatile float*>(base + Smem::kStats);
      const uint32_t ocol = tmem + lane_base + kColO + 256 * sub;
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
        const int pb = i & 1;
        ok = __all_sync(0xffffffffu, mbar_wait_cluster(&bar[B_PFULL + pb], (i >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        const uint8_t* pblk = base + Smem::kP + pb * kPStride;
        if (reinterpret_cast<const volatile uint32_t*>(pblk + kPFlags)[quad] != 0u) {
          // P(i) was shipped after MMA2(i-2) completed, so B_ODONE is at most one phase behind:
          // the parity wait below really waits for MMA2(i-1).
          ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ODONE], (i - 1) & 1, p.status, kDevErrTimeout));
          if (!ok) break;
          tc_fence_after();
          const float a = reinterpret_cast<const float*>(pblk + kPAlpha)[h];
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t o[32];
            tmem_ld32_sync(ocol + 32 * c, o);
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * a);
            tmem_st32(ocol + 32 * c, o);
          }
          tmem_wait_st();
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_OREADY + pb]);
      }
      ok = __all_sync(0xffffffffu, ok);
      // B_OFINAL, not B_ODONE: here the per-tile barrier may still be two phases behind, and a
      // parity wait cannot tell phase ntiles-1 from ntiles-3.
      if (ok && ntiles > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_OFINAL], 0, p.status, kDevErrTimeout));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_cluster(&bar[B_STATS], 0, p.status, kDevErrTimeout));
      tc_fence_after();
      const float m_ref = stats[h], l = stats[128 + h], lr = stats[256 + h];
      const bool have_o = ok && ntiles > 0;
      const float inv = (have_o && lr > 0.f) ? 1.f / lr : 0.f;
      const float lse_nat = (have_o && l > 0.f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
      if (p.nsplit == 1) {
        // normalised bf16 O -> the V ring (idle once every P V product has completed) as 8 boxes of
        // [H heads][64 dims], 128-byte swizzled; one thread writes the boxes out with TMA stores
        uint8_t* ost = base + Smem::kVRing;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          if (have_o) {
            tmem_ld32_sync(ocol + 32 * c, o);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
          if (h < H) {
            uint8_t* rowp = ost + (4 * sub + (c >> 1)) * kBlk + h * 128;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(o[8 * j + 0]) * inv, __uint_as_float(o[8 * j + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(o[8 * j + 2]) * inv, __uint_as_float(o[8 * j + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(o[8 * j + 4]) * inv, __uint_as_float(o[8 * j + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(o[8 * j + 6]) * inv, __uint_as_float(o[8 * j + 7]) * inv);
              const int chunk = 4 * (c & 1) + j;
              *reinterpret_cast<uint4*>(rowp + ((chunk ^ (h & 7)) << 4)) = w;
            }
          }
        }
        if (sub == 0 && h < H && p.lse) p.lse[static_cast<int64_t>(t) * H + h] = lse_nat;
        fence_proxy_async_smem();  // staging writes (generic proxy) -> TMA store reads (async proxy)
        named_bar_sync(1, 32 * kSoftWarps);
        if (warp == kSoftWarp0 && lane == 0) {
          for (int box = 0; box < 8; ++box) tma_store_3d(&omap, ost + box * kBlk, 64 * box, 0, t);
          bulk_commit_group();
          bulk_wait_all();
        }
      } else {
        const int64_t prow = (static_cast<int64_t>(t) * p.nsplit + split) * H + h;
        float* dst = p.part_o + prow * kDV + 256 * sub;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          if (have_o) {
            tmem_ld32_sync(ocol + 32 * c, o);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
          if (h < H) {
            float4* d4 = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              d4[j] = make_float4(__uint_as_float(o[4 * j]) * inv, __uint_as_float(o[4 * j + 1]) * inv,
                                  __uint_as_float(o[4 * j + 2]) * inv, __uint_as_float(o[4 * j + 3]) * inv);
          }
        }
        if (sub == 0 && h < H) p.part_lse[prow] = lse_nat;
      }
    }
  }
  // the Q boxes may still be landing if an error ended the pipeline before Q was consumed
  if (threadIdx.x == 0 && is_s && ntiles > 0) mbar_drain(&bar[B_QROPE], 0, p.status);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the peer may still touch its shared memory
  if (warp == kMmaWarp) {
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
  pdl_trigger();
  pdl_wait();  // the partial results of the sparse MLA kernel
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
  const int clusters_per_wave = 74;  // 148 SMs, two per cluster
  int n = 1;  // as many splits as keep every cluster of the launch in one wave
  if (T > 0 && T < clusters_per_wave) n = clusters_per_wave / T;
  const int max_by_tiles = (k + kTile - 1) / kTile;
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
  prm.kv = static_cast<const uint8_t*>(kv_cache);
  prm.S = S;
  prm.k = k;
  prm.H = H;
  prm.nsplit = sparse_mla_splits(b.T, k);
  const int per = (k + prm.nsplit - 1) / prm.nsplit;
  prm.chunk = (per + kTile - 1) / kTile * kTile;
  prm.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634);
  prm.out = static_cast<uint16_t*>(out);
  prm.lse = lse;
  if (prm.nsplit > 1) {
    prm.part_o = static_cast<float*>(ws);
    prm.part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                            align16(sizeof(float) * static_cast<size_t>(b.T) * prm.nsplit * H * kDV));
  }
  prm.status = &pv.hdr->status;

  CUtensorMap qmap, kvmap, omap;
  int e = make_tmap_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, kDLat, static_cast<uint64_t>(b.T) * H,
                       kDLat * 2, 64, 128);
  if (e) return e;
  // latent rows, one row high boxes of 64 dims (TMA gather of the rope block)
  e = make_tmap_2d(&kvmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kv_cache, kDLat,
                   static_cast<uint64_t>(b.num_pages) * kPage, kDLat * 2, 64, 1);
  if (e) return e;
  memset(&omap, 0, sizeof(omap));
  if (prm.nsplit == 1) {  // out [T][H][512] bf16, boxes of 64 dims x H heads of one row
    e = make_tmap_3d(&omap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, kDV, static_cast<uint64_t>(H),
                     static_cast<uint64_t>(b.T), kDV * 2, static_cast<uint64_t>(H) * kDV * 2, 64,
                     static_cast<uint32_t>(H), 1);
    if (e) return e;
  }
  cudaError_t ce =
      cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem::kDynamic);
  if (ce != cudaSuccess) return static_cast<int>(ce);
  ce = launch_pdl(sparse_mla_kernel, dim3(2 * b.T * prm.nsplit), dim3(kThreads), Smem::kDynamic, stream, qmap, kvmap,
                  omap, prm);
  if (ce != cudaSuccess) return static_cast<int>(ce);
  if (prm.nsplit > 1) {
    const int warps = b.T * H;
    ce = launch_pdl(mla_combine_kernel, dim3((warps + 7) / 8), dim3(256), 0, stream, prm.part_o, prm.part_lse, b.T, H,
                    prm.nsplit, prm.out, lse);
  }
  return static_cast<int>(ce);
}

}  // namespace dsa
