// Sparse MLA on the selected positions (sm_100a).
//
// For query row t with index set S_t and every head h:
//   z_hj = scale * q_th . c_j  (576 dims),   o_th = sum_{j in S_t} softmax_j(z_hj) * c_j[0:512]
// ("DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section "Sparse Attention", the masked
// softmax with M = 0 on S_t, computed by reading only the selected rows; absorbed MLA with a
// 576-wide latent shared by all heads per "MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与
// DSA". S_t is shared by all heads.)
//
// Persistent clusters of two CTAs (on two SMs): as many clusters as fit on the GPU at once, each
// taking the units (query row, split of S_t) u = cluster, cluster + clusters, ... in turn. The
// pipelines run on across units: while one unit's last tiles, its softmax and its output are
// finishing, the next unit's index rows, Q and first gathers are already under way.
//
//   S-CTA (rank 0): S = Q C^T and the softmax.
//     * Q (128 heads x 576 bf16): dims 0..511 in TMEM as the A operand (256 columns), the 64 rope
//       dims in shared memory (one 128-byte-swizzled block). A unit's Q arrives by TMA in the
//       latent ring once the previous unit's MMAs have completed; the softmax warps move it into
//       TMEM.
//     * 8 producer warps gather latent dims 0..511 of the selected rows with 16-byte cp.async (8
//       lanes per 128-byte row segment, XOR-swizzled on the way into the canonical 128-byte-swizzled
//       K-major UMMA layout) into an 8-slot ring (slot = 64-dim block of the current tile); another
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
//       At the end of a unit they send its maximum and sums to the O-CTA.
//   O-CTA (rank 1): O = P V.
//     * O (128 heads x 512 fp32) fills its whole TMEM. V = c[0:512] of the same rows (mostly L2
//       hits: the S-CTA fetched them) is gathered by 8 producer warps in units of 128 keys x 128
//       dims (4 per tile).
//     * Per tile: 32 tcgen05.mma (M=128, N=128 dims, K=16 keys), A = P (shared memory, K-major),
//       B = V (MN-major). Completion is multicast back to the S-CTA to free the P buffer.
//     * Eight correction warps rescale O rows in TMEM when a quadrant is flagged (rare), and at the
//       end of a unit normalise O; the bf16 rows are staged in the V ring and leave with TMA
//       stores, after which the ring takes the next unit's rows.
//   Both: one warp reads the index rows (S_t -> block table -> physical rows) of the cluster's
//   next unit into the other half of a double buffer while the current unit runs.
//
// Splits (several units over one S_t) write normalised partial outputs and their log-sum-exp to
// the workspace; a combine kernel merges them: o = sum_s exp(lse_s - lse) o_s.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
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
constexpr int kMaxKeysPerCta = 2048;         // S_t entries one unit covers
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
constexpr int kRowsWarp = kRopeWarp + 1;            // warp 18: index rows of the cluster's next units
constexpr int kThreads = 32 * (kRowsWarp + 1);
constexpr int kRowIters = (kMaxKeysPerCta + kThreads - 1) / kThreads;
constexpr float kRescaleThreshold = 8.0f;    // log2 units
// warps that read a unit's rows, masks or info and release them (ROWSFREE arrivals)
constexpr int kRowUsersS = kProdWarps + 1 + kSoftWarps + 1;  // producers, MMA, softmax, rope
constexpr int kRowUsersO = kProdWarps + 1 + kSoftWarps;      // producers, MMA, correction

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
  static constexpr int kKRing = kQRope + kBlk;                   // 8 x 16 KB (a unit's Q dims 0..511 first)
  static constexpr int kRRing = kKRing + kKSlots * kBlk;         // 2 x 16 KB
  static constexpr int kRed = kRRing + kRSlots * kBlk;           // float [2][kSubs][128]: tile maxima
  static constexpr int kRedL = kRed + 2 * kSubs * 128 * 4;       // float [2][2][kSubs][128]: l, lr per unit parity
  static constexpr int kSEnd = kRedL + 4 * kSubs * 128 * 4;
  // O-CTA
  static constexpr int kP = 0;                                   // 2 P blocks, kPStride apart
  static constexpr int kVRing = kP + 2 * kPStride;               // 4 x 32 KB; output staging after a unit
  static constexpr int kStats = kVRing + kVSlots * 2 * kBlk;     // float [2][3][128]: m, l, lr per unit parity
  static constexpr int kOEnd = kStats + 2 * 3 * 128 * 4;
  // both
  static constexpr int kCommon = (kSEnd > kOEnd ? kSEnd : kOEnd);
  static constexpr int kRows = kCommon;                          // int32 [2][2048] physical rows
  static constexpr int kMasks = kRows + 2 * kMaxKeysPerCta * 4;  // u32 [2][64] validity bits
  static constexpr int kInfo = kMasks + 2 * kMaxTiles * 4 * 4;   // int4 [2]: row t, split, tiles
  static constexpr int kBars = kInfo + 2 * 16;
  static constexpr int kNumBars = 80;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kTotal = kTmemSlot + 16;
  static constexpr int kDynamic = kTotal + 1024;
};
static_assert(Smem::kDynamic <= 232448, "sparse MLA shared memory exceeds the 227 KB limit");
static_assert(Smem::kBars % 8 == 0 && Smem::kInfo % 16 == 0, "barrier and info alignment");
static_assert(kPShip <= kPStride && kPShip % 16 == 0, "P block");
static_assert(kKSlots % kSGroups == 0 && kVSlots % kOGroups == 0, "every ring slot needs a single owner group");
static_assert(kKSlots == 8, "one cp.async slot per latent block of a tile");
static_assert(kVSlots == 4, "one V slot per 128-dim quarter of a tile");
static_assert(kTile == 32 * 2 * kSubs, "softmax warps cover a tile");

// Barrier indices (same offsets in both CTAs; each CTA initialises the ones it owns). Phases are
// counted per tile over the whole kernel (tiles of all units in turn), per unit, or per unit
// with tiles, as noted; every waiter follows the same sequence, so a parity names one phase.
enum : int {
  // S-CTA
  B_KFULL = 0,                      // [8]  per tile: cp.async arrivals of one producer group
  B_KEMPTY = B_KFULL + kKSlots,     // [8]  per tile: MMA commit
  B_RFULL = B_KEMPTY + kKSlots,     // [2]  per tile: TMA bytes of a rope block
  B_REMPTY = B_RFULL + kRSlots,     // [2]  per tile: MMA commit
  B_QROPE = B_REMPTY + kRSlots,     // 1    per unit with tiles: TMA of Q
  B_QCONS = B_QROPE + 1,            // 1    per unit with tiles: softmax warps moved Q out of the ring
  B_QRED = B_QCONS + 1,             // [2][4] per tile: partial maxima of one quadrant written
  B_QEND = B_QRED + 8,              // [4]  per unit: partial sums of one quadrant written
  B_SFULL = B_QEND + 4,             // [2]  per tile: MMA -> softmax
  B_SFREE = B_SFULL + 2,            // [2]  per tile: softmax -> MMA (8 warps)
  B_PFREE = B_SFREE + 2,            // [2]  per tile: O-CTA MMA -> S-CTA (multicast commit)
  B_SDONE = B_PFREE + 2,            // 1    per unit with tiles: the unit's MMAs completed
  B_STATSFREE = B_SDONE + 1,        // [2]  per unit: the O-CTA read the statistics buffer
  // O-CTA
  B_VFULL = B_STATSFREE + 2,        // [4]  per tile: cp.async arrivals of one producer group
  B_VEMPTY = B_VFULL + kVSlots,     // [4]  per tile: MMA commit
  B_PFULL = B_VEMPTY + kVSlots,     // [2]  per tile: one remote arrival + the P block's bytes
  B_OREADY = B_PFULL + 2,           // [2]  per tile: correction warps -> MMA (8 warps)
  B_ODONE = B_OREADY + 2,           // 1    per tile: MMA -> correction warps
  B_OFINAL = B_ODONE + 1,           // 1    per unit with tiles: MMA -> epilogue
  B_STATS = B_OFINAL + 1,           // [2]  per unit: S-CTA statistics (128 remote arrivals)
  B_OFREE = B_STATS + 2,            // 1    per unit: the epilogue read O out of TMEM (8 warps)
  B_STAGED = B_OFREE + 1,           // 1    per unit: the output left the V ring
  B_EPI = B_STAGED + 1,             // 1    per unit: the correction warps staged the output (8 warps)
  // both
  B_ROWSFULL = B_EPI + 1,        // [2]  per unit: index rows, masks and info of a unit (32 lanes)
  B_ROWSFREE = B_ROWSFULL + 2,      // [2]  per unit: every reader is done with them
  B_MDONE = B_ROWSFREE + 2,         // 1    the MMA issuer's last commit (drained before TMEM is freed)
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
  int units;          // T * nsplit
  int chunk;          // S_t entries per split (multiple of kTile)
  float scale_log2;   // softmax scale * log2(e)
  uint16_t* out;
  float* lse;
  float* part_o;      // [T, nsplit, H, 512] when nsplit > 1
  float* part_lse;    // [T, nsplit, H]
  uint32_t* status;
};

struct UnitInfo {
  int t, split, b, pos, nkeys, ntiles;
};

__device__ __forceinline__ UnitInfo unit_info(const MlaParams& p, int u) {
  UnitInfo ui;
  ui.t = u / p.nsplit;
  ui.split = u % p.nsplit;
  ui.b = __ldg(p.row_req + ui.t);
  ui.pos = __ldg(p.row_pos + ui.t);
  const int nvis = min(p.k, ui.pos + 1);
  ui.nkeys = max(0, min(nvis - ui.split * p.chunk, p.chunk));
  ui.ntiles = (ui.nkeys + kTile - 1) / kTile;
  return ui;
}

// Physical latent row of index entry j (a position of request b, page lookup pg), or -1 for an
// entry to skip; reports entries outside the visible positions or the page pool.
__device__ __forceinline__ int physical_row(const MlaParams& p, const UnitInfo& ui, int n_b, int j, int pg) {
  if (j < 0) return -1;
  if (j > ui.pos || j >= n_b) {
    report_error(p.status, kDevErrIndex);
    return -1;
  }
  if (pg < 0 || pg >= p.bd.num_pages) {
    report_error(p.status, kDevErrIndex);
    return -1;
  }
  return pg * kPage + (j % kPage);
}

// 19 warps: the busiest of the SM's four schedulers holds 5 of them, whose registers must fit its
// quarter of the register file (16384), so 96 per thread at most
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kvmap,
                      const __grid_constant__ CUtensorMap omap, const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  int32_t* rows = reinterpret_cast<int32_t*>(base + Smem::kRows);
  uint32_t* masks = reinterpret_cast<uint32_t*>(base + Smem::kMasks);
  int4* info = reinterpret_cast<int4*>(base + Smem::kInfo);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + Smem::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + Smem::kTmemSlot);

  const uint32_t rank = cluster_ctarank();
  const bool is_s = rank == 0;
  const int warp = warp_id(), lane = lane_id();
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;  // this cluster, clusters in the launch
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
        mbar_init(&bar[B_STATSFREE + i], kSoftWarps);
        mbar_init(&bar[B_ROWSFREE + i], kRowUsersS);
      }
      mbar_init(&bar[B_SDONE], 1);
    } else {
      for (int i = 0; i < kVSlots; ++i) {
        mbar_init(&bar[B_VFULL + i], 32 * kOGroupWarps);
        mbar_init(&bar[B_VEMPTY + i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&bar[B_PFULL + i], 1);
        mbar_init(&bar[B_OREADY + i], kSoftWarps);
        mbar_init(&bar[B_STATS + i], 128);
        mbar_init(&bar[B_ROWSFREE + i], kRowUsersO);
      }
      mbar_init(&bar[B_ODONE], 1);
      mbar_init(&bar[B_OFINAL], 1);
      mbar_init(&bar[B_OFREE], kSoftWarps);
      mbar_init(&bar[B_STAGED], 1);
      mbar_init(&bar[B_EPI], kSoftWarps);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&bar[B_ROWSFULL + i], 32);
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

  // ---------- the cluster's first unit, prepared by every thread ----------
  const UnitInfo u0 = unit_info(p, cid);
  if (threadIdx.x == 0 && is_s && u0.ntiles > 0) {  // its Q: 9 boxes of 128 heads x 64 dims; dims 0..511 -> ring
    mbar_arrive_expect_tx(&bar[B_QROPE], 9 * kBlk);
    for (int blk = 0; blk < 8; ++blk)
      tma_load_2d(base + Smem::kKRing + blk * kBlk, &qmap, 64 * blk, u0.t * H, &bar[B_QROPE]);
    tma_load_2d(base + Smem::kQRope, &qmap, 512, u0.t * H, &bar[B_QROPE]);
  }
  {
    // all index loads first, then all page lookups: two dependent round trips to memory in total
    const int32_t* S_row = p.S + static_cast<int64_t>(u0.t) * p.k + u0.split * p.chunk;
    const int32_t* bt_row = p.bd.block_table + static_cast<int64_t>(u0.b) * p.bd.max_pages;
    const int n_b = __ldg(p.bd.seq_lens + u0.b);
    int jv[kRowIters], pg[kRowIters];
#pragma unroll
    for (int it = 0; it < kRowIters; ++it) {
      const int e = threadIdx.x + it * kThreads;
      jv[it] = (e < u0.nkeys) ? __ldg(S_row + e) : -1;
    }
#pragma unroll
    for (int it = 0; it < kRowIters; ++it) {
      const int j = jv[it];
      pg[it] = (j >= 0 && j <= u0.pos && j < n_b) ? __ldg(bt_row + j / kPage) : -1;
    }
#pragma unroll
    for (int it = 0; it < kRowIters; ++it) {
      const int e = threadIdx.x + it * kThreads;
      if (e < u0.ntiles * kTile) rows[e] = physical_row(p, u0, n_b, jv[it], pg[it]);
    }
  }
  if (threadIdx.x == 0) info[0] = make_int4(u0.t, u0.split, u0.ntiles, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (is_s && static_cast<int>(threadIdx.x) < u0.ntiles * 4) {  // mask word w of tile i covers keys 32w..32w+31
    const int i = threadIdx.x >> 2, w = threadIdx.x & 3;
    uint32_t m = 0;
    for (int c = 0; c < 32; ++c) m |= (rows[i * kTile + 32 * w + c] >= 0 ? 1u : 0u) << c;
    masks[threadIdx.x] = m;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int quad = warp & 3;
  const int sub = (warp - kSoftWarp0) >> 2;  // softmax / correction warps: which column half
  const int h = quad * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
  const volatile int4* vinfo = reinterpret_cast<const volatile int4*>(info);

  if (warp == kRowsWarp) {
    // ---------- rows warp: announces unit 0, then prepares units 1, 2, ... in the other buffer ----------
    mbar_arrive(&bar[B_ROWSFULL + 0]);
    bool ok = true;
    for (int qn = 1; ok; ++qn) {
      const int buf = qn & 1;
      if (qn >= 2) {  // every reader released this buffer (unit qn - 2)
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ROWSFREE + buf], ((qn - 2) >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
      }
      const int u = cid + qn * ncl;
      int4 inf = make_int4(0, 0, -1, 0);  // no more units
      if (u < p.units) {
        const UnitInfo ui = unit_info(p, u);
        inf = make_int4(ui.t, ui.split, ui.ntiles, 0);
        if (is_s && lane == 0 && ui.ntiles > 0)  // its Q is read when the unit starts: bring it into L2 now
          bulk_prefetch_l2(p.q + static_cast<int64_t>(ui.t) * H * kDLat, static_cast<uint32_t>(H * kRowBytes));
        const int32_t* S_row = p.S + static_cast<int64_t>(ui.t) * p.k + ui.split * p.chunk;
        const int32_t* bt_row = p.bd.block_table + static_cast<int64_t>(ui.b) * p.bd.max_pages;
        const int n_b = __ldg(p.bd.seq_lens + ui.b);
        int32_t* rws = rows + buf * kMaxKeysPerCta;
        uint32_t* msk = masks + buf * kMaxTiles * 4;
        for (int e0 = 0; e0 < ui.ntiles * kTile; e0 += 16 * 32) {  // 16 entries per lane per round
          int jv[16], pg[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int e = e0 + 32 * j + lane;
            jv[j] = (e < ui.nkeys) ? __ldg(S_row + e) : -1;
          }
#pragma unroll
          for (int j = 0; j < 16; ++j)
            pg[j] = (jv[j] >= 0 && jv[j] <= ui.pos && jv[j] < n_b) ? __ldg(bt_row + jv[j] / kPage) : -1;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int e = e0 + 32 * j + lane;
            if (e0 + 32 * j < ui.ntiles * kTile) {  // warp-uniform: e0 + 32j and the bound are multiples of 32
              const int r = physical_row(p, ui, n_b, jv[j], pg[j]);
              rws[e] = r;
              const uint32_t m = __ballot_sync(0xffffffffu, r >= 0);
              if (lane == 0) msk[(e0 >> 5) + j] = m;
            }
          }
        }
      }
      if (lane == 0) info[buf] = inf;
      mbar_arrive(&bar[B_ROWSFULL + buf]);  // each lane releases its own writes
      if (u >= p.units) break;
    }
  } else if (is_s) {
    if (warp < kProdWarps) {
      // ---------- S-CTA producers: latent blocks 0..7; group g fills blocks g and g + 4 of every tile ----------
      // lane l of warp wg copies 16-byte chunk (l & 7) of rows r_lo + 4j + (l >> 3) of its half of the block
      const int g = warp / kSGroupWarps, wg = warp % kSGroupWarps;
      const int r_lo = (wg * kTile) / kSGroupWarps, r_hi = ((wg + 1) * kTile) / kSGroupWarps;
      const int c = lane & 7;
      int gt = 0, nq = 0;  // tiles and units with tiles before the current unit
      bool ok = true;
      for (int qn = 0; ok; ++qn) {
        const int buf = qn & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        const int ntiles = vinfo[buf].z;
        if (ntiles < 0) break;
        if (ntiles > 0) {
          // the unit's Q went through the ring slots: wait until the softmax warps moved it to TMEM
          ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_QCONS], nq & 1, p.status, kDevErrTimeout));
          if (!ok) break;
          const int32_t* rws = rows + buf * kMaxKeysPerCta;
          for (int u = g; u < ntiles * kKSlots && ok; u += kSGroups) {
            const int i = u / kKSlots, blk = u % kKSlots, gi = gt + i;  // the slot is the block
            ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_KEMPTY + blk], (gi & 1) ^ 1, p.status, kDevErrTimeout));
            if (!ok) break;
            const uint32_t sbase = smem_u32(base + Smem::kKRing + blk * kBlk);
#pragma unroll 4
            for (int r = r_lo + (lane >> 3); r < r_hi; r += 4) {
              const int prow = max(rws[i * kTile + r], 0);
              cp_async_16(sbase + r * 128 + ((c ^ (r & 7)) << 4),
                          p.kv + static_cast<int64_t>(prow) * kRowBytes + blk * 128 + c * 16);
            }
            cp_async_mbar_arrive_noinc(&bar[B_KFULL + blk]);
          }
          if (!ok) break;
          gt += ntiles;
          ++nq;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_ROWSFREE + buf]);
      }
      if (!ok) asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == kMmaWarp) {
      // ---------- S-CTA MMA issuer: S[h, key] = Q . C^T over 9 blocks of 64 dims ----------
      if (lane == 0) {
        const uint32_t idesc = umma_idesc(128, kTile, 1, 0, 0);
        const uint64_t kdesc0 = umma_desc_sw128(smem_u32(base + Smem::kKRing), 16, 1024);
        const uint64_t rrdesc0 = umma_desc_sw128(smem_u32(base + Smem::kRRing), 16, 1024);
        const uint64_t rdesc = umma_desc_sw128(smem_u32(base + Smem::kQRope), 16, 1024);
        int gt = 0, nq = 0;
        int q_issued = u0.ntiles > 0 ? 1 : 0;  // Q loads started (the first unit's in the prologue)
        bool ok = true;
        for (int qn = 0; ok; ++qn) {
          const int buf = qn & 1;
          ok = mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout);
          if (!ok) break;
          const int4 inf = make_int4(vinfo[buf].x, 0, vinfo[buf].z, 0);
          const int ntiles = inf.z;
          if (ntiles < 0) break;
          if (ntiles > 0) {
            if (q_issued == nq) {  // this unit's Q is not on its way yet
              // the previous unit's MMAs (readers of Q in TMEM, of the rope block and of the ring)
              // have completed: the unit's Q may take their place
              if (nq > 0) ok = mbar_wait(&bar[B_SDONE], (nq - 1) & 1, p.status, kDevErrTimeout);
              if (!ok) break;
              mbar_arrive_expect_tx(&bar[B_QROPE], 9 * kBlk);
              for (int blk = 0; blk < 8; ++blk)
                tma_load_2d(base + Smem::kKRing + blk * kBlk, &qmap, 64 * blk, inf.x * H, &bar[B_QROPE]);
              tma_load_2d(base + Smem::kQRope, &qmap, 512, inf.x * H, &bar[B_QROPE]);
              ++q_issued;
            }
            // Q rope in shared memory (TMA) and Q dims 0..511 in TMEM (softmax warps) before the first MMA
            ok = mbar_wait(&bar[B_QROPE], nq & 1, p.status, kDevErrTimeout) &&
                 mbar_wait(&bar[B_QCONS], nq & 1, p.status, kDevErrTimeout);
            if (!ok) break;
            tc_fence_after();
            for (int i = 0; i < ntiles && ok; ++i) {
              const int gi = gt + i, sb = gi & 1;
              ok = mbar_wait(&bar[B_SFREE + sb], ((gi >> 1) & 1) ^ 1, p.status, kDevErrTimeout);
              if (!ok) break;
              const uint32_t d = tmem + kColS + kTile * sb;
              for (int blk = 0; blk < kKSlots && ok; ++blk) {  // latent dims 0..511: A = Q from TMEM
                ok = mbar_wait(&bar[B_KFULL + blk], gi & 1, p.status, kDevErrTimeout);
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
                const int rs = gi % kRSlots;
                ok = mbar_wait(&bar[B_RFULL + rs], (gi / kRSlots) & 1, p.status, kDevErrTimeout);
                if (!ok) break;
                tc_fence_after();
                const uint64_t bd = rrdesc0 + static_cast<uint64_t>((rs * kBlk) >> 4);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) mma_bf16_ss(d, rdesc + 2 * kk, bd + 2 * kk, idesc, 1u);
                mma_commit(&bar[B_REMPTY + rs]);
              }
              mma_commit(&bar[B_SFULL + sb]);
            }
            if (!ok) break;
            mma_commit(&bar[B_SDONE]);
            gt += ntiles;
            ++nq;
          }
          mbar_arrive(&bar[B_ROWSFREE + buf]);
        }
        // every MMA this thread issued has completed before TMEM is freed (also after an error),
        // and no Q box is still landing
        mma_commit(&bar[B_MDONE]);
        mbar_drain(&bar[B_MDONE], 0, p.status);
        if (q_issued > 0) mbar_drain(&bar[B_QROPE], (q_issued - 1) & 1, p.status);
      }
      __syncwarp();
    } else if (warp == kRopeWarp) {
      // ---------- S-CTA rope producer: dims 512..575 of a tile's 128 rows, 32 TMA gathers of 4 rows ----------
      // (the TMA engine runs beside the cp.async path and adds to the gather rate of this SM)
      bool ok = true;
      int gt = 0;  // tiles whose gathers went out
      if (lane == 0) tma_prefetch_desc(&kvmap);
      for (int qn = 0; ok; ++qn) {
        const int buf = qn & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        const int ntiles = vinfo[buf].z;
        if (ntiles < 0) break;
        const int32_t* rws = rows + buf * kMaxKeysPerCta;
        for (int i = 0; i < ntiles && ok; ++i) {
          const int gi = gt, rs = gi % kRSlots;
          const int32_t* rr = rws + i * kTile + 4 * lane;
          bool w = true;
          if (lane == 0) {
            w = mbar_wait(&bar[B_REMPTY + rs], ((gi / kRSlots) & 1) ^ 1, p.status, kDevErrTimeout);
            if (w) mbar_arrive_expect_tx(&bar[B_RFULL + rs], kBlk);
          }
          ok = __shfl_sync(0xffffffffu, w, 0);
          if (!ok) break;
          tma_gather4(base + Smem::kRRing + rs * kBlk + lane * 512, &kvmap, 512, max(rr[0], 0), max(rr[1], 0),
                      max(rr[2], 0), max(rr[3], 0), &bar[B_RFULL + rs]);
          ++gt;
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_ROWSFREE + buf]);
      }
      // no gather may still be landing when the CTA exits, also after an error (the MMA normally
      // consumed them all)
      if (lane == 0)
        for (int gi = max(0, gt - kRSlots); gi < gt; ++gi)
          mbar_drain(&bar[B_RFULL + gi % kRSlots], (gi / kRSlots) & 1, p.status);
      __syncwarp();
    } else if (warp >= kSoftWarp0 && warp < kSoftWarp0 + kSoftWarps) {
      // ---------- S-CTA softmax (warps 9..16: thread = head h, keys 64*sub .. 64*sub+63) ----------
      float* red = reinterpret_cast<float*>(base + Smem::kRed);    // [2][kSubs][128]
      float* redl = reinterpret_cast<float*>(base + Smem::kRedL);  // [2][2][kSubs][128]: l, lr
      const uint32_t peer_p = peer_addr(smem_u32(base + Smem::kP), 1);
      const uint32_t peer_pfull = peer_addr(smem_u32(&bar[B_PFULL]), 1);
      const uint32_t peer_stats = peer_addr(smem_u32(base + Smem::kStats), 1);
      const uint32_t peer_sbar = peer_addr(smem_u32(&bar[B_STATS]), 1);
      int gt = 0, nq = 0;
      bool ok = true;
      for (int qn = 0; ok; ++qn) {
        const int buf = qn & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        const int ntiles = vinfo[buf].z;
        if (ntiles < 0) break;
        const uint32_t* msk = masks + buf * kMaxTiles * 4;
        float m_ref = -INFINITY, l = 0.f, lr = 0.f;
        if (ntiles > 0) {
          // Q dims 0..511: blocks 4*sub .. 4*sub+3 (ring slots) -> TMEM columns (lane = head). The
          // previous unit's MMAs completed before this Q was loaded.
          ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_QROPE], nq & 1, p.status, kDevErrTimeout));
          if (!ok) break;
          tc_fence_after();
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
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_QCONS]);  // ring slots may be refilled, the MMA may start
        }
        for (int i = 0; i < ntiles && ok; ++i) {
          const int gi = gt + i, sb = gi & 1;
          ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_SFULL + sb], (gi >> 1) & 1, p.status, kDevErrTimeout));
          if (!ok) break;
          tc_fence_after();
          const uint32_t srow = tmem + lane_base + kColS + kTile * sb + 64 * sub;
          // pass 1: maximum over this warp's 64 keys (scaled, log2 units)
          float pmax = -INFINITY;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            tmem_ld32_sync(srow + 32 * c, v);
            const uint32_t m = msk[4 * i + 2 * sub + c];
            if (m == 0xFFFFFFFFu) {  // every key of the chunk selected (the usual case; warp-uniform)
              // the scale is positive and rounding is monotonic: max(v) * s == max(v * s)
              float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
              for (int j = 0; j < 32; ++j) mx[j & 3] = fmaxf(mx[j & 3], __uint_as_float(v[j]));
              pmax = fmaxf(pmax, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if ((m >> j) & 1u) pmax = fmaxf(pmax, __uint_as_float(v[j]) * p.scale_log2);
            }
          }
          // tile maximum of head h across this quadrant's warps (shared memory + mbarrier)
          red[(sb * kSubs + sub) * 128 + h] = pmax;
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_QRED + sb * 4 + quad]);
          ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_QRED + sb * 4 + quad], (gi >> 1) & 1, p.status, kDevErrTimeout));
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
          // the O-CTA's product of tile gi - 2 must have released its P buffer sb
          ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_PFREE + sb], ((gi >> 1) & 1) ^ 1, p.status, kDevErrTimeout));
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
            const uint32_t m = msk[4 * i + 2 * sub + c];
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
        if (!ok) break;
        gt += ntiles;
        if (ntiles > 0) ++nq;
        // per-head sums over the quadrant's warps, then the unit's statistics to the O-CTA
        float* rl = redl + buf * 2 * kSubs * 128;
        rl[(0 * kSubs + sub) * 128 + h] = l;
        rl[(1 * kSubs + sub) * 128 + h] = lr;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_QEND + quad]);
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_QEND + quad], qn & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        if (sub == 0) {
          float lt = 0.f, lrt = 0.f;
          for (int s2 = 0; s2 < kSubs; ++s2) {
            lt += rl[(0 * kSubs + s2) * 128 + h];
            lrt += rl[(1 * kSubs + s2) * 128 + h];
          }
          // the O-CTA read this statistics buffer for unit qn - 2
          ok = __all_sync(0xffffffffu,
                          mbar_wait_cluster(&bar[B_STATSFREE + buf], ((qn >> 1) & 1) ^ 1, p.status, kDevErrTimeout));
          if (!ok) break;
          const uint32_t st = peer_stats + static_cast<uint32_t>(buf * 3 * 128 * 4);
          st_cluster_f32(st + static_cast<uint32_t>(h * 4), m_ref);
          st_cluster_f32(st + static_cast<uint32_t>((128 + h) * 4), lt);
          st_cluster_f32(st + static_cast<uint32_t>((256 + h) * 4), lrt);
          mbar_arrive_remote(peer_sbar + static_cast<uint32_t>(buf * 8));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_ROWSFREE + buf]);
      }
      // the O-CTA's last multicast commits land in this CTA's barriers: wait for them before exit
      if (ok && gt > 0 && warp == kSoftWarp0 && lane == 0) {
        const int i1 = gt - 1;
        mbar_wait(&bar[B_PFREE + (i1 & 1)], (i1 >> 1) & 1, p.status, kDevErrTimeout);
        if (gt > 1) mbar_wait(&bar[B_PFREE + ((i1 - 1) & 1)], ((i1 - 1) >> 1) & 1, p.status, kDevErrTimeout);
      }
      __syncwarp();
    }
  } else {
    if (warp < kProdWarps) {
      // ---------- O-CTA producers: V in units of 128 keys x 128 dims (2 blocks), one unit per group ----
      // lane l copies 16-byte chunk (l & 15) of rows r_lo + 2j + (l >> 4) of its warp's share of the unit
      const int g = warp / kOGroupWarps, wg = warp % kOGroupWarps;
      const int r_lo = (wg * kTile) / kOGroupWarps, r_hi = ((wg + 1) * kTile) / kOGroupWarps;
      const int c = lane & 15;
      int gt = 0;
      bool ok = true;
      for (int qn = 0; ok; ++qn) {
        const int buf = qn & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        const int ntiles = vinfo[buf].z;
        if (ntiles < 0) break;
        if (qn > 0) {  // the previous unit's output, staged in the V ring, has left it
          ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_STAGED], (qn - 1) & 1, p.status, kDevErrTimeout));
          if (!ok) break;
        }
        const int32_t* rws = rows + buf * kMaxKeysPerCta;
        for (int u = g; u < ntiles * kVSlots && ok; u += kOGroups) {
          const int i = u / kVSlots, qd = u % kVSlots, slot = qd, gi = gt + i;
          ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_VEMPTY + slot], (gi & 1) ^ 1, p.status, kDevErrTimeout));
          if (!ok) break;
          const uint32_t sbase = smem_u32(base + Smem::kVRing + slot * 2 * kBlk);
#pragma unroll 4
          for (int r = r_lo + (lane >> 4); r < r_hi; r += 2) {  // 16 lanes per 256-byte row segment
            const int prow = max(rws[i * kTile + r], 0);
            cp_async_16(sbase + (c >> 3) * kBlk + r * 128 + (((c & 7) ^ (r & 7)) << 4),
                        p.kv + static_cast<int64_t>(prow) * kRowBytes + qd * 256 + c * 16);
          }
          cp_async_mbar_arrive_noinc(&bar[B_VFULL + slot]);
        }
        if (!ok) break;
        gt += ntiles;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_ROWSFREE + buf]);
      }
      if (!ok) asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == kMmaWarp) {
      // ---------- O-CTA MMA issuer: O[:, 128qd..] += P . V[:, 128qd..] ----------
      if (lane == 0) {
        const uint32_t idesc = umma_idesc(128, 128, 1, 0, 1);  // bf16, A K-major, B MN-major
        const uint64_t pdesc0 = umma_desc_sw128(smem_u32(base + Smem::kP), 16, 1024);
        const uint64_t vdesc0 = umma_desc_sw128(smem_u32(base + Smem::kVRing), kBlk, 1024);
        int gt = 0;
        bool ok = true;
        for (int qn = 0; ok; ++qn) {
          const int buf = qn & 1;
          ok = mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout);
          if (!ok) break;
          const int ntiles = vinfo[buf].z;
          if (ntiles < 0) break;
          if (qn > 0) {  // the epilogue of the previous unit read O out of TMEM
            ok = mbar_wait(&bar[B_OFREE], (qn - 1) & 1, p.status, kDevErrTimeout);
            if (!ok) break;
            tc_fence_after();
          }
          for (int i = 0; i < ntiles && ok; ++i) {
            const int gi = gt + i, pb = gi & 1;
            ok = mbar_wait(&bar[B_OREADY + pb], (gi >> 1) & 1, p.status, kDevErrTimeout) &&
                 mbar_wait_cluster(&bar[B_PFULL + pb], (gi >> 1) & 1, p.status, kDevErrTimeout);
            if (!ok) break;
            fence_proxy_async_smem();  // P arrived by st.async -> tensor-core reads
            tc_fence_after();
            const uint64_t pd = pdesc0 + static_cast<uint64_t>((pb * kPStride) >> 4);
            for (int qd = 0; qd < kVSlots; ++qd) {
              const int slot = qd;
              ok = mbar_wait(&bar[B_VFULL + slot], gi & 1, p.status, kDevErrTimeout);
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
          if (!ok) break;
          gt += ntiles;
          mbar_arrive(&bar[B_ROWSFREE + buf]);
        }
        // every MMA this thread issued has completed before TMEM is freed (also after an error)
        mma_commit(&bar[B_MDONE]);
        mbar_drain(&bar[B_MDONE], 0, p.status);
      }
      __syncwarp();
    } else if (warp >= kSoftWarp0 && warp < kSoftWarp0 + kSoftWarps) {
      // ---------- O-CTA correction + epilogue (warps 9..16: head h, O columns 256*sub .. +255) ------
      const volatile float* stats = reinterpret_cast<const volatile float*>(base + Smem::kStats);
      const uint32_t ocol = tmem + lane_base + kColO + 256 * sub;
      const uint32_t peer_sfree = peer_addr(smem_u32(&bar[B_STATSFREE]), 0);
      int gt = 0, no = 0;  // tiles, units with tiles before the current unit
      bool ok = true;
      for (int qn = 0; ok; ++qn) {
        const int buf = qn & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        const int t = vinfo[buf].x, split = vinfo[buf].y, ntiles = vinfo[buf].z;
        if (ntiles < 0) break;
        for (int i = 0; i < ntiles && ok; ++i) {
          const int gi = gt + i, pb = gi & 1;
          ok = __all_sync(0xffffffffu, mbar_wait_cluster(&bar[B_PFULL + pb], (gi >> 1) & 1, p.status, kDevErrTimeout));
          if (!ok) break;
          const uint8_t* pblk = base + Smem::kP + pb * kPStride;
          if (reinterpret_cast<const volatile uint32_t*>(pblk + kPFlags)[quad] != 0u) {
            // P(gi) was shipped after the product of tile gi - 2 completed, so B_ODONE is at most
            // one phase behind: the parity wait below really waits for the product of tile gi - 1
            // (a flag is never set on a unit's first tile).
            ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ODONE], (gi - 1) & 1, p.status, kDevErrTimeout));
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
        if (!ok) break;
        gt += ntiles;
        // B_OFINAL, not B_ODONE: here the per-tile barrier may still be two phases behind, and a
        // parity wait cannot tell phase gt-1 from gt-3.
        if (ntiles > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_OFINAL], no & 1, p.status, kDevErrTimeout));
          ++no;
          if (!ok) break;
        }
        ok = __all_sync(0xffffffffu, mbar_wait_cluster(&bar[B_STATS + buf], (qn >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        tc_fence_after();
        const volatile float* stu = stats + buf * 3 * 128;
        const float m_ref = stu[h], l = stu[128 + h], lr = stu[256 + h];
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(peer_sfree + static_cast<uint32_t>(buf * 8));  // buffer free again
        const bool have_o = ntiles > 0;
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
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_OFREE]);  // TMEM may take the next unit's products
          if (sub == 0 && h < H && p.lse) p.lse[static_cast<int64_t>(t) * H + h] = lse_nat;
          fence_proxy_async_smem();  // staging writes (generic proxy) -> TMA store reads (async proxy)
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_EPI]);
          if (warp == kSoftWarp0 && lane == 0) {
            // all eight warps staged their rows (a bounded wait, unlike a named barrier, so a warp
            // that gave up after an error cannot hold the others)
            if (mbar_wait(&bar[B_EPI], qn & 1, p.status, kDevErrTimeout)) {
              for (int box = 0; box < 8; ++box) tma_store_3d(&omap, ost + box * kBlk, 64 * box, 0, t);
              bulk_commit_group();
              bulk_wait_read_all();  // the ring may be refilled once the stores have read it
              mbar_arrive(&bar[B_STAGED]);
            }
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
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_OFREE]);
          if (sub == 0 && h < H) p.part_lse[prow] = lse_nat;
          if (warp == kSoftWarp0 && lane == 0) mbar_arrive(&bar[B_STAGED]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_ROWSFREE + buf]);
      }
    }
  }
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

// Clusters of the sparse MLA kernel that are resident on this GPU at once (its shared memory and
// TMEM allow one CTA per SM); asked of the runtime once per device.
static int mla_resident_clusters() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] > 0) return cached[dev];
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * std::max(1, sms / 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Smem::kDynamic;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaOccupancyMaxActiveClusters(&n, sparse_mla_kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();  // clear a failed query; fall back to one cluster per SM pair
    n = std::max(1, sms / 2);
  }
  cached[dev] = n;
  return n;
}

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
  prm.units = b.T * prm.nsplit;
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
  // Persistent clusters (as many as are resident at once, each taking every ncl-th unit) save a
  // unit's start-up and tail, ~9 us, but keep every SM gathering all the time. Long units over many
  // waves (a long prefill) are bound by the GPU-wide rate of random L2 gathers either way, and
  // there one cluster per unit, whose start-up gaps lower that contention, measured ~2% faster.
  const int resident = mla_resident_clusters();
  const bool long_units = prm.chunk >= 14 * kTile && prm.units > 4 * resident;
  const int ncl = long_units ? prm.units : std::min(prm.units, resident);
  ce = launch_pdl(sparse_mla_kernel, dim3(2 * ncl), dim3(kThreads), Smem::kDynamic, stream, qmap, kvmap, omap, prm);
  if (ce != cudaSuccess) return static_cast<int>(ce);
  if (prm.nsplit > 1) {
    const int warps = b.T * H;
    ce = launch_pdl(mla_combine_kernel, dim3((warps + 7) / 8), dim3(256), 0, stream, prm.part_o, prm.part_lse, b.T, H,
                    prm.nsplit, prm.out, lse);
  }
  return static_cast<int>(ce);
}

}  // namespace dsa
