// Sparse MLA for few heads (H <= 16) on sm_100a.
//
// The operation is that of sparse_mla.cu: for query row t with index set S_t and every head h,
//   z_hj = scale * q_th . c_j  (576 dims),   o_th = sum_{j in S_t} softmax_j(z_hj) * c_j[0:512]
// ("DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section "Sparse Attention": the masked
// softmax with M = 0 on S_t, computed by reading only the selected rows; "MTP 与稀疏注意力：NSA 与
// DSA", section "稀疏注意力：NSA 与 DSA": the absorbed MLA, one 576-wide latent row per position
// shared by all heads, V = its first 512 dims.)
//
// With the heads on the MMA's M axis (128 rows) a 16-head query would leave 112 rows of every MMA
// empty and still fill a whole SM's TMEM with O. Here the selected keys and the value dimensions
// take the M axis and the heads the N axis (N = 16):
//   S^T[key, h]  = C Q^T        M = 128 keys of a tile, K = 576 dims: 36 MMAs of K = 16
//   O^T[dim, h] += V^T P^T      M = 128 dims (four of them), K = 128 keys: 8 MMAs each
// so every accumulator row is a real key or a real value dimension; S^T and O^T take 160 TMEM
// columns and one CTA (one SM) runs the whole of a unit (query row, split of S_t).
// Measured on B200: a tcgen05.mma of N <= 32 costs ~46 cycles whether M is 64 or 128 (64 cycles at
// N = 128, 128 at N = 256), so a tile's 68 MMAs take ~1.6 us. The tile period (~4.7 us) is set by
// the ring instead: a tile's V slots stay until its P V MMAs complete, so the next tile's last
// three slots are gathered only after the softmax and the products of this one. (Tiles of 64 keys
// with a 2.5-tile ring, and two softmax groups on alternating tiles, were measured slower.)
//
// Persistent CTAs, one per SM, each taking the units u = cta, cta + ctas, ... in turn:
//   * warps 0..7 gather the rows of each tile of 128 keys with 16-byte cp.async (8 lanes per
//     128-byte row segment, XOR-swizzled into the canonical 128-byte-swizzled layout, zero-filled
//     for entries to skip): dims 0..511 in pairs of 64-dim blocks into a 5-slot ring (a slot is
//     128 dims of one tile, the M extent of one P V MMA), dims 512..575 into a 1-slot rope ring.
//     A tile's four V slots stay until its P V MMAs complete; the fifth takes the next tile's first
//     slot, the rope slot frees as soon as the tile's S MMAs complete.
//   * warp 8 issues the S MMAs (B = Q, 9 blocks of [16 heads][64 dims] that one TMA per block
//     brings in per unit, once the previous unit's S MMAs completed); it also owns the TMEM.
//   * warp 9 issues the P V MMAs (A = V^T straight from the ring slots, MN-major; B = P^T).
//   * warps 10..13 (one per TMEM lane quadrant: 32 keys of a tile each) run the online softmax:
//     the tile maximum of every head over the 128 keys (warp reduction, then across the four warps
//     through shared memory), a reference maximum that only moves when a tile's maximum exceeds it
//     by more than 2^8 (then O^T is rescaled in TMEM once the previous tile's product completed),
//     the exponentials, per-lane running sums, and P^T in bf16 (two buffers, alternating by tile).
//   * warps 14..17 (one per quadrant: 32 value dimensions of each 128) normalise O^T and write the
//     unit's output; O^T is double-buffered by unit, so this overlaps the next unit.
//   * warp 18 reads the index rows of the CTA's next unit (S_t -> block table -> physical rows).
// Every wait is an mbarrier wait bounded in time (dsa_ptx.cuh); phases are counted per tile over
// the whole kernel, per unit, or per unit with tiles, as noted below, so a parity names one phase.
//
// Splits (several units over one S_t, as many as sparse_mla_splits gives for the batch) write
// normalised partial outputs and their log-sum-exp; a combine kernel merges them.
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

namespace {

constexpr int kNH = kNarrowHeads;        // MMA N: head columns (heads >= H are padding)
constexpr int kRowBytes = kDLat * 2;     // 1152
constexpr int kTile = 128;               // keys per tile: M of the S MMAs, K extent of the P V MMAs
constexpr int kMaxKeys = 2048;           // S_t entries of one unit
constexpr int kMaxTiles = kMaxKeys / kTile;
constexpr int kBlk = kTile * 128;        // 64 dims of a tile: 128 rows x 128 bytes = 16 KB
constexpr int kPairBytes = 2 * kBlk;     // a V ring slot: dims 128 s .. 128 s + 127 of a tile
constexpr int kVSlots = 5;
constexpr int kQBlk = kNH * 128;         // 64 dims of Q: 16 rows x 128 bytes
constexpr int kPBlk = kNH * 128;         // 64 keys of P^T: 16 rows x 128 bytes
constexpr int kPBuf = 2 * kPBlk;         // P^T of one tile
constexpr int kProdWarps = 8;
constexpr int kProdThreads = 32 * kProdWarps;
constexpr int kSWarp = 8, kPVWarp = 9, kSoftWarp0 = 10, kEpiWarp0 = 14, kRowsWarp = 18;
constexpr int kThreads = 32 * (kRowsWarp + 1);
constexpr int kRowUsers = kProdWarps + 2 + 4 + 4;  // warps that read a unit's rows or info
constexpr float kRescaleThreshold = 8.0f;          // log2 units

// TMEM columns
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;   // S^T: two buffers of kNH columns (tile parity)
constexpr uint32_t kColO = 64;  // O^T: two buffers (unit parity) of 4 x kNH columns

static_assert(kNH == 16, "the P^T and output packing below assume 16 head columns");
static_assert(kProdThreads == 2 * kTile, "8 lanes per 128-byte row segment, 32 rows per pass");

struct NSmem {
  static constexpr int kV = 0;                                 // 5 x 32 KB
  static constexpr int kRope = kV + kVSlots * kPairBytes;      // 16 KB
  static constexpr int kQ = kRope + kBlk;                      // 9 x 2 KB
  static constexpr int kP = kQ + 9 * kQBlk;                    // 2 x 4 KB
  static constexpr int kRows = kP + 2 * kPBuf;                 // int32 [2][2048] physical rows
  static constexpr int kMasks = kRows + 2 * kMaxKeys * 4;      // u32 [2][64] validity bits
  static constexpr int kRed = kMasks + 2 * kMaxTiles * 4 * 4;  // float [2][4][kNH] tile maxima
  static constexpr int kStats = kRed + 2 * 4 * kNH * 4;        // float [2][5][kNH]: m, l of each softmax warp
  static constexpr int kInfo = kStats + 2 * 5 * kNH * 4;       // int4 [2]: row t, split, tiles
  static constexpr int kBars = kInfo + 2 * 16;
  static constexpr int kNumBars = 48;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kTotal = kTmemSlot + 16;
  static constexpr int kDynamic = kTotal + 1024;
};
static_assert(NSmem::kDynamic <= 232448, "shared memory exceeds the 227 KB limit");
static_assert(NSmem::kRope % 1024 == 0 && NSmem::kQ % 1024 == 0 && NSmem::kP % 1024 == 0,
              "128-byte-swizzled operands start on 1024-byte boundaries");
static_assert(NSmem::kBars % 8 == 0 && NSmem::kInfo % 16 == 0 && NSmem::kRed % 16 == 0, "alignment");

enum : int {
  B_VFULL = 0,                      // [5] per use of a slot: cp.async arrivals of the 256 producer lanes
  B_VEMPTY = B_VFULL + kVSlots,     // [5] per use of a slot: P V MMA commit
  B_RFULL = B_VEMPTY + kVSlots,     // 1   per tile: cp.async arrivals (rope block)
  B_REMPTY = B_RFULL + 1,           // 1   per tile: S MMA commit
  B_QFULL = B_REMPTY + 1,           // 1   per unit with tiles: TMA bytes of Q
  B_QFREE = B_QFULL + 1,            // 1   per unit with tiles: its S MMAs completed
  B_SFULL = B_QFREE + 1,            // [2] per tile: S MMAs -> softmax
  B_SFREE = B_SFULL + 2,            // [2] per tile: softmax read S (4 warps)
  B_RED = B_SFREE + 2,              // [2] per tile: tile maxima written (4 warps)
  B_PFULL = B_RED + 2,              // [2] per tile: P^T written (4 warps)
  B_PFREE = B_PFULL + 2,            // [2] per tile: P V MMA commit
  B_ODONE = B_PFREE + 2,            // 1   per tile: P V MMA commit
  B_OFULL = B_ODONE + 1,            // [2] per unit with tiles: the unit's last P V MMAs completed
  B_OFREE = B_OFULL + 2,            // [2] per unit with tiles: the epilogue read O^T (4 warps)
  B_STATS = B_OFREE + 2,            // [2] per unit with tiles: softmax statistics written (4 warps)
  B_STATSFREE = B_STATS + 2,        // [2] per unit with tiles: the epilogue read them (4 warps)
  B_ROWSFULL = B_STATSFREE + 2,     // [2] per unit: index rows, masks and info (32 lanes)
  B_ROWSFREE = B_ROWSFULL + 2,      // [2] per unit: every reader is done with them
  B_SDRAIN = B_ROWSFREE + 2,        // 1   the S issuer's last commit
  B_PVDRAIN = B_SDRAIN + 1,         // 1   the P V issuer's last commit
  B_COUNT = B_PVDRAIN + 1
};
static_assert(B_COUNT <= NSmem::kNumBars, "barrier space");

struct NarrowParams {
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

struct Unit {
  int t, split, b, pos, nkeys, ntiles;
};

__device__ __forceinline__ Unit narrow_unit(const NarrowParams& p, int u) {
  Unit ui;
  ui.t = u / p.nsplit;
  ui.split = u - ui.t * p.nsplit;
  ui.b = __ldg(p.row_req + ui.t);
  ui.pos = __ldg(p.row_pos + ui.t);
  const int nvis = min(p.k, ui.pos + 1);
  ui.nkeys = max(0, min(nvis - ui.split * p.chunk, p.chunk));
  ui.ntiles = (ui.nkeys + kTile - 1) / kTile;
  return ui;
}

// Physical latent row of index entry j (request b: n_b positions, page id pg), or -1 for an entry
// to skip; an entry outside the visible positions or the page pool is reported and skipped.
__device__ __forceinline__ int narrow_row(const NarrowParams& p, const Unit& ui, int n_b, int j, int pg) {
  if (j < 0) return -1;
  if (j > ui.pos || j >= n_b || pg < 0 || pg >= p.bd.num_pages) {
    report_error(p.status, kDevErrIndex);
    return -1;
  }
  return pg * kPage + (j & (kPage - 1));
}

__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 19 warps: the busiest of the SM's four schedulers holds 5 of them, whose registers must fit its
// quarter of the register file (16384), so 96 per thread at most
__global__ void __launch_bounds__(kThreads, 1)
    sparse_mla_narrow_kernel(const __grid_constant__ CUtensorMap qmap, const NarrowParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  int32_t* rows = reinterpret_cast<int32_t*>(base + NSmem::kRows);
  uint32_t* masks = reinterpret_cast<uint32_t*>(base + NSmem::kMasks);
  int4* info = reinterpret_cast<int4*>(base + NSmem::kInfo);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + NSmem::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + NSmem::kTmemSlot);
  const volatile int4* vinfo = reinterpret_cast<const volatile int4*>(info);
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int i = 0; i < kVSlots; ++i) {
      mbar_init(&bar[B_VFULL + i], kProdThreads);  // one cp.async arrival per producer lane
      mbar_init(&bar[B_VEMPTY + i], 1);
    }
    mbar_init(&bar[B_RFULL], kProdThreads);
    mbar_init(&bar[B_REMPTY], 1);
    mbar_init(&bar[B_QFULL], 1);
    mbar_init(&bar[B_QFREE], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[B_SFULL + i], 1);
      mbar_init(&bar[B_SFREE + i], 4);
      mbar_init(&bar[B_RED + i], 4);
      mbar_init(&bar[B_PFULL + i], 4);
      mbar_init(&bar[B_PFREE + i], 1);
      mbar_init(&bar[B_OFULL + i], 1);
      mbar_init(&bar[B_OFREE + i], 4);
      mbar_init(&bar[B_STATS + i], 4);
      mbar_init(&bar[B_STATSFREE + i], 4);
      mbar_init(&bar[B_ROWSFULL + i], 32);
      mbar_init(&bar[B_ROWSFREE + i], kRowUsers);
    }
    mbar_init(&bar[B_ODONE], 1);
    mbar_init(&bar[B_SDRAIN], 1);
    mbar_init(&bar[B_PVDRAIN], 1);
    fence_barrier_init();
    tma_prefetch_desc(&qmap);
  }
  if (warp == kSWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything above stays inside this CTA; from here on the kernel reads the plan and S_t
  pdl_trigger();
  pdl_wait();

  if (warp == kRowsWarp) {
    // ---------- index rows of units 0, 1, 2, ... into alternating buffers ----------
    bool ok = true;
    for (int qn = 0; ok; ++qn) {
      const int buf = qn & 1;
      if (qn >= 2) {  // every reader released this buffer (unit qn - 2)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bar[B_ROWSFREE + buf], ((qn >> 1) & 1) ^ 1, p.status, kDevErrTimeout));
        if (!ok) break;
      }
      const int u = static_cast<int>(blockIdx.x) + qn * static_cast<int>(gridDim.x);
      int4 inf = make_int4(0, 0, -1, 0);  // no more units
      if (u < p.units) {
        const Unit ui = narrow_unit(p, u);
        inf = make_int4(ui.t, ui.split, ui.ntiles, 0);
        if (lane == 0 && ui.ntiles > 0)  // its Q is read when the unit starts: bring it into L2 now
          bulk_prefetch_l2(p.q + static_cast<int64_t>(ui.t) * p.H * kDLat, static_cast<uint32_t>(p.H * kRowBytes));
        const int32_t* S_row = p.S + static_cast<int64_t>(ui.t) * p.k + ui.split * p.chunk;
        const int32_t* bt_row = p.bd.block_table + static_cast<int64_t>(ui.b) * p.bd.max_pages;
        const int n_b = __ldg(p.bd.seq_lens + ui.b);
        int32_t* rws = rows + buf * kMaxKeys;
        uint32_t* msk = masks + buf * kMaxTiles * 4;
        const int nent = ui.ntiles * kTile;
        for (int e0 = 0; e0 < nent; e0 += 8 * 32) {  // 8 entries per lane per round: two round trips
          int jv[8], pg[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int e = e0 + 32 * j + lane;
            jv[j] = (e < ui.nkeys) ? __ldg(S_row + e) : -1;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j)
            pg[j] = (jv[j] >= 0 && jv[j] <= ui.pos && jv[j] < n_b) ? __ldg(bt_row + (jv[j] >> 6)) : -1;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (e0 + 32 * j < nent) {  // warp-uniform: both sides are multiples of 32
              const int r = narrow_row(p, ui, n_b, jv[j], pg[j]);
              rws[e0 + 32 * j + lane] = r;
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
  } else if (warp < kProdWarps) {
    // ---------- producers: lane l copies chunk l & 7 of rows (l >> 3) + 32 j of every block ----------
    const int tid = static_cast<int>(threadIdx.x);
    const int c = tid & 7, r0 = tid >> 3;
    uint32_t vslot = 0, vround = 0;  // next V slot, and how often the ring went round
    int gt = 0;                      // tiles before the current one
    bool ok = true;
    for (int qn = 0; ok; ++qn) {
      const int buf = qn & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout));
      if (!ok) break;
      const int ntiles = vinfo[buf].z;
      if (ntiles < 0) break;
      const int32_t* rws = rows + buf * kMaxKeys;
      for (int i = 0; i < ntiles && ok; ++i, ++gt) {
        const uint8_t* src[4];
        uint32_t nbytes[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = rws[i * kTile + r0 + 32 * j];
          src[j] = p.kv + static_cast<int64_t>(max(r, 0)) * kRowBytes + c * 16;
          nbytes[j] = r >= 0 ? 16u : 0u;  // entries to skip read nothing and land as zeros
        }
        for (int pr = 0; pr < 4; ++pr) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&bar[B_VEMPTY + vslot], (vround & 1) ^ 1, p.status, kDevErrTimeout));
          if (!ok) break;
          const uint32_t sb = smem_u32(base + NSmem::kV + vslot * kPairBytes);
#pragma unroll
          for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int r = r0 + 32 * j;
              cp_async_16_zfill(sb + s * kBlk + r * 128 + ((c ^ (r & 7)) << 4), src[j] + pr * 256 + s * 128,
                                nbytes[j]);
            }
          cp_async_mbar_arrive_noinc(&bar[B_VFULL + vslot]);
          if (++vslot == kVSlots) vslot = 0, ++vround;
        }
        if (!ok) break;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_REMPTY], (gt & 1) ^ 1, p.status, kDevErrTimeout));
        if (!ok) break;
        const uint32_t rb = smem_u32(base + NSmem::kRope);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = r0 + 32 * j;
          cp_async_16_zfill(rb + r * 128 + ((c ^ (r & 7)) << 4), src[j] + 1024, nbytes[j]);
        }
        cp_async_mbar_arrive_noinc(&bar[B_RFULL]);
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_ROWSFREE + buf]);
    }
    if (!ok) asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == kSWarp) {
    // ---------- S issuer: S^T[key, h] = C . Q^T over 9 blocks of 64 dims ----------
    if (lane == 0) {
      const uint32_t idesc = umma_idesc(128, kNH, 1, 0, 0);  // bf16, A and B K-major
      const uint32_t vbase = smem_u32(base + NSmem::kV), rbase = smem_u32(base + NSmem::kRope);
      const uint32_t qbase = smem_u32(base + NSmem::kQ);
      uint32_t vslot = 0, vround = 0;
      int gt = 0, nq = 0;  // tiles, units with tiles before the current one
      bool ok = true, q_in_flight = false;
      for (int qn = 0; ok; ++qn) {
        const int buf = qn & 1;
        ok = mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout);
        if (!ok) break;
        const int t = vinfo[buf].x, ntiles = vinfo[buf].z;
        if (ntiles < 0) break;
        if (ntiles > 0) {
          if (nq > 0) {  // the previous unit's S MMAs have read Q
            ok = mbar_wait(&bar[B_QFREE], (nq - 1) & 1, p.status, kDevErrTimeout);
            if (!ok) break;
          }
          mbar_arrive_expect_tx(&bar[B_QFULL], 9 * kQBlk);
          for (int blk = 0; blk < 9; ++blk)
            tma_load_2d(base + NSmem::kQ + blk * kQBlk, &qmap, 64 * blk, t * p.H, &bar[B_QFULL]);
          q_in_flight = true;
          ok = mbar_wait(&bar[B_QFULL], nq & 1, p.status, kDevErrTimeout);
          if (!ok) break;
          q_in_flight = false;
          for (int i = 0; i < ntiles && ok; ++i, ++gt) {
            const int sb = gt & 1;
            ok = mbar_wait(&bar[B_SFREE + sb], ((gt >> 1) & 1) ^ 1, p.status, kDevErrTimeout);
            if (!ok) break;
            tc_fence_after();
            const uint32_t d = tmem + kColS + sb * kNH;
            for (int pr = 0; pr < 4 && ok; ++pr) {
              ok = mbar_wait(&bar[B_VFULL + vslot], vround & 1, p.status, kDevErrTimeout);
              if (!ok) break;
              fence_proxy_async_smem();  // cp.async writes -> tensor-core reads
              tc_fence_after();
              const uint32_t a0 = vbase + vslot * kPairBytes;
#pragma unroll
              for (int s = 0; s < 2; ++s)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_bf16_ss(d, umma_desc_sw128(a0 + s * kBlk + kk * 32, 16, 1024),
                              umma_desc_sw128(qbase + (2 * pr + s) * kQBlk + kk * 32, 16, 1024), idesc,
                              (pr | s | kk) ? 1u : 0u);
              if (++vslot == kVSlots) vslot = 0, ++vround;
            }
            if (!ok) break;
            ok = mbar_wait(&bar[B_RFULL], gt & 1, p.status, kDevErrTimeout);
            if (!ok) break;
            fence_proxy_async_smem();
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(d, umma_desc_sw128(rbase + kk * 32, 16, 1024),
                          umma_desc_sw128(qbase + 8 * kQBlk + kk * 32, 16, 1024), idesc, 1u);
            mma_commit(&bar[B_REMPTY]);
            mma_commit(&bar[B_SFULL + sb]);
            if (i == ntiles - 1) mma_commit(&bar[B_QFREE]);
          }
          if (!ok) break;
          ++nq;
        }
        mbar_arrive(&bar[B_ROWSFREE + buf]);
      }
      if (q_in_flight) mbar_drain(&bar[B_QFULL], nq & 1, p.status);  // no TMA may land after the exit
      // every MMA this thread issued has completed before TMEM is freed (also after an error)
      mma_commit(&bar[B_SDRAIN]);
      mbar_drain(&bar[B_SDRAIN], 0, p.status);
    }
    __syncwarp();
  } else if (warp == kPVWarp) {
    // ---------- P V issuer: O^T[128 db .., h] += V^T . P^T, four M blocks of 128 dims ----------
    if (lane == 0) {
      const uint32_t idesc = umma_idesc(128, kNH, 1, 1, 0);  // bf16, A MN-major (V^T), B K-major (P^T)
      const uint32_t vbase = smem_u32(base + NSmem::kV), pbase = smem_u32(base + NSmem::kP);
      uint32_t vslot = 0;
      int gt = 0, nq = 0;
      bool ok = true;
      for (int qn = 0; ok; ++qn) {
        const int buf = qn & 1;
        ok = mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout);
        if (!ok) break;
        const int ntiles = vinfo[buf].z;
        if (ntiles < 0) break;
        if (ntiles > 0) {
          const int ob = nq & 1;
          ok = mbar_wait(&bar[B_OFREE + ob], ((nq >> 1) & 1) ^ 1, p.status, kDevErrTimeout);  // unit nq - 2 read out
          if (!ok) break;
          tc_fence_after();
          const uint32_t dO = tmem + kColO + ob * 4 * kNH;
          for (int i = 0; i < ntiles && ok; ++i, ++gt) {
            const int pb = gt & 1;
            ok = mbar_wait(&bar[B_PFULL + pb], (gt >> 1) & 1, p.status, kDevErrTimeout);
            if (!ok) break;
            fence_proxy_async_smem();  // P^T written by the softmax warps -> tensor-core reads
            tc_fence_after();
            const uint32_t b0 = pbase + pb * kPBuf;
            for (int db = 0; db < 4; ++db) {
              const uint32_t a0 = vbase + vslot * kPairBytes;
#pragma unroll
              for (int kk = 0; kk < kTile / 16; ++kk)
                mma_bf16_ss(dO + db * kNH, umma_desc_sw128(a0 + kk * 2048, kBlk, 1024),
                            umma_desc_sw128(b0 + (kk >> 2) * kPBlk + (kk & 3) * 32, 16, 1024), idesc,
                            (i > 0 || kk > 0) ? 1u : 0u);
              mma_commit(&bar[B_VEMPTY + vslot]);
              if (++vslot == kVSlots) vslot = 0;
            }
            // B_ODONE before B_PFREE: a softmax warp that saw P^T buffer pb free (this tile's
            // product complete) then finds B_ODONE at most one phase behind
            mma_commit(&bar[B_ODONE]);
            mma_commit(&bar[B_PFREE + pb]);
            if (i == ntiles - 1) mma_commit(&bar[B_OFULL + ob]);
          }
          if (!ok) break;
          ++nq;
        }
        mbar_arrive(&bar[B_ROWSFREE + buf]);
      }
      mma_commit(&bar[B_PVDRAIN]);
      mbar_drain(&bar[B_PVDRAIN], 0, p.status);
    }
    __syncwarp();
  } else if (warp < kSoftWarp0 + 4) {
    // ---------- softmax: keys 32 q .. 32 q + 31 of every tile, all 16 head columns ----------
    const int q = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    float* red = reinterpret_cast<float*>(base + NSmem::kRed);
    float* stats = reinterpret_cast<float*>(base + NSmem::kStats);
    // this lane's bf16 pair (keys 2m, 2m + 1) in a row of P^T: 16-byte chunk and byte in it
    const int chunk = 4 * (q & 1) + (lane >> 3);
    const int word = ((lane & 7) >> 1) * 4;
    uint8_t* pq = base + NSmem::kP + (q >> 1) * kPBlk;  // keys 0..63 -> block 0, 64..127 -> block 1
    int gt = 0, nq = 0;
    bool ok = true;
    for (int qn = 0; ok; ++qn) {
      const int buf = qn & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout));
      if (!ok) break;
      const int ntiles = vinfo[buf].z;
      if (ntiles < 0) break;
      if (ntiles > 0) {
        const int ob = nq & 1;
        const uint32_t* msk = masks + buf * kMaxTiles * 4;
        float m_ref[kNH], l[kNH];
#pragma unroll
        for (int h = 0; h < kNH; ++h) m_ref[h] = -INFINITY, l[h] = 0.f;
        for (int i = 0; i < ntiles && ok; ++i, ++gt) {
          const int sb = gt & 1;
          ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_SFULL + sb], (gt >> 1) & 1, p.status, kDevErrTimeout));
          if (!ok) break;
          tc_fence_after();
          uint32_t sr[kNH];
          tmem_ld16_sync(tmem + lane_base + kColS + sb * kNH, sr);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_SFREE + sb]);
          const bool valid = (msk[i * 4 + q] >> lane) & 1u;
          float v[kNH];
#pragma unroll
          for (int h = 0; h < kNH; ++h) v[h] = valid ? __uint_as_float(sr[h]) * p.scale_log2 : -INFINITY;
          // the tile's maximum of every head: over this warp's keys, then over the four warps
          float* rd = red + sb * 4 * kNH;
          {
            float mine = 0.f;
#pragma unroll
            for (int h = 0; h < kNH; ++h) {
              const float wm = warp_max(v[h]);
              if (lane == h) mine = wm;
            }
            if (lane < kNH) rd[q * kNH + lane] = mine;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_RED + sb]);
          ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_RED + sb], (gt >> 1) & 1, p.status, kDevErrTimeout));
          if (!ok) break;
          float alpha[kNH];  // the tile maxima, then the rescale factors
#pragma unroll
          for (int h4 = 0; h4 < kNH / 4; ++h4) {
            float4 m4 = reinterpret_cast<const float4*>(rd)[h4];
#pragma unroll
            for (int w = 1; w < 4; ++w) {
              const float4 x = reinterpret_cast<const float4*>(rd + w * kNH)[h4];
              m4.x = fmaxf(m4.x, x.x), m4.y = fmaxf(m4.y, x.y), m4.z = fmaxf(m4.z, x.z), m4.w = fmaxf(m4.w, x.w);
            }
            alpha[4 * h4 + 0] = m4.x, alpha[4 * h4 + 1] = m4.y, alpha[4 * h4 + 2] = m4.z, alpha[4 * h4 + 3] = m4.w;
          }
          bool resc = false;  // the same decision in every lane of the four warps
#pragma unroll
          for (int h = 0; h < kNH; ++h) {
            const float tm = alpha[h];
            alpha[h] = 1.f;
            if (tm > m_ref[h] + kRescaleThreshold) {
              alpha[h] = fast_exp2(m_ref[h] - tm);  // 0 on the unit's first valid tile
              m_ref[h] = tm;
              resc = true;
            }
          }
          // P^T buffer sb was read by the product of tile gt - 2, which has completed: O^T holds
          // every product up to that tile
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&bar[B_PFREE + sb], ((gt >> 1) & 1) ^ 1, p.status, kDevErrTimeout));
          if (!ok) break;
          if (resc) {
            if (i > 0) {  // rescale O^T once the product of tile gt - 1 has completed too
              ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ODONE], (gt - 1) & 1, p.status, kDevErrTimeout));
              if (!ok) break;
              tc_fence_after();
#pragma unroll 1
              for (int db = 0; db < 4; ++db) {
                const uint32_t ta = tmem + lane_base + kColO + ob * 4 * kNH + db * kNH;
                uint32_t o[kNH];
                tmem_ld16_sync(ta, o);
#pragma unroll
                for (int h = 0; h < kNH; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
                tmem_st16(ta, o);
              }
              tmem_wait_st();
              tc_fence_before();
            }
#pragma unroll
            for (int h = 0; h < kNH; ++h) l[h] *= alpha[h];
          }
#pragma unroll
          for (int h = 0; h < kNH; ++h) {
            v[h] = valid ? fast_exp2(v[h] - m_ref[h]) : 0.f;
            l[h] += v[h];
          }
          // P^T in bf16: even lanes write heads 0..7 and odd lanes heads 8..15, each a pair of keys;
          // the odd lanes' head order (8 + (j ^ 4)) puts the two halves in different banks
          uint8_t* pt = pq + sb * kPBuf;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int ho = 8 + (j ^ 4);
            const float send = (lane & 1) ? v[j] : v[ho];
            const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
            const int h = (lane & 1) ? ho : j;
            const uint32_t w = (lane & 1) ? pack_bf16x2(recv, v[ho]) : pack_bf16x2(v[j], recv);
            *reinterpret_cast<uint32_t*>(pt + (h >> 3) * 1024 + (h & 7) * 128 + ((chunk ^ (h & 7)) << 4) + word) = w;
          }
          fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_PFULL + sb]);
        }
        if (!ok) break;
        // the unit's reference maxima and this warp's share of the sums, for the epilogue
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bar[B_STATSFREE + ob], ((nq >> 1) & 1) ^ 1, p.status, kDevErrTimeout));
        if (!ok) break;
        float* st = stats + ob * 5 * kNH;
        float mine_l = 0.f, mine_m = 0.f;
#pragma unroll
        for (int h = 0; h < kNH; ++h) {
          const float ls = warp_sum(l[h]);
          if (lane == h) mine_l = ls, mine_m = m_ref[h];
        }
        if (lane < kNH) {
          st[(1 + q) * kNH + lane] = mine_l;
          if (q == 0) st[lane] = mine_m;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_STATS + ob]);
        ++nq;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_ROWSFREE + buf]);
    }
  } else if (warp < kEpiWarp0 + 4) {
    // ---------- epilogue: value dims 128 db + 32 q + lane of every O^T block ----------
    const int q = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const float* stats = reinterpret_cast<const float*>(base + NSmem::kStats);
    const int H = p.H;
    int nq = 0;
    bool ok = true;
    for (int qn = 0; ok; ++qn) {
      const int buf = qn & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_ROWSFULL + buf], (qn >> 1) & 1, p.status, kDevErrTimeout));
      if (!ok) break;
      const int t = vinfo[buf].x, split = vinfo[buf].y, ntiles = vinfo[buf].z;
      if (ntiles < 0) break;
      const bool have_o = ntiles > 0;
      const int ob = nq & 1;
      float inv[kNH], lse_mine = -INFINITY;  // lse of head `lane`
      if (have_o) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_STATS + ob], (nq >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        const float* st = stats + ob * 5 * kNH;
#pragma unroll
        for (int h = 0; h < kNH; ++h) {
          const float m = st[h];
          const float l = (st[kNH + h] + st[2 * kNH + h]) + (st[3 * kNH + h] + st[4 * kNH + h]);
          inv[h] = l > 0.f ? 1.f / l : 0.f;
          if (lane == h && l > 0.f) lse_mine = (m + log2f(l)) * 0.69314718055994531f;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_STATSFREE + ob]);
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_OFULL + ob], (nq >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        tc_fence_after();
      } else {
#pragma unroll
        for (int h = 0; h < kNH; ++h) inv[h] = 0.f;
      }
#pragma unroll 1
      for (int db = 0; db < 4; ++db) {
        float o[kNH];
        if (have_o) {
          uint32_t r[kNH];
          tmem_ld16_sync(tmem + lane_base + kColO + ob * 4 * kNH + db * kNH, r);
#pragma unroll
          for (int h = 0; h < kNH; ++h) o[h] = __uint_as_float(r[h]) * inv[h];
        } else {
#pragma unroll
          for (int h = 0; h < kNH; ++h) o[h] = 0.f;
        }
        const int d = 128 * db + 32 * q + lane;
        if (p.nsplit == 1) {
          // bf16 pairs of dims (d, d + 1): even lanes heads 0..7, odd lanes heads 8..15
          uint16_t* orow = p.out + static_cast<int64_t>(t) * H * kDV + (d & ~1);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float send = (lane & 1) ? o[j] : o[8 + j];
            const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
            const int h = (lane & 1) ? 8 + j : j;
            const uint32_t w = (lane & 1) ? pack_bf16x2(recv, o[8 + j]) : pack_bf16x2(o[j], recv);
            if (h < H) *reinterpret_cast<uint32_t*>(orow + static_cast<int64_t>(h) * kDV) = w;
          }
        } else {
          float* prow = p.part_o + (static_cast<int64_t>(t) * p.nsplit + split) * H * kDV + d;
#pragma unroll
          for (int h = 0; h < kNH; ++h)
            if (h < H) prow[static_cast<int64_t>(h) * kDV] = o[h];
        }
      }
      if (have_o) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_OFREE + ob]);
        ++nq;
      }
      if (q == 0 && lane < H) {
        if (p.nsplit == 1) {
          if (p.lse) p.lse[static_cast<int64_t>(t) * H + lane] = lse_mine;
        } else {
          p.part_lse[(static_cast<int64_t>(t) * p.nsplit + split) * H + lane] = lse_mine;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_ROWSFREE + buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kSWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// One warp per (row, head): o = sum_s exp(lse_s - lse) o_s, lse = log sum_s exp(lse_s).
__global__ void __launch_bounds__(256) narrow_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_lse, int T, int H,
                                                             int nsplit, uint16_t* __restrict__ out,
                                                             float* __restrict__ lse) {
  const int gw = static_cast<int>(blockIdx.x) * 8 + static_cast<int>(threadIdx.x >> 5);
  const int lane = static_cast<int>(threadIdx.x & 31);
  pdl_trigger();
  pdl_wait();  // the partial results of the sparse MLA kernel
  if (gw >= T * H) return;
  const int t = gw / H, h = gw - t * H;
  const int64_t r0 = static_cast<int64_t>(t) * nsplit * H + h;  // split s of (t, h): row r0 + s * H
  float mx = -INFINITY;
  for (int s = 0; s < nsplit; ++s) mx = fmaxf(mx, __ldg(part_lse + r0 + static_cast<int64_t>(s) * H));
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (mx > -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const int64_t r = r0 + static_cast<int64_t>(s) * H;
      const float w = expf(__ldg(part_lse + r) - mx);
      wsum += w;
      const float4* src = reinterpret_cast<const float4*>(part_o + r * kDV) + lane * 4;
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

int launch_sparse_mla_narrow(const BatchDev& b, const void* plan, const void* q, int H, const void* kv_cache,
                             const int32_t* S, int k, float softmax_scale, void* out, float* lse, void* ws,
                             void* stream) {
  if (b.T == 0) return 0;
  if (H < 1 || H > kNH) return static_cast<int>(cudaErrorInvalidValue);
  PlanView pv = plan_view(const_cast<void*>(plan), b.B, b.T);
  NarrowParams prm{};
  prm.bd = b;
  prm.row_req = pv.row_req;
  prm.row_pos = pv.row_pos;
  prm.q = static_cast<const uint16_t*>(q);
  prm.kv = static_cast<const uint8_t*>(kv_cache);
  prm.S = S;
  prm.k = k;
  prm.H = H;
  // the same splits (and so the same workspace) as the many-head kernel
  prm.nsplit = sparse_mla_splits(b.T, k);
  prm.units = b.T * prm.nsplit;
  const int per = (k + prm.nsplit - 1) / prm.nsplit;
  prm.chunk = (per + kTile - 1) / kTile * kTile;
  if (prm.chunk > kMaxKeys) return static_cast<int>(cudaErrorInvalidValue);
  prm.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634);
  prm.out = static_cast<uint16_t*>(out);
  prm.lse = lse;
  if (prm.nsplit > 1) {
    prm.part_o = static_cast<float*>(ws);
    prm.part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                            align16(sizeof(float) * static_cast<size_t>(b.T) * prm.nsplit * H * kDV));
  }
  prm.status = &pv.hdr->status;

  // Q [T * H rows][576] bf16, boxes of 64 dims x 16 rows (rows past a query's H heads belong to
  // the next query, or lie past the tensor and read as zeros; their columns are never used)
  CUtensorMap qmap;
  int e = make_tmap_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, kDLat, static_cast<uint64_t>(b.T) * H,
                       kDLat * 2, 64, kNH);
  if (e) return e;
  cudaError_t ce = cudaFuncSetAttribute(sparse_mla_narrow_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        NSmem::kDynamic);
  if (ce != cudaSuccess) return static_cast<int>(ce);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ctas = std::min(prm.units, std::max(1, sms));  // one CTA per SM (shared memory), persistent
  ce = launch_pdl(sparse_mla_narrow_kernel, dim3(ctas), dim3(kThreads), NSmem::kDynamic, stream, qmap, prm);
  if (ce != cudaSuccess) return static_cast<int>(ce);
  if (prm.nsplit > 1) {
    const int warps = b.T * H;
    ce = launch_pdl(narrow_combine_kernel, dim3((warps + 7) / 8), dim3(256), 0, stream, prm.part_o, prm.part_lse,
                    b.T, H, prm.nsplit, prm.out, lse);
  }
  return static_cast<int>(ce);
}

}  // namespace dsa
