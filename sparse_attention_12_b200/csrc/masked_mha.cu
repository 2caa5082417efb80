// Masked MHA mode for short prefill (sm_100a).
//
// For a short prefill the pages note that sparse attention in the absorbed MQA form costs more than
// dense attention in the expanded multi-head form, and that DeepSeek-V3.2 therefore emulates DSA
// there with a multi-head attention under a mask ("MTP 与稀疏注意力：NSA 与 DSA", section
// "稀疏注意力：NSA 与 DSA": 2H(128+64) + 2H*128 FLOPs per pair instead of 2H(512+64) + 2H*512). The
// mask is the DSA mask of "DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section
// "Sparse Attention": M_tj = 0 for j in S_t, -inf otherwise. For query row t and head h:
//   z_hj = scale * q_th . k_jh (192 dims) + M_tj,   o_th = sum_j softmax_j(z_hj) v_jh (128 dims).
//
// Every request is a whole prefill (m_b = n_b), so position j of request b is row cu_q[b] + j of k
// and v, and the query tile's rows are its own positions.
//
// Two kernels:
//   * mha_mask_kernel: the bitmap of S_t, one row of 32-bit words per query row (bit j of word w is
//     position 32w + j), one warp per row, built in shared memory with atomics, then stored with
//     16-byte stores.
//   * masked_mha_kernel: one CTA per (head, 128-query tile, request), a flash-attention pass over the
//     key tiles 0 .. the tile's last position (causal by construction: S_t only holds j <= t).
//       - warp 0: TMA producers. Lane 0: Q (3 boxes of 128 rows x 64 dims, 128-byte swizzle) once,
//         then K (3 boxes per key tile) into a two-stage ring; lane 1: V (2 boxes per key tile) into
//         its own two-stage ring.
//       - warp 1: TMEM allocator and the single MMA-issuing thread. S = Q K^T is 12 tcgen05.mma
//         (M = 128 queries, N = 128 keys, K = 16) from shared memory into one of two S buffers in
//         TMEM; O += P V is 8 tcgen05.mma with P read from TMEM (the A operand) and V from shared
//         memory (MN-major), into O in TMEM. Order: S0, S1, then P V(i), S(i+2) per tile.
//       - warps 2..9: softmax, two warps per TMEM lane quadrant (thread = query row, 64 keys each;
//         four warps of 32 keys measured slower: the per-tile exchange and waits outweigh the extra
//         latency hiding). They mask with the bitmap, keep an online softmax whose reference maximum
//         moves only when a tile's maximum exceeds it by more than 2^8 (then they rescale their half
//         of O's row), and write bf16 P into TMEM (two buffers). At the end they normalise O and
//         store bf16 rows.
//   TMEM: S at columns 0 and 128, O at 256, P at 384 and 448 (bf16 pairs): all 512 columns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"

namespace dsa {

int make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2);

namespace {

constexpr int kTile = 128;             // queries per CTA, keys per tile
constexpr int kDqk = DSA_D_QK_MHA;     // 192
constexpr int kDvh = DSA_D_V_MHA;      // 128
constexpr int kBlk = kTile * 128;      // 128 rows x 64 bf16 dims (128 bytes), 16 KB
constexpr int kQBlks = kDqk / 64;      // 3
constexpr int kVBlks = kDvh / 64;      // 2
constexpr int kStages = 2;             // K and V ring depth
constexpr int kSoftWarp0 = 2;
constexpr int kSoftWarps = 8;
constexpr int kSubs = kSoftWarps / 4;  // softmax warps per TMEM lane quadrant
constexpr int kCols = kTile / kSubs;   // keys of a tile per softmax warp (64)
constexpr int kWords = kCols / 32;     // mask words (and 32-column TMEM loads) per softmax warp and tile
constexpr int kOCols = kDvh / kSubs;   // O columns per softmax warp (64)
constexpr int kThreads = 32 * (kSoftWarp0 + kSoftWarps);
constexpr float kRescaleThreshold = 8.0f;  // log2 units

constexpr uint32_t kColS = 0;    // S tiles, 128 fp32 columns each, at 0 and 128
constexpr uint32_t kColO = 256;  // O, 128 fp32 columns
constexpr uint32_t kColP = 384;  // P tiles, 64 columns of bf16 pairs each, at 384 and 448

struct Smem {
  static constexpr int kQ = 0;                                      // 3 blocks
  static constexpr int kK = kQ + kQBlks * kBlk;                     // kStages x 3 blocks
  static constexpr int kV = kK + kStages * kQBlks * kBlk;           // kStages x 2 blocks
  static constexpr int kRed = kV + kStages * kVBlks * kBlk;         // float [2][kSubs][128]: tile maxima
  static constexpr int kRedL = kRed + 2 * kSubs * 128 * 4;          // float [2][kSubs][128]: l, lr
  static constexpr int kBars = kRedL + 2 * kSubs * 128 * 4;
  static constexpr int kNumBars = 32;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kTotal = kTmemSlot + 16;
  static constexpr int kDynamic = kTotal + 1024;
};
static_assert(Smem::kDynamic <= 232448, "masked MHA shared memory exceeds the 227 KB limit");
static_assert(kDqk % 64 == 0 && kDvh % 64 == 0, "head widths in 64-dim blocks");
static_assert(kCols % 32 == 0 && kOCols % 32 == 0, "softmax warps work in 32-column TMEM loads");

enum : int {
  B_QFULL = 0,                 // 1    TMA bytes of Q
  B_KFULL = B_QFULL + 1,       // [2]  TMA bytes of a K stage
  B_KEMPTY = B_KFULL + 2,      // [2]  MMA commit
  B_VFULL = B_KEMPTY + 2,      // [2]  TMA bytes of a V stage
  B_VEMPTY = B_VFULL + 2,      // [2]  MMA commit
  B_SFULL = B_VEMPTY + 2,      // [2]  MMA -> softmax: S tile ready
  B_PFULL = B_SFULL + 2,       // [2]  softmax (8 warps) -> MMA: P tile in TMEM, O rescaled
  B_PVDONE = B_PFULL + 2,      // [2]  MMA commit after P V: P buffer free, O up to date
  B_RED = B_PVDONE + 2,        // [2][4] partial maxima of one quadrant written (kSubs warps)
  B_LEND = B_RED + 8,          // [4]  partial sums of one quadrant written (kSubs warps)
  B_OFINAL = B_LEND + 4,       // 1    MMA -> epilogue after the last P V
  B_MDONE = B_OFINAL + 1,      // 1    the MMA issuer's last commit (drained before TMEM is freed)
  B_COUNT = B_MDONE + 1
};
static_assert(B_COUNT <= Smem::kNumBars, "barrier space");

struct MhaParams {
  BatchDev bd;
  const uint32_t* mask;  // [T][ldw] bitmap of S_t
  int ldw;               // words per mask row (multiple of 4)
  int H;
  float scale_log2;      // softmax scale * log2(e)
  uint16_t* out;         // bf16 [T][H][128]
  float* lse;            // [T][H] or null
  uint32_t* status;
};

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int32_t x, int32_t y, int32_t z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Bitmap of S_t for every query row: bit (j & 31) of word j / 32 set for j in S_t. Entries below 0
// are padding; an entry above the row's position is reported and skipped. One warp per row, each
// warp with its own ldw words of shared memory (no block-wide synchronisation).
__global__ void __launch_bounds__(256) mha_mask_kernel(const int32_t* __restrict__ row_pos,
                                                       const int32_t* __restrict__ S, int k, int ldw, int T,
                                                       uint32_t* __restrict__ mask, uint32_t* status) {
  extern __shared__ uint32_t words[];
  pdl_trigger();
  pdl_wait();  // S_t and the plan come from earlier kernels
  const int rows = static_cast<int>(blockDim.x >> 5);
  const int warp = warp_id(), lane = lane_id();
  const int t = blockIdx.x * rows + warp;
  if (t >= T) return;
  uint32_t* wrow = words + warp * ldw;
  for (int w = lane; w < ldw; w += 32) wrow[w] = 0u;
  __syncwarp();
  const int p = __ldg(row_pos + t);
  const int32_t* St = S + static_cast<int64_t>(t) * k;
  for (int e0 = 0; e0 < k; e0 += 32 * 8) {
    int jv[8];  // eight loads in flight per lane before the first atomic
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + 32 * u + lane;
      jv[u] = (e < k) ? __ldg(St + e) : -1;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = jv[u];
      if (j < 0) continue;
      if (j > p || j >= 32 * ldw) {
        report_error(status, kDevErrIndex);
        continue;
      }
      atomicOr(&wrow[j >> 5], 1u << (j & 31));
    }
  }
  __syncwarp();
  uint4* dst = reinterpret_cast<uint4*>(mask + static_cast<int64_t>(t) * ldw);
  for (int w4 = lane; w4 < ldw / 4; w4 += 32)
    dst[w4] = make_uint4(wrow[4 * w4], wrow[4 * w4 + 1], wrow[4 * w4 + 2], wrow[4 * w4 + 3]);
}

__global__ void __launch_bounds__(kThreads, 1)
    masked_mha_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const MhaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + Smem::kBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + Smem::kTmemSlot);
  const int warp = warp_id(), lane = lane_id();
  const int h = blockIdx.x;
  const int qi = static_cast<int>(gridDim.y) - 1 - static_cast<int>(blockIdx.y);  // longest tiles first
  const int b = blockIdx.z;

  if (threadIdx.x == 0) {
    mbar_init(&bar[B_QFULL], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[B_KFULL + i], 1);
      mbar_init(&bar[B_KEMPTY + i], 1);
      mbar_init(&bar[B_VFULL + i], 1);
      mbar_init(&bar[B_VEMPTY + i], 1);
      mbar_init(&bar[B_SFULL + i], 1);
      mbar_init(&bar[B_PFULL + i], kSoftWarps);
      mbar_init(&bar[B_PVDONE + i], 1);
    }
    for (int i = 0; i < 8; ++i) mbar_init(&bar[B_RED + i], kSubs);
    for (int i = 0; i < 4; ++i) mbar_init(&bar[B_LEND + i], kSubs);
    mbar_init(&bar[B_OFINAL], 1);
    mbar_init(&bar[B_MDONE], 1);
    fence_barrier_init();
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();  // the mask kernel's bitmap
  const int row0 = __ldg(p.bd.cu_q + b);
  const int nq = __ldg(p.bd.cu_q + b + 1) - row0;
  const int n_b = __ldg(p.bd.seq_lens + b);
  const int q0 = qi * kTile;  // first position (and row within the request) of this query tile
  const int nrows = min(kTile, nq - q0);
  int nkt = 0;  // key tiles: positions 0 .. q0 + nrows - 1
  if (nrows > 0) {
    if (n_b != nq) {
      if (threadIdx.x == 0) report_error(p.status, kDevErrIndex);  // not a whole prefill
    } else {
      nkt = (q0 + nrows - 1) / kTile + 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------- TMA producers: lane 0 Q and the K ring, lane 1 the V ring ----------
    // (independent loops: K(i+2) goes out as soon as S(i) has consumed its stage, without waiting
    // behind V(i+1), whose stage frees only after P V(i-1))
    if (lane < 2 && nkt > 0) {
      const bool is_k = lane == 0;
      const int nblk = is_k ? kQBlks : kVBlks;
      const CUtensorMap* map = is_k ? &kmap : &vmap;
      uint8_t* ring = base + (is_k ? Smem::kK : Smem::kV);
      uint64_t* full = &bar[is_k ? B_KFULL : B_VFULL];
      uint64_t* empty = &bar[is_k ? B_KEMPTY : B_VEMPTY];
      if (is_k) {
        mbar_arrive_expect_tx(&bar[B_QFULL], kQBlks * kBlk);
        for (int blk = 0; blk < kQBlks; ++blk)
          tma_load_3d(base + Smem::kQ + blk * kBlk, &qmap, 64 * blk, h, row0 + q0, &bar[B_QFULL]);
      }
      bool ok = true;
      int issued = 0;  // tiles whose loads went out
      for (int i = 0; i < nkt && ok; ++i) {
        const int s = i & 1;
        ok = mbar_wait(&empty[s], ((i >> 1) & 1) ^ 1, p.status, kDevErrTimeout);
        if (!ok) break;
        mbar_arrive_expect_tx(&full[s], nblk * kBlk);
        for (int blk = 0; blk < nblk; ++blk)
          tma_load_3d(ring + (s * nblk + blk) * kBlk, map, 64 * blk, h, row0 + i * kTile, &full[s]);
        issued = i + 1;
      }
      // no copy may still be landing when the CTA exits, also after an error
      if (is_k) mbar_drain(&bar[B_QFULL], 0, p.status);
      for (int i = max(0, issued - kStages); i < issued; ++i) mbar_drain(&full[i & 1], (i >> 1) & 1, p.status);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------- MMA issuer ----------
    if (lane == 0 && nkt > 0) {
      const uint32_t idesc_s = umma_idesc(128, kTile, 1, 0, 0);  // bf16, A and B K-major
      const uint32_t idesc_o = umma_idesc(128, kDvh, 1, 0, 1);   // bf16, A (TMEM) K-major, B MN-major
      const uint64_t qdesc = umma_desc_sw128(smem_u32(base + Smem::kQ), 16, 1024);
      const uint64_t kdesc0 = umma_desc_sw128(smem_u32(base + Smem::kK), 16, 1024);
      const uint64_t vdesc0 = umma_desc_sw128(smem_u32(base + Smem::kV), kBlk, 1024);
      bool ok = mbar_wait(&bar[B_QFULL], 0, p.status, kDevErrTimeout);
      // S(i) = Q K(i)^T into S buffer i % 2
      auto issue_qk = [&](int i) -> bool {
        const int s = i & 1;
        if (!mbar_wait(&bar[B_KFULL + s], (i >> 1) & 1, p.status, kDevErrTimeout)) return false;
        tc_fence_after();
        const uint32_t d = tmem + kColS + kTile * s;
        const uint64_t kd = kdesc0 + static_cast<uint64_t>((s * kQBlks * kBlk) >> 4);
#pragma unroll
        for (int blk = 0; blk < kQBlks; ++blk)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t off = static_cast<uint64_t>((blk * kBlk) >> 4) + 2 * kk;
            mma_bf16_ss(d, qdesc + off, kd + off, idesc_s, (blk | kk) ? 1u : 0u);
          }
        mma_commit(&bar[B_KEMPTY + s]);
        mma_commit(&bar[B_SFULL + s]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      if (ok && nkt > 1) ok = issue_qk(1);
      for (int i = 0; i < nkt && ok; ++i) {
        const int s = i & 1;
        ok = mbar_wait(&bar[B_PFULL + s], (i >> 1) & 1, p.status, kDevErrTimeout) &&
             mbar_wait(&bar[B_VFULL + s], (i >> 1) & 1, p.status, kDevErrTimeout);
        if (!ok) break;
        tc_fence_after();
        const uint64_t vd = vdesc0 + static_cast<uint64_t>((s * kVBlks * kBlk) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)  // 16 keys: 8 P columns, 16 rows of V (2048 bytes)
          mma_bf16_ts(tmem + kColO, tmem + kColP + 64 * s + 8 * kk, vd + static_cast<uint64_t>((kk * 2048) >> 4),
                      idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar[B_VEMPTY + s]);
        mma_commit(&bar[B_PVDONE + s]);
        if (i == nkt - 1) mma_commit(&bar[B_OFINAL]);
        // S buffer s was read by the softmax of tile i before it signalled P(i)
        if (i + 2 < nkt) ok = issue_qk(i + 2);
      }
      // every MMA this thread issued has completed before TMEM is freed (also after an error)
      mma_commit(&bar[B_MDONE]);
      mbar_drain(&bar[B_MDONE], 0, p.status);
    }
    __syncwarp();
  } else {
    // ---------- softmax + epilogue (warps 2..9: thread = query row r, keys kCols*sub .. +kCols-1) ----------
    const int quad = warp & 3;
    const int sub = (warp - kSoftWarp0) >> 2;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const bool row_ok = r < nrows;
    const int64_t t = static_cast<int64_t>(row0) + q0 + r;
    // words 4i + kWords*sub .. + kWords-1 cover this warp's keys of tile i
    const uint32_t* mrow = p.mask + (row_ok ? t : 0) * p.ldw + kWords * sub;
    float* red = reinterpret_cast<float*>(base + Smem::kRed);
    float* redl = reinterpret_cast<float*>(base + Smem::kRedL);
    const float sl2 = p.scale_log2;
    float m_ref = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    uint32_t mk[kWords], mk_next[kWords];
#pragma unroll
    for (int w = 0; w < kWords; ++w) mk[w] = (row_ok && nkt > 0) ? __ldg(mrow + w) : 0u;
    for (int i = 0; i < nkt && ok; ++i) {
      const int s = i & 1;
#pragma unroll
      for (int w = 0; w < kWords; ++w) mk_next[w] = (row_ok && i + 1 < nkt) ? __ldg(mrow + 4 * (i + 1) + w) : 0u;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_SFULL + s], (i >> 1) & 1, p.status, kDevErrTimeout));
      if (!ok) break;
      tc_fence_after();
      // this warp's kCols scores of the row, -inf where the position is not in S_t
      float x[kCols];
#pragma unroll
      for (int w = 0; w < kWords; ++w) {
        uint32_t v[32];
        tmem_ld32_sync(tmem + lane_base + kColS + kTile * s + kCols * sub + 32 * w, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) x[32 * w + j] = ((mk[w] >> j) & 1u) ? __uint_as_float(v[j]) : -INFINITY;
      }
      // maximum as a tree (short dependency chains)
      static_assert(kCols == 64, "the tree below covers 64 scores");
      float mx[8];
#pragma unroll
      for (int a = 0; a < 8; ++a)
        mx[a] = fmaxf(fmaxf(fmaxf(x[a], x[a + 8]), fmaxf(x[a + 16], x[a + 24])),
                      fmaxf(fmaxf(x[a + 32], x[a + 40]), fmaxf(x[a + 48], x[a + 56])));
      float pmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      pmax *= sl2;  // positive scale: the maximum commutes with it (-inf stays -inf)
      red[(s * kSubs + sub) * 128 + r] = pmax;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_RED + s * 4 + quad]);
      ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_RED + s * 4 + quad], (i >> 1) & 1, p.status, kDevErrTimeout));
      if (!ok) break;
      float tmax = -INFINITY;
#pragma unroll
      for (int s2 = 0; s2 < kSubs; ++s2) tmax = fmaxf(tmax, red[(s * kSubs + s2) * 128 + r]);
      const bool need = tmax > m_ref + kRescaleThreshold;
      const float alpha = need ? exp2f(m_ref - tmax) : 1.f;  // 0 when m_ref is -inf
      if (need) {
        l *= alpha;
        lr *= alpha;
        m_ref = tmax;
      }
      if (__any_sync(0xffffffffu, need && i > 0)) {
        // rescale this warp's part of the O rows once P V(i-1) has landed (rows without a new
        // reference maximum multiply by 1)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bar[B_PVDONE + ((i - 1) & 1)], ((i - 1) >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        tc_fence_after();
        const uint32_t ocol = tmem + lane_base + kColO + kOCols * sub;
#pragma unroll 1
        for (int c = 0; c < kOCols / 32; ++c) {
          uint32_t o[32];
          tmem_ld32_sync(ocol + 32 * c, o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(ocol + 32 * c, o);
        }
        tmem_wait_st();
      }
      // P buffer s was last read by P V(i-2)
      if (i >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_PVDONE + s], ((i - 2) >> 1) & 1, p.status, kDevErrTimeout));
        if (!ok) break;
        tc_fence_after();
      }
      const float m_use = (m_ref > -INFINITY) ? m_ref : 0.f;  // m_ref = -inf: every key so far masked
      // p = 2^(scale' x - m): masked entries give 2^-inf = 0. Sums on four independent accumulators:
      // l of the fp32 weights (for the log-sum-exp), lr of the bf16-rounded weights the MMA uses.
      uint32_t pk[kCols / 2];
      float la[4] = {0.f, 0.f, 0.f, 0.f}, lra[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j2 = 0; j2 < kCols / 2; ++j2) {
        const float a0 = fast_exp2(fmaf(x[2 * j2], sl2, -m_use));
        const float a1 = fast_exp2(fmaf(x[2 * j2 + 1], sl2, -m_use));
        const uint32_t w = pack_bf16x2(a0, a1);
        la[j2 & 3] += a0 + a1;
        lra[j2 & 3] += __uint_as_float(w << 16) + __uint_as_float(w & 0xFFFF0000u);
        pk[j2] = w;
      }
      l += (la[0] + la[1]) + (la[2] + la[3]);
      lr += (lra[0] + lra[1]) + (lra[2] + lra[3]);
      static_assert(kCols == 64, "one 32-column TMEM store of P per softmax warp");
      tmem_st32(tmem + lane_base + kColP + 64 * s + (kCols / 2) * sub, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_PFULL + s]);
#pragma unroll
      for (int w = 0; w < kWords; ++w) mk[w] = mk_next[w];
    }
    // row sums over the quadrant's warps
    redl[(0 * kSubs + sub) * 128 + r] = l;
    redl[(1 * kSubs + sub) * 128 + r] = lr;
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar[B_LEND + quad]);
    const bool sums_ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_LEND + quad], 0, p.status, kDevErrTimeout));
    float lt = 0.f, lrt = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < kSubs; ++s2) {
      lt += redl[(0 * kSubs + s2) * 128 + r];
      lrt += redl[(1 * kSubs + s2) * 128 + r];
    }
    ok = __all_sync(0xffffffffu, ok && sums_ok);
    if (ok && nkt > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_OFINAL], 0, p.status, kDevErrTimeout));
    tc_fence_after();
    if (nkt > 0) {
      const float inv = (ok && lrt > 0.f) ? 1.f / lrt : 0.f;
      const float lse_nat = (ok && lt > 0.f) ? (m_ref + log2f(lt)) * 0.69314718055994531f : -INFINITY;
      uint4* dst = reinterpret_cast<uint4*>(p.out + (t * p.H + h) * kDvh + kOCols * sub);
#pragma unroll 1
      for (int c = 0; c < kOCols / 32; ++c) {
        uint32_t o[32];
        tmem_ld32_sync(tmem + lane_base + kColO + kOCols * sub + 32 * c, o);
        if (row_ok) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * j + 0]) * inv, __uint_as_float(o[8 * j + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * j + 2]) * inv, __uint_as_float(o[8 * j + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * j + 4]) * inv, __uint_as_float(o[8 * j + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * j + 6]) * inv, __uint_as_float(o[8 * j + 7]) * inv);
            dst[4 * c + j] = w;
          }
        }
      }
      if (row_ok && sub == 0 && p.lse) p.lse[t * p.H + h] = lse_nat;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

int masked_mha_ldw(int max_seq_len) { return (max_seq_len + kTile - 1) / kTile * 4; }

size_t masked_mha_ws_bytes(int T, int max_seq_len) {
  return sizeof(uint32_t) * static_cast<size_t>(T) * static_cast<size_t>(masked_mha_ldw(max_seq_len));
}

int launch_masked_mha(const BatchDev& b, const void* plan, const void* q, const void* k, const void* v, int H,
                      const int32_t* S, int topk, float softmax_scale, void* out, float* lse, void* ws, void* stream) {
  if (b.T == 0) return 0;
  PlanView pv = plan_view(const_cast<void*>(plan), b.B, b.T);
  const int ldw = masked_mha_ldw(b.max_seq_len);
  uint32_t* mask = static_cast<uint32_t*>(ws);
  // rows per mask block: up to 8, within 48 KB of shared memory (ldw <= 2048 words)
  const int mrows = std::max(1, std::min(8, 12288 / ldw));
  cudaError_t ce = launch_pdl(mha_mask_kernel, dim3((b.T + mrows - 1) / mrows), dim3(32 * mrows),
                              sizeof(uint32_t) * mrows * ldw, stream, static_cast<const int32_t*>(pv.row_pos), S,
                              topk, ldw, b.T, mask, &pv.hdr->status);
  if (ce != cudaSuccess) return static_cast<int>(ce);

  MhaParams prm{};
  prm.bd = b;
  prm.mask = mask;
  prm.ldw = ldw;
  prm.H = H;
  prm.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634);
  prm.out = static_cast<uint16_t*>(out);
  prm.lse = lse;
  prm.status = &pv.hdr->status;
  // [T][H][d] bf16, boxes of 64 dims x 1 head x 128 rows (128-byte swizzle)
  CUtensorMap qmap, kmap, vmap;
  const uint64_t Hu = static_cast<uint64_t>(H), Tu = static_cast<uint64_t>(b.T);
  int e = make_tmap_3d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, kDqk, Hu, Tu, kDqk * 2, Hu * kDqk * 2, 64, 1, kTile);
  if (e) return e;
  e = make_tmap_3d(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, kDqk, Hu, Tu, kDqk * 2, Hu * kDqk * 2, 64, 1, kTile);
  if (e) return e;
  e = make_tmap_3d(&vmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v, kDvh, Hu, Tu, kDvh * 2, Hu * kDvh * 2, 64, 1, kTile);
  if (e) return e;
  ce = cudaFuncSetAttribute(masked_mha_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem::kDynamic);
  if (ce != cudaSuccess) return static_cast<int>(ce);
  const int qtiles = (b.max_q + kTile - 1) / kTile;
  ce = launch_pdl(masked_mha_kernel, dim3(H, qtiles, b.B), dim3(kThreads), Smem::kDynamic, stream, qmap, kmap, vmap,
                  prm);
  return static_cast<int>(ce);
}

}  // namespace dsa
