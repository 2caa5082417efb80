// Exact top-k selection over one score row whose keys are spread over the shared memory of the
// CTAs of a thread-block cluster (used by the cluster top-k kernel and by the fused indexer and
// top-k kernel).
//
//   S_t = TopK_{j<=t}(I_tj, k)  ("DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section
//   "Lightning Indexer", TopK formula); ties: the smaller position wins; positions come out in
//   increasing order.
//
// CTA r of a cluster of C holds the order-preserving keys of positions base_r .. base_r + n_r - 1,
// with base_r increasing in r. The steps are those of a single-CTA radix select, run over the whole
// row:
//   1. the row's smallest and largest key (every CTA pushes its own into every peer);
//   2. a 2048-bin histogram linear in the score value between them: each CTA reduces its local
//      histogram into the CTA that sums bin b (b / (2048 / C)) with remote reductions, then reads
//      the summed bins (vector remote loads) and finds the bin b* of the k-th largest key;
//   3. the keys of b* (normally a handful; at most kCandCap) go to rank 0 (one remote atomic per CTA
//      reserves a range), together with every CTA's count of keys above b*; every CTA then reads
//      them, finds the k-th largest key theta exactly, and from the candidates' ranks and the counts
//      above b* computes how many keys above / equal to theta every lower rank emits;
//   4. emission of this CTA's keys above theta and its share of the ties, in position order.
// Rows the value bins cannot split (infinities, NaN, heavy ties, an overfull b*) narrow further in
// key space (more exchanges of the same kind). Every decision depends only on values every CTA of
// the cluster holds identically, so all of them pass the same cluster barriers.
//
// Protocol (remote accesses happen only between two cluster barriers: every peer has started and
// none has left): before the first call each CTA clears its state (clear_state) and issues
// cluster_arrive(). A call opens with the matching cluster_wait(), clears its state again after its
// last remote access, issues cluster_arrive() and then emits. After the last call, cluster_wait()
// before the CTA exits.
#pragma once
#include <cstdint>

#include "dsa_ptx.cuh"

namespace dsa {
namespace sel {

constexpr int kBins = 2048;
constexpr int kCandCap = 128;    // boundary-bin keys resolved by counting
constexpr int kMaxCluster = 8;
constexpr int kMaxChunks = 16;   // chunks of 4 * NT keys per CTA

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;  // NaN ranks below every other score, -inf included
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;  // -0 ranks as +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t u) {  // inverse of order_key (-0 -> +0, NaN -> a NaN)
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_barrier() {
  cluster_arrive();
  cluster_wait();
}
__device__ __forceinline__ uint4 ld_cluster_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

template <int NT>
struct Shared {
  static constexpr int kW = NT / 32;
  uint32_t mm[kMaxCluster][2];      // every rank's smallest and largest key (pushed by that rank)
  uint32_t above[kMaxCluster];      // every rank's keys above the candidate range (pushed)
  uint32_t rc[kMaxCluster][2];      // every rank's keys above / equal to theta (rare path, pushed)
  uint32_t cand_count;              // rank 0: candidates pushed so far
  uint32_t cand_key[kCandCap];      // rank 0: the candidates
  uint32_t cand_rank[kCandCap];     //   and the rank that holds each
  alignas(16) uint32_t lkey[kCandCap];  // this CTA's copy of the candidates (read 16 bytes at a time)
  uint32_t lrank[kCandCap];
  uint32_t rgt[kMaxCluster], req[kMaxCluster];  // candidates above / equal to theta per rank
  uint32_t lo, remaining, ncand, slot, w0;
  int scan_scratch[kW];
  uint32_t red_a[kW], red_b[kW];
  int2 cnt[kMaxChunks][kW];         // per (chunk, warp): keys above / equal to theta, then offsets
};

// Shared-memory words of the histograms: the local one (kBins) and three buffers of this CTA's
// share of the row's (3 * kBins / C).
__host__ __device__ constexpr int hist_words(int C) { return kBins + 3 * (kBins / C); }

template <int NT>
__device__ __forceinline__ void clear_state(Shared<NT>& sh, uint32_t* hist, uint32_t C) {
  const uint32_t words = kBins + 3u * (kBins / C);
  for (uint32_t i = threadIdx.x; i < words; i += NT) hist[i] = 0u;
  if (threadIdx.x == 0) sh.cand_count = 0u;
}

// Block-wide inclusive scan of one value per thread; also returns the total.
template <int NT>
__device__ __forceinline__ int block_scan(int v, int* scratch, int* total) {
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
    int s = lane < NT / 32 ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NT / 32) scratch[lane] = s;
  }
  __syncthreads();
  const int r = x + (wid > 0 ? scratch[wid - 1] : 0);
  *total = scratch[NT / 32 - 1];
  __syncthreads();
  return r;
}

// Sum over the CTA of one value per thread (every thread gets it).
template <int NT>
__device__ __forceinline__ uint32_t block_sum(uint32_t v, Shared<NT>& sh) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  v = __reduce_add_sync(0xffffffffu, v);
  if (lane == 0) sh.red_a[wid] = v;
  __syncthreads();
  uint32_t s = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) s += sh.red_a[w];
  __syncthreads();
  return s;
}

// Selects the k largest of the L keys of one row (L > k) and writes their positions to out[0..k).
// keys: this CTA's n keys (positions base .. base + n - 1; 16-byte aligned; n <= 4 * NT * kMaxChunks).
// hist: hist_words(C) words, cleared (see the protocol above).
template <int NT>
__device__ void select_topk(const uint32_t* keys, int n, int base, int k, int32_t* out, Shared<NT>& sh,
                            uint32_t* hist, uint32_t C, uint32_t rank) {
  constexpr int kChunk = 4 * NT;
  constexpr int kBPT = kBins / NT;  // summed bins each thread reads in a find step
  static_assert(kBins % NT == 0 && kBPT % 4 == 0 && kCandCap <= NT, "select_topk thread count");
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const uint32_t bpr = kBins / C;
  uint32_t* gh = hist + kBins;  // [3][bpr]
  const int nchunks = (n + kChunk - 1) / kChunk;

  auto load4 = [&](int c, uint32_t (&r)[4]) -> int {
    const int j0 = c * kChunk + 4 * tid;
    const int nv = max(0, min(4, n - j0));
    if (nv > 0) {
      const uint4 v = *reinterpret_cast<const uint4*>(keys + j0);
      r[0] = v.x, r[1] = v.y, r[2] = v.z, r[3] = v.w;
    } else {
      r[0] = r[1] = r[2] = r[3] = 0u;
    }
    return nv;
  };
  // this CTA's keys satisfying pred
  auto count_local = [&](auto pred) -> uint32_t {
    uint32_t c0 = 0;
    for (int c = 0; c < nchunks; ++c) {
      uint32_t r[4];
      const int nv = load4(c, r);
#pragma unroll
      for (int e = 0; e < 4; ++e) c0 += (e < nv && pred(r[e])) ? 1u : 0u;
    }
    return block_sum<NT>(c0, sh);
  };

  // ---- 1. the row's smallest and largest key ----
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int c = 0; c < nchunks; ++c) {
    uint32_t r[4];
    const int nv = load4(c, r);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (e < nv) kmin = min(kmin, r[e]), kmax = max(kmax, r[e]);
  }
  auto cluster_minmax = [&](uint32_t& mn, uint32_t& mx) {  // pushes, a barrier, a local reduction
    mn = __reduce_min_sync(0xffffffffu, mn);
    mx = __reduce_max_sync(0xffffffffu, mx);
    if (lane == 0) sh.red_a[wid] = mn, sh.red_b[wid] = mx;
    __syncthreads();
    if (wid == 0) {
      uint32_t a = lane < NT / 32 ? sh.red_a[lane] : 0xffffffffu, b = lane < NT / 32 ? sh.red_b[lane] : 0u;
      a = __reduce_min_sync(0xffffffffu, a);
      b = __reduce_max_sync(0xffffffffu, b);
      if (static_cast<uint32_t>(lane) < C) {
        st_cluster_u32(peer_addr(smem_u32(&sh.mm[rank][0]), lane), a);
        st_cluster_u32(peer_addr(smem_u32(&sh.mm[rank][1]), lane), b);
      }
    }
    cluster_barrier();
    mn = 0xffffffffu, mx = 0u;
    for (uint32_t q = 0; q < C; ++q) mn = min(mn, sh.mm[q][0]), mx = max(mx, sh.mm[q][1]);
  };
  cluster_wait();  // every peer has started and cleared its state
  cluster_minmax(kmin, kmax);

  uint32_t lo = kmin, wmax = kmax - kmin;
  uint32_t remaining = static_cast<uint32_t>(k);
  uint32_t theta = kmax;
  bool found = false, via_cands = false;
  int pass = 0;

  // local hist[bin(key)] += 1 for bin(key) < kBins: one shared-memory atomic per key, no warp-wide
  // steps (their latency per key costs more than the rare collisions of random bins)
  auto histogram = [&](auto bin_of) {
    for (int c = 0; c < nchunks; ++c) {
      uint32_t r[4];
      const int nv = load4(c, r);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t bin = e < nv ? bin_of(r[e]) : 0xffffffffu;
        if (bin < static_cast<uint32_t>(kBins)) atomicAdd(&hist[bin], 1u);
      }
    }
    __syncthreads();
  };
  // the row's histogram of nb bins from every CTA's local one; then the bin of the remaining-th
  // largest key, counted from the top: sh.lo = b, sh.remaining = remaining - keys in higher bins,
  // sh.ncand = keys in b. The local histogram is kept (the caller clears it).
  auto exchange_and_find = [&](uint32_t nb) {
    uint32_t* buf = gh + (pass % 3) * bpr;
    for (uint32_t b = tid; b < nb; b += NT) {
      const uint32_t c = hist[b];
      if (c) red_cluster_add_u32(peer_addr(smem_u32(buf + b % bpr), b / bpr), c);
    }
    cluster_barrier();
    uint32_t cnts[kBPT], sum = 0;
    const uint32_t d0 = static_cast<uint32_t>(kBPT * tid);  // descending index of this thread's first bin
    if (nb == static_cast<uint32_t>(kBins)) {  // kBPT consecutive bins of one owner, 16-byte aligned
#pragma unroll
      for (int q = 0; q < kBPT; q += 4) {
        const uint32_t b = nb - 4 - d0 - q;  // lowest of the four bins
        const uint4 v = ld_cluster_v4(peer_addr(smem_u32(buf + b % bpr), b / bpr));
        cnts[q] = v.w, cnts[q + 1] = v.z, cnts[q + 2] = v.y, cnts[q + 3] = v.x;
      }
    } else {
#pragma unroll
      for (int q = 0; q < kBPT; ++q) {
        const uint32_t d = d0 + q, b = nb - 1 - d;
        cnts[q] = d < nb ? ld_cluster_u32(peer_addr(smem_u32(buf + b % bpr), b / bpr)) : 0u;
      }
    }
#pragma unroll
    for (int q = 0; q < kBPT; ++q) sum += cnts[q];
    // this CTA's share of the buffer used two exchanges from now was last read one exchange ago
    uint32_t* next = gh + ((pass + 2) % 3) * bpr;
    for (uint32_t i = tid; i < bpr; i += NT) next[i] = 0u;
    ++pass;
    int total;
    const int incl = block_scan<NT>(static_cast<int>(sum), sh.scan_scratch, &total);
    uint32_t before = static_cast<uint32_t>(incl) - sum;
#pragma unroll
    for (int q = 0; q < kBPT; ++q) {
      if (before < remaining && remaining <= before + cnts[q]) {
        sh.lo = nb - 1 - (d0 + q);
        sh.remaining = remaining - before;
        sh.ncand = cnts[q];
      }
      before += cnts[q];
    }
    __syncthreads();
  };
  auto clear_local_hist = [&]() {
    for (int i = tid; i < kBins; i += NT) hist[i] = 0u;
    __syncthreads();
  };
  // The row's ncand (<= kCandCap) keys satisfying is_cand go to rank 0 with their ranks, and every
  // rank's count of keys satisfying is_above (the keys above the candidates) to every peer; then
  // every CTA finds theta = the largest candidate v with #(candidates >= v) >= remaining, leaves in
  // `remaining` the keys equal to theta that are taken, and in sh.rgt / sh.req every rank's
  // candidates above / equal to theta.
  auto resolve_candidates = [&](auto is_cand, uint32_t above_local, uint32_t ncand) {
    const uint32_t mine = count_local(is_cand);
    if (tid == 0) sh.slot = mine ? atom_cluster_add_u32(peer_addr(smem_u32(&sh.cand_count), 0), mine) : 0u;
    if (wid == 0 && static_cast<uint32_t>(lane) < C)
      st_cluster_u32(peer_addr(smem_u32(&sh.above[rank]), lane), above_local);
    if (tid == 0) sh.w0 = 0u;
    __syncthreads();
    const uint32_t key0 = peer_addr(smem_u32(sh.cand_key), 0), rank0 = peer_addr(smem_u32(sh.cand_rank), 0);
    if (mine) {
      for (int c = 0; c < nchunks; ++c) {
        uint32_t r[4];
        const int nv = load4(c, r);
        bool any = false;
#pragma unroll
        for (int e = 0; e < 4; ++e) any |= e < nv && is_cand(r[e]);
        if (!__any_sync(0xffffffffu, any)) continue;  // the common case: no candidate in this chunk
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool in = e < nv && is_cand(r[e]);
          const uint32_t act = __ballot_sync(0xffffffffu, in);
          if (act == 0u) continue;
          const int first = __ffs(act) - 1;
          uint32_t at = 0;
          if (lane == first) at = atomicAdd(&sh.w0, static_cast<uint32_t>(__popc(act)));
          at = __shfl_sync(0xffffffffu, at, first) + __popc(act & ((1u << lane) - 1u)) + sh.slot;
          if (in) {
            st_cluster_u32(key0 + 4u * at, r[e]);
            st_cluster_u32(rank0 + 4u * at, rank);
          }
        }
      }
    }
    cluster_barrier();
    if (static_cast<uint32_t>(tid) < ncand) {
      sh.lkey[tid] = ld_cluster_u32(key0 + 4u * tid);
      sh.lrank[tid] = ld_cluster_u32(rank0 + 4u * tid);
    }
    if (tid < kMaxCluster) sh.rgt[tid] = 0u, sh.req[tid] = 0u;
    __syncthreads();
    if (static_cast<uint32_t>(tid) >= ncand && tid < ((ncand + 3) & ~3u)) sh.lkey[tid] = 0u;  // padding
    __syncthreads();
    uint32_t best = 0u;
    bool have = false;
    if (static_cast<uint32_t>(tid) < ncand) {
      const uint32_t v = sh.lkey[tid];
      uint32_t ge = 0;
      for (uint32_t j = 0; j < ncand; j += 4) {  // 16-byte broadcast loads, four compares each
        const uint4 w = *reinterpret_cast<const uint4*>(&sh.lkey[j]);
        ge += (w.x >= v ? 1u : 0u) + (w.y >= v ? 1u : 0u) + (w.z >= v ? 1u : 0u) + (w.w >= v ? 1u : 0u);
      }
      if (v == 0u) ge -= ((ncand + 3) & ~3u) - ncand;  // the zero padding counted as >= 0
      if (ge >= remaining) best = v, have = true;
    }
    best = __reduce_max_sync(0xffffffffu, have ? best : 0u);
    if (lane == 0) sh.red_a[wid] = best;
    __syncthreads();
    theta = 0u;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) theta = max(theta, sh.red_a[w]);
    if (static_cast<uint32_t>(tid) < ncand) {
      const uint32_t v = sh.lkey[tid];
      if (v > theta) atomicAdd(&sh.rgt[sh.lrank[tid]], 1u);
      if (v == theta) atomicAdd(&sh.req[sh.lrank[tid]], 1u);
    }
    __syncthreads();
    uint32_t gt = 0;
    for (uint32_t q = 0; q < C; ++q) gt += sh.rgt[q];
    remaining -= gt;
  };

  // ---- 2. value-linear first pass ----
  uint32_t cand_lo = 0, cand_hi = 0;  // key range of the candidates once resolved in key space
  {
    const float fmin = key_value(kmin), fmax = key_value(kmax);
    const float range = fmax - fmin;
    const float vscale = static_cast<float>(kBins) / range;
    if (isfinite(fmin) && isfinite(fmax) && isfinite(range) && range > 0.f && isfinite(vscale)) {
      auto vbin = [&](uint32_t u) -> uint32_t {
        const int b = static_cast<int>((key_value(u) - fmin) * vscale);  // >= 0: key >= kmin
        return static_cast<uint32_t>(min(b, kBins - 1));
      };
      histogram(vbin);
      exchange_and_find(kBins);
      const uint32_t bstar = sh.lo, ncand = sh.ncand;
      remaining = sh.remaining;
      if (ncand <= static_cast<uint32_t>(kCandCap)) {
        uint32_t above = 0;  // this CTA's keys in bins above b*, from its local histogram
        for (int b = static_cast<int>(bstar) + 1 + tid; b < kBins; b += NT) above += hist[b];
        above = block_sum<NT>(above, sh);
        resolve_candidates([&](uint32_t u) { return vbin(u) == bstar; }, above, ncand);
        found = via_cands = true;
      } else {
        // the boundary bin is a contiguous key interval: its exact bounds, then key-space passes
        uint32_t bmin = 0xffffffffu, bmax = 0u;
        for (int c = 0; c < nchunks; ++c) {
          uint32_t r[4];
          const int nv = load4(c, r);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (e < nv && vbin(r[e]) == bstar) bmin = min(bmin, r[e]), bmax = max(bmax, r[e]);
        }
        clear_local_hist();
        cluster_minmax(bmin, bmax);
        lo = bmin;
        wmax = bmax - bmin;
        kmax = bmax;
        if (wmax == 0u) {
          theta = lo;
          found = true;
        }
      }
    }
  }

  // ---- 3. key-space narrowing of [lo, lo + wmax] down to the k-th largest key theta ----
  for (int it = 0; it < 4 && !found; ++it) {
    int sft = 0;
    while ((wmax >> sft) >= static_cast<uint32_t>(kBins)) ++sft;
    const uint32_t lo0 = lo, w0 = wmax;
    histogram([&](uint32_t u) -> uint32_t {
      const uint32_t d = u - lo0;
      return d <= w0 ? (d >> sft) : 0xffffffffu;
    });
    exchange_and_find((wmax >> sft) + 1u);
    clear_local_hist();
    lo = lo + (sh.lo << sft);
    remaining = sh.remaining;
    const uint32_t ncand = sh.ncand;
    wmax = min((1u << sft) - 1u, kmax - lo);
    if (sft == 0 || wmax == 0) {
      theta = lo;
      found = true;
      break;
    }
    if (ncand <= static_cast<uint32_t>(kCandCap)) {
      cand_lo = lo, cand_hi = lo + wmax;
      const uint32_t clo = cand_lo, chi = cand_hi;
      const uint32_t above = count_local([&](uint32_t u) { return u > chi; });
      resolve_candidates([&](uint32_t u) { return u >= clo && u <= chi; }, above, ncand);
      found = via_cands = true;
      break;
    }
  }
  // theta: the row's k-th largest key; remaining: how many keys equal to theta are taken

  // ---- 4. keys above / equal to theta before this CTA (every lower rank) ----
  uint32_t gt0 = 0, eq0 = 0;
  if (via_cands) {
    for (uint32_t q = 0; q < rank; ++q) gt0 += sh.above[q] + sh.rgt[q], eq0 += sh.req[q];
  } else {  // theta found without candidates: every rank's counts through one more exchange
    const uint32_t gl = count_local([&](uint32_t u) { return u > theta; });
    const uint32_t el = count_local([&](uint32_t u) { return u == theta; });
    if (wid == 0 && static_cast<uint32_t>(lane) < C) {
      st_cluster_u32(peer_addr(smem_u32(&sh.rc[rank][0]), lane), gl);
      st_cluster_u32(peer_addr(smem_u32(&sh.rc[rank][1]), lane), el);
    }
    cluster_barrier();
    for (uint32_t q = 0; q < rank; ++q) gt0 += sh.rc[q][0], eq0 += sh.rc[q][1];
  }
  // no remote access of this call remains: clear the state for the next call, release the peers
  __syncthreads();
  clear_state<NT>(sh, hist, C);
  cluster_arrive();

  // ---- 5. ordered emission of this CTA's share ----
  for (int c = 0; c < nchunks; ++c) {
    uint32_t r[4];
    const int nv = load4(c, r);
    int gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      gt += (e < nv && r[e] > theta) ? 1 : 0;
      eq += (e < nv && r[e] == theta) ? 1 : 0;
    }
    gt = __reduce_add_sync(0xffffffffu, gt);
    eq = __reduce_add_sync(0xffffffffu, eq);
    if (lane == 0) sh.cnt[c][wid] = make_int2(gt, eq);
  }
  __syncthreads();
  {  // exclusive prefix over (chunk, warp) in position order: one block scan, entry tid = (chunk, warp)
    static_assert(kMaxChunks * (NT / 32) <= NT, "one (chunk, warp) entry per thread");
    const int c = tid / (NT / 32), w = tid % (NT / 32);
    const int2 v = c < nchunks ? sh.cnt[c][w] : make_int2(0, 0);
    const int packed = (v.y << 16) | v.x;  // a CTA holds fewer than 65536 keys
    int total;
    const int incl = block_scan<NT>(packed, sh.scan_scratch, &total);
    const uint32_t ex = static_cast<uint32_t>(incl - packed);  // the two 16-bit halves, unsigned
    if (c < nchunks)
      sh.cnt[c][w] = make_int2(static_cast<int>(gt0 + (ex & 0xffffu)), static_cast<int>(eq0 + (ex >> 16)));
  }
  __syncthreads();
  const int ties = static_cast<int>(remaining);
  for (int c = 0; c < nchunks; ++c) {
    uint32_t r[4];
    const int nv = load4(c, r);
    int gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      gt += (e < nv && r[e] > theta) ? 1 : 0;
      eq += (e < nv && r[e] == theta) ? 1 : 0;
    }
    if (!__any_sync(0xffffffffu, gt + eq > 0)) continue;
    const int packed = (eq << 16) | gt;  // each <= 128 per warp and chunk
    int x = packed;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    x -= packed;
    const int2 cb = sh.cnt[c][wid];
    int gt_before = cb.x + (x & 0xffff);
    int eq_before = cb.y + (x >> 16);
    const int j0 = c * kChunk + 4 * tid;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (e >= nv) break;
      const uint32_t u = r[e];
      if (u > theta) {
        out[gt_before + min(eq_before, ties)] = base + j0 + e;
        ++gt_before;
      } else if (u == theta) {
        if (eq_before < ties) out[gt_before + eq_before] = base + j0 + e;
        ++eq_before;
      }
    }
  }
}

}  // namespace sel
}  // namespace dsa
