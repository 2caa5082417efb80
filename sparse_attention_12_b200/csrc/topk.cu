// Per-query TopK over the indexer scores:  S_t = TopK_{j<=t}(I_tj, k)
// ("DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section "Lightning Indexer", TopK
// formula; when the prefix holds no more than k positions all of them are taken, the handbook's
// k = min(L, TOPK) in "MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与 DSA").
//
// Two kernels share the steps below. Batches of many rows (prefill) run one CTA of 1024 threads
// per row. Batches of few rows (decode) would leave most SMs idle that way and pay one CTA's
// latency chain per row, so there one cluster of up to 8 CTAs takes each row (topk_cluster_kernel,
// further down). L = p + 1 visible scores.
//  1. Scores become order-preserving uint32 keys (one float4 per thread per chunk of 4096
//     positions, four chunks in flight); the row's smallest and largest key bound the search.
//  2. A 2048-bin histogram linear in the score value between the row's minimum and maximum
//     (floating-point subtraction and scaling are monotonic, so bins stay ordered) locates the bin
//     holding the k-th largest score; real score rows spread over many bins, so plain shared-memory
//     atomics rarely collide and the boundary bin holds a handful of keys. Rows this cannot split
//     (infinities, NaN, heavy ties, an overfull boundary bin) narrow further in key space: bins
//     (key - lo) >> s over the bin's exact key interval [lo, lo + W), s the smallest shift that
//     fits W into 2048 bins, until the boundary bin is small or a single key value.
//  3. Once that bin holds at most kCandCap keys, they are copied out and the k-th largest key
//     theta is found exactly by counting, for each candidate, the candidates at least as large.
//  4. Emission in increasing position order: every key above theta, then the first
//     `ties` keys equal to theta (equal scores: the smaller position wins), so the result is
//     deterministic. Per-(chunk, warp) counts and one warp-level scan give each warp its offsets.
// Keys always sit in shared memory (at most kSlice = 32768 of them per CTA). A row longer than
// kSlice is split into slices of kSlice positions, one CTA each, each selecting its own top k; a
// merge CTA per row then selects among the slices' winners (at most 8k candidates, their scores
// gathered from the row). This is exact: an element of the row's top k has fewer than k elements
// above it in its own slice too (same order: score, then position).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "dsa_internal.h"
#include "dsa_ptx.cuh"
#include "select_cluster.cuh"

namespace dsa {
namespace {

constexpr int kWarps = 32;            // warps of a 1024-thread CTA (the block scan's default)
constexpr int kBins = 2048;
constexpr int kSlice = 32768;         // most positions per CTA: their keys sit in shared memory (128 KB)
constexpr int kSliceMany = 16384;     // slice for batches of many rows (64 KB: three CTAs per SM)
constexpr int kCandCap = 128;         // candidates resolved by counting
constexpr int kLoadGroup = 4;         // chunks whose global loads are in flight together
constexpr int kMaxSlices = kMaxTopKRow / kSlice;  // rows up to 262144 positions: 8 slices of kSlice
static_assert(kMaxSlices * kMaxTopK <= kSlice, "a merge of kSlice-position slices fits one CTA");

__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;  // NaN ranks below every other score, -inf included
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;  // -0 ranks as +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t u) {  // inverse of order_key (-0 -> +0, NaN -> a NaN)
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// Block-wide inclusive scan of one value per thread over NW warps; `scratch` holds NW ints.
template <int NW = kWarps>
__device__ __forceinline__ int block_inclusive_scan(int v, int* scratch, int* total) {
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
    int s = lane < NW ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NW) scratch[lane] = s;
  }
  __syncthreads();
  const int r = x + (wid > 0 ? scratch[wid - 1] : 0);
  *total = scratch[NW - 1];
  __syncthreads();
  return r;
}

struct Keys4 {
  uint32_t k[4];
};

// kMerge = false (slice mode): CTA (t, s) of a T x nsl_max grid selects among positions
//   [s*kSlice, min(L, (s+1)*kSlice)) of row t. A row of one slice writes S_t itself; otherwise the
//   slice's k winners (increasing positions, -1 padded) go to block (t, s) of the candidate space,
//   and their keys to the same block of the key space that follows it.
// kMerge = true: CTA t selects among the candidates of row t (keys read from the key space), in
//   candidate order = increasing position; rows of one slice have nothing to do here.
// NT threads per CTA (1024 for batches of few rows: the shortest chain per row; 512 for batches of
// many rows, whose 16384-position slices then leave room for three CTAs per SM). `slice`: positions
// per slice CTA (kSlice or kSliceMany); a row of nsl slices has nsl * k <= kSlice candidates.
template <bool kMerge, int NT>
__global__ void __launch_bounds__(NT) topk_kernel(const int32_t* __restrict__ row_pos,
                                                  const float* __restrict__ scores, int64_t ld, int k,
                                                  int32_t* __restrict__ S, int32_t* __restrict__ cand_ws,
                                                  int nsl_max, int kpad, int slice) {
  constexpr int kThreads = NT;
  constexpr int kWarps = NT / 32;
  constexpr int kChunk = 4 * NT;                 // positions per chunk (one float4 per thread)
  constexpr int kMaxChunks = kSlice / kChunk;    // 8 (NT = 1024) or 16 (NT = 512) chunks per CTA
  constexpr int kBinsPerThread = kBins / NT;     // descending bins owned by one thread in the scan
  static_assert(kMaxChunks % kLoadGroup == 0 && kCandCap <= NT && kBins % NT == 0 && kWarps <= 32, "top-k CTA");
  extern __shared__ __align__(16) uint32_t tk_smem[];
  uint32_t* hist = tk_smem;                 // [kBins]
  uint32_t* cand = tk_smem + kBins;         // [kCandCap]
  uint32_t* cache = cand + kCandCap;        // [slice] keys of this CTA's positions
  __shared__ int scan_scratch[kWarps];
  __shared__ uint32_t red_min[kWarps], red_max[kWarps];
  __shared__ uint32_t sh_lo, sh_remaining, sh_ncand, sh_done;
  __shared__ int2 cnt[kMaxChunks][kWarps];  // per (chunk, warp): (above theta, equal to theta)

  const int t = kMerge ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x) / nsl_max;
  const int sl = kMerge ? 0 : static_cast<int>(blockIdx.x) % nsl_max;
  pdl_trigger();
  pdl_wait();  // scores, plan and candidates from the previous kernels
  const int L = __ldg(row_pos + t) + 1;
  const int nsl = (L + slice - 1) / slice;
  if (kMerge ? nsl <= 1 : sl >= nsl) return;
  const float* row = scores + static_cast<int64_t>(t) * ld;
  const int base = sl * slice;
  // the n elements this CTA selects from: positions base + i, or the candidates of row t
  const int n = kMerge ? (nsl - 1) * k + min(k, L - (nsl - 1) * slice) : min(slice, L - base);
  // candidate space: positions [T][nsl_max][kpad], then their keys in the same layout
  const int64_t key_off = static_cast<int64_t>(gridDim.x / (kMerge ? 1 : nsl_max)) * nsl_max * kpad;
  const int32_t* cands = cand_ws + static_cast<int64_t>(t) * nsl_max * kpad;
  const uint32_t* cand_keys = reinterpret_cast<const uint32_t*>(cands + key_off);
  // candidate i of the merge sits at slice i / k, entry i % k (rows of kpad entries; kpad == k for
  // k a multiple of 4, where the index is i itself)
  const bool packed = kpad == k;
  auto cand_at = [&](int i) -> int { return packed ? i : (i / k) * kpad + i % k; };
  auto position = [&](int i) -> int { return kMerge ? __ldg(cands + cand_at(i)) : base + i; };
  const bool to_cands = !kMerge && nsl > 1;
  int32_t* out = to_cands ? cand_ws + (static_cast<int64_t>(t) * nsl_max + sl) * kpad : S + static_cast<int64_t>(t) * k;
  uint32_t* out_key = to_cands ? reinterpret_cast<uint32_t*>(out + key_off) : nullptr;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;

  if (n <= k) {
    for (int j = tid; j < k; j += kThreads) {
      out[j] = (j < n) ? position(j) : -1;
      if (out_key) out_key[j] = (j < n) ? order_key(__ldg(row + base + j)) : 0u;
    }
    return;
  }
  const int nchunks = (n + kChunk - 1) / kChunk;

  // keys of this thread in chunks cg .. cg + G - 1 from shared memory; elements >= n report nv = 0
  constexpr int G = 1;
  auto load_group = [&](int cg, Keys4 (&r)[G], int (&nv)[G]) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int j0 = (cg + g) * kChunk + 4 * tid;
      nv[g] = max(0, min(4, n - j0));
      if (nv[g] > 0) {
        const uint4 v = *reinterpret_cast<const uint4*>(cache + j0);
        r[g].k[0] = v.x, r[g].k[1] = v.y, r[g].k[2] = v.z, r[g].k[3] = v.w;
      } else {
        r[g].k[0] = r[g].k[1] = r[g].k[2] = r[g].k[3] = 0u;
      }
    }
  };

  // ---- 1. keys, row minimum and maximum ----
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int cg = 0; cg < nchunks; cg += kLoadGroup) {
    float4 f[kLoadGroup];
    int nv[kLoadGroup];
#pragma unroll
    for (int g = 0; g < kLoadGroup; ++g) {
      const int j0 = (cg + g) * kChunk + 4 * tid;
      nv[g] = max(0, min(4, n - j0));
      if (nv[g] > 0) {
        if (kMerge) {  // the candidates' keys, as the slice CTAs wrote them
          float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (e < nv[g]) v[e] = key_value(__ldg(cand_keys + cand_at(j0 + e)));
          f[g] = make_float4(v[0], v[1], v[2], v[3]);
        } else {  // base + j0 + 3 < ld: base and j0 are multiples of 4, ld % 4 == 0, base + j0 < L <= ld
          f[g] = __ldg(reinterpret_cast<const float4*>(row + base + j0));
        }
      }
    }
#pragma unroll
    for (int g = 0; g < kLoadGroup; ++g) {
      if (nv[g] == 0) continue;
      const uint32_t u[4] = {order_key(f[g].x), order_key(f[g].y), order_key(f[g].z), order_key(f[g].w)};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (e < nv[g]) kmin = min(kmin, u[e]), kmax = max(kmax, u[e]);
      *reinterpret_cast<uint4*>(cache + (cg + g) * kChunk + 4 * tid) = make_uint4(u[0], u[1], u[2], u[3]);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) red_min[wid] = kmin, red_max[wid] = kmax;
  for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
  __syncthreads();
  kmin = __reduce_min_sync(0xffffffffu, lane < kWarps ? red_min[lane] : 0xffffffffu);
  kmax = __reduce_max_sync(0xffffffffu, lane < kWarps ? red_max[lane] : 0u);

  uint32_t lo = kmin, wmax = kmax - kmin;  // key-space range [lo, lo + wmax]
  uint32_t remaining = static_cast<uint32_t>(k);
  uint32_t theta = kmax;
  bool found = false;

  // theta = the largest candidate value v with #(candidates >= v) >= remaining; on return
  // `remaining` counts the keys equal to theta that are taken. cand[0 .. ncand) holds the keys.
  auto resolve_candidates = [&](uint32_t ncand) {
    if (static_cast<uint32_t>(tid) >= ncand && tid < ((ncand + 3) & ~3u)) cand[tid] = 0u;  // padding
    __syncthreads();
    uint32_t best = 0u;
    bool have = false;
    if (static_cast<uint32_t>(tid) < ncand) {
      const uint32_t v = cand[tid];
      uint32_t ge = 0;
      for (uint32_t j = 0; j < ncand; j += 4) {  // 16-byte broadcast loads, four compares each
        const uint4 w = *reinterpret_cast<const uint4*>(&cand[j]);
        ge += (w.x >= v ? 1u : 0u) + (w.y >= v ? 1u : 0u) + (w.z >= v ? 1u : 0u) + (w.w >= v ? 1u : 0u);
      }
      if (v == 0u) ge -= ((ncand + 3) & ~3u) - ncand;  // the zero padding counted as >= 0
      if (ge >= remaining) best = v, have = true;
    }
    best = __reduce_max_sync(0xffffffffu, have ? best : 0u);
    if (lane == 0) red_max[wid] = best;
    __syncthreads();
    theta = __reduce_max_sync(0xffffffffu, lane < kWarps ? red_max[lane] : 0u);
    const uint32_t v = (static_cast<uint32_t>(tid) < ncand) ? cand[tid] : 0u;
    const int gt = __syncthreads_count(static_cast<uint32_t>(tid) < ncand && v > theta);
    remaining -= static_cast<uint32_t>(gt);
  };
  // copies the keys satisfying `pred` into cand (their number is known to be <= kCandCap)
  auto compact = [&](auto pred) {
    for (int cg = 0; cg < nchunks; cg += G) {
      Keys4 r[G];
      int nv[G];
      load_group(cg, r, nv);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        bool any = false;
#pragma unroll
        for (int e = 0; e < 4; ++e) any |= e < nv[g] && pred(r[g].k[e]);
        if (!__any_sync(0xffffffffu, any)) continue;  // the common case: no candidate in this chunk
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool in = e < nv[g] && pred(r[g].k[e]);
          const uint32_t act = __ballot_sync(0xffffffffu, in);
          if (act == 0u) continue;
          const int first = __ffs(act) - 1;
          uint32_t base = 0;
          if (lane == first) base = atomicAdd(&sh_done, static_cast<uint32_t>(__popc(act)));
          base = __shfl_sync(0xffffffffu, base, first);
          if (in) cand[base + __popc(act & ((1u << lane) - 1u))] = r[g].k[e];
        }
      }
    }
    __syncthreads();
  };
  // hist[bin(key)] += 1 over the keys with bin(key) < kBins: one shared-memory atomic per key, no
  // warp-wide steps (their latency per key costs more than the rare collisions of random bins)
  auto histogram = [&](auto bin_of) {
    for (int cg = 0; cg < nchunks; cg += G) {
      Keys4 r[G];
      int nv[G];
      load_group(cg, r, nv);
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t bin = e < nv[g] ? bin_of(r[g].k[e]) : 0xffffffffu;
          if (bin < static_cast<uint32_t>(kBins)) atomicAdd(&hist[bin], 1u);
        }
      }
    }
    __syncthreads();
  };
  // the bin b (of nb, counted from the top) holding the remaining-th largest key:
  // sh_bin = b, sh_remaining = remaining - (keys in higher bins), sh_ncand = keys in b
  auto find_bin = [&](uint32_t nb) {
    // thread i owns descending bins kBinsPerThread*i .. +kBinsPerThread-1 (counted from the top)
    uint32_t cnts[kBinsPerThread], sum = 0;
#pragma unroll
    for (int q = 0; q < kBinsPerThread; ++q) {
      const uint32_t d = static_cast<uint32_t>(kBinsPerThread * tid + q);
      cnts[q] = d < nb ? hist[nb - 1 - d] : 0u;
      sum += cnts[q];
    }
    int total;
    const int incl = block_inclusive_scan<kWarps>(static_cast<int>(sum), scan_scratch, &total);
    uint32_t before = static_cast<uint32_t>(incl) - sum;
#pragma unroll
    for (int q = 0; q < kBinsPerThread; ++q) {
      if (before < remaining && remaining <= before + cnts[q]) {
        sh_lo = nb - 1 - static_cast<uint32_t>(kBinsPerThread * tid + q);
        sh_remaining = remaining - before;
        sh_ncand = cnts[q];
      }
      before += cnts[q];
    }
    if (tid == 0) sh_done = 0u;
    __syncthreads();
  };

  // ---- 2. value-linear first pass ----
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
      find_bin(kBins);
      const uint32_t bstar = sh_lo, ncand = sh_ncand;
      remaining = sh_remaining;
      if (ncand <= static_cast<uint32_t>(kCandCap)) {
        compact([&](uint32_t u) { return vbin(u) == bstar; });
        resolve_candidates(ncand);
        found = true;
      } else {
        // the boundary bin is a contiguous key interval: narrow it in key space
        uint32_t bmin = 0xffffffffu, bmax = 0u;
        for (int cg = 0; cg < nchunks; cg += G) {
          Keys4 r[G];
          int nv[G];
          load_group(cg, r, nv);
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (e < nv[g] && vbin(r[g].k[e]) == bstar) bmin = min(bmin, r[g].k[e]), bmax = max(bmax, r[g].k[e]);
        }
        bmin = __reduce_min_sync(0xffffffffu, bmin);
        bmax = __reduce_max_sync(0xffffffffu, bmax);
        if (lane == 0) red_min[wid] = bmin, red_max[wid] = bmax;
        for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
        __syncthreads();
        lo = __reduce_min_sync(0xffffffffu, lane < kWarps ? red_min[lane] : 0xffffffffu);
        wmax = __reduce_max_sync(0xffffffffu, lane < kWarps ? red_max[lane] : 0u) - lo;
        kmax = lo + wmax;
        __syncthreads();  // red_min / red_max are reused below
        if (wmax == 0u) {
          theta = lo;
          found = true;
        }
      }
    }
  }

  // ---- 3. key-space narrowing of [lo, lo + wmax] down to the k-th largest key theta ----
  for (int pass = 0; pass < 4 && !found; ++pass) {
    int s = 0;
    while ((wmax >> s) >= static_cast<uint32_t>(kBins)) ++s;
    histogram([&](uint32_t u) -> uint32_t {
      const uint32_t d = u - lo;
      return d <= wmax ? (d >> s) : 0xffffffffu;
    });
    find_bin((wmax >> s) + 1u);
    lo = lo + (sh_lo << s);
    remaining = sh_remaining;
    const uint32_t ncand = sh_ncand;
    // the new range is bin b* of this pass, clipped to the largest key
    wmax = min((1u << s) - 1u, kmax - lo);
    if (s == 0 || wmax == 0) {  // one key value left: theta found
      theta = lo;
      found = true;
      break;
    }
    if (ncand <= static_cast<uint32_t>(kCandCap)) {
      const uint32_t clo = lo, cw = wmax;
      compact([&](uint32_t u) { return (u - clo) <= cw; });
      resolve_candidates(ncand);
      found = true;
      break;
    }
    for (int i = tid; i < kBins; i += kThreads) hist[i] = 0u;
    __syncthreads();
  }
  // theta: the k-th largest key; remaining: how many keys equal to theta are taken

  // ---- 4. ordered emission ----
  for (int cg = 0; cg < nchunks; cg += G) {
    Keys4 r[G];
    int nv[G];
    load_group(cg, r, nv);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      int gt = 0, eq = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        gt += (e < nv[g] && r[g].k[e] > theta) ? 1 : 0;
        eq += (e < nv[g] && r[g].k[e] == theta) ? 1 : 0;
      }
      gt = __reduce_add_sync(0xffffffffu, gt);
      eq = __reduce_add_sync(0xffffffffu, eq);
      if (lane == 0 && cg + g < nchunks) cnt[cg + g][wid] = make_int2(gt, eq);
    }
  }
  __syncthreads();
  {  // exclusive prefix over (chunk, warp) in position order: one block scan, entry tid = (chunk, warp)
    static_assert(kMaxChunks * kWarps <= kThreads, "one (chunk, warp) entry per thread");
    const int c = tid / kWarps, w = tid % kWarps;
    const int2 v = c < nchunks ? cnt[c][w] : make_int2(0, 0);
    const int packed = (v.y << 16) | v.x;  // a CTA holds fewer than 65536 keys
    int total;
    const int incl = block_inclusive_scan<kWarps>(packed, scan_scratch, &total);
    const uint32_t ex = static_cast<uint32_t>(incl - packed);  // the two 16-bit halves, unsigned
    if (c < nchunks) cnt[c][w] = make_int2(static_cast<int>(ex & 0xffffu), static_cast<int>(ex >> 16));
  }
  __syncthreads();
  const int ties = static_cast<int>(remaining);
  for (int cg = 0; cg < nchunks; cg += G) {
    Keys4 r[G];
    int nv[G];
    load_group(cg, r, nv);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int c = cg + g;
      int gt = 0, eq = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        gt += (e < nv[g] && r[g].k[e] > theta) ? 1 : 0;
        eq += (e < nv[g] && r[g].k[e] == theta) ? 1 : 0;
      }
      if (!__any_sync(0xffffffffu, gt + eq > 0)) continue;
      // exclusive prefix of (gt, eq) over the lanes below, packed into one word (each <= 128)
      const int packed = (eq << 16) | gt;
      int x = packed;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      x -= packed;
      const int2 base = cnt[c][wid];  // c < nchunks: a chunk past the row has no selected key
      int gt_before = base.x + (x & 0xffff);
      int eq_before = base.y + (x >> 16);
      const int j0 = c * kChunk + 4 * tid;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (e >= nv[g]) break;
        const uint32_t u = r[g].k[e];
        if (u > theta) {
          const int at = gt_before + min(eq_before, ties);
          out[at] = position(j0 + e);
          if (out_key) out_key[at] = u;
          ++gt_before;
        } else if (u == theta) {
          if (eq_before < ties) {
            out[gt_before + eq_before] = position(j0 + e);
            if (out_key) out_key[gt_before + eq_before] = u;
          }
          ++eq_before;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Cluster top-k for batches of few rows (decode): one cluster of C CTAs (C = 1, 2, 4 or 8) per row,
// so that one row's latency chain is spread over C SMs. CTA r loads the scores of positions
// [r*s, min(L, (r+1)*s)) into its shared memory as order-preserving keys, s = ceil(L/C) rounded up
// to a multiple of 4; the selection over the whole row then runs in sel::select_topk, which
// exchanges what it combines across the row through distributed shared memory.

constexpr int kCThreads = 512;
constexpr int kCChunk = 4 * kCThreads;             // positions per chunk (one float4 per thread)
constexpr int kCMaxSlice = 16384;                  // positions per CTA
constexpr int kCMaxCluster = sel::kMaxCluster;     // 8
constexpr int kCMaxRow = kCMaxSlice * kCMaxCluster;  // 131072
static_assert(kCMaxSlice <= kCChunk * sel::kMaxChunks && kBins == sel::kBins, "cluster top-k");

__global__ void __launch_bounds__(kCThreads) topk_cluster_kernel(const int32_t* __restrict__ row_pos,
                                                                 const float* __restrict__ scores, int64_t ld,
                                                                 int k, int32_t* __restrict__ S, int slice_cap) {
  extern __shared__ __align__(16) uint32_t tc_smem[];
  __shared__ sel::Shared<kCThreads> sh;
  const uint32_t C = cluster_nctarank(), rank = cluster_ctarank();
  uint32_t* cache = tc_smem;             // [slice_cap] keys of this CTA's positions
  uint32_t* hist = tc_smem + slice_cap;  // [sel::hist_words(C)]
  const int t = static_cast<int>(blockIdx.x / C);
  const int tid = threadIdx.x;

  sel::clear_state<kCThreads>(sh, hist, C);
  sel::cluster_arrive();  // waited for at the start of the selection (or before an early exit)
  pdl_trigger();
  pdl_wait();  // scores and plan from the previous kernels
  const int L = __ldg(row_pos + t) + 1;
  int32_t* out = S + static_cast<int64_t>(t) * k;
  if (L <= k) {  // every visible position, then padding (the same branch in every CTA of the row)
    const int per = (k + static_cast<int>(C) - 1) / static_cast<int>(C);
    const int j1 = min(k, static_cast<int>(rank + 1) * per);
    for (int j = static_cast<int>(rank) * per + tid; j < j1; j += kCThreads) out[j] = j < L ? j : -1;
    sel::cluster_wait();
    return;
  }
  const int s = ((L + static_cast<int>(C) - 1) / static_cast<int>(C) + 3) & ~3;
  const int base = static_cast<int>(rank) * s;
  const int n = max(0, min(L - base, s));
  const float* row = scores + static_cast<int64_t>(t) * ld + base;
  const int nchunks = (n + kCChunk - 1) / kCChunk;
  for (int cg = 0; cg < nchunks; cg += kLoadGroup) {
    float4 f[kLoadGroup];
    int nv[kLoadGroup];
#pragma unroll
    for (int g = 0; g < kLoadGroup; ++g) {
      const int j0 = (cg + g) * kCChunk + 4 * tid;
      nv[g] = max(0, min(4, n - j0));
      // base + j0 + 3 < ld: base and j0 are multiples of 4, ld % 4 == 0, base + j0 < L <= ld
      if (nv[g] > 0) f[g] = __ldg(reinterpret_cast<const float4*>(row + j0));
    }
#pragma unroll
    for (int g = 0; g < kLoadGroup; ++g) {
      if (nv[g] == 0) continue;
      *reinterpret_cast<uint4*>(cache + (cg + g) * kCChunk + 4 * tid) =
          make_uint4(sel::order_key(f[g].x), sel::order_key(f[g].y), sel::order_key(f[g].z), sel::order_key(f[g].w));
    }
  }
  __syncthreads();
  sel::select_topk<kCThreads>(cache, n, base, k, out, sh, hist, C, rank);
  sel::cluster_wait();  // no CTA leaves while a peer may still address its shared memory
}

}  // namespace

// Cluster size of the cluster kernel for this batch, or 0 for the single-CTA kernel. Measured on
// B200: for rows that fit one CTA (<= kSlice positions) the cluster's exchanges cost about what
// splitting the row saves, so one CTA per row it is; rows above kSlice need the single-CTA kernel's
// slices and a merge launch, which the cluster kernel avoids when all its clusters fit in one wave
// (two CTAs per SM).
int topk_cluster_size(int T, int max_seq_len) {
  constexpr int kOneWave = 2 * 148;
  if (max_seq_len <= kSlice || max_seq_len > kCMaxRow) return 0;
  int c = 1;
  while (c < kCMaxCluster && (max_seq_len + c - 1) / c > kCMaxSlice) c <<= 1;
  return (T * c <= kOneWave) ? c : 0;
}

// Slice size of the single-CTA kernel: 16384 positions (512-thread CTAs, three per SM) for batches
// of many rows, whose throughput is what counts, when the slices' winners still fit one merge CTA;
// else 32768 (1024-thread CTAs: the shortest chain per row).
namespace {
constexpr int kManyRows = 8 * 148;
int single_cta_slice(int T, int max_seq_len, int k) {
  const int nsl = (max_seq_len + kSliceMany - 1) / kSliceMany;
  return (T >= kManyRows && nsl * k <= kSlice) ? kSliceMany : kSlice;
}
}  // namespace

size_t topk_ws_bytes(int T, int max_seq_len, int k) {
  if (topk_cluster_size(T, max_seq_len) > 0) return 0;
  const int slice = single_cta_slice(T, max_seq_len, k);
  const int nsl = (max_seq_len + slice - 1) / slice;
  if (nsl <= 1) return 0;  // positions and keys of every slice's winners
  return 2 * sizeof(int32_t) * static_cast<size_t>(T) * static_cast<size_t>(nsl) * static_cast<size_t>((k + 3) & ~3);
}

namespace {
template <int NT>
int launch_topk_single(const BatchDev& b, const PlanView& pv, const float* scores, int64_t ld, int k, int32_t* S,
                       void* ws, int slice, void* stream) {
  const int nsl = (b.max_seq_len + slice - 1) / slice;
  const int kpad = (k + 3) & ~3;
  if (nsl > 1 && !ws) return static_cast<int>(cudaErrorInvalidValue);
  int32_t* cand_ws = static_cast<int32_t*>(ws);
  const int max_smem = static_cast<int>(sizeof(uint32_t) * (kBins + kCandCap + kSlice));
  for (auto kern : {topk_kernel<false, NT>, topk_kernel<true, NT>}) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  const int capA = std::min(slice, (b.max_seq_len + 3) & ~3);
  cudaError_t e = launch_pdl(topk_kernel<false, NT>, dim3(b.T * nsl), dim3(NT),
                             sizeof(uint32_t) * (kBins + kCandCap + static_cast<size_t>(capA)), stream, pv.row_pos,
                             scores, ld, k, S, cand_ws, nsl, kpad, slice);
  if (e != cudaSuccess || nsl == 1) return static_cast<int>(e);
  const int capB = std::min(kSlice, (nsl * k + 3) & ~3);
  e = launch_pdl(topk_kernel<true, NT>, dim3(b.T), dim3(NT),
                 sizeof(uint32_t) * (kBins + kCandCap + static_cast<size_t>(capB)), stream, pv.row_pos, scores, ld, k,
                 S, cand_ws, nsl, kpad, slice);
  return static_cast<int>(e);
}
}  // namespace

int launch_topk(const BatchDev& b, const void* plan, const float* scores, int64_t ld, int k, int32_t* S, void* ws,
                void* stream) {
  if (b.T == 0) return 0;
  if (b.max_seq_len > kMaxTopKRow) return static_cast<int>(cudaErrorInvalidValue);
  PlanView pv = plan_view(const_cast<void*>(plan), b.B, b.T);
  const int C = topk_cluster_size(b.T, b.max_seq_len);
  if (C > 0) {
    const int slice_cap = ((b.max_seq_len + C - 1) / C + 3) & ~3;
    const size_t smem = sizeof(uint32_t) * (static_cast<size_t>(slice_cap) + sel::hist_words(C));
    cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
    return static_cast<int>(launch_pdl_cluster(topk_cluster_kernel, dim3(b.T * C), dim3(kCThreads), smem, stream,
                                               static_cast<unsigned>(C), pv.row_pos, scores, ld, k, S, slice_cap));
  }
  const int slice = single_cta_slice(b.T, b.max_seq_len, k);
  return slice == kSliceMany ? launch_topk_single<512>(b, pv, scores, ld, k, S, ws, slice, stream)
                             : launch_topk_single<1024>(b, pv, scores, ld, k, S, ws, slice, stream);
}

}  // namespace dsa
