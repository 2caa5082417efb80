// Internal layout shared by the kernels and the C-ABI layer (not part of the public ABI).
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/dsa.h"

#if defined(__CUDACC__)
#include <cuda_runtime.h>
#endif

#if defined(__CUDACC__)
#define DSA_HD __host__ __device__
#else
#define DSA_HD
#endif

namespace dsa {

constexpr int kPage = DSA_PAGE_SIZE;     // positions per page
constexpr int kDIdx = DSA_D_INDEX;       // indexer head width (bytes per FP8 key)
constexpr int kDLat = DSA_D_LATENT;      // latent width
constexpr int kDV = DSA_D_V;             // value width
constexpr int kIdxTileKeys = 128;        // keys per indexer MMA tile (2 pages)
constexpr int kIdxCols = 256;            // query-head columns per indexer group (MMA N <= 256)
constexpr int kMaxTopK = 4096;
constexpr int kMaxTopKRow = 262144;  // longest score row the top-k kernel takes

// Device status bits recorded by kernels (dsa_status_read maps them to dsa_status_t).
constexpr uint32_t kDevErrTimeout = 1u;
constexpr uint32_t kDevErrIndex = 2u;
constexpr uint32_t kDevErrValue = 4u;

// ---- plan workspace --------------------------------------------------------------------
// header (64 B) then int32 arrays, each starting on a 16-byte boundary:
//   row_req[T], row_pos[T]                      request and position of every query row
//   req_goff[B+1]                               first indexer group of each request
//   grp_row0[T], grp_nq[T], grp_req[T], grp_pos0[T], grp_tile0[T+1]
//                                               indexer groups (at most T of them) and the
//                                               exclusive prefix of their key tiles
struct PlanHeader {
  uint32_t status;      // device status word
  int32_t total_tiles;  // indexer work units
  int32_t num_groups;
  int32_t nhI;
  int32_t qpg;          // queries per indexer group = 256 / nhI
  int32_t T;
  int32_t B;
  int32_t pad[9];
};
static_assert(sizeof(PlanHeader) == 64, "plan header is 64 bytes");

struct PlanView {
  PlanHeader* hdr;
  int32_t* row_req;
  int32_t* row_pos;
  int32_t* req_goff;
  int32_t* grp_row0;
  int32_t* grp_nq;
  int32_t* grp_req;
  int32_t* grp_pos0;
  int32_t* grp_tile0;
};

DSA_HD inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

DSA_HD inline size_t plan_bytes(int B, int T) {
  size_t s = sizeof(PlanHeader);
  s += 2 * align16(sizeof(int32_t) * size_t(T));
  s += align16(sizeof(int32_t) * size_t(B + 1));
  s += 4 * align16(sizeof(int32_t) * size_t(T));
  s += align16(sizeof(int32_t) * size_t(T + 1));
  return s;
}

DSA_HD inline PlanView plan_view(void* base, int B, int T) {
  char* p = static_cast<char*>(base);
  PlanView v;
  v.hdr = reinterpret_cast<PlanHeader*>(p);
  p += sizeof(PlanHeader);
  auto take = [&](size_t n) {
    int32_t* r = reinterpret_cast<int32_t*>(p);
    p += align16(sizeof(int32_t) * n);
    return r;
  };
  v.row_req = take(T);
  v.row_pos = take(T);
  v.req_goff = take(B + 1);
  v.grp_row0 = take(T);
  v.grp_nq = take(T);
  v.grp_req = take(T);
  v.grp_pos0 = take(T);
  v.grp_tile0 = take(T + 1);
  return v;
}

// Every check dsa_layer makes before it launches, except those of the workspace (shared with
// dsa_layer_noalloc). DSA_OK also for an empty batch with valid sizes.
dsa_status_t check_layer_args(const dsa_batch_t* batch, const uint8_t* qI, const float* qI_scale, const float* wI,
                              int nhI, const uint8_t* kI_cache, const float* kI_scale, const void* q, int H,
                              const void* kv_cache, int k, float softmax_scale, const void* out);

// ---- launchers (defined in the .cu files; return cudaError_t as int) ---------------------
struct BatchDev {
  int B, T, max_q, max_seq_len, max_pages, num_pages;
  const int32_t* seq_lens;
  const int32_t* cu_q;
  const int32_t* block_table;
};

int launch_plan(const BatchDev& b, int nhI, void* plan, void* stream);
int launch_cache_write(const BatchDev& b, const void* plan, const float* k_new, const void* c_new, uint8_t* kI_cache,
                       float* kI_scale, void* kv_cache, void* stream);
int launch_index_scores(const BatchDev& b, const void* plan, const uint8_t* qI, const float* qI_scale,
                        const float* wI, int nhI, const uint8_t* kI_cache, const float* kI_scale, float* scores,
                        int64_t ld, void* stream);
int index_topk_cluster_size(int B, int max_q, int max_seq_len, int nhI);
int launch_index_topk(const BatchDev& b, const void* plan, const uint8_t* qI, const float* qI_scale, const float* wI,
                      int nhI, const uint8_t* kI_cache, const float* kI_scale, int k, int32_t* S, void* stream);
size_t topk_ws_bytes(int T, int max_seq_len, int k);
int launch_topk(const BatchDev& b, const void* plan, const float* scores, int64_t ld, int k, int32_t* S, void* ws,
                void* stream);
size_t sparse_mla_ws_bytes(int T, int H, int k);
int sparse_mla_splits(int T, int k);
int launch_sparse_mla(const BatchDev& b, const void* plan, const void* q, int H, const void* kv_cache,
                      const int32_t* S, int k, float softmax_scale, void* out, float* lse, void* ws, void* stream);
// Head counts up to kNarrowHeads run the keys-on-M kernel (sparse_mla_narrow.cu), with the same
// splits and workspace as launch_sparse_mla.
constexpr int kNarrowHeads = 16;
int launch_sparse_mla_narrow(const BatchDev& b, const void* plan, const void* q, int H, const void* kv_cache,
                             const int32_t* S, int k, float softmax_scale, void* out, float* lse, void* ws,
                             void* stream);
constexpr int kMaxMhaSeqLen = 65536;  // longest request the masked MHA mode takes
size_t masked_mha_ws_bytes(int T, int max_seq_len);
int launch_masked_mha(const BatchDev& b, const void* plan, const void* q, const void* k, const void* v, int H,
                      const int32_t* S, int topk, float softmax_scale, void* out, float* lse, void* ws, void* stream);

#if defined(__CUDACC__)
// Launches every kernel of the library with programmatic stream serialization: its CTAs may be
// scheduled while the previous kernel in the stream finishes (once all of that kernel's CTAs have
// started), run their set-up, and wait in griddepcontrol.wait before touching memory an earlier
// kernel writes or reads. Each kernel calls pdl_wait() before its first such access.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, void* stream,
                              Args&&... args) {
  // one shared-memory carveout (the largest) for every kernel of the path: consecutive kernels
  // then need no L1/shared-memory reconfiguration of the SMs between them
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       static_cast<int>(cudaSharedmemCarveoutMaxShared));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// The same, with thread-block clusters of `cluster_x` CTAs along x (grid.x a multiple of it).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, void* stream,
                                      unsigned cluster_x, Args&&... args) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       static_cast<int>(cudaSharedmemCarveoutMaxShared));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
#endif

}  // namespace dsa
