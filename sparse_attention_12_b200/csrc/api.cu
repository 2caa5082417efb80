// C ABI of the DSA hot path: host-side argument checks, workspace carving and launches.
// Every function validates before touching the GPU and never synchronises the host, except
// dsa_status_read, whose job is to read the device status word back.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "dsa_internal.h"

using namespace dsa;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool valid_nhI(int nhI) { return nhI == 16 || nhI == 32 || nhI == 64 || nhI == 128; }

// Checks shared by every call. Returns DSA_OK or the status to return.
dsa_status_t check_batch(const dsa_batch_t* b) {
  if (!b) return DSA_ERR_INVALID_ARG;
  if (b->num_requests < 0 || b->total_q < 0) return DSA_ERR_INVALID_ARG;
  if (b->total_q == 0) return DSA_OK;
  if (b->num_requests < 1 || b->max_q < 1 || b->max_seq_len < 1 || b->max_pages < 1 || b->num_pages < 1)
    return DSA_ERR_INVALID_ARG;
  if (b->max_q > b->total_q || b->max_q > b->max_seq_len) return DSA_ERR_INVALID_ARG;
  if (b->max_pages < (b->max_seq_len + DSA_PAGE_SIZE - 1) / DSA_PAGE_SIZE) return DSA_ERR_INVALID_ARG;
  if (!b->seq_lens || !b->cu_q || !b->block_table) return DSA_ERR_INVALID_ARG;
  if (b->num_pages > (1 << 25)) return DSA_ERR_UNSUPPORTED;  // page * 64 stays an int32 row index
  return DSA_OK;
}

BatchDev to_dev(const dsa_batch_t* b) {
  BatchDev d;
  d.B = b->num_requests;
  d.T = b->total_q;
  d.max_q = b->max_q;
  d.max_seq_len = b->max_seq_len;
  d.max_pages = b->max_pages;
  d.num_pages = b->num_pages;
  d.seq_lens = b->seq_lens;
  d.cu_q = b->cu_q;
  d.block_table = b->block_table;
  return d;
}

dsa_status_t from_cuda(int e) { return e == 0 ? DSA_OK : DSA_ERR_CUDA; }

// The sparse MLA step: keys on the MMA's M axis for a few heads, heads on it otherwise.
int launch_mla(const BatchDev& b, const void* plan, const void* q, int H, const void* kv_cache, const int32_t* S,
               int k, float softmax_scale, void* out, float* lse, void* ws, void* stream) {
  if (H <= kNarrowHeads)
    return launch_sparse_mla_narrow(b, plan, q, H, kv_cache, S, k, softmax_scale, out, lse, ws, stream);
  return launch_sparse_mla(b, plan, q, H, kv_cache, S, k, softmax_scale, out, lse, ws, stream);
}

size_t scores_ld(const dsa_batch_t* b) {
  return (static_cast<size_t>(b->max_seq_len) + 127) / 128 * 128;
}

}  // namespace

namespace dsa {

dsa_status_t check_layer_args(const dsa_batch_t* batch, const uint8_t* qI, const float* qI_scale, const float* wI,
                              int nhI, const uint8_t* kI_cache, const float* kI_scale, const void* q, int H,
                              const void* kv_cache, int k, float softmax_scale, const void* out) {
  dsa_status_t st = check_batch(batch);
  if (st != DSA_OK) return st;
  if (!valid_nhI(nhI)) return DSA_ERR_UNSUPPORTED;
  if (H < 1 || H > 128 || k < 1 || k > kMaxTopK) return DSA_ERR_UNSUPPORTED;
  if (batch->total_q == 0) return DSA_OK;
  if (!qI || !qI_scale || !wI || !kI_cache || !kI_scale || !q || !kv_cache || !out) return DSA_ERR_INVALID_ARG;
  if (!aligned16(qI) || !aligned16(kI_cache) || !aligned16(kI_scale) || !aligned16(q) || !aligned16(kv_cache) ||
      !aligned16(out))
    return DSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f)) return DSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(batch->total_q) * nhI > (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

}  // namespace dsa

extern "C" {

int dsa_abi_version(void) { return DSA_ABI_VERSION; }

const char* dsa_status_string(dsa_status_t s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported size";
    case DSA_ERR_WORKSPACE: return "workspace too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "a kernel wait timed out";
    case DSA_ERR_DEVICE_INDEX: return "a kernel met an out-of-range index";
    case DSA_ERR_DEVICE_VALUE: return "a kernel met a non-finite input value";
  }
  return "unknown status";
}

size_t dsa_plan_workspace_size(const dsa_batch_t* batch, int nhI) {
  if (check_batch(batch) != DSA_OK || !valid_nhI(nhI)) return 0;
  return plan_bytes(batch->num_requests, batch->total_q);
}

dsa_status_t dsa_plan(const dsa_batch_t* batch, int nhI, void* plan, size_t plan_bytes_given, void* stream) {
  dsa_status_t st = check_batch(batch);
  if (st != DSA_OK) return st;
  if (!valid_nhI(nhI)) return DSA_ERR_UNSUPPORTED;
  if (!plan || !aligned16(plan)) return DSA_ERR_INVALID_ARG;
  if (plan_bytes_given < plan_bytes(batch->num_requests, batch->total_q)) return DSA_ERR_WORKSPACE;
  return from_cuda(launch_plan(to_dev(batch), nhI, plan, stream));
}

dsa_status_t dsa_status_read(void* plan, void* stream) {
  if (!plan) return DSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, plan, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (word != 0 && cudaMemset(plan, 0, sizeof(word)) != cudaSuccess) return DSA_ERR_CUDA;
  if (word & kDevErrTimeout) return DSA_ERR_TIMEOUT;
  if (word & kDevErrIndex) return DSA_ERR_DEVICE_INDEX;
  if (word & kDevErrValue) return DSA_ERR_DEVICE_VALUE;
  return DSA_OK;
}

dsa_status_t dsa_index_scores(const dsa_batch_t* batch, const void* plan, const uint8_t* qI, const float* qI_scale,
                              const float* wI, int nhI, const uint8_t* kI_cache, const float* kI_scale,
                              float* scores, int64_t ld, void* stream) {
  dsa_status_t st = check_batch(batch);
  if (st != DSA_OK) return st;
  if (!valid_nhI(nhI)) return DSA_ERR_UNSUPPORTED;
  if (batch->total_q == 0) return DSA_OK;
  if (!plan || !qI || !qI_scale || !wI || !kI_cache || !kI_scale || !scores) return DSA_ERR_INVALID_ARG;
  if (!aligned16(plan) || !aligned16(qI) || !aligned16(kI_cache) || !aligned16(kI_scale) || !aligned16(scores))
    return DSA_ERR_INVALID_ARG;
  if (ld < batch->max_seq_len || ld % 4 != 0) return DSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(batch->total_q) * nhI > (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  return from_cuda(launch_index_scores(to_dev(batch), plan, qI, qI_scale, wI, nhI, kI_cache, kI_scale, scores, ld,
                                       stream));
}

int dsa_index_topk_supported(const dsa_batch_t* batch, int nhI, int k) {
  if (check_batch(batch) != DSA_OK || !valid_nhI(nhI) || k < 1 || k > kMaxTopK) return 0;
  if (batch->total_q == 0) return 1;
  return index_topk_cluster_size(batch->num_requests, batch->max_q, batch->max_seq_len, nhI) > 0 ? 1 : 0;
}

dsa_status_t dsa_index_topk(const dsa_batch_t* batch, const void* plan, const uint8_t* qI, const float* qI_scale,
                            const float* wI, int nhI, const uint8_t* kI_cache, const float* kI_scale, int k,
                            int32_t* S, void* stream) {
  dsa_status_t st = check_batch(batch);
  if (st != DSA_OK) return st;
  if (!valid_nhI(nhI) || k < 1 || k > kMaxTopK) return DSA_ERR_UNSUPPORTED;
  if (batch->total_q == 0) return DSA_OK;
  if (!plan || !qI || !qI_scale || !wI || !kI_cache || !kI_scale || !S) return DSA_ERR_INVALID_ARG;
  if (!aligned16(plan) || !aligned16(qI) || !aligned16(kI_cache) || !aligned16(kI_scale) || !aligned16(wI))
    return DSA_ERR_INVALID_ARG;
  if (!dsa_index_topk_supported(batch, nhI, k)) return DSA_ERR_UNSUPPORTED;
  return from_cuda(launch_index_topk(to_dev(batch), plan, qI, qI_scale, wI, nhI, kI_cache, kI_scale, k, S, stream));
}

size_t dsa_topk_workspace_size(const dsa_batch_t* batch, int k) {
  if (check_batch(batch) != DSA_OK || k < 1 || k > kMaxTopK || batch->max_seq_len > kMaxTopKRow) return 0;
  return topk_ws_bytes(batch->total_q, batch->max_seq_len, k);
}

dsa_status_t dsa_topk(const dsa_batch_t* batch, const void* plan, const float* scores, int64_t ld, int k,
                      int32_t* S, void* ws, size_t ws_bytes, void* stream) {
  dsa_status_t st = check_batch(batch);
  if (st != DSA_OK) return st;
  if (k < 1 || k > kMaxTopK) return DSA_ERR_UNSUPPORTED;
  if (batch->total_q == 0) return DSA_OK;
  if (batch->max_seq_len > kMaxTopKRow) return DSA_ERR_UNSUPPORTED;
  if (!plan || !scores || !S || !aligned16(plan) || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  if (ld < batch->max_seq_len || ld % 4 != 0) return DSA_ERR_INVALID_ARG;
  const size_t need = topk_ws_bytes(batch->total_q, batch->max_seq_len, k);
  if (need > 0 && (!ws || !aligned16(ws))) return DSA_ERR_INVALID_ARG;
  if (ws_bytes < need) return DSA_ERR_WORKSPACE;
  return from_cuda(launch_topk(to_dev(batch), plan, scores, ld, k, S, ws, stream));
}

size_t dsa_sparse_mla_workspace_size(const dsa_batch_t* batch, int H, int k) {
  if (check_batch(batch) != DSA_OK || H < 1 || H > 128 || k < 1 || k > kMaxTopK) return 0;
  return sparse_mla_ws_bytes(batch->total_q, H, k);
}

dsa_status_t dsa_sparse_mla(const dsa_batch_t* batch, const void* plan, const void* q, int H, const void* kv_cache,
                            const int32_t* S, int k, float softmax_scale, void* out, float* lse, void* ws,
                            size_t ws_bytes, void* stream) {
  dsa_status_t st = check_batch(batch);
  if (st != DSA_OK) return st;
  if (H < 1 || H > 128 || k < 1 || k > kMaxTopK) return DSA_ERR_UNSUPPORTED;
  if (batch->total_q == 0) return DSA_OK;
  if (!plan || !q || !kv_cache || !S || !out) return DSA_ERR_INVALID_ARG;
  if (!aligned16(plan) || !aligned16(q) || !aligned16(kv_cache) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || softmax_scale != softmax_scale) return DSA_ERR_INVALID_ARG;
  const size_t need = sparse_mla_ws_bytes(batch->total_q, H, k);
  if (need > 0 && (!ws || !aligned16(ws))) return DSA_ERR_INVALID_ARG;
  if (ws_bytes < need) return DSA_ERR_WORKSPACE;
  return from_cuda(launch_mla(to_dev(batch), plan, q, H, kv_cache, S, k, softmax_scale, out, lse, ws, stream));
}

dsa_status_t dsa_cache_write(const dsa_batch_t* batch, const void* plan, const float* k_new, const void* c_new,
                             uint8_t* kI_cache, float* kI_scale, void* kv_cache, void* stream) {
  dsa_status_t st = check_batch(batch);
  if (st != DSA_OK) return st;
  if (batch->total_q == 0) return DSA_OK;
  if (!plan || !k_new || !c_new || !kI_cache || !kI_scale || !kv_cache) return DSA_ERR_INVALID_ARG;
  if (!aligned16(plan) || !aligned16(k_new) || !aligned16(c_new) || !aligned16(kI_cache) || !aligned16(kI_scale) ||
      !aligned16(kv_cache))
    return DSA_ERR_INVALID_ARG;
  return from_cuda(launch_cache_write(to_dev(batch), plan, k_new, c_new, kI_cache, kI_scale, kv_cache, stream));
}

size_t dsa_masked_mha_workspace_size(const dsa_batch_t* batch, int H, int topk) {
  if (check_batch(batch) != DSA_OK || H < 1 || H > 128 || topk < 1 || topk > kMaxTopK ||
      batch->max_seq_len > kMaxMhaSeqLen)
    return 0;
  return masked_mha_ws_bytes(batch->total_q, batch->max_seq_len);
}

dsa_status_t dsa_masked_mha(const dsa_batch_t* batch, const void* plan, const void* q, const void* k, const void* v,
                            int H, const int32_t* S, int topk, float softmax_scale, void* out, float* lse, void* ws,
                            size_t ws_bytes, void* stream) {
  dsa_status_t st = check_batch(batch);
  if (st != DSA_OK) return st;
  if (H < 1 || H > 128 || topk < 1 || topk > kMaxTopK) return DSA_ERR_UNSUPPORTED;
  if (batch->total_q == 0) return DSA_OK;
  if (batch->max_seq_len > kMaxMhaSeqLen || batch->num_requests > 65535) return DSA_ERR_UNSUPPORTED;
  if (!plan || !q || !k || !v || !S || !out || !ws) return DSA_ERR_INVALID_ARG;
  if (!aligned16(plan) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(ws))
    return DSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || softmax_scale != softmax_scale) return DSA_ERR_INVALID_ARG;
  if (ws_bytes < masked_mha_ws_bytes(batch->total_q, batch->max_seq_len)) return DSA_ERR_WORKSPACE;
  return from_cuda(
      launch_masked_mha(to_dev(batch), plan, q, k, v, H, S, topk, softmax_scale, out, lse, ws, stream));
}

size_t dsa_layer_workspace_size(const dsa_batch_t* batch, int nhI, int H, int k) {
  if (check_batch(batch) != DSA_OK || !valid_nhI(nhI) || H < 1 || H > 128 || k < 1 || k > kMaxTopK) return 0;
  const size_t T = static_cast<size_t>(batch->total_q);
  size_t s = align256(plan_bytes(batch->num_requests, batch->total_q));
  s += align256(sizeof(float) * T * scores_ld(batch));
  s += align256(sizeof(int32_t) * T * static_cast<size_t>(k));
  // one scratch region: the top-k candidates, then (after top-k is done) the split partials
  s += align256(std::max(sparse_mla_ws_bytes(batch->total_q, H, k),
                         topk_ws_bytes(batch->total_q, batch->max_seq_len, k)));
  return s;
}

dsa_status_t dsa_layer(const dsa_batch_t* batch, const uint8_t* qI, const float* qI_scale, const float* wI, int nhI,
                       const uint8_t* kI_cache, const float* kI_scale, const void* q, int H, const void* kv_cache,
                       int k, float softmax_scale, void* out, float* lse, int32_t* S_out, void* ws, size_t ws_bytes,
                       void* stream) {
  const dsa_status_t st = check_layer_args(batch, qI, qI_scale, wI, nhI, kI_cache, kI_scale, q, H, kv_cache, k,
                                           softmax_scale, out);
  if (st != DSA_OK || batch->total_q == 0) return st;
  if (!ws || !aligned16(ws)) return DSA_ERR_INVALID_ARG;
  if (ws_bytes < dsa_layer_workspace_size(batch, nhI, H, k)) return DSA_ERR_WORKSPACE;

  const size_t T = static_cast<size_t>(batch->total_q);
  char* p = static_cast<char*>(ws);
  void* plan = p;
  p += align256(plan_bytes(batch->num_requests, batch->total_q));
  float* scores = reinterpret_cast<float*>(p);
  const int64_t ld = static_cast<int64_t>(scores_ld(batch));
  p += align256(sizeof(float) * T * static_cast<size_t>(ld));
  int32_t* S = reinterpret_cast<int32_t*>(p);
  p += align256(sizeof(int32_t) * T * static_cast<size_t>(k));
  void* mla_ws = p;  // also the top-k candidate space (the two are never live together)
  if (S_out) S = S_out;

  const BatchDev bd = to_dev(batch);
  int e = launch_plan(bd, nhI, plan, stream);
  if (!e) e = launch_index_scores(bd, plan, qI, qI_scale, wI, nhI, kI_cache, kI_scale, scores, ld, stream);
  if (!e) e = launch_topk(bd, plan, scores, ld, k, S, mla_ws, stream);
  if (!e) e = launch_mla(bd, plan, q, H, kv_cache, S, k, softmax_scale, out, lse, mla_ws, stream);
  return from_cuda(e);
}

}  // extern "C"
