/*
 * dsa.h — C ABI of the B200 (sm_100a) DeepSeek Sparse Attention hot path.
 *
 * The path has three steps, each defined on the pages this library follows:
 *
 *   1. Lightning-Indexer scores. "DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section
 *      "Lightning Indexer：为历史位置打分并选出 top-k", formula for I_tj:
 *          I_tj = sum_r w_tr * ReLU(q_tr . k_j)   for every visible position j <= t,
 *      with one shared key k_j per position. The page "MTP 与稀疏注意力：NSA 与 DSA", section
 *      "稀疏注意力：NSA 与 DSA", fixes 64 heads of width 128 computed in FP8 and a key cache of
 *      128 FP8 bytes plus a 4-byte scale per token. Here q_tr = s^q_t * e4m3(qI[t][r]) and
 *      k_j = s^k_j * e4m3(kI[j]) (per-token fp32 scales).
 *   2. TopK. Same section: S_t = TopK_{j<=t}(I_tj, k); k = 2048 on the pages; when the prefix holds
 *      no more than k positions every position is taken (the handbook's k = min(L, TOPK)).
 *   3. Sparse MLA. Same page, section "Sparse Attention：在选中位置上计算 Attention": attention on the
 *      rows in S_t only, equivalent to softmax(QK^T/sqrt(d_h) + M) V with M = 0 on S_t and -inf
 *      elsewhere; S_t is shared by all heads. The handbook computes it in the absorbed MLA form:
 *      a 576-wide bf16 latent row c_j per position (512 + 64 rope) shared by all 128 heads, with
 *      V = c_j[0:512].
 *
 * Conventions for every entry point:
 *   - Positions are 0-based. Request b has n_b cached positions (its own query tokens included)
 *     and m_b query tokens; query i of request b sits at position p = n_b - m_b + i and sees
 *     j in [0, p].
 *   - All data pointers are DEVICE pointers owned by the caller; the library allocates no memory
 *     and keeps no global state (thread-safe), except dsa_layer_noalloc's static device array.
 *     Workspace is caller-provided, sized by the *_workspace_size functions.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *     default stream). Nothing synchronises the host.
 *   - Arguments are checked on the host before anything is launched; a bad argument returns
 *     DSA_ERR_INVALID_ARG (or DSA_ERR_UNSUPPORTED for a valid but unsupported size) and launches
 *     nothing. A failed launch returns DSA_ERR_CUDA. Errors found by a kernel at run time (a wait
 *     that gave up, an index out of range) are recorded in the status word of the plan and read
 *     back with dsa_status_read.
 *   - Tensors are dense and row-major in the shapes given; the paged caches use pages of
 *     DSA_PAGE_SIZE positions; page ids come from block_table.
 *   - Pointers must be 16-byte aligned.
 */
#ifndef DSA_B200_H_
#define DSA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_ABI_VERSION 4
#define DSA_PAGE_SIZE 64   /* positions per cache page */
#define DSA_D_INDEX 128    /* indexer head width d_h^I */
#define DSA_D_LATENT 576   /* latent width: 512 + 64 rope */
#define DSA_D_V 512        /* value width: first 512 latent dims */
#define DSA_D_QK_MHA 192   /* masked MHA mode: expanded q/k head width, 128 + 64 rope */
#define DSA_D_V_MHA 128    /* masked MHA mode: expanded v head width */

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer, small workspace */
  DSA_ERR_UNSUPPORTED = 2,  /* a size outside what the kernels are built for */
  DSA_ERR_WORKSPACE = 3,    /* workspace smaller than *_workspace_size */
  DSA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  DSA_ERR_TIMEOUT = 5,      /* a kernel wait gave up (read back by dsa_status_read) */
  DSA_ERR_DEVICE_INDEX = 6, /* a kernel met an index outside its buffers (dsa_status_read) */
  DSA_ERR_DEVICE_VALUE = 7  /* a kernel met a non-finite input value (dsa_status_read) */
} dsa_status_t;

/* A ragged batch of requests. Shared by every call. */
typedef struct dsa_batch {
  int32_t num_requests;      /* B >= 0 */
  int32_t total_q;           /* T = sum_b m_b, host copy of cu_q[B] */
  int32_t max_q;             /* max_b m_b (host), >= 1 when T > 0 */
  int32_t max_seq_len;       /* max_b n_b (host) */
  int32_t max_pages;         /* columns of block_table, >= ceil(max_seq_len / 64) */
  int32_t num_pages;         /* pages in the pool: rows of both paged caches */
  const int32_t* seq_lens;   /* device int32 [B]: n_b, 1 <= n_b <= max_seq_len, n_b >= m_b */
  const int32_t* cu_q;       /* device int32 [B+1]: query-row offsets, cu_q[0] = 0 */
  const int32_t* block_table;/* device int32 [B, max_pages]: physical page of logical page i */
} dsa_batch_t;

/* ---- batch plan --------------------------------------------------------------------------
 * Per-batch metadata shared by the steps (row -> request/position, indexer work list, status
 * word). Compute it once per batch; it stays valid while seq_lens/cu_q do not change.
 * nhI: indexer heads the plan is made for (16, 32, 64 or 128). */
size_t dsa_plan_workspace_size(const dsa_batch_t* batch, int nhI);
dsa_status_t dsa_plan(const dsa_batch_t* batch, int nhI, void* plan, size_t plan_bytes, void* stream);

/* Synchronises `stream`, then returns the status word the kernels of the last calls that used
 * `plan` recorded (DSA_OK, DSA_ERR_TIMEOUT, DSA_ERR_DEVICE_INDEX or DSA_ERR_DEVICE_VALUE; the first of
 * these when several were recorded) and clears it. */
dsa_status_t dsa_status_read(void* plan, void* stream);

/* ---- writing new positions into the caches (the step before step 1) ----------------------
 * Every query row t (request b, position p) is a new token; its indexer key and its latent row are
 * stored at slot p % 64 of page block_table[b][p / 64] of the two caches:
 *   kI_scale[page][slot]    = s = max_d |k_new[t][d]| / 448 (fp32; 1 when the key is all zeros)
 *   kI_cache[page][slot][d] = e4m3(k_new[t][d] / s)   division in fp32; OCP E4M3, nearest with
 *                                                      ties to even, saturating at +-448
 *   kv_cache[page][slot][:] = c_new[t][:]            576 bf16, copied
 * ("MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与 DSA": per token the latent vector and the
 * indexer key as FP8 + a 4-byte scale, both paged; "DeepSeek Sparse Attention：从 SWA 到稀疏
 * Attention 计算", Lightning Indexer section: one shared indexer key per position in its own key
 * cache.) The plan must be made for this batch (dsa_plan).
 * k_new f32 [T, 128], c_new bf16 [T, 576]; caches as for dsa_index_scores / dsa_sparse_mla.
 * A page id outside [0, num_pages) is recorded as DSA_ERR_DEVICE_INDEX (dsa_status_read) and its
 * row is skipped. A key with an infinite or NaN element has no FP8 encoding (it would store e4m3 NaN
 * codes): it is recorded as DSA_ERR_DEVICE_VALUE and its row is skipped (neither cache is written
 * there). The latent row is copied as given. */
dsa_status_t dsa_cache_write(const dsa_batch_t* batch, const void* plan, const float* k_new, const void* c_new,
                             uint8_t* kI_cache, float* kI_scale, void* kv_cache, void* stream);

/* ---- step 1: indexer scores -------------------------------------------------------------
 * qI       e4m3 [T, nhI, 128]   indexer queries (FP8 codes)
 * qI_scale f32  [T]             s^q_t
 * wI       f32  [T, nhI]        head weights w_t
 * kI_cache e4m3 [P, 64, 128]    indexer keys, paged (FP8 codes)
 * kI_scale f32  [P, 64]         s^k per cached position
 * scores   f32  [T, ld]         out: I_tj for j <= p; -inf for p < j < min(ld, 128*ceil((p+1)/128));
 *                               other entries untouched. ld >= max_seq_len, ld % 4 == 0.
 * Runs as an FP8 tcgen05 GEMM (keys x query-heads) with ReLU, w and the head sum in the epilogue.
 * The caches must hold no e4m3 NaN codes (0x7F, 0xFF; dsa_cache_write never writes them): scores
 * computed from them are undefined. */
dsa_status_t dsa_index_scores(const dsa_batch_t* batch, const void* plan, const uint8_t* qI,
                              const float* qI_scale, const float* wI, int nhI, const uint8_t* kI_cache,
                              const float* kI_scale, float* scores, int64_t ld, void* stream);

/* ---- step 2: top-k ----------------------------------------------------------------------
 * scores f32 [T, ld] as written by dsa_index_scores (row t read at j <= p only); ld % 4 == 0,
 *        ld >= max_seq_len. max_seq_len <= 262144 (else DSA_ERR_UNSUPPORTED).
 * S      int32 [T, k] out: the min(k, p+1) positions with the largest scores, followed by -1.
 *        Among equal scores the smaller position wins; -0 equals +0; a NaN score ranks below every
 *        other score (-inf included). Selected positions are listed in increasing position order.
 *        1 <= k <= 4096.
 * ws/ws_bytes: dsa_topk_workspace_size bytes (0 when max_seq_len <= 32768): rows longer than 32768
 *        positions select per slice of 32768 first, then among the slices' winners. */
size_t dsa_topk_workspace_size(const dsa_batch_t* batch, int k);
dsa_status_t dsa_topk(const dsa_batch_t* batch, const void* plan, const float* scores, int64_t ld, int k,
                      int32_t* S, void* ws, size_t ws_bytes, void* stream);

/* ---- steps 1 and 2 fused, for decode batches ---------------------------------------------
 * The score rows never reach memory: one cluster of CTAs per request scores its keys into shared
 * memory (the indexer's FP8 tcgen05 GEMM and epilogue) and selects there, the CTAs exchanging
 * histograms, candidates and counts through distributed shared memory. ("MTP 与稀疏注意力：NSA 与
 * DSA", section "对推理引擎的新要求": FP8 scoring and a per-query top-k over tens of thousands of
 * positions are the kernels DSA asks of an engine; "DeepSeek Sparse Attention：从 SWA 到稀疏
 * Attention 计算", Lightning Indexer section, formulas for I_tj and S_t.)
 * Arguments as for dsa_index_scores and dsa_topk; S int32 [T, k] receives what dsa_topk writes for
 * the scores dsa_index_scores computes (the same fp32 arithmetic: the same sets). The plan must be
 * made for this batch (its status word records run-time faults). No workspace.
 * Supported when every request's queries fit one indexer MMA group (max_q <= 256 / nhI) and a
 * request's scores fit the shared memory of at most 8 CTAs (max_seq_len <= 131072 for one query
 * per request, less for more); dsa_index_topk_supported returns 1 then (and for an empty batch),
 * else 0, and dsa_index_topk returns DSA_ERR_UNSUPPORTED without launching. */
int dsa_index_topk_supported(const dsa_batch_t* batch, int nhI, int k);
dsa_status_t dsa_index_topk(const dsa_batch_t* batch, const void* plan, const uint8_t* qI, const float* qI_scale,
                            const float* wI, int nhI, const uint8_t* kI_cache, const float* kI_scale, int k,
                            int32_t* S, void* stream);

/* ---- step 3: sparse MLA -----------------------------------------------------------------
 * q        bf16 [T, H, 576]     absorbed MLA queries, 1 <= H <= 128
 * kv_cache bf16 [P, 64, 576]    latent rows, paged
 * S        int32 [T, k]         positions per query row (as dsa_topk writes them: the first
 *                               min(k, p+1) entries are read, negative entries are skipped)
 * out      bf16 [T, H, 512]     softmax(scale * q . c_j) weighted sum of c_j[0:512] over S_t
 * lse      f32  [T, H] or NULL  natural-log sum of exp(scale * q . c_j) over S_t (-inf if empty)
 * ws/ws_bytes: workspace of dsa_sparse_mla_workspace_size bytes (split partial results). */
size_t dsa_sparse_mla_workspace_size(const dsa_batch_t* batch, int H, int k);
dsa_status_t dsa_sparse_mla(const dsa_batch_t* batch, const void* plan, const void* q, int H,
                            const void* kv_cache, const int32_t* S, int k, float softmax_scale, void* out,
                            float* lse, void* ws, size_t ws_bytes, void* stream);

/* ---- masked MHA mode for short prefill (an alternative to step 3) -------------------------
 * "MTP 与稀疏注意力：NSA 与 DSA", section "稀疏注意力：NSA 与 DSA": in a short prefill the absorbed
 * form costs 2H(512+64) + 2H*512 FLOPs per (query, key) pair against 2H(128+64) + 2H*128 for the
 * expanded multi-head form, so DeepSeek-V3.2 emulates DSA there with a masked multi-head attention.
 * The mask is the DSA mask of "DeepSeek Sparse Attention：从 SWA 到稀疏 Attention 计算", section
 * "Sparse Attention": M_tj = 0 for j in S_t, -inf elsewhere. For query row t and head h:
 *     out[t][h] = sum_j softmax_j(scale * q[t][h] . k[j][h] + M_tj) v[j][h]
 * Every request must be a whole prefill (m_b = n_b): row cu_q[b] + j of k and v holds position j of
 * request b. A request with n_b != m_b is recorded as DSA_ERR_DEVICE_INDEX and its rows are not
 * written.
 * q, k     bf16 [T, H, 192]   expanded queries and keys (128 "nope" + 64 rope dims per head)
 * v        bf16 [T, H, 128]   expanded values
 * S        int32 [T, topk]    index sets as dsa_topk writes them (entries < 0 skipped; a position
 *                             listed twice counts once; an entry above the row's position is
 *                             recorded as DSA_ERR_DEVICE_INDEX and skipped)
 * out      bf16 [T, H, 128]   lse f32 [T, H] or NULL (natural log; -inf for an empty set)
 * 1 <= H <= 128, 1 <= topk <= 4096, max_seq_len <= 65536. The plan must be made for this batch.
 * ws/ws_bytes: dsa_masked_mha_workspace_size bytes (the bitmap of S_t, T * max_seq_len / 8 bytes
 * rounded up). Dense tiles of 128 queries x 128 keys over each query tile's causal range, tcgen05
 * MMAs with S, P and O in TMEM. */
size_t dsa_masked_mha_workspace_size(const dsa_batch_t* batch, int H, int topk);
dsa_status_t dsa_masked_mha(const dsa_batch_t* batch, const void* plan, const void* q, const void* k,
                            const void* v, int H, const int32_t* S, int topk, float softmax_scale, void* out,
                            float* lse, void* ws, size_t ws_bytes, void* stream);

/* ---- the whole path ---------------------------------------------------------------------
 * Plan, indexer, top-k and sparse MLA in one call (four to five kernel launches, no host
 * synchronisation). S_out (int32 [T, k]) receives the index sets when not NULL. The plan lives in
 * `ws`; dsa_status_read takes `ws` as the plan. */
size_t dsa_layer_workspace_size(const dsa_batch_t* batch, int nhI, int H, int k);
dsa_status_t dsa_layer(const dsa_batch_t* batch, const uint8_t* qI, const float* qI_scale, const float* wI,
                       int nhI, const uint8_t* kI_cache, const float* kI_scale, const void* q, int H,
                       const void* kv_cache, int k, float softmax_scale, void* out, float* lse, int32_t* S_out,
                       void* ws, size_t ws_bytes, void* stream);

/* ---- the whole path without caller-provided workspace --------------------------------------
 * No counterpart on the pages: this exists for callers that cannot allocate device memory where
 * they run a layer (a locked or defragmenting memory pool, allocator-free runtimes, hooks that
 * must not call cudaMalloc). Same arguments and results as dsa_layer, minus ws/ws_bytes: the
 * workspace comes from a file-scope device array of 64 MiB that every GPU loading the library
 * holds until exit. Arguments are checked exactly as dsa_layer checks them (same statuses); then
 * requests needing more than 64 MiB (dsa_layer_workspace_size) return DSA_ERR_WORKSPACE and launch
 * nothing. Allocates nothing. Every call looks up the array's device address on the current device
 * (cudaGetSymbolAddress, host side); the first call on a device also loads the library's device
 * code there: make it before any stream capture. All calls share the array, which keeps the last
 * call's contents; calls whose kernels overlap on the GPU race on it. */
dsa_status_t dsa_layer_noalloc(const dsa_batch_t* batch, const uint8_t* qI, const float* qI_scale, const float* wI,
                               int nhI, const uint8_t* kI_cache, const float* kI_scale, const void* q, int H,
                               const void* kv_cache, int k, float softmax_scale, void* out, float* lse,
                               int32_t* S_out, void* stream);

/* The status word of the last dsa_layer_noalloc call on the current device (its plan lives in the
 * static array): synchronises `stream`, returns DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_DEVICE_INDEX as
 * dsa_status_read does, and clears the word. Read it before the next dsa_layer_noalloc call, whose
 * plan kernel rewrites the word. No counterpart on the pages. */
dsa_status_t dsa_layer_noalloc_status_read(void* stream);

const char* dsa_status_string(dsa_status_t status);
int dsa_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DSA_B200_H_ */
