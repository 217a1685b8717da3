// C-ABI entry points of libkara: host-side argument checks, workspace carving, launches.
// Semantics of every call are documented in include/kara.h.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "internal.h"
#include "kara.h"

using namespace kara;

namespace {

thread_local char g_last_error[512] = "";
std::atomic<uint64_t> g_launches{0};

}  // namespace

namespace kara {

void set_last_error(const char* where, const char* what) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, what);
}

void count_launch(cudaError_t err) {
  if (err == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
}

int device_slot() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

kara_status check_launch(const char* where) {
  const cudaError_t err = cudaGetLastError();
  if (err == cudaSuccess) return KARA_OK;
  set_last_error(where, cudaGetErrorString(err));
  return KARA_ERR_CUDA;
}

}  // namespace kara

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

kara_status check_pool(const kara_pool* pool) {
  if (pool == nullptr) return KARA_ERR_INVALID_ARG;
  if (pool->block_table == nullptr || pool->ctx_len == nullptr) return KARA_ERR_INVALID_ARG;
  if (pool->batch < 0 || pool->max_blocks_per_seq <= 0 || pool->num_blocks <= 0)
    return KARA_ERR_INVALID_ARG;
  if (pool->page_size != 16) return KARA_ERR_UNSUPPORTED;
  if (pool->head_dim != 64 && pool->head_dim != 128) return KARA_ERR_UNSUPPORTED;
  if (pool->num_kv_heads <= 0) return KARA_ERR_INVALID_ARG;
  return KARA_OK;
}

// Token2Chunk step (a): the anchors are the top ceil(anchor_frac * k) of the selection. The
// product is rounded to 6 decimals before the ceiling, so that a float fraction such as 0.2f
// (0.2000000030) gives ceil(0.2 * 5) = 1 as the decimal fraction would. Returns -1 for a
// fraction outside [0, 1] (or NaN).
int anchors_from_frac(float anchor_frac, int32_t k) {
  if (!(anchor_frac >= 0.f && anchor_frac <= 1.f)) return -1;
  const double x = std::nearbyint(static_cast<double>(anchor_frac) * k * 1e6) / 1e6;
  const int n = static_cast<int>(std::ceil(x));
  return n < 0 ? 0 : (n > k ? k : n);
}

kara_status check_heads(const kara_pool* pool, int32_t num_q_heads) {
  if (num_q_heads <= 0 || num_q_heads % pool->num_kv_heads != 0) return KARA_ERR_INVALID_ARG;
  if (num_q_heads / pool->num_kv_heads > 8) return KARA_ERR_UNSUPPORTED;
  return KARA_OK;
}

kara_status fill_layers(const kara_layer_kv* layers, int32_t num_layers, LayerPtrs* out) {
  if (layers == nullptr || num_layers < 1 || num_layers > KARA_MAX_LAYERS)
    return KARA_ERR_INVALID_ARG;
  std::memset(out, 0, sizeof(*out));
  for (int i = 0; i < num_layers; ++i) {
    if (layers[i].k == nullptr || layers[i].v == nullptr) return KARA_ERR_INVALID_ARG;
    if (!aligned16(layers[i].k) || !aligned16(layers[i].v)) return KARA_ERR_INVALID_ARG;
    out->k[i] = layers[i].k;
    out->v[i] = layers[i].v;
  }
  return KARA_OK;
}


kara_status score_impl(const void* q_win, int ring, const void* k_cache, const kara_pool* pool,
                       const int32_t* seq_ids, int32_t num_seqs, int32_t window,
                       int32_t num_q_heads, float scale, int32_t agg, float* scores,
                       void* workspace, size_t workspace_bytes, int32_t* dev_status,
                       cudaStream_t stream) {
  if (agg != KARA_AGG_SUM && agg != KARA_AGG_MEAN && agg != KARA_AGG_MAX)
    return KARA_ERR_INVALID_ARG;
  kara_status st = check_pool(pool);
  if (st != KARA_OK) return st;
  if ((st = check_heads(pool, num_q_heads)) != KARA_OK) return st;
  if (num_seqs < 0 || window < 1 || window > KARA_MAX_WINDOW) return KARA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KARA_OK;
  if (q_win == nullptr || k_cache == nullptr || scores == nullptr || dev_status == nullptr)
    return KARA_ERR_INVALID_ARG;
  if (!aligned16(q_win) || !aligned16(k_cache) || !aligned16(scores)) return KARA_ERR_INVALID_ARG;
  const size_t need = kara_workspace_bytes(KARA_OP_SCORE, pool, num_seqs, window, num_q_heads, 0);
  if (workspace == nullptr || workspace_bytes < need || !aligned256(workspace))
    return KARA_ERR_WORKSPACE;
  ScoreLaunch L;
  L.q_win = q_win;
  L.k_cache = k_cache;
  L.block_table = pool->block_table;
  L.ctx_len = pool->ctx_len;
  L.seq_ids = seq_ids;
  L.lse = static_cast<float*>(workspace);
  L.scores = scores;
  L.status = dev_status;
  L.R = num_seqs;
  L.W = window;
  L.Hq = num_q_heads;
  L.Hkv = pool->num_kv_heads;
  L.D = pool->head_dim;
  L.batch = pool->batch;
  L.max_blocks = pool->max_blocks_per_seq;
  L.num_blocks = pool->num_blocks;
  L.scale = scale;
  L.ring = ring;
  L.agg = agg;
  return launch_score_kernels(L, stream);
}


kara_status decode_impl(const void* q, const void* k_new, const void* v_new, const void* k_cache,
                        const void* v_cache, const kara_pool* pool, int32_t num_q_heads,
                        float scale, void* q_ring, int32_t window, void* out, void* workspace,
                        size_t workspace_bytes, int32_t* dev_status, cudaStream_t stream) {
  kara_status st = check_pool(pool);
  if (st != KARA_OK) return st;
  if ((st = check_heads(pool, num_q_heads)) != KARA_OK) return st;
  if (pool->batch == 0) return KARA_OK;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || out == nullptr ||
      dev_status == nullptr)
    return KARA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return KARA_ERR_INVALID_ARG;
  const size_t need = kara_workspace_bytes(KARA_OP_DECODE, pool, 0, 0, num_q_heads, 0);
  if (workspace == nullptr || workspace_bytes < need || !aligned256(workspace))
    return KARA_ERR_WORKSPACE;
  DecodeLaunch L;
  L.q = q;
  L.k_cache = k_cache;
  L.v_cache = v_cache;
  L.block_table = pool->block_table;
  L.ctx_len = pool->ctx_len;
  L.out = out;
  L.partial = static_cast<float*>(workspace);
  L.status = dev_status;
  L.B = pool->batch;
  L.Hq = num_q_heads;
  L.Hkv = pool->num_kv_heads;
  L.D = pool->head_dim;
  L.max_blocks = pool->max_blocks_per_seq;
  L.num_blocks = pool->num_blocks;
  L.scale = scale;
  L.k_new = k_new;
  L.v_new = v_new;
  L.q_ring = q_ring;
  L.ring_w = window;
  return launch_decode(L, stream);
}

}  // namespace

extern "C" {

const char* kara_status_str(int32_t status) {
  switch (status) {
    case KARA_OK: return "ok";
    case KARA_ERR_INVALID_ARG: return "invalid argument";
    case KARA_ERR_UNSUPPORTED: return "unsupported configuration";
    case KARA_ERR_OUT_OF_BLOCKS: return "out of free blocks";
    case KARA_ERR_CUDA: return "CUDA error";
    case KARA_ERR_TIMEOUT: return "on-device wait timed out";
    case KARA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case KARA_ERR_BAD_BLOCK: return "block id out of range";
    default: return "unknown status";
  }
}

const char* kara_version(void) { return "kara-b200 0.1"; }

const char* kara_last_error(void) { return g_last_error; }

uint64_t kara_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t kara_workspace_bytes(kara_op op, const kara_pool* pool, int32_t num_seqs, int32_t window,
                            int32_t num_q_heads, int32_t k_or_budget) {
  switch (op) {
    case KARA_OP_SCORE:
      if (num_seqs <= 0 || window <= 0 || num_q_heads <= 0) return 0;
      return score_workspace_bytes(num_seqs, window, num_q_heads);
    case KARA_OP_COMPACT:
      if (num_seqs <= 0 || k_or_budget <= 0) return 0;
      return compact_workspace_bytes(num_seqs, window, k_or_budget);
    case KARA_OP_DECODE:
      if (pool == nullptr || pool->batch <= 0 || num_q_heads <= 0) return 0;
      return decode_workspace_bytes(pool->batch, num_q_heads, pool->head_dim,
                                    pool->max_blocks_per_seq);
    case KARA_OP_LACACHE:
      if (num_seqs <= 0 || k_or_budget <= 0) return 0;
      return lacache_workspace_bytes(num_seqs, k_or_budget);
    default:
      return 0;
  }
}


kara_status kara_score(const void* q_win, const void* k_cache, const kara_pool* pool,
                       const int32_t* seq_ids, int32_t num_seqs, int32_t window,
                       int32_t num_q_heads, float scale, float* scores, void* workspace,
                       size_t workspace_bytes, int32_t* dev_status, cudaStream_t stream) {
  return score_impl(q_win, 0, k_cache, pool, seq_ids, num_seqs, window, num_q_heads, scale,
                    KARA_AGG_SUM, scores, workspace, workspace_bytes, dev_status, stream);
}

kara_status kara_score_ex(const void* q, int32_t q_is_ring, const void* k_cache,
                          const kara_pool* pool, const int32_t* seq_ids, int32_t num_seqs,
                          int32_t window, int32_t num_q_heads, float scale, int32_t agg,
                          float* scores, void* workspace, size_t workspace_bytes,
                          int32_t* dev_status, cudaStream_t stream) {
  return score_impl(q, q_is_ring != 0 ? 1 : 0, k_cache, pool, seq_ids, num_seqs, window,
                    num_q_heads, scale, agg, scores, workspace, workspace_bytes, dev_status,
                    stream);
}

kara_status kara_sum_heads(const float* scores, int32_t rows, int32_t num_kv_heads,
                           int32_t window, float* out, cudaStream_t stream) {
  if (rows < 0 || num_kv_heads < 1 || window < 1 || window > KARA_MAX_WINDOW)
    return KARA_ERR_INVALID_ARG;
  if (rows == 0) return KARA_OK;
  if (scores == nullptr || out == nullptr) return KARA_ERR_INVALID_ARG;
  return launch_sum_heads(scores, rows, num_kv_heads, window, out, stream);
}

kara_status kara_expand_keep(const int32_t* keep_shared, int32_t rows, int32_t num_kv_heads,
                             int32_t k, int32_t* keep, cudaStream_t stream) {
  if (rows < 0 || num_kv_heads < 1 || k < 1) return KARA_ERR_INVALID_ARG;
  if (rows == 0) return KARA_OK;
  if (keep_shared == nullptr || keep == nullptr) return KARA_ERR_INVALID_ARG;
  return launch_expand_keep(keep_shared, rows, num_kv_heads, k, keep, stream);
}

kara_status kara_score_ring(const void* q_ring, const void* k_cache, const kara_pool* pool,
                            const int32_t* seq_ids, int32_t num_seqs, int32_t window,
                            int32_t num_q_heads, float scale, float* scores, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, cudaStream_t stream) {
  return score_impl(q_ring, 1, k_cache, pool, seq_ids, num_seqs, window, num_q_heads, scale,
                    KARA_AGG_SUM, scores, workspace, workspace_bytes, dev_status, stream);
}

kara_status kara_select(const float* scores, int32_t rows, int32_t window, int32_t k,
                        int32_t* sel, cudaStream_t stream) {
  if (rows < 0 || window < 1 || window > KARA_MAX_WINDOW || k < 1 || k > window)
    return KARA_ERR_INVALID_ARG;
  if (rows == 0) return KARA_OK;
  if (scores == nullptr || sel == nullptr) return KARA_ERR_INVALID_ARG;
  return launch_select(scores, rows, window, k, sel, stream);
}

kara_status kara_token2chunk_ex(const float* scores, const int32_t* sel, int32_t rows,
                                int32_t window, int32_t k, float anchor_frac, int32_t gap_limit,
                                int32_t widen, int32_t trim, int32_t* keep, cudaStream_t stream) {
  if (rows < 0 || window < 1 || window > KARA_MAX_WINDOW || k < 1 || k > window)
    return KARA_ERR_INVALID_ARG;
  const int num_anchors = anchors_from_frac(anchor_frac, k);
  if (num_anchors < 0 || gap_limit < 0 || widen < 0) return KARA_ERR_INVALID_ARG;
  if (trim != KARA_TRIM_TOKEN && trim != KARA_TRIM_CHUNK) return KARA_ERR_INVALID_ARG;
  if (rows == 0) return KARA_OK;
  if (scores == nullptr || sel == nullptr || keep == nullptr) return KARA_ERR_INVALID_ARG;
  return launch_token2chunk(scores, sel, rows, window, k, num_anchors, gap_limit, widen, keep,
                            stream, trim);
}

kara_status kara_token2chunk(const float* scores, const int32_t* sel, int32_t rows,
                             int32_t window, int32_t k, float anchor_frac, int32_t gap_limit,
                             int32_t widen, int32_t* keep, cudaStream_t stream) {
  return kara_token2chunk_ex(scores, sel, rows, window, k, anchor_frac, gap_limit, widen,
                             KARA_TRIM_TOKEN, keep, stream);
}

kara_status kara_select_chunks_ex(const float* scores, int32_t rows, int32_t window, int32_t k,
                                  float anchor_frac, int32_t gap_limit, int32_t widen,
                                  int32_t trim, int32_t* sel, int32_t* keep,
                                  cudaStream_t stream) {
  if (rows < 0 || window < 1 || window > KARA_MAX_WINDOW || k < 1 || k > window)
    return KARA_ERR_INVALID_ARG;
  const int num_anchors = anchors_from_frac(anchor_frac, k);
  if (num_anchors < 0 || gap_limit < 0 || widen < 0) return KARA_ERR_INVALID_ARG;
  if (trim != KARA_TRIM_TOKEN && trim != KARA_TRIM_CHUNK) return KARA_ERR_INVALID_ARG;
  if (rows == 0) return KARA_OK;
  if (scores == nullptr || keep == nullptr) return KARA_ERR_INVALID_ARG;
  return launch_select_chunks(scores, rows, window, k, num_anchors, gap_limit, widen, sel, keep,
                              stream, trim);
}

kara_status kara_select_chunks(const float* scores, int32_t rows, int32_t window, int32_t k,
                               float anchor_frac, int32_t gap_limit, int32_t widen,
                               int32_t* sel, int32_t* keep, cudaStream_t stream) {
  return kara_select_chunks_ex(scores, rows, window, k, anchor_frac, gap_limit, widen,
                               KARA_TRIM_TOKEN, sel, keep, stream);
}

kara_status kara_compact(const kara_layer_kv* layers, int32_t num_layers, const kara_pool* pool,
                         const int32_t* seq_ids, int32_t num_seqs, int32_t window, int32_t k,
                         const int32_t* keep, void* workspace, size_t workspace_bytes,
                         int32_t* dev_status, cudaStream_t stream) {
  kara_status st = check_pool(pool);
  if (st != KARA_OK) return st;
  if (pool->free_list == nullptr || pool->free_top == nullptr) return KARA_ERR_INVALID_ARG;
  if (num_seqs < 0 || window < 1 || window > KARA_MAX_WINDOW || k < 1 || k > window)
    return KARA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KARA_OK;
  if (keep == nullptr || dev_status == nullptr) return KARA_ERR_INVALID_ARG;
  CompactLaunch L;
  if ((st = fill_layers(layers, num_layers, &L.layers)) != KARA_OK) return st;
  const size_t need = kara_workspace_bytes(KARA_OP_COMPACT, pool, num_seqs, window, 0, k);
  if (workspace == nullptr || workspace_bytes < need || !aligned256(workspace))
    return KARA_ERR_WORKSPACE;
  L.L = num_layers;
  L.block_table = pool->block_table;
  L.ctx_len = pool->ctx_len;
  L.free_list = pool->free_list;
  L.free_top = pool->free_top;
  L.seq_ids = seq_ids;
  L.keep = keep;
  L.plan = static_cast<int32_t*>(workspace);
  L.status = dev_status;
  L.R = num_seqs;
  L.W = window;
  L.k = k;
  L.Hkv = pool->num_kv_heads;
  L.D = pool->head_dim;
  L.batch = pool->batch;
  L.max_blocks = pool->max_blocks_per_seq;
  L.num_blocks = pool->num_blocks;
  return launch_compact(L, stream);
}

kara_status kara_compress(const float* scores, const kara_layer_kv* layers, int32_t num_layers,
                          const kara_pool* pool, const int32_t* seq_ids, int32_t num_seqs,
                          int32_t window, int32_t k, float anchor_frac, int32_t gap_limit,
                          int32_t widen, int32_t* keep, void* workspace, size_t workspace_bytes,
                          int32_t* dev_status, cudaStream_t stream) {
  kara_status st = check_pool(pool);
  if (st != KARA_OK) return st;
  if (pool->free_list == nullptr || pool->free_top == nullptr) return KARA_ERR_INVALID_ARG;
  if (num_seqs < 0 || window < 1 || window > KARA_MAX_WINDOW || k < 1 || k > window)
    return KARA_ERR_INVALID_ARG;
  const int num_anchors = anchors_from_frac(anchor_frac, k);
  if (num_anchors < 0 || gap_limit < 0 || widen < 0) return KARA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KARA_OK;
  if (scores == nullptr || dev_status == nullptr) return KARA_ERR_INVALID_ARG;
  CompactLaunch L;
  if ((st = fill_layers(layers, num_layers, &L.layers)) != KARA_OK) return st;
  const size_t need = kara_workspace_bytes(KARA_OP_COMPACT, pool, num_seqs, window, 0, k);
  if (workspace == nullptr || workspace_bytes < need || !aligned256(workspace))
    return KARA_ERR_WORKSPACE;
  L.L = num_layers;
  L.block_table = pool->block_table;
  L.ctx_len = pool->ctx_len;
  L.free_list = pool->free_list;
  L.free_top = pool->free_top;
  L.seq_ids = seq_ids;
  L.keep = nullptr;
  L.plan = static_cast<int32_t*>(workspace);
  L.status = dev_status;
  L.R = num_seqs;
  L.W = window;
  L.k = k;
  L.Hkv = pool->num_kv_heads;
  L.D = pool->head_dim;
  L.batch = pool->batch;
  L.max_blocks = pool->max_blocks_per_seq;
  L.num_blocks = pool->num_blocks;
  L.scores = scores;
  L.keep_out = keep;
  L.num_anchors = num_anchors;
  L.gap_limit = gap_limit;
  L.widen = widen;
  return launch_compact(L, stream);
}


kara_status paged_decode_attn(const void* q, const void* k_cache, const void* v_cache,
                              const kara_pool* pool, int32_t num_q_heads, float scale, void* out,
                              void* workspace, size_t workspace_bytes, int32_t* dev_status,
                              cudaStream_t stream) {
  return decode_impl(q, nullptr, nullptr, k_cache, v_cache, pool, num_q_heads, scale, nullptr, 0,
                     out, workspace, workspace_bytes, dev_status, stream);
}

kara_status kara_decode_append(const void* q, const void* k_new, const void* v_new,
                               void* k_cache, void* v_cache, const kara_pool* pool,
                               int32_t num_q_heads, float scale, void* q_ring, int32_t window,
                               void* out, void* workspace, size_t workspace_bytes,
                               int32_t* dev_status, cudaStream_t stream) {
  if (k_new == nullptr || v_new == nullptr || !aligned16(k_new) || !aligned16(v_new))
    return KARA_ERR_INVALID_ARG;
  if (q_ring != nullptr && (window < 1 || window > KARA_MAX_WINDOW || !aligned16(q_ring)))
    return KARA_ERR_INVALID_ARG;
  return decode_impl(q, k_new, v_new, k_cache, v_cache, pool, num_q_heads, scale, q_ring,
                     window, out, workspace, workspace_bytes, dev_status, stream);
}

kara_status kara_step_begin(const kara_pool* pool, int32_t* dev_status, cudaStream_t stream) {
  kara_status st = check_pool(pool);
  if (st != KARA_OK) return st;
  if (pool->free_list == nullptr || pool->free_top == nullptr || dev_status == nullptr)
    return KARA_ERR_INVALID_ARG;
  if (pool->batch == 0) return KARA_OK;
  return launch_step_begin(pool, dev_status, stream);
}

kara_status kara_step_end(const kara_pool* pool, int32_t* tail, int32_t window,
                          int32_t capacity, int32_t check, int32_t* due, int32_t* due_count,
                          cudaStream_t stream) {
  kara_status st = check_pool(pool);
  if (st != KARA_OK) return st;
  if (window < 0 || capacity < 0 || (window > 0 && tail == nullptr)) return KARA_ERR_INVALID_ARG;
  if (check != 0 && (due == nullptr || due_count == nullptr || (window == 0 && capacity == 0)))
    return KARA_ERR_INVALID_ARG;
  if (pool->batch == 0) return KARA_OK;
  return launch_step_end(pool, tail, window, capacity, check != 0 ? 1 : 0, due, due_count,
                         stream);
}

kara_status kara_reset_tails(int32_t* tail, const int32_t* seq_ids, int32_t num_seqs,
                             int32_t batch, cudaStream_t stream) {
  if (num_seqs < 0 || batch < 0) return KARA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KARA_OK;
  if (tail == nullptr || seq_ids == nullptr) return KARA_ERR_INVALID_ARG;
  return launch_reset_tails(tail, seq_ids, num_seqs, batch, stream);
}

kara_status lacache_compact(const kara_layer_kv* layers, int32_t num_layers,
                            const kara_pool* pool, const int32_t* seq_ids, int32_t num_seqs,
                            const kara_lacache_params* params, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, cudaStream_t stream) {
  kara_status st = check_pool(pool);
  if (st != KARA_OK) return st;
  if (pool->free_list == nullptr || pool->free_top == nullptr || params == nullptr)
    return KARA_ERR_INVALID_ARG;
  const int S = params->span, O = params->overlap;
  if (S < 1 || S > num_layers || O < 0 || O >= S || params->rung < 1) return KARA_ERR_INVALID_ARG;
  const int stride = S - O;
  if (S % stride != 0 || num_layers % stride != 0) return KARA_ERR_INVALID_ARG;
  const int region_budget = params->budget - params->sink - params->recent;
  if (params->sink < 0 || params->recent < 0 || region_budget <= 0) return KARA_ERR_INVALID_ARG;
  if (region_budget % (params->rung * S / stride) != 0) return KARA_ERR_INVALID_ARG;
  if (num_seqs < 0) return KARA_ERR_INVALID_ARG;
  if (num_seqs == 0) return KARA_OK;
  if (dev_status == nullptr) return KARA_ERR_INVALID_ARG;
  LacacheLaunch L;
  if ((st = fill_layers(layers, num_layers, &L.layers)) != KARA_OK) return st;
  const size_t need =
      kara_workspace_bytes(KARA_OP_LACACHE, pool, num_seqs, 0, 0, params->budget);
  if (workspace == nullptr || workspace_bytes < need || !aligned256(workspace))
    return KARA_ERR_WORKSPACE;
  L.L = num_layers;
  L.block_table = pool->block_table;
  L.ctx_len = pool->ctx_len;
  L.free_list = pool->free_list;
  L.free_top = pool->free_top;
  L.seq_ids = seq_ids;
  L.plan = static_cast<int32_t*>(workspace);
  L.status = dev_status;
  L.R = num_seqs;
  L.Hkv = pool->num_kv_heads;
  L.D = pool->head_dim;
  L.batch = pool->batch;
  L.max_blocks = pool->max_blocks_per_seq;
  L.num_blocks = pool->num_blocks;
  L.span = S;
  L.overlap = O;
  L.rung = params->rung;
  L.budget = params->budget;
  L.sink = params->sink;
  L.recent = params->recent;
  return launch_lacache(L, stream);
}

}  // extern "C"
