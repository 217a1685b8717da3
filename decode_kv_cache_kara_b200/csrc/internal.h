// Internal launch interface between the C-ABI entry points (api.cu) and the kernel files.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kara.h"

namespace kara {

// Counts a kernel launch call that returned cudaSuccess (kara_launch_count). Defined in api.cu.
void count_launch(cudaError_t err);

// Kernel attributes (shared-memory limits) and occupancy are set and measured per device: every
// device holds its own instance of the library's kernels. Tables indexed by device_slot() hold
// that per-device state for device ordinals 0 .. kMaxDevices - 1.
constexpr int kMaxDevices = 64;
// The current CUDA device's index into such tables, or -1 (no current device, or an ordinal of
// kMaxDevices or more). Defined in api.cu.
int device_slot();

// Launches `kernel` as a programmatic dependent of the previous kernel in `stream`: it may
// start while that kernel finishes, and it must execute griddepcontrol.wait (which returns once
// the previous kernel has completed and its memory is visible) before it touches memory.
// Every library kernel launched this way does so at entry, so stream order holds as usual.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, args...);
  count_launch(err);
  return err;
}

// 4-D bf16 tensor map (innermost dimension first), 128-byte swizzle, box {64, 1, rows, 1}.
// Defined in score.cu.
bool make_bf16_map_4d(CUtensorMap* map, const void* base, const uint64_t dims[4],
                      const uint64_t strides[3], uint32_t box_rows);

// Records the pending CUDA error (if any) under `where` for kara_last_error() and returns
// KARA_OK or KARA_ERR_CUDA. Defined in api.cu.
kara_status check_launch(const char* where);
void set_last_error(const char* where, const char* what);

struct ScoreLaunch {
  const void* q_win;
  const void* k_cache;
  const int32_t* block_table;
  const int32_t* ctx_len;
  const int32_t* seq_ids;
  float* lse;
  float* scores;
  int32_t* status;
  int R, W, Hq, Hkv, D;
  int batch, max_blocks, num_blocks;
  float scale;
  int ring = 0;   // q_win is the window-query ring [batch, 2W, Hq, d]
  int agg = 0;    // KARA_AGG_SUM / MEAN / MAX
};
int score_lse_stride(int W);
int score_chunks(int W);
size_t score_workspace_bytes(int R, int W, int Hq);
kara_status launch_score_kernels(const ScoreLaunch& L, cudaStream_t stream);

kara_status launch_select(const float* scores, int rows, int W, int k, int32_t* sel,
                          cudaStream_t stream);
kara_status launch_select_chunks(const float* scores, int rows, int W, int k, int num_anchors,
                                 int gap_limit, int widen, int32_t* sel, int32_t* keep,
                                 cudaStream_t stream, int trim = KARA_TRIM_TOKEN);
kara_status launch_sum_heads(const float* scores, int rows, int hkv, int W, float* out,
                             cudaStream_t stream);
kara_status launch_expand_keep(const int32_t* keep_shared, int rows, int hkv, int k,
                               int32_t* keep, cudaStream_t stream);
kara_status launch_token2chunk(const float* scores, const int32_t* sel, int rows, int W, int k,
                               int num_anchors, int gap_limit, int widen, int32_t* keep,
                               cudaStream_t stream, int trim = KARA_TRIM_TOKEN);

struct LayerPtrs {
  void* k[KARA_MAX_LAYERS];
  void* v[KARA_MAX_LAYERS];
};

struct CompactLaunch {
  LayerPtrs layers;
  int L;
  int32_t* block_table;
  int32_t* ctx_len;
  int32_t* free_list;
  int32_t* free_top;
  const int32_t* seq_ids;
  const int32_t* keep;
  int32_t* plan;     // workspace
  int32_t* status;
  int R, W, k, Hkv, D;
  int batch, max_blocks, num_blocks;
  // fused compression (kara_compress): the keep sets come from these scores [L, R, Hkv, W]
  // through selection and Token2Chunk in the gather's CTAs (keep may then be an output)
  const float* scores = nullptr;
  int32_t* keep_out = nullptr;
  int num_anchors = 0, gap_limit = 0, widen = 0;
};
size_t compact_workspace_bytes(int R, int W, int k);
kara_status launch_compact(const CompactLaunch& L, cudaStream_t stream);

struct LacacheLaunch {
  LayerPtrs layers;
  int L;
  int32_t* block_table;
  int32_t* ctx_len;
  int32_t* free_list;
  int32_t* free_top;
  const int32_t* seq_ids;
  int32_t* plan;
  int32_t* status;
  int R, Hkv, D;
  int batch, max_blocks, num_blocks;
  int span, overlap, rung, budget, sink, recent;
};
size_t lacache_workspace_bytes(int R, int budget);
kara_status launch_lacache(const LacacheLaunch& L, cudaStream_t stream);

struct DecodeLaunch {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_table;
  const int32_t* ctx_len;
  void* out;
  float* partial;    // workspace
  int32_t* status;
  int B, Hq, Hkv, D;
  int max_blocks, num_blocks;
  float scale;
  // fused decode step: the new token (null for plain decode) and the window-query ring
  const void* k_new = nullptr;
  const void* v_new = nullptr;
  void* q_ring = nullptr;
  int ring_w = 0;
};
int decode_num_splits(int max_blocks);
size_t decode_workspace_bytes(int B, int Hq, int D, int max_blocks);
kara_status launch_decode(const DecodeLaunch& L, cudaStream_t stream);
kara_status launch_step_begin(const kara_pool* pool, int32_t* dev_status, cudaStream_t stream);
kara_status launch_step_end(const kara_pool* pool, int32_t* tail, int32_t window,
                            int32_t capacity, int32_t check, int32_t* due, int32_t* due_count,
                            cudaStream_t stream);
kara_status launch_reset_tails(int32_t* tail, const int32_t* seq_ids, int32_t num_seqs,
                               int32_t batch, cudaStream_t stream);

}  // namespace kara
