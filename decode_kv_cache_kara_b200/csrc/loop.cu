// Decode-loop bookkeeping around the fused decode step (decode.cu): blocks for the new slots,
// the length and tail counters, the periodic tail-W trigger.
//
// "Kara: Efficient Reasoning LLM Serving via Sliding-Window KV Cache Compression", English
// abstract: compression runs during decoding on the recently generated context, and a
// threshold trigger is what the method avoids; gist.science explainer (German), section 3
// "Der 'Periodische' Zeitplan (KvLLM)": on a fixed schedule (every 100 steps) the oldest part
// of the current reasoning of some selected requests is cleaned up. Here a sequence is due at
// a check step when the tokens appended since its last compression (its tail) reach the
// window W; its window is then its last W slots, the window of kara_score / kara_compact.
// LaCache in the same loop ("LaCache: Ladder-Shaped KV Caching ...", iterative compaction with
// a fixed budget per layer): a sequence is due when its length reaches the capacity
// sink + recent + R_max, at which one ladder pass keeps exactly the budget in every layer.
//
// One CTA of 1024 threads per call: the counts are one int per sequence, and allocation in
// ascending sequence order is a block-wide prefix sum.
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace kara {

namespace {

constexpr int kLoopThreads = 1024;

struct LoopArgs {
  int32_t* block_table;
  int32_t* ctx_len;
  const int32_t* free_list;
  int32_t* free_top;
  int32_t* tail;        // may be null (step_end then only advances ctx_len)
  int32_t* due;         // check steps: ascending due sequences
  int32_t* due_count;
  int32_t* status;
  int B, max_blocks, num_blocks, window, capacity, check;
};

// Sequences whose next slot n = ctx_len starts a page take the block for page n / 16, in
// ascending order from the top of the free list (stack[top - 1] first). All or nothing: a slot
// past the table or a free-list top outside [0, num_blocks] (KARA_ERR_INVALID_ARG), or too few
// free blocks (KARA_ERR_OUT_OF_BLOCKS), changes nothing.
__global__ void __launch_bounds__(kLoopThreads) step_begin_kernel(const LoopArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ int buf[33];
  __shared__ int s_top;
  if (threadIdx.x == 0) s_top = *a.free_top;
  __syncthreads();
  int bad = s_top < 0 || s_top > a.num_blocks ? 1 : 0;
  int count = 0;
  for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
    const int n = a.ctx_len[b];
    if (n < 0 || n >= a.max_blocks * 16) bad = 1;
    else if (n % 16 == 0) ++count;
  }
  if (__syncthreads_or(bad)) {
    if (threadIdx.x == 0) report(a.status, KARA_ERR_INVALID_ARG);
    return;
  }
  int total;
  block_scan_add(count, buf, &total);
  const int top = s_top;
  if (total > top) {
    if (threadIdx.x == 0) report(a.status, KARA_ERR_OUT_OF_BLOCKS);
    return;
  }
  int carry = 0;
  for (int base = 0; base < a.B; base += blockDim.x) {   // chunks keep the ascending order
    const int b = base + static_cast<int>(threadIdx.x);
    const int n = b < a.B ? a.ctx_len[b] : 1;
    const int need = n % 16 == 0 ? 1 : 0;
    int chunk;
    const int ex = block_scan_add(need, buf, &chunk);
    if (need)
      a.block_table[static_cast<size_t>(b) * a.max_blocks + n / 16] =
          a.free_list[top - 1 - (carry + ex)];
    carry += chunk;
  }
  if (threadIdx.x == 0) *a.free_top = top - total;
}

// ctx_len += 1 and tail += 1 for every sequence; on a check step the sequences with
// tail >= W (W > 0) or ctx_len >= capacity (capacity > 0), ascending, and their count.
__global__ void __launch_bounds__(kLoopThreads) step_end_kernel(const LoopArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ int buf[33];
  int carry = 0;
  for (int base = 0; base < a.B; base += blockDim.x) {
    const int b = base + static_cast<int>(threadIdx.x);
    int is_due = 0;
    if (b < a.B) {
      const int n = a.ctx_len[b] + 1;
      a.ctx_len[b] = n;
      if (a.tail != nullptr) {
        const int t = a.tail[b] + 1;
        a.tail[b] = t;
        is_due = a.check && a.window > 0 && t >= a.window ? 1 : 0;
      }
      if (a.check && a.capacity > 0 && n >= a.capacity) is_due = 1;
    }
    if (a.check) {
      int chunk;
      const int ex = block_scan_add(is_due, buf, &chunk);
      if (is_due) a.due[carry + ex] = b;
      carry += chunk;
    }
  }
  if (a.check && threadIdx.x == 0) *a.due_count = carry;
}

__global__ void reset_tails_kernel(int32_t* tail, const int32_t* seq_ids, int n, int batch) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int b = seq_ids[i];
    if (b >= 0 && b < batch) tail[b] = 0;
  }
}

}  // namespace

kara_status launch_step_begin(const kara_pool* pool, int32_t* dev_status, cudaStream_t stream) {
  LoopArgs a = {};
  a.block_table = pool->block_table;
  a.ctx_len = pool->ctx_len;
  a.free_list = pool->free_list;
  a.free_top = pool->free_top;
  a.status = dev_status;
  a.B = pool->batch;
  a.max_blocks = pool->max_blocks_per_seq;
  a.num_blocks = pool->num_blocks;
  launch_pdl(step_begin_kernel, dim3(1), dim3(kLoopThreads), 0, stream, a);
  return check_launch("kara_step_begin");
}

kara_status launch_step_end(const kara_pool* pool, int32_t* tail, int32_t window,
                            int32_t capacity, int32_t check, int32_t* due, int32_t* due_count,
                            cudaStream_t stream) {
  LoopArgs a = {};
  a.ctx_len = pool->ctx_len;
  a.tail = tail;
  a.due = due;
  a.due_count = due_count;
  a.B = pool->batch;
  a.window = window;
  a.capacity = capacity;
  a.check = check;
  launch_pdl(step_end_kernel, dim3(1), dim3(kLoopThreads), 0, stream, a);
  return check_launch("kara_step_end");
}

kara_status launch_reset_tails(int32_t* tail, const int32_t* seq_ids, int32_t num_seqs,
                               int32_t batch, cudaStream_t stream) {
  const int blocks = (num_seqs + 255) / 256;
  launch_pdl(reset_tails_kernel, dim3(blocks < 1 ? 1 : blocks), dim3(256), 0, stream, tail,
             seq_ids, num_seqs, batch);
  return check_launch("kara_reset_tails");
}

}  // namespace kara
