// Top-k selection and Token2Chunk, one CTA per window row, everything in shared memory (the
// block-level device code is in select_row.cuh); the shared-selection helpers.
#include <cstdint>

#include "common.cuh"
#include "internal.h"
#include "select_row.cuh"

namespace kara {

namespace {

__global__ void __launch_bounds__(kSelThreads)
select_kernel(const float* __restrict__ scores, int W, int k, int32_t* __restrict__ sel) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // previous kernel done (PDL launch)
  extern __shared__ __align__(16) uint8_t smem[];
  SelectSmem* ss = reinterpret_cast<SelectSmem*>(smem);
  uint32_t* key = reinterpret_cast<uint32_t*>(smem + sizeof(SelectSmem));
  uint8_t* cand = reinterpret_cast<uint8_t*>(key + W);
  uint8_t* flag = cand + W;
  const int row = blockIdx.x;
  const float* s = scores + static_cast<size_t>(row) * W;
  const int E = (W + kSelThreads - 1) / kSelThreads;
  for (int j = threadIdx.x; j < W; j += kSelThreads) {
    key[j] = order_key(s[j]);
    cand[j] = 1;
    flag[j] = 0;
  }
  __syncthreads();
  block_select(key, cand, flag, W, E, k, ss);
  block_compact_write(flag, W, E, sel + static_cast<size_t>(row) * k, ss->ibuf);
}

__global__ void __launch_bounds__(kSelThreads)
token2chunk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ sel, int W,
                   int k, int num_anchors, int gap_limit, int widen, int32_t* __restrict__ keep,
                   int trim) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // previous kernel done (PDL launch)
  extern __shared__ __align__(16) uint8_t smem[];
  const size_t row = blockIdx.x;
  token2chunk_row(scores + row * W, sel + row * k, nullptr, W, k, num_anchors, gap_limit, widen,
                  keep + row * k, smem, trim);
}

__global__ void __launch_bounds__(kSelThreads)
select_chunks_kernel(const float* __restrict__ scores, int32_t* __restrict__ sel, int W, int k,
                     int num_anchors, int gap_limit, int widen, int32_t* __restrict__ keep,
                     int trim) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // previous kernel done (PDL launch)
  extern __shared__ __align__(16) uint8_t smem[];
  const size_t row = blockIdx.x;
  token2chunk_row(scores + row * W, nullptr, sel != nullptr ? sel + row * k : nullptr, W, k,
                  num_anchors, gap_limit, widen, keep + row * k, smem, trim);
}


}  // namespace

kara_status launch_select(const float* scores, int rows, int W, int k, int32_t* sel,
                          cudaStream_t stream) {
  if (rows == 0) return KARA_OK;
  launch_pdl(select_kernel, dim3(rows), dim3(kSelThreads), select_smem(W), stream, scores, W, k,
             sel);
  return check_launch(__func__);
}

// Windows above about 3400 keys (about 1500 with the chunk-aware trim) need more than the
// default 48 KB of dynamic shared memory.
size_t t2c_launch_smem(int W, int trim) {
  return t2c_smem(W) + (trim == KARA_TRIM_CHUNK ? chunk_smem(W) : 0);
}

// Per device (every device holds its own instance of the kernels).
void allow_t2c_smem() {
  static std::atomic<int> done[kMaxDevices];
  const int dev = device_slot();
  if (dev < 0 || done[dev].load()) return;   // no device: the launch reports the error
  const int bytes = static_cast<int>(t2c_launch_smem(KARA_MAX_WINDOW, KARA_TRIM_CHUNK));
  cudaFuncSetAttribute(token2chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  cudaFuncSetAttribute(select_chunks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  done[dev].store(1);
}

kara_status launch_token2chunk(const float* scores, const int32_t* sel, int rows, int W, int k,
                               int num_anchors, int gap_limit, int widen, int32_t* keep,
                               cudaStream_t stream, int trim) {
  if (rows == 0) return KARA_OK;
  allow_t2c_smem();
  launch_pdl(token2chunk_kernel, dim3(rows), dim3(kSelThreads), t2c_launch_smem(W, trim), stream,
             scores, sel, W, k, num_anchors, gap_limit, widen, keep, trim);
  return check_launch(__func__);
}

kara_status launch_select_chunks(const float* scores, int rows, int W, int k, int num_anchors,
                                 int gap_limit, int widen, int32_t* sel, int32_t* keep,
                                 cudaStream_t stream, int trim) {
  if (rows == 0) return KARA_OK;
  allow_t2c_smem();
  launch_pdl(select_chunks_kernel, dim3(rows), dim3(kSelThreads), t2c_launch_smem(W, trim),
             stream, scores, sel, W, k, num_anchors, gap_limit, widen, keep, trim);
  return check_launch(__func__);
}

namespace {

// A selection shared by the KV heads of a layer: the head-summed scores (heads added in
// ascending order, so the result is reproducible) ...
__global__ void sum_heads_kernel(const float* __restrict__ scores, int rows, int hkv, int W,
                                 float* __restrict__ out) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const size_t total = static_cast<size_t>(rows) * W;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t r = i / W, j = i - r * W;
    const float* p = scores + r * hkv * W + j;
    float s = 0.f;
    for (int g = 0; g < hkv; ++g) s += p[static_cast<size_t>(g) * W];
    out[i] = s;
  }
}

// ... and the one keep set copied to every head.
__global__ void expand_keep_kernel(const int32_t* __restrict__ keep_shared, int rows, int hkv,
                                   int k, int32_t* __restrict__ keep) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const size_t total = static_cast<size_t>(rows) * hkv * k;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t t = i % k, r = i / (static_cast<size_t>(hkv) * k);
    keep[i] = keep_shared[r * k + t];
  }
}

int grid_for(size_t n) {
  const size_t b = (n + 255) / 256;
  return static_cast<int>(b < 1 ? 1 : (b > 4096 ? 4096 : b));
}

}  // namespace

kara_status launch_sum_heads(const float* scores, int rows, int hkv, int W, float* out,
                             cudaStream_t stream) {
  launch_pdl(sum_heads_kernel, dim3(grid_for(static_cast<size_t>(rows) * W)), dim3(256), 0,
             stream, scores, rows, hkv, W, out);
  return check_launch("kara_sum_heads");
}

kara_status launch_expand_keep(const int32_t* keep_shared, int rows, int hkv, int k,
                               int32_t* keep, cudaStream_t stream) {
  launch_pdl(expand_keep_kernel, dim3(grid_for(static_cast<size_t>(rows) * hkv * k)), dim3(256),
             0, stream, keep_shared, rows, hkv, k, keep);
  return check_launch("kara_expand_keep");
}

}  // namespace kara
