// kara_wait_probe: the bounded-wait failure path of the tcgen05 kernels, run on its own.
//
// Every mbarrier wait in the library gives up after a clock budget, reports KARA_ERR_TIMEOUT
// and raises a shared abort flag so that the other roles of the CTA unwind. This kernel waits
// on barriers that nothing arrives on: warp 0 with a short budget (it times out), warp 1 with
// the default budget (it must leave through the abort flag long before its own budget ends).
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace kara {
namespace {

__global__ void __launch_bounds__(64) wait_probe_kernel(int32_t* status, long long budget) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_wait_for(&bars[0], 0, &abort_flag, status, budget);      // times out
  } else if (threadIdx.x == 32) {
    if (mbar_wait(&bars[1], 0, &abort_flag, status)) report(status, KARA_ERR_INVALID_ARG);
  }
  __syncthreads();
}

}  // namespace
}  // namespace kara

extern "C" kara_status kara_wait_probe(int32_t wait_ms, int32_t* dev_status, cudaStream_t stream) {
  using namespace kara;
  if (wait_ms < 1 || wait_ms > 2000 || dev_status == nullptr) return KARA_ERR_INVALID_ARG;
  int dev = 0, khz = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev) != cudaSuccess || khz <= 0)
    return check_launch("kara_wait_probe");
  const long long budget = static_cast<long long>(wait_ms) * khz;   // cycles at the rated clock
  wait_probe_kernel<<<1, 64, 0, stream>>>(dev_status, budget);
  const kara_status st = check_launch("kara_wait_probe");
  if (st == KARA_OK) count_launch(cudaSuccess);
  return st;
}
