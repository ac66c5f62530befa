// selftest.cu -- checks, on the GPU, the failure-detection path every pipeline
// wait of the kernels relies on: a bounded mbarrier wait whose phase never
// completes gives up after its limit, records TRA_DEV_TIMEOUT in the CTA's
// error word (so the other waiters drain at once) and the kernel returns
// normally, leaving the context usable.
#include "tra_device.cuh"
#include "tra_launch.h"

namespace tra {
namespace {

__global__ void __launch_bounds__(64) wait_selftest_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int err;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);  // one arrival expected; nobody arrives
    err = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* e = &err;
  // one thread waits first: its wait expires and sets the error word
  if (threadIdx.x == 0) mbar_wait_for(b, 0, e, limit_ns);
  __syncthreads();
  // the others then see the error word and return without waiting the limit again
  if (threadIdx.x != 0 && mbar_wait_for(b, 0, e, limit_ns)) atomicOr(status, 0x100);
  __syncthreads();
  if (threadIdx.x == 0 && *e) atomicOr(status, *e);
}

}  // namespace

cudaError_t launch_wait_selftest(int32_t* status, uint64_t limit_ns, cudaStream_t s) {
  wait_selftest_kernel<<<1, 64, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace tra
