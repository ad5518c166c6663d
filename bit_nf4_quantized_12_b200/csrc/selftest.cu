// selftest.cu -- a self-test of the bounded device wait.  Every kernel of the
// library waits on shared-memory barriers (TMA data, ring slots, tensor-core
// completion) through mbar_wait (common.cuh), which gives up after a limit,
// sets the timeout bit of the call's status word and lets the kernel return,
// so that a lost arrival ends in a status bit rather than a hung GPU.  This
// entry runs that same wait on a barrier nothing arrives at, with a short
// caller-chosen limit, so the give-up path can be exercised on a device
// without disturbing it.  The pages have no counterpart.
#include <cstdint>
#include <cuda_runtime.h>

#include "qlora_nf4.h"
#include "common.cuh"

namespace nf4 {
namespace {

__global__ void wait_selftest_kernel(uint32_t* status, long long limit_cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);          // one arrival expected; none will come
  abort_flag = 0;
  fence_mbar_init();
  mbar_wait(&bar, 0, status, &abort_flag, limit_cycles);
}

}  // namespace
}  // namespace nf4

extern "C" nf4_status nf4_wait_selftest(int32_t* d_status, int64_t limit_cycles, void* stream) {
  if (!d_status || limit_cycles < 1 || limit_cycles > (int64_t(1) << 40)) return NF4_ERR_INVALID_ARG;
  nf4::wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(reinterpret_cast<uint32_t*>(d_status),
                                                                              (long long)limit_cycles);
  return cudaGetLastError() == cudaSuccess ? NF4_OK : NF4_ERR_CUDA;
}
