// repitch.cu -- copies an activation-side matrix into a row pitch that TMA
// can address (a multiple of 16 bytes), for linear-layer shapes whose K or N
// is not a multiple of 8 ("QLoRA 原理精讲" robustness of the layer to any
// weight shape; the frozen weight itself is never copied: its packed codes
// are read in place).  Bandwidth-bound: one coalesced read and write of the
// matrix; the padding columns are not written (TMA never reads past the
// logical extent, it fills zeros there instead).
#include <cstdint>
#include <cuda_runtime.h>
#include "kernels.h"

namespace nf4 {
namespace {

// one row per CTA iteration, the threads along the row: coalesced on both sides
__global__ void __launch_bounds__(256) repitch_kernel(const uint16_t* __restrict__ src, int64_t rows, int64_t cols,
                                                      uint16_t* __restrict__ dst, int64_t ld) {
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint16_t* s = src + r * cols;
    uint16_t* d = dst + r * ld;
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x) d[c] = __ldcs(s + c);
  }
}

}  // namespace

cudaError_t launch_repitch(const uint16_t* src, int64_t rows, int64_t cols, uint16_t* dst, int64_t ld, int num_sms,
                           cudaStream_t stream) {
  if (rows < 1 || cols < 1 || ld < cols) return cudaErrorInvalidValue;
  int64_t grid = rows;
  const int64_t cap = int64_t(num_sms) * 8;
  if (grid > cap) grid = cap;
  repitch_kernel<<<unsigned(grid), 256, 0, stream>>>(src, rows, cols, dst, ld);
  return cudaGetLastError();
}

}  // namespace nf4
