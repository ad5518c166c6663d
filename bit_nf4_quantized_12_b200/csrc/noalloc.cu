// noalloc.cu -- qlora_linear_fwd_noalloc: the QLoRA linear forward with its
// scratch taken from a fixed device array of this module instead of a
// caller-supplied workspace.
//
// Who needs it: callers that cannot allocate device memory at the point of
// the call.  One example is a token-by-token decode loop driven from C whose
// memory budget is fixed at start-up and that has no device allocator of its
// own.  There, cudaMalloc / cudaFree would synchronize the device between
// tokens and could fail once the budget is committed.  Another example is a
// host that only hands out input and output buffers and owns no allocator.
// Those callers run the forward with no cudaMalloc, cudaFree or allocating
// library routine on this path.  The kernels and the launch sequence are
// those of qlora_linear_fwd; only the origin of the scratch differs.
//
// The scratch is one array per device, shared by every call:
//  * set-up: the first call on a device (with that device current) looks up
//    the array's device address once.  Make that first call before any stream
//    capture begins.
//  * capacity: requests whose workspace exceeds QLORA_NOALLOC_SCRATCH_BYTES
//    are rejected with NF4_ERR_WORKSPACE before anything is launched.
//  * zeroing: the 256-byte status header is cleared on the stream by every
//    call.  The rest is fully written by the kernels before it is read.
//  * status: the first 4 bytes of the array are the call's status word (bit 1:
//    a bounded device wait gave up).  qlora_linear_fwd_noalloc_info returns
//    its device address; read it after the stream synchronizes and before the
//    next call, which clears it.
//  * overlapping calls race: two calls in flight at once on one device
//    (different streams or host threads) share the array.  Order them.
//  * device reset: the cached address belongs to the device's current
//    context.  After cudaDeviceReset (or any teardown of the primary context)
//    the module is loaded anew and the array may move; do not use this entry
//    point across such a reset.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "qlora_nf4.h"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's copy of the scratch array (set-up on first
// use).  nullptr when the address cannot be obtained.
void* scratch_for_current_device(nf4_status* why) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    *why = NF4_ERR_CUDA;
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    *why = NF4_ERR_UNSUPPORTED;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      *why = NF4_ERR_CUDA;
      return nullptr;
    }
    if ((reinterpret_cast<uintptr_t>(ptr) & 255u) != 0) {
      *why = NF4_ERR_MISALIGNED;
      return nullptr;
    }
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" nf4_status qlora_linear_fwd_noalloc_info(int32_t** d_status_word, size_t* scratch_bytes) {
  if (scratch_bytes) *scratch_bytes = size_t(QLORA_NOALLOC_SCRATCH_BYTES);
  if (!d_status_word) return NF4_OK;
  nf4_status why = NF4_OK;
  void* scratch = scratch_for_current_device(&why);
  if (scratch == nullptr) return why;
  *d_status_word = static_cast<int32_t*>(scratch);
  return NF4_OK;
}

extern "C" nf4_status qlora_linear_fwd_noalloc(const uint16_t* X, int64_t M, nf4_weight w, const uint16_t* A,
                                               const uint16_t* B, int32_t r, float s, uint16_t* Y,
                                               uint16_t* T_out, void* stream) {
  // Size check first: an oversize request fails on the host, before set-up.
  const size_t need = qlora_workspace_bytes(M, w.rows, w.cols, r);
  if (need == 0) return NF4_ERR_INVALID_ARG;
  if (need > size_t(QLORA_NOALLOC_SCRATCH_BYTES)) return NF4_ERR_WORKSPACE;
  nf4_status why = NF4_OK;
  void* scratch = scratch_for_current_device(&why);
  if (scratch == nullptr) return why;
  return qlora_linear_fwd(X, M, w, A, B, r, s, Y, T_out, scratch, size_t(QLORA_NOALLOC_SCRATCH_BYTES), stream);
}
