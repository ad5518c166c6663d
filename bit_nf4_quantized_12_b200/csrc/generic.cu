// generic.cu -- the QLoRA linear layer for shapes the fused tensor-core path
// does not take (K % 64 != 0, N % 8 != 0 or r % 8 != 0), for example a
// weight whose rows do not start on an NF4 block ("从LoRA到QLoRA" §3.1;
// "LoRA、Q-LoRA 与 PortLLM" §3.4 for the layer):
//   forward : T = rnd(X A),  Y = rnd(X Wd^T + s T B)
//   backward: G = s dY B^T,  dX = rnd(dY Wd + G A^T),  dA = X^T G,  dB = s T^T dY
// (rnd: round to the compute type, bf16 or fp16)
// The weight is first dequantized exactly into the workspace by the
// standalone dequant kernel (any shape), so unlike the fused path Wd reaches
// memory here.  Every product then runs through one tiled CUDA-core kernel:
// a 16 x 16 output tile per CTA, up to two reduction segments, operands read
// through strided accessors (bf16, fp16 or fp32), fp32 accumulation in a
// fixed order, bf16 / fp16 (round to nearest even) or fp32 output.  Correctness first:
// this path serves shapes outside the fused kernels, not throughput.
#include <cstdint>
#include <cuda_runtime.h>
#include "common.cuh"
#include "kernels.h"

namespace nf4 {
namespace {

constexpr int kTile = 16;

__device__ __forceinline__ float load_operand(const GenericOperand& o, int64_t i, int64_t p) {
  const int64_t idx = i * o.si + p * o.sp;
  if (o.kind == kOpF32) return static_cast<const float*>(o.base)[idx];
  return half_lo_to_f32(o.kind == kOpF16, uint32_t(static_cast<const uint16_t*>(o.base)[idx]));
}

// tile[il][pl] = o(i0 + il, p0 + pl), zero outside [0, I) x [0, P); the
// thread-to-element map follows the operand's contiguous dimension so that
// neighbouring threads read neighbouring elements
__device__ __forceinline__ void load_tile(float (&tile)[kTile][kTile + 1], const GenericOperand& o, int64_t i0,
                                          int64_t I, int64_t p0, int64_t P, int tx, int ty) {
  const int il = (o.sp == 1) ? ty : tx;
  const int pl = (o.sp == 1) ? tx : ty;
  const int64_t i = i0 + il, p = p0 + pl;
  tile[il][pl] = (i < I && p < P) ? load_operand(o, i, p) : 0.0f;
}

// One CTA walks output tiles t = blockIdx.x, blockIdx.x + gridDim.x, ...
// (row-major over the tile grid); the trip count is uniform across the CTA,
// so every thread meets every barrier.
__global__ void __launch_bounds__(kTile * kTile) generic_gemm_kernel(const __grid_constant__ GenericGemm g) {
  __shared__ float as[kTile][kTile + 1];
  __shared__ float bs[kTile][kTile + 1];
  const int tx = threadIdx.x % kTile, ty = threadIdx.x / kTile;
  const int64_t tiles_j = (g.J + kTile - 1) / kTile;
  const int64_t tiles = (g.I + kTile - 1) / kTile * tiles_j;
  for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
    const int64_t i0 = t / tiles_j * kTile, j0 = t % tiles_j * kTile;
    float total = 0.0f;
    for (int s = 0; s < g.nseg; ++s) {
      const GenericSegment& seg = g.seg[s];
      float acc = 0.0f;
      for (int64_t p0 = 0; p0 < seg.P; p0 += kTile) {
        load_tile(as, seg.a, i0, g.I, p0, seg.P, tx, ty);
        load_tile(bs, seg.b, j0, g.J, p0, seg.P, tx, ty);
        __syncthreads();
#pragma unroll
        for (int q = 0; q < kTile; ++q) acc = fmaf(as[ty][q], bs[tx][q], acc);
        __syncthreads();
      }
      total = fmaf(seg.scale, acc, total);
    }
    const int64_t i = i0 + ty, j = j0 + tx;
    if (i < g.I && j < g.J) {
      if (g.out_kind == kOpF32) static_cast<float*>(g.out)[i * g.J + j] = total;
      else static_cast<uint16_t*>(g.out)[i * g.J + j] = uint16_t(pack2(g.out_kind == kOpF16, total, 0.0f) & 0xFFFFu);
    }
  }
}

}  // namespace

cudaError_t launch_generic_gemm(const GenericGemm& g, int num_sms, cudaStream_t stream) {
  if (g.I < 1 || g.J < 1 || g.nseg < 1 || g.nseg > 2) return cudaErrorInvalidValue;
  for (int s = 0; s < g.nseg; ++s)
    if (g.seg[s].P < 0) return cudaErrorInvalidValue;
  const int64_t tiles = (g.I + kTile - 1) / kTile * ((g.J + kTile - 1) / kTile);
  const int64_t grid = tiles < int64_t(num_sms) * 8 ? tiles : int64_t(num_sms) * 8;
  generic_gemm_kernel<<<unsigned(grid), kTile * kTile, 0, stream>>>(g);
  return cudaGetLastError();
}

}  // namespace nf4
