// gemv.cu -- the QLoRA linear forward for one token (decode) on CUDA cores.
//
//   y[n] = bf16( sum_k x[k] Wd[n, k]  +  s * sum_j T[j] B[j, n] ),
//
// with Wd the NF4 weight dequantized on the fly ("LoRA、Q-LoRA 与 PortLLM"
// §3.4; "从LoRA到QLoRA" §3.1: NF4 storage, BF16 compute) and T = bf16(x A)
// from the previous kernel of the stream.  With one token the product is a
// matrix-vector product bound by reading the packed weight once, so it runs
// on the CUDA cores rather than being padded into tensor-core tiles.
//
// Work: each warp owns a group of up to kRows rows (n = first + r * stride)
// and walks the K dimension in passes of 32 NF4 blocks, one block (64
// weights, 32 packed bytes) per lane.  The 1 KB row piece of a pass comes
// through a per-warp ring of shared-memory slots (one per row) filled by the
// bulk-copy engine a pass ahead, so enough bytes are in flight to cover
// memory latency without holding them in registers.  One CTA of 32 warps
// per SM keeps the issue slots busy.  x is staged once per CTA in
// shared memory, each 64-element block with its 16-byte chunks rotated so
// that the 32 lanes of a warp read it without bank conflicts.  Each block is
// dequantized with the per-block table lookup shared with the tensor-core
// GEMM and accumulated by fp32 fmas on bf16 operands, so no integer work
// goes into widening x or the weights (the integer pipe, busy with the table
// lookups, is what bounds the kernel).  The low-rank term is added per lane
// before the warp reduction; only that part waits for T.
#include <cstdint>
#include <cuda_runtime.h>
#include "common.cuh"
#include "kernels.h"
#include "nf4_lut.cuh"

namespace nf4 {
namespace {

constexpr int kGemvThreads = 1024;  // 32 warps: one CTA per SM, x staged once per SM
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kRows = 4;            // rows per warp group, one ring slot each
constexpr int kSlots = kRows;       // ring depth per warp (row pieces in flight)
constexpr int kPiece = 1024;        // bytes of one row piece: 32 blocks x 32 bytes

struct GemvParams {
  Nf4GemvArgs a;
  CodeTable code;
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
// byte offset of 16-byte chunk i (eight bf16 values) of x block kb in the
// staged copy: 128 bytes a block, chunks rotated by the block index
__device__ __forceinline__ uint32_t x_chunk(int64_t kb, int i) {
  return uint32_t(kb) * 128u + uint32_t((i ^ int(kb & 7)) * 16);
}
// acc += x.lo * w.lo, then acc += x.hi * w.hi, for two bf16 (or fp16) pairs:
// an fp32 fma on 16-bit operands, equal to widening them first (their product
// is exact in fp32) but without the integer work of the widening
template <bool F16>
__device__ __forceinline__ float fma2_half(uint32_t x2, uint32_t w2, float acc) {
  if (F16) {
    asm("{\n\t.reg .b16 xl, xh, wl, wh;\n\t"
        "mov.b32 {xl, xh}, %1;\n\t"
        "mov.b32 {wl, wh}, %2;\n\t"
        "fma.rn.f32.f16 %0, xl, wl, %0;\n\t"
        "fma.rn.f32.f16 %0, xh, wh, %0;\n\t}"
        : "+f"(acc)
        : "r"(x2), "r"(w2));
  } else {
    asm("{\n\t.reg .b16 xl, xh, wl, wh;\n\t"
        "mov.b32 {xl, xh}, %1;\n\t"
        "mov.b32 {wl, wh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, xl, wl, %0;\n\t"
        "fma.rn.f32.bf16 %0, xh, wh, %0;\n\t}"
        : "+f"(acc)
        : "r"(x2), "r"(w2));
  }
  return acc;
}

// sum over the 64 weights of block kb of x[k] * Wd[n, k]; (q, c2) are the
// block's first-level constant parts in storage format dq
template <bool F16>
__device__ __forceinline__ float block_dot(const CodeTable& code, const uint4& p0, const uint4& p1, int dq,
                                           uint32_t q, float c2, uint32_t xs, int64_t kb, float acc) {
  const BlockTable t = make_table(code, scale_from_parts(dq, q, c2), F16);
  const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t o[4];
    lookup4(t, w[i] & 0xFFFFu, o[0], o[1]);   // weights 8i .. 8i+3
    lookup4(t, w[i] >> 16, o[2], o[3]);       // weights 8i+4 .. 8i+7
    const uint4 xv = lds128(xs + x_chunk(kb, i));
    acc = fma2_half<F16>(xv.x, o[0], acc);
    acc = fma2_half<F16>(xv.y, o[1], acc);
    acc = fma2_half<F16>(xv.z, o[2], acc);
    acc = fma2_half<F16>(xv.w, o[3], acc);
  }
  return acc;
}

template <bool F16>
__global__ void __launch_bounds__(kGemvThreads, 1) nf4_gemv_kernel(const __grid_constant__ GemvParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Nf4GemvArgs& a = P.a;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t KB = a.K / kBlock;
  const int64_t npass = (KB + 31) / 32;
  uint8_t* x_s = smem;                                          // K bf16, chunk-rotated
  uint8_t* ring = smem + a.K * 2 + warp * (kSlots * kPiece);    // this warp's slots
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.K * 2 + kGemvWarps * kSlots * kPiece) + warp * kSlots;
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(smem + a.K * 2 + kGemvWarps * kSlots * kPiece + kGemvWarps * kSlots * 8);

  if (lane < kSlots) mbar_init(&full[lane], 1);
  if (threadIdx.x == 0) *abort_flag = 0;
  fence_mbar_init();
  // stage x: 16-byte chunk c holds x[8c .. 8c+7], block c / 8, chunk c % 8
  for (int64_t c = threadIdx.x; c < a.K / 8; c += kGemvThreads) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.X) + c);
    *reinterpret_cast<uint4*>(x_s + x_chunk(c / 8, int(c % 8))) = v;
  }
  __syncthreads();
  griddep_launch();
  const uint32_t xs = smem_u32(x_s);
  const int64_t warp0 = int64_t(blockIdx.x) * kGemvWarps + warp;
  const int64_t stride = int64_t(gridDim.x) * kGemvWarps;
  uint32_t ph = 0;            // per-slot parity of completed fills
  bool ok = true, have_T = false;

  // issue the row piece (pass p, row r of the group) into slot r, with the
  // block scales of this lane's block into (q, c2)
  auto issue = [&](int64_t first, int nrows, int64_t p, int r, uint32_t& q, float& c2) {
    if (p >= npass || r >= nrows) return;
    const int64_t n = first + int64_t(r) * stride;
    const int64_t kb0 = p * 32;
    const int64_t nb = (KB - kb0 < 32) ? (KB - kb0) : 32;
    const int s = r;
    if (lane == 0) {
      mbar_arrive_expect_tx(&full[s], uint32_t(nb) * 32u);
      bulk_load(ring + s * kPiece, a.packed + n * (a.K / 2) + kb0 * 32, uint32_t(nb) * 32u, &full[s]);
    }
    const int64_t b = n * KB + kb0 + lane;
    if (kb0 + lane < KB) load_scale_parts(a.dq, a.c1q, a.c2, b, q, c2);
  };

  for (int64_t first = warp0; first < a.N && ok; first += stride * kRows) {
    int nrows = 0;
    while (nrows < kRows && first + int64_t(nrows) * stride < a.N) ++nrows;
    float acc[kRows];
    uint32_t q[kSlots];
    float c2[kSlots];
#pragma unroll
    for (int r = 0; r < kRows; ++r) acc[r] = 0.0f;
#pragma unroll
    for (int s = 0; s < kSlots; ++s) { q[s] = 0u; c2[s] = 0.0f; }
#pragma unroll
    for (int r = 0; r < kSlots; ++r) issue(first, nrows, 0, r, q[r], c2[r]);
    for (int64_t p = 0; p < npass && ok; ++p) {
      const int64_t kb = p * 32 + lane;
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        const int s = r;
        if (r < nrows) {
          if (!(ok = mbar_wait(&full[s], (ph >> s) & 1u, a.status, abort_flag))) break;
          ph ^= 1u << s;
          uint4 p0 = make_uint4(0, 0, 0, 0), p1 = p0;
          if (kb < KB) {
            p0 = lds128(smem_u32(ring + s * kPiece + lane * 32));
            p1 = lds128(smem_u32(ring + s * kPiece + lane * 32 + 16));
          }
          // the slot is refilled by the bulk-copy engine (async proxy):
          // order these generic reads before it
          fence_proxy_async_smem();
          __syncwarp();
          const uint32_t qc = q[s];
          const float cc = c2[s];
          // next piece of this slot: the same row, next pass
          issue(first, nrows, p + 1, r, q[s], c2[s]);
          if (kb < KB) acc[r] = block_dot<F16>(P.code, p0, p1, a.dq, qc, cc, xs, kb, acc[r]);
        }
      }
    }
    if (!ok) break;
    if (!have_T) {   // T comes from the previous kernel of the stream
      griddep_wait();
      have_T = true;
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      if (r < nrows) {
        const int64_t n = first + int64_t(r) * stride;
        float v = acc[r];
        for (int j = lane; j < a.r; j += 32)
          v = fmaf(a.s * half_lo_to_f32(F16, uint32_t(a.T[j])), half_lo_to_f32(F16, uint32_t(a.B[int64_t(j) * a.N + n])),
                   v);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) a.Y[n] = uint16_t(pack2(F16, v, 0.0f) & 0xFFFFu);
      }
    }
  }
  if (!ok) {   // let copies already issued land before the CTA exits (bounded)
#pragma unroll
    for (int s = 0; s < kSlots; ++s) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&full[s], (ph >> s) & 1u) && clock64() - t0 < 200000000ll) {
      }
    }
  }
  if (!have_T) griddep_wait();   // complete only after the previous kernel
}

size_t gemv_smem(int64_t K) {
  return size_t(K) * 2 + size_t(kGemvWarps) * kSlots * kPiece + size_t(kGemvWarps) * kSlots * 8 + 16;
}

}  // namespace

bool gemv_supported(int64_t M, int64_t K) {
  return M == 1 && K % kBlock == 0 && gemv_smem(K) <= size_t(220 * 1024);
}

cudaError_t launch_nf4_gemv(const Nf4GemvArgs& a, const float code[16], int num_sms, cudaStream_t stream,
                            bool pdl) {
  if (!gemv_supported(a.M, a.K)) return cudaErrorInvalidValue;
  GemvParams P;
  P.a = a;
  for (int i = 0; i < 16; ++i) P.code.v[i] = code[i];
  const size_t smem = gemv_smem(a.K);
  void (*kern)(const GemvParams) = a.f16 ? nf4_gemv_kernel<true> : nf4_gemv_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  // one CTA per SM, fewer when there are not enough rows for every warp
  int64_t blocks = int64_t(num_sms);
  const int64_t by_rows = (a.N + kGemvWarps - 1) / kGemvWarps;
  if (blocks > by_rows) blocks = by_rows;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(blocks));
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, P);
}

}  // namespace nf4
