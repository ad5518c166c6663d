// decode.cu -- the QLoRA linear forward for decode-shaped inputs, 1 to 16
// tokens ("QLoRA 原理精讲" §三 误区3 ①: serve with the adapter kept
// separate, dequantizing the NF4 weight on the fly):
//
//   Y[m, n] = round( sum_k X[m, k] Wd[n, k]  +  s sum_j T[m, j] B[j, n] ),
//
// T = round(X A) from the previous kernel of the stream.  The call is bound by
// reading the packed weight once (0.5 byte per weight plus the block
// constants), and in practice by the integer work of decoding it; so each
// weight is decoded exactly once, in registers, and multiplied with every
// token by the tensor cores (mma.sync m16n8k16, fp32 accumulation): the
// weights are the 16-row A operand, the tokens the 8-wide N dimension.
//
// Fragment order.  Within one MMA the reduction order is free, so the 16
// reduction slots of lane (g, c) over 16 consecutive MMAs are mapped onto one
// whole NF4 block: over a unit of 4 blocks (256 columns of W), lane (g, c)
// decodes block c of rows g and g + 8 of its warp's 16-row strip, four
// consecutive weights per MMA (MMA t takes weights 4t .. 4t+3 of the block as
// its slots 2c, 2c+1, 2c+8, 2c+9).  So every lane builds one 16-entry table
// per block and row (the same byte-permute lookup as the tensor-core GEMM),
// and the B fragment is four consecutive x values of that block; one 16-byte
// shared load gives the x values of two consecutive MMAs.
//
// Work split.  A tile is 256 rows of W (16 consumer warps x 16 rows); a unit
// is one tile x 256 columns.  Persistent CTAs (one per SM) take contiguous
// ranges of the units in tile-major order (stream-K), so the SMs get equal
// work for any shape.  A tile whose columns are split between CTAs is summed
// by the CTA that finishes last: the others leave fp32 partials in the
// workspace, and the last one adds them in CTA order (a fixed order, so the
// result does not depend on timing).  One producer warp streams the units
// through a ring of shared-memory stages with TMA: the 256 x 128-byte box of
// packed codes and the 4 boxes of X (64 columns each), both with the 128-byte
// swizzle.  The X box of block c is loaded from token row -2c (rows before
// token 0 and past the last token read as zeros), so token m sits in shared
// row m + 2c and the eight lanes that share a 128-byte phase of a load (two
// token rows x four blocks) meet eight different swizzle phases: the loads
// are free of bank conflicts.  Every wait is bounded and reports
// kStatusTimeout instead of hanging.
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include "common.cuh"
#include "kernels.h"
#include "nf4_lut.cuh"

namespace nf4 {
namespace {

constexpr int kDecWarps = 16;                        // consumer warps, one 16-row strip each
constexpr int kDecThreads = (kDecWarps + 1) * 32;    // + one producer warp
constexpr int kDecTileRows = 16 * kDecWarps;         // 256 rows of W per tile
constexpr int kDecChunk = 256;                       // columns of W per unit (4 NF4 blocks)
constexpr int kDecStages = 4;
constexpr uint32_t kPkBytes = kDecTileRows * 128;    // packed box: 256 rows x 128 bytes

struct DecodeParams {
  CUtensorMap tm_pk;   // packed [N, K/2] bytes, box {128, 256}, 128-byte swizzle
  CUtensorMap tm_x;    // X [M, K] 2-byte, box {64, M}, 128-byte swizzle
  Nf4DecodeArgs a;
  CodeTable code;
  ShiftMuls km;
  int64_t tiles, nk, units;
  uint32_t xrows;       // rows of an X box: 8 per token tile + 6 for the block offsets
  uint32_t xbox_bytes;  // shared bytes per X box (xrows x 128, a multiple of 1024)
  uint32_t stage_bytes;
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void consumer_sync() {   // the 16 consumer warps
  asm volatile("bar.sync 1, %0;" ::"n"(kDecWarps * 32) : "memory");
}

template <bool F16>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  if (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

// Stream-K partition: CTA p takes units [begin(p), begin(p + 1)).
__device__ __forceinline__ int64_t unit_begin(int64_t p, int64_t U, int64_t P) { return p * U / P; }
__device__ __forceinline__ int64_t unit_owner(int64_t u, int64_t U, int64_t P) {
  int64_t p = u * P / U;
  while (p + 1 < P && unit_begin(p + 1, U, P) <= u) ++p;
  while (p > 0 && unit_begin(p, U, P) > u) --p;
  return p;
}

template <bool F16, int NT>
__global__ void __launch_bounds__(kDecThreads, 1) nf4_decode_kernel(const __grid_constant__ DecodeParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Nf4DecodeArgs& a = P.a;
  float* red = reinterpret_cast<float*>(smem + kDecStages * P.stage_bytes);      // [16 tokens][256 rows]
  uint64_t* full = reinterpret_cast<uint64_t*>(red + 16 * kDecTileRows);
  uint64_t* empty = full + kDecStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kDecStages);
  int* bcast = const_cast<int*>(abort_flag) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t p = blockIdx.x, NP = gridDim.x;
  const int64_t u0 = unit_begin(p, P.units, NP), u1 = unit_begin(p + 1, P.units, NP);
  const int64_t KB = a.K / kBlock;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == kDecWarps * 32) {
    tma_prefetch_desc(&P.tm_pk);
    tma_prefetch_desc(&P.tm_x);
  }
  __syncthreads();
  griddep_launch();

  if (warp == kDecWarps) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      int64_t issued = 0;
      for (int64_t u = u0; u < u1; ++u) {
        const int64_t i = u - u0;
        const int s = int(i % kDecStages);
        if (i >= kDecStages && !mbar_wait(&empty[s], uint32_t(i / kDecStages - 1) & 1u, a.status, abort_flag)) break;
        const int64_t tile = u / P.nk, kc = u % P.nk;
        uint8_t* st = smem + s * P.stage_bytes;
        mbar_arrive_expect_tx(&full[s], kPkBytes + 4u * P.xrows * 128u);
        tma_load_2d(st, &P.tm_pk, &full[s], int32_t(kc * 128), int32_t(tile * kDecTileRows));
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tma_load_2d(st + kPkBytes + c * P.xbox_bytes, &P.tm_x, &full[s], int32_t(kc * kDecChunk + c * 64),
                      -2 * c);
        issued = i + 1;
      }
      if (*abort_flag) {   // let copies already in flight land before the CTA exits
        for (int64_t i = (issued > kDecStages ? issued - kDecStages : 0); i < issued; ++i) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&full[i % kDecStages], uint32_t(i / kDecStages) & 1u) &&
                 clock64() - t0 < 200000000ll) {
          }
        }
      }
    }
    __syncwarp();
    return;
  }

  // -------------------------------------------------------------- consumers
  const int g = lane >> 2, c = lane & 3;
  const int row0 = warp * 16 + g;           // rows row0 and row0 + 8 of the tile
  bool ok = true, have_T = false;
  // two accumulators per token tile (even and odd MMAs), so that two chains
  // of dependent MMAs are in flight; summed when a segment ends
  float acc[NT][4], acc2[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[nt][q] = acc2[nt][q] = 0.0f;

  // block constants of (row, block c of unit (tile, kc)), loaded one unit ahead
  auto load_scales = [&](bool valid, int64_t tile, int64_t kc, uint32_t (&q)[2], float (&s2)[2]) {
    q[0] = q[1] = 0u;
    s2[0] = s2[1] = 0.0f;
    const int64_t kb = kc * 4 + c;
    if (!valid || kb >= KB) return;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t n = tile * kDecTileRows + row0 + 8 * h;
      if (n < a.N) load_scale_parts(a.dq, a.c1q, a.c2, n * KB + kb, q[h], s2[h]);
    }
  };
  const uint32_t xph = uint32_t((g + 2 * c) & 7) << 4;   // swizzle phase of this lane's token rows
  uint32_t cq[2], nq[2];
  float cs[2], ns[2];
  int64_t tile = u0 / P.nk, kc = u0 % P.nk;          // unit u = tile * nk + kc, advanced without division
  load_scales(true, tile, kc, cq, cs);

  // Every consumer warp walks the same units and meets the same barriers,
  // whatever happens: after a failed wait (ok == false) a warp skips the work
  // but still takes part in each segment's barriers, so no warp can wait on
  // one that left.  The status word then says the outputs are unspecified.
  int64_t seg_first_kc = u0 % P.nk;
  bool first_segment = true;
  for (int64_t u = u0; u < u1; ++u) {
    const int64_t i = u - u0;
    const int s = int(i % kDecStages);
    {
      const bool last_kc = kc + 1 == P.nk;
      load_scales(u + 1 < u1, last_kc ? tile + 1 : tile, last_kc ? 0 : kc + 1, nq, ns);
    }
    if (ok) ok = mbar_wait(&full[s], uint32_t(i / kDecStages) & 1u, a.status, abort_flag);
    if (ok) {
      const uint32_t st = smem_u32(smem + s * P.stage_bytes);
      // packed codes of block c, rows row0 and row0 + 8 (128-byte swizzle:
      // the 16-byte chunk index is XORed with the row index mod 8, here g)
      uint32_t w0[8], w1[8];
      {
        const uint32_t r0 = st + uint32_t(row0) * 128u, r1 = r0 + 8u * 128u;
        const uint32_t ca = (uint32_t(2 * c) ^ uint32_t(g)) << 4, cb = (uint32_t(2 * c + 1) ^ uint32_t(g)) << 4;
        const uint4 x0 = lds128(r0 + ca), x1 = lds128(r0 + cb);
        const uint4 y0 = lds128(r1 + ca), y1 = lds128(r1 + cb);
        w0[0] = x0.x; w0[1] = x0.y; w0[2] = x0.z; w0[3] = x0.w;
        w0[4] = x1.x; w0[5] = x1.y; w0[6] = x1.z; w0[7] = x1.w;
        w1[0] = y0.x; w1[1] = y0.y; w1[2] = y0.z; w1[3] = y0.w;
        w1[4] = y1.x; w1[5] = y1.y; w1[6] = y1.z; w1[7] = y1.w;
      }
      const BlockTable t0 = make_table(P.code, scale_from_parts(a.dq, cq[0], cs[0]), F16);
      const BlockTable t1 = make_table(P.code, scale_from_parts(a.dq, cq[1], cs[1]), F16);
      // X box c: token nt * 8 + g sits in shared row nt * 8 + g + 2c
      // (the row starts on 128 bytes, so chunk i of it is at row ^ ((i << 4) ^ xph))
      const uint32_t xb = (st + kPkBytes + uint32_t(c) * P.xbox_bytes + uint32_t(g + 2 * c) * 128u) | xph;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        // word i: weights 8i .. 8i + 7 of the block, MMAs 2i and 2i + 1
        uint32_t p0, p1, p2, p3, q0, q1, q2, q3;
        lookup8(t0, w0[i], P.km, p0, p1, p2, p3);
        lookup8(t1, w1[i], P.km, q0, q1, q2, q3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint4 b = lds128((xb ^ uint32_t(i << 4)) + uint32_t(nt) * 1024u);
          mma16816<F16>(acc[nt], p0, q0, p1, q1, b.x, b.y);
          mma16816<F16>(acc2[nt], p2, q2, p3, q3, b.z, b.w);
        }
      }
      // the stage is refilled by TMA (async proxy): order these reads first
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    cq[0] = nq[0]; cq[1] = nq[1]; cs[0] = ns[0]; cs[1] = ns[1];

    // ---------------------------------------------------------- tile segment end
    if (kc != P.nk - 1 && u != u1 - 1) {
      ++kc;
      continue;
    }
    const bool whole = seg_first_kc == 0 && kc == P.nk - 1;
    // park the accumulators as red[token][row]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int tk = nt * 8 + 2 * c;
      red[tk * kDecTileRows + row0] = acc[nt][0] + acc2[nt][0];
      red[(tk + 1) * kDecTileRows + row0] = acc[nt][1] + acc2[nt][1];
      red[tk * kDecTileRows + row0 + 8] = acc[nt][2] + acc2[nt][2];
      red[(tk + 1) * kDecTileRows + row0 + 8] = acc[nt][3] + acc2[nt][3];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[nt][q] = acc2[nt][q] = 0.0f;
    }
    consumer_sync();
    const int tid = threadIdx.x;   // 0 .. 511
    const int64_t n0 = tile * kDecTileRows;
    const int64_t per_slot = int64_t(a.M) * kDecTileRows;
    bool finalize = whole;
    int64_t pa = p, pb = p;
    if (!whole) {
      // leave this CTA's partial, then count the contributors that are done
      const int slot = first_segment ? 0 : 1;
      float* mine = a.partial + (p * 2 + slot) * per_slot;
      for (int64_t e = tid; e < per_slot; e += kDecWarps * 32) mine[e] = red[e];
      __threadfence();
      consumer_sync();
      pa = unit_owner(tile * P.nk, P.units, NP);
      pb = unit_owner(tile * P.nk + P.nk - 1, P.units, NP);
      if (tid == 0) {
        const int prev = atomicAdd(a.counters + tile, 1);
        *bcast = (prev == int(pb - pa)) ? 1 : 0;
      }
      consumer_sync();
      finalize = *bcast != 0;
      if (finalize) __threadfence();
    }
    if (finalize) {
      if (!have_T) {   // T comes from the previous kernel of the stream
        griddep_wait();
        have_T = true;
      }
      // this thread's outputs: e = tid + 512 j (token e / 256, row e % 256)
      constexpr int kPer = 16 * kDecTileRows / (kDecWarps * 32);   // 8
      float v[kPer];
#pragma unroll
      for (int jj = 0; jj < kPer; ++jj) {
        const int64_t e = tid + int64_t(jj) * (kDecWarps * 32);
        v[jj] = (whole && e < per_slot) ? red[e] : 0.0f;
      }
      if (!whole) {   // contributors in CTA order: a fixed summation order
        for (int64_t q = pa; q <= pb; ++q) {
          const int slot = unit_begin(q, P.units, NP) >= tile * P.nk ? 0 : 1;
          const float* part = a.partial + (q * 2 + slot) * per_slot;
#pragma unroll
          for (int jj = 0; jj < kPer; ++jj) {
            const int64_t e = tid + int64_t(jj) * (kDecWarps * 32);
            if (e < per_slot) v[jj] += __ldcg(part + e);
          }
        }
      }
#pragma unroll
      for (int jj = 0; jj < kPer; ++jj) {
        const int64_t e = tid + int64_t(jj) * (kDecWarps * 32);
        const int tk = int(e / kDecTileRows), row = int(e % kDecTileRows);
        const int64_t n = n0 + row;
        if (e >= per_slot || n >= a.N) continue;
        float lr = 0.0f;
        for (int j = 0; j < a.r; ++j)
          lr = fmaf(half_lo_to_f32(F16, a.T[int64_t(tk) * a.r + j]), half_lo_to_f32(F16, a.B[int64_t(j) * a.N + n]),
                    lr);
        a.Y[int64_t(tk) * a.N + n] = uint16_t(pack2(F16, fmaf(a.s, lr, v[jj]), 0.0f) & 0xFFFFu);
      }
      if (!whole && tid == 0) a.counters[tile] = 0;   // ready for the next call
    }
    consumer_sync();   // red is reused by the next segment
    first_segment = false;
    seg_first_kc = 0;
    if (kc + 1 == P.nk) {
      ++tile;
      kc = 0;
    } else {
      ++kc;
    }
  }
  if (!have_T) griddep_wait();   // complete only after the previous kernel
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

bool decode_supported(int64_t M, int64_t K) { return M >= 1 && M <= 16 && K % kBlock == 0; }

DecodePlan plan_decode(int64_t M, int64_t N, int64_t K, int num_sms) {
  DecodePlan d{};
  d.tiles = cdiv(N, kDecTileRows);
  d.nk = cdiv(K, kDecChunk);
  d.units = d.tiles * d.nk;
  d.ctas = d.units < num_sms ? d.units : num_sms;
  d.partial_floats = d.ctas * 2 * M * kDecTileRows;
  return d;
}

uint32_t decode_xrows(int64_t M) { return uint32_t(cdiv(M, 8)) * 8u + 6u; }
uint32_t decode_xbox_bytes(int64_t M) { return uint32_t(cdiv(decode_xrows(M) * 128, 1024)) * 1024u; }

size_t decode_smem_bytes(int64_t M) {
  const uint32_t xbox = decode_xbox_bytes(M);
  const size_t stage = kPkBytes + 4 * size_t(xbox);
  return 1024 + kDecStages * stage + 16 * kDecTileRows * 4 + 2 * kDecStages * 8 + 16;
}

cudaError_t launch_nf4_decode(const DecodePlan& plan, const Nf4DecodeArgs& a, const float code[16],
                              cudaStream_t stream, bool pdl) {
  if (!decode_supported(a.M, a.K)) return cudaErrorInvalidValue;
  DecodeParams P;
  memset(&P, 0, sizeof(P));
  P.a = a;
  for (int i = 0; i < 16; ++i) P.code.v[i] = code[i];
  P.tiles = plan.tiles;
  P.nk = plan.nk;
  P.units = plan.units;
  P.km = make_shift_muls();
  P.xrows = decode_xrows(a.M);
  P.xbox_bytes = decode_xbox_bytes(a.M);
  P.stage_bytes = kPkBytes + 4 * P.xbox_bytes;
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;   // 2-byte elements (bf16 or fp16)
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  const uint64_t M = a.M, N = a.N, K = a.K;
  bool ok = encode_tmap_2d(&P.tm_pk, U8, a.packed, K / 2, N, K / 2, 128, kDecTileRows, SW);
  ok &= encode_tmap_2d(&P.tm_x, BF, a.X, K, M, K * 2, 64, P.xrows, SW);
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = decode_smem_bytes(a.M);
  void (*kern)(const DecodeParams);
  if (a.f16) kern = a.M > 8 ? nf4_decode_kernel<true, 2> : nf4_decode_kernel<true, 1>;
  else kern = a.M > 8 ? nf4_decode_kernel<false, 2> : nf4_decode_kernel<false, 1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(plan.ctas));
  cfg.blockDim = dim3(kDecThreads);
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
