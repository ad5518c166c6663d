// merge.cu -- merging the LoRA adapter into the frozen weight for serving:
//
//     W' = round(Wd + s (A B)^T),   Wd = dequant(packed, scale1, scale2),
//
// "QLoRA 原理精讲" §2.5 (after merging, the weights are BF16 again and
// inference runs at the original speed) and §三 误区3 (deployment path ②:
// merge the adapter back, then re-quantize for inference).
//
// Per element: wd = round(fp32(code[q] * scale1')) exactly as the standalone
// dequantization; p = sum_j A[k,j] B[j,n] in fp32 on the tensor cores (exact
// products, fp32 accumulation); v = fma(s, p, wd) in fp32; W' = round(v) to
// the compute type.  The bound is HBM: 0.5 byte of packed code read and the
// 2-byte result written per weight; the rank-r product adds 2 r flops per
// weight, which the tensor cores absorb.
//
// Two kernels.  nf4_merge_tc_kernel takes the common shapes (K a multiple of
// 64, so every NF4 block lies in one row; N and r multiples of 8, so rows of
// A and B can be TMA boxes): p on the tensor cores (tcgen05) and one row of
// the tile per thread in the epilogue; see the kernel.  nf4_merge_kernel
// takes every other shape: one CTA per 128 x 128 tile, 8 warps; B^T and A
// slices staged in shared memory (zero padded), each warp forms a 32 x 64
// part of p with ldmatrix + mma.sync, the whole tile of p is parked in
// shared memory, and the epilogue walks each row in 8-column pieces of
// element loads and stores.
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include "common.cuh"
#include "kernels.h"
#include "nf4_lut.cuh"

namespace nf4 {
namespace {

constexpr int kMergeThreads = 256;
constexpr int kTile = 128;             // rows and columns of W per CTA
constexpr int kPStride = kTile + 4;    // floats per row of the parked product

struct MergeParams {
  MergeArgs a;
  float code[16];
  int rp;                              // r rounded up to 16
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

template <bool F16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

template <bool F16>
__global__ void __launch_bounds__(kMergeThreads, 3) nf4_merge_kernel(const __grid_constant__ MergeParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  const MergeArgs& a = P.a;
  const int rp = P.rp;
  const int srow = (rp + 8) * 2;                 // bytes per staged operand row (ldmatrix conflict-free)
  uint8_t* bt_s = smem;                          // B^T slice [128 rows of W][rp]
  uint8_t* a_s = smem + kTile * srow;            // A slice   [128 columns of W][rp]
  float* p_s = reinterpret_cast<float*>(smem);   // parked product [128][kPStride], after the MMAs
  __shared__ float code_s[16];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t k0 = int64_t(blockIdx.x) * kTile;
  const int64_t n0 = int64_t(blockIdx.y) * kTile;
  if (tid < 16) code_s[tid] = P.code[tid];

  // ---- stage the operand slices (zero padded past r, N and K), four 16-byte
  // loads in flight per thread
  const int jc = rp / 8;                         // 8-wide chunks per operand row
  for (int i0 = tid; i0 < kTile * jc; i0 += 4 * kMergeThreads) {   // A[k0 + row][8c .. 8c+7]
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kMergeThreads;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (i >= kTile * jc) continue;
      const int row = i / jc, c = i % jc;
      const int64_t k = k0 + row;
      if (k >= a.K) continue;
      const uint16_t* src = a.A + k * a.r + c * 8;
      if (c * 8 + 8 <= a.r && (a.r % 8) == 0) {
        v[u] = __ldg(reinterpret_cast<const uint4*>(src));
      } else {
        uint32_t t[4] = {0u, 0u, 0u, 0u};
        for (int j = 0; j < 8; ++j)
          if (c * 8 + j < a.r) t[j >> 1] |= uint32_t(src[j]) << (16 * (j & 1));
        v[u] = make_uint4(t[0], t[1], t[2], t[3]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kMergeThreads;
      if (i < kTile * jc) *reinterpret_cast<uint4*>(a_s + (i / jc) * srow + (i % jc) * 16) = v[u];
    }
  }
  // B's slice goes in transposed: thread (c, jp) loads 8 columns of rows 2jp
  // and 2jp + 1 and writes them as 32-bit pairs down the rows of B^T, so the
  // lanes of a warp write neighbouring words of one B^T row (no bank conflicts)
  constexpr int nc = kTile / 8;                  // 8-wide chunks of a row of B's slice
  const int jp_n = rp / 2;
  for (int i0 = tid; i0 < nc * jp_n; i0 += 2 * kMergeThreads) {
    uint4 v[2][2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + u * kMergeThreads;
      const int c = i / jp_n, jp = i % jp_n;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = 2 * jp + h;
        v[u][h] = make_uint4(0u, 0u, 0u, 0u);
        if (i >= nc * jp_n || j >= a.r) continue;
        const int64_t nb = n0 + c * 8;
        const uint16_t* src = a.B + int64_t(j) * a.N + nb;
        if (nb + 8 <= a.N && (a.N % 8) == 0) {
          v[u][h] = __ldg(reinterpret_cast<const uint4*>(src));
        } else {
          uint32_t t[4] = {0u, 0u, 0u, 0u};
          for (int q = 0; q < 8; ++q)
            if (nb + q < a.N) t[q >> 1] |= uint32_t(src[q]) << (16 * (q & 1));
          v[u][h] = make_uint4(t[0], t[1], t[2], t[3]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + u * kMergeThreads;
      if (i >= nc * jp_n) continue;
      const int c = i / jp_n, jp = i % jp_n;
      const uint32_t w0[4] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w};
      const uint32_t w1[4] = {v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t lo = (w0[q >> 1] >> (16 * (q & 1))) & 0xFFFFu, hi = (w1[q >> 1] >> (16 * (q & 1))) & 0xFFFFu;
        *reinterpret_cast<uint32_t*>(bt_s + (c * 8 + q) * srow + jp * 4) = lo | (hi << 16);
      }
    }
  }
  __syncthreads();

  // ---- p = B^T A^T over the rank: warp (wn, wk) owns rows wn*32.. and columns wk*64..
  const int wn = warp & 3, wk = warp >> 2;
  float acc[2][8][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[mt][nt][q] = 0.0f;
  const uint32_t bt_base = smem_u32(bt_s), a_base = smem_u32(a_s);
  for (int kk = 0; kk < rp / 16; ++kk) {
    uint32_t af[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const int row = wn * 32 + mt * 16 + (lane & 15);
      const int col = kk * 16 + (lane >> 4) * 8;
      ldsm_x4(bt_base + row * srow + col * 2, af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
    }
#pragma unroll
    for (int np = 0; np < 4; ++np) {               // pairs of 8-column MMA tiles
      const int row = wk * 64 + np * 16 + (lane & 7) + ((lane >> 4) << 3);
      const int col = kk * 16 + ((lane >> 3) & 1) * 8;
      uint32_t b0, b1, b2, b3;
      ldsm_x4(a_base + row * srow + col * 2, b0, b1, b2, b3);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        mma16816<F16>(acc[mt][2 * np], af[mt], b0, b1);
        mma16816<F16>(acc[mt][2 * np + 1], af[mt], b2, b3);
      }
    }
  }
  __syncthreads();                                  // operand slices are dead: park p over them
  {
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int row = wn * 32 + mt * 16 + g;
        const int col = wk * 64 + nt * 8 + 2 * c;
        *reinterpret_cast<float2*>(p_s + row * kPStride + col) = make_float2(acc[mt][nt][0], acc[mt][nt][1]);
        *reinterpret_cast<float2*>(p_s + (row + 8) * kPStride + col) = make_float2(acc[mt][nt][2], acc[mt][nt][3]);
      }
  }
  __syncthreads();

  // ---- the epilogue's packed codes and block constants, all eight pieces'
  // loads in flight at once (after the MMAs, so that the accumulators and
  // these registers are never live together: three CTAs fit an SM).  Thread
  // tid handles the 8-column piece pc = tid % 16 of rows tid / 16 + 16 j.
  const bool vec = (a.K % 8) == 0;
  const int pc = tid & 15;
  constexpr int kPieces = kTile * (kTile / 8) / kMergeThreads;   // 8
  uint32_t pw[kPieces];
  float ps[kPieces];
  if (vec) {
#pragma unroll
    for (int j = 0; j < kPieces; ++j) {
      const int64_t n = n0 + (tid >> 4) + 16 * j;
      const int64_t k = k0 + pc * 8;
      pw[j] = 0u;
      ps[j] = 0.0f;
      if (n < a.N && k < a.K) {
        const int64_t e0 = n * a.K + k;
        pw[j] = __ldcs(reinterpret_cast<const unsigned int*>(a.packed + (e0 >> 1)));
        ps[j] = block_scale(a.double_quant, a.c1, a.c2, e0 >> 6);
      }
    }
  }

  // ---- epilogue: W' = round(fma(s, p, wd)), 8 columns of one row per piece
  if (vec) {
    // K % 8 == 0: the 8 weights of a piece share one packed word and one block
#pragma unroll
    for (int j = 0; j < kPieces; ++j) {
      const int row = (tid >> 4) + 16 * j;
      const int64_t n = n0 + row;
      const int64_t k = k0 + pc * 8;
      if (n >= a.N || k >= a.K) continue;
      const float* pr = p_s + row * kPStride + pc * 8;
      const uint32_t w = pw[j];
      uint32_t o[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float wd0 = round_to(F16, code_s[(w >> (8 * h)) & 0xFu] * ps[j]);
        const float wd1 = round_to(F16, code_s[(w >> (8 * h + 4)) & 0xFu] * ps[j]);
        o[h] = pack2(F16, fmaf(a.s, pr[2 * h], wd0), fmaf(a.s, pr[2 * h + 1], wd1));
      }
      __stcs(reinterpret_cast<uint4*>(a.out + n * a.K + k), make_uint4(o[0], o[1], o[2], o[3]));
    }
  } else {
    for (int i = tid; i < kTile * (kTile / 8); i += kMergeThreads) {
      const int row = i >> 4, pcc = i & 15;
      const int64_t n = n0 + row;
      const int64_t k = k0 + pcc * 8;
      if (n >= a.N || k >= a.K) continue;
      const float* pr = p_s + row * kPStride + pcc * 8;
      for (int q = 0; q < 8 && k + q < a.K; ++q) {
        const int64_t e = n * a.K + k + q;
        const uint32_t byte = a.packed[e >> 1];
        const uint32_t code = (e & 1) ? (byte >> 4) : (byte & 0xFu);
        const float wd = round_to(F16, code_s[code] * block_scale(a.double_quant, a.c1, a.c2, e >> 6));
        a.out[e] = uint16_t(pack2(F16, fmaf(a.s, pr[q], wd), 0.0f) & 0xFFFFu);
      }
    }
  }
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ---------------------------------------------------------------------------
// nf4_merge_tc_kernel: p on the tensor cores (tcgen05, accumulator in tensor
// memory), the epilogue one row per thread.
//
// One CTA per 128 (rows of W) x 128 (columns) tile, 4 warps.  One thread
// loads by TMA, per 64 ranks, the B slice as two rank-major boxes [64 ranks x
// 64 rows of W] (the MMA's A operand, MN-major) and the A slice [128 columns
// x 64 ranks] (its B operand, K-major), both with the 128-byte swizzle (ranks
// past r read as zeros), and issues p[128 x 128] = B^T A^T as M128 N128 K16
// MMAs into 128 tensor-memory columns.  Meanwhile every thread loads the
// packed codes (64 bytes) and the two block constants of its row: warp w owns
// tensor-memory lanes 32w .. 32w + 31, i.e. rows 32w + lane.  Per NF4 block a
// thread then reads its row's 64 values of p (two 32-column loads), decodes
// the block's 64 codes with its 16-entry table, forms round(fma(s, p, wd)),
// and writes the 128-byte row piece into a 128-byte-swizzled TMA tile that
// leaves as one TMA store per warp and block.  The waits are bounded: a lost
// arrival leaves the output unspecified instead of hanging.
constexpr int kTcThreads = 128;
constexpr int kTcTile = 128;
constexpr uint32_t kTcStage = 4 * 2 * 4096;   // per warp and block a 32-row x 128-byte tile
constexpr uint32_t kTcChunk = 32768;          // per 64 ranks: B slice 2 x 8 KB, A slice 16 KB

struct MergeTcParams {
  MergeArgs a;
  CodeTable code;
  ShiftMuls km;
  CUtensorMap tm_b;     // B [r x N], box {64 columns, 64 ranks}, 128-byte swizzle
  CUtensorMap tm_a;     // A [K x r], box {64 ranks, 128 rows}, 128-byte swizzle
  CUtensorMap tm_out;   // out [N x K], box {64, 32}, 128-byte swizzle
  int nch;              // 64-rank chunks: ceil(r / 64)
  int64_t ktiles;
};

template <bool F16>
__global__ void __launch_bounds__(kTcThreads, 1) nf4_merge_tc_kernel(const __grid_constant__ MergeTcParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const MergeArgs& a = P.a;
  uint8_t* stage = smem;
  uint8_t* ops = smem + kTcStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(ops + P.nch * kTcChunk);
  uint64_t* done = full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t nt_i = int64_t(blockIdx.x) / P.ktiles;
  const int64_t n0 = nt_i * kTcTile;
  const int64_t k0 = (int64_t(blockIdx.x) - nt_i * P.ktiles) * kTcTile;

  if (tid == 0) {
    tma_prefetch_desc(&P.tm_b);
    tma_prefetch_desc(&P.tm_a);
    mbar_init(full, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }

  // this thread's row: packed codes of both blocks and their constants,
  // loaded while the operands arrive and the MMAs run
  const int64_t n = n0 + warp * 32 + lane;
  const int64_t kblocks = a.K >> 6;
  uint4 pk[4];
  uint32_t q[2];
  float s2[2];
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    const int64_t k = k0 + 64 * b;
    pk[2 * b] = pk[2 * b + 1] = make_uint4(0u, 0u, 0u, 0u);
    q[b] = 0u;
    s2[b] = 0.0f;
    if (n < a.N && k < a.K) {
      const uint4* src = reinterpret_cast<const uint4*>(a.packed + ((n * a.K + k) >> 1));
      pk[2 * b] = __ldcs(src);
      pk[2 * b + 1] = __ldcs(src + 1);
      load_scale_parts(a.double_quant, a.c1, a.c2, n * kblocks + (k >> 6), q[b], s2[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (elect_one()) {
      const uint32_t bytes = uint32_t(P.nch) * kTcChunk;
      mbar_arrive_expect_tx(full, bytes);
      for (int ch = 0; ch < P.nch; ++ch) {
        uint8_t* o = ops + ch * kTcChunk;
        tma_load_2d(o, &P.tm_b, full, int32_t(n0), int32_t(64 * ch));
        tma_load_2d(o + 8192, &P.tm_b, full, int32_t(n0 + 64), int32_t(64 * ch));
        tma_load_2d(o + 16384, &P.tm_a, full, int32_t(64 * ch), int32_t(k0));
      }
      const bool ok = mbar_wait(full, 0u, nullptr, abort_flag);
      if (ok) {
        tc_fence_after();
        const uint32_t idesc = make_idesc(128, 128, 1, 0, F16);
        for (int ch = 0; ch < P.nch; ++ch) {
          const uint32_t o = smem_u32(ops + ch * kTcChunk);
          mma_ss_k64(tmem_base, make_sdesc_sw128(o, 8192, 1024), 128u, make_sdesc_sw128(o + 16384, 16, 1024), 2u,
                     idesc, ch > 0 ? 1u : 0u);
        }
      }
      mma_commit(done);   // arrives once the MMAs above are complete (at once if none)
      if (!ok) {          // let the loads land before the CTA exits
        const long long t0 = clock64();
        while (!mbar_try_wait(full, 0u) && clock64() - t0 < 200000000ll) {
        }
      }
    }
    __syncwarp();
  }

  // warp-uniform: the tensor-memory loads below are collective
  const bool ok = __all_sync(0xffffffffu, mbar_wait(done, 0u, nullptr, abort_flag) && !*abort_flag);
  tc_fence_after();
  if (ok && n0 + warp * 32 < a.N) {
    const uint32_t taddr = tmem_base + (uint32_t(warp * 32) << 16);
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      if (k0 + 64 * b >= a.K) break;
      const BlockTable t = make_table(P.code, scale_from_parts(a.double_quant, q[b], s2[b]), F16);
      uint8_t* tile = stage + (warp * 2 + b) * 4096;
      const uint32_t row = smem_u32(tile) + uint32_t(lane) * 128u;
      const uint32_t w[8] = {pk[2 * b].x, pk[2 * b].y, pk[2 * b].z, pk[2 * b].w,
                             pk[2 * b + 1].x, pk[2 * b + 1].y, pk[2 * b + 1].z, pk[2 * b + 1].w};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + uint32_t(64 * b + 32 * h), v);   // columns 64b + 32h .. + 31 of p
#pragma unroll
        for (int i = 0; i < 4; ++i) {   // word 4h + i: columns 8 (4h + i) .. + 7
          uint32_t o[4];
          lookup8(t, w[4 * h + i], P.km, o[0], o[1], o[2], o[3]);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            o[e] = pack2(F16, fmaf(a.s, __uint_as_float(v[8 * i + 2 * e]), half_lo_to_f32(F16, o[e])),
                         fmaf(a.s, __uint_as_float(v[8 * i + 2 * e + 1]), half_hi_to_f32(F16, o[e])));
          const uint32_t chunk = uint32_t(4 * h + i) ^ uint32_t(lane & 7);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(row + (chunk << 4)), "r"(o[0]), "r"(o[1]),
                       "r"(o[2]), "r"(o[3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();   // generic-proxy writes, read next by the TMA engine
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&P.tm_out, tile, int32_t(k0 + 64 * b), int32_t(n0 + warp * 32));
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 128);
  }
}

size_t merge_tc_smem_bytes(int nch) { return 1024 + size_t(kTcStage) + size_t(nch) * kTcChunk + 32; }

}  // namespace

size_t merge_smem_bytes(int r) {
  const int rp = (r + 15) / 16 * 16;
  const size_t operands = size_t(2) * kTile * (rp + 8) * 2;
  const size_t parked = size_t(kTile) * kPStride * 4;
  return operands > parked ? operands : parked;
}

cudaError_t launch_merge(const MergeArgs& a, const float code[16], cudaStream_t stream) {
  const int64_t tc_ktiles = (a.K + kTcTile - 1) / kTcTile;
  const int64_t tc_tiles = tc_ktiles * ((a.N + kTcTile - 1) / kTcTile);
  if (a.K % 64 == 0 && a.N % 8 == 0 && a.r % 8 == 0 && a.K < (int64_t(1) << 31) && a.N < (int64_t(1) << 31) &&
      tc_tiles < (int64_t(1) << 31)) {
    MergeTcParams P;
    memset(&P, 0, sizeof(P));
    P.a = a;
    for (int i = 0; i < 16; ++i) P.code.v[i] = code[i];
    P.km = make_shift_muls();
    P.nch = (a.r + 63) / 64;
    P.ktiles = tc_ktiles;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;   // 2-byte elements (bf16 or fp16)
    const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
    bool ok = encode_tmap_2d(&P.tm_b, BF, a.B, uint64_t(a.N), uint64_t(a.r), uint64_t(a.N) * 2, 64, 64, SW);
    ok &= encode_tmap_2d(&P.tm_a, BF, a.A, uint64_t(a.r), uint64_t(a.K), uint64_t(a.r) * 2, 64, 128, SW);
    ok &= encode_tmap_2d(&P.tm_out, BF, a.out, uint64_t(a.K), uint64_t(a.N), uint64_t(a.K) * 2, 64, 32, SW);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = merge_tc_smem_bytes(P.nch);
    void (*kern)(const MergeTcParams) = a.f16 ? nf4_merge_tc_kernel<true> : nf4_merge_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    kern<<<unsigned(tc_tiles), kTcThreads, smem, stream>>>(P);
    return cudaGetLastError();
  }
  MergeParams P;
  P.a = a;
  for (int i = 0; i < 16; ++i) P.code[i] = code[i];
  P.rp = (a.r + 15) / 16 * 16;
  const size_t smem = merge_smem_bytes(a.r);
  void (*kern)(const MergeParams) = a.f16 ? nf4_merge_kernel<true> : nf4_merge_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(unsigned((a.K + kTile - 1) / kTile), unsigned((a.N + kTile - 1) / kTile));
  kern<<<grid, kMergeThreads, smem, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace nf4
