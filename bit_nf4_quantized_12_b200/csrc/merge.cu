// merge.cu -- merging the LoRA adapter into the frozen weight for serving:
//
//     W' = round(Wd + s (A B)^T),   Wd = dequant(packed, scale1, scale2),
//
// "QLoRA 原理精讲" §2.5 (after merging, the weights are BF16 again and
// inference runs at the original speed) and §三 误区3 (deployment path ②:
// merge the adapter back, then re-quantize for inference).
//
// Per element: wd = round(fp32(code[q] * scale1')) exactly as the standalone
// dequantization; p = sum_j A[k,j] B[j,n] in fp32 on the tensor cores
// (mma.sync m16n8k16, exact products, fp32 accumulation); v = fma(s, p, wd)
// in fp32; W' = round(v) to the compute type.  The kernel is bound by HBM:
// it reads 0.5 byte of packed code per weight and writes the 2-byte result;
// the rank-r product adds 2 r flops per weight, which the tensor cores absorb.
//
// Two kernels.  nf4_merge_frag_kernel takes the common shapes (K a multiple
// of 64, so every NF4 block lies in one row; N and r multiples of 8, so rows
// of A and B are 16-byte aligned); nf4_merge_kernel takes every other shape.
//
// nf4_merge_frag_kernel: one CTA per 64 (rows of W) x 128 (columns) tile, 4
// warps, each owning 32 rows x 64 columns -- one NF4 block per row.  The
// tile's B slice [r x 64], A slice [128 x r] and packed codes arrive by
// cp.async; p is formed 16 rows at a time with ldmatrix (.trans for B, which
// is stored rank-major) and mma.sync, and the epilogue runs on the MMA
// fragments where they are: a thread holds columns 2c, 2c+1 of each 8-column
// tile of a row, i.e. byte c of each of the block's eight packed words, so
// three byte permutes gather its 16 codes into two words and the block's
// 16-entry table (byte permutes, as in the fused GEMM) decodes them.  The
// results go to shared memory by stmatrix in the 128-byte-swizzled layout of
// a TMA tile and leave as one TMA store per warp (rows and columns past the
// weight are not written).
//
// nf4_merge_kernel: one CTA per 128 x 128 tile, 8 warps; B^T and A slices
// staged in shared memory (zero padded), each warp forms a 32 x 64 part of p
// with ldmatrix + mma.sync, the whole tile of p is parked in shared memory,
// and the epilogue walks each row in 8-column pieces of element loads and
// stores.
#include <cstdint>
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

// ---------------------------------------------------------------------------
// nf4_merge_frag_kernel
constexpr int kFragThreads = 128;
constexpr int kFragRows = 64;           // rows of W per CTA
constexpr int kFragCols = 128;          // columns of W per CTA (two NF4 blocks per row)
constexpr int kFragStage = 4 * 4096;    // per warp a 32-row x 128-byte swizzled TMA tile
constexpr int kFragBRow = kFragRows * 2 + 16;   // bytes per staged B row (ldmatrix conflict-free)
constexpr int kFragPkRow = 80;          // bytes per staged row of packed codes (64 + 16)

struct MergeFragParams {
  MergeArgs a;
  CodeTable code;
  ShiftMuls km;
  CUtensorMap tm_out;                   // out [N x K], 2-byte elements, box {64, 32}, 128-byte swizzle
  int rp;                               // r rounded up to 16
  uint32_t a_chunks;                    // 16-byte chunks per staged A row (rp / 8)
  uint32_t a_magic;                     // ceil(2^32 / a_chunks): exact quotients for indices < 2^16
  int64_t ktiles;                       // column tiles per row of tiles
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void stsm_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r0), "r"(r1),
               "r"(r2), "r"(r3)
               : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

template <bool F16>
__global__ void __launch_bounds__(kFragThreads, 4) nf4_merge_frag_kernel(const __grid_constant__ MergeFragParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const MergeArgs& a = P.a;
  const int rp = P.rp;
  const int a_row = rp * 2 + 16;                     // bytes per staged A row (ldmatrix conflict-free)
  uint8_t* stage = smem;                             // 4 x 4 KB TMA tiles
  uint8_t* bs = stage + kFragStage;                  // B slice [rp][64 columns of out's rows]
  uint8_t* as = bs + rp * kFragBRow;                 // A slice [128 columns of W][rp]
  uint8_t* pk = as + kFragCols * a_row;              // packed codes [64 rows][64 bytes]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t nt_i = int64_t(blockIdx.x) / P.ktiles;
  const int64_t n0 = nt_i * kFragRows;
  const int64_t k0 = (int64_t(blockIdx.x) - nt_i * P.ktiles) * kFragCols;

  // ---- stage the B slice, the A slice and the packed codes (zero fill past
  // r, N and K)
  const uint32_t bs_u = smem_u32(bs), as_u = smem_u32(as), pk_u = smem_u32(pk);
  for (int i = tid; i < rp * 8; i += kFragThreads) {         // B[j][n0 + 8c .. + 7]
    const int j = i >> 3, c = i & 7;
    const int64_t n = n0 + 8 * c;
    const bool ok = j < a.r && n < a.N;
    cp_async16(bs_u + j * kFragBRow + c * 16, ok ? a.B + int64_t(j) * a.N + n : a.B, ok ? 16u : 0u);
  }
  for (int i = tid; i < kFragCols * int(P.a_chunks); i += kFragThreads) {   // A[k0 + row][8c .. 8c + 7]
    const int row = int(__umulhi(uint32_t(i), P.a_magic));
    const int c = i - row * int(P.a_chunks);
    const int64_t k = k0 + row;
    const bool ok = 8 * c < a.r && k < a.K;
    cp_async16(as_u + row * a_row + c * 16, ok ? a.A + k * a.r + 8 * c : a.A, ok ? 16u : 0u);
  }
  for (int i = tid; i < kFragRows * 4; i += kFragThreads) {   // row n0 + row, columns k0 + 32c .. + 31
    const int row = i >> 2, c = i & 3;
    const int64_t n = n0 + row, k = k0 + 32 * c;
    const bool ok = n < a.N && k < a.K;
    cp_async16(pk_u + row * kFragPkRow + c * 16, ok ? a.packed + ((n * a.K + k) >> 1) : a.packed, ok ? 16u : 0u);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");

  // ---- this thread's four block constants (rows g, g + 8 of each 16-row half)
  const int wn = warp & 1, wk = warp >> 1;
  const int g = lane >> 2, c = lane & 3;
  const int64_t kb = k0 + wk * 64;                   // the warp's NF4 block column
  const int64_t kblocks = a.K >> 6;
  uint32_t q[4];
  float s2[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t n = n0 + wn * 32 + (u >> 1) * 16 + (u & 1) * 8 + g;
    q[u] = 0u;
    s2[u] = 0.0f;
    if (n < a.N && kb < a.K) load_scale_parts(a.double_quant, a.c1, a.c2, n * kblocks + (kb >> 6), q[u], s2[u]);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  if (kb >= a.K || n0 + wn * 32 >= a.N) return;      // the warp's tile lies past the weight

  const uint32_t st_u = smem_u32(stage + warp * 4096);
  const uint32_t sel = uint32_t(c) | (uint32_t(c + 4) << 4);   // byte c of two words
#pragma unroll 1
  for (int mt = 0; mt < 2; ++mt) {
    float acc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
    const int mrow = wn * 32 + mt * 16;              // first row of W (in the tile) of this half
    for (int kk = 0; kk < rp / 16; ++kk) {
      // A operand (rows of W x rank) from B stored rank-major: matrix i of
      // the four is rank 8 (i >> 1) .. + 7 by rows 8 (i & 1) .. + 7
      uint32_t af[4];
      {
        const int i = lane >> 3;
        const int j = kk * 16 + (i >> 1) * 8 + (lane & 7);
        ldsm_x4_trans(bs_u + j * kFragBRow + (mrow + (i & 1) * 8) * 2, af[0], af[1], af[2], af[3]);
      }
#pragma unroll
      for (int np = 0; np < 4; ++np) {               // pairs of 8-column tiles
        const int row = wk * 64 + np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int col = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(as_u + row * a_row + col * 2, b0, b1, b2, b3);
        mma16816<F16>(acc[2 * np], af, b0, b1);
        mma16816<F16>(acc[2 * np + 1], af, b2, b3);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = mrow + h * 8 + g;
      const uint32_t qu = mt ? q[2 + h] : q[h];   // selects: the arrays stay in registers
      const float s2u = mt ? s2[2 + h] : s2[h];
      const BlockTable t = make_table(P.code, scale_from_parts(a.double_quant, qu, s2u), F16);
      const uint32_t src = pk_u + row * kFragPkRow + wk * 32;
      const uint4 lo = lds128(src), hi = lds128(src + 16);
      // byte c of each of the block's eight words: columns 8 nt + 2c, + 1
      const uint32_t w0 = prmt(prmt(lo.x, lo.y, sel), prmt(lo.z, lo.w, sel), 0x5410u);
      const uint32_t w1 = prmt(prmt(hi.x, hi.y, sel), prmt(hi.z, hi.w, sel), 0x5410u);
      uint32_t o[8];
      lookup8(t, w0, P.km, o[0], o[1], o[2], o[3]);
      lookup8(t, w1, P.km, o[4], o[5], o[6], o[7]);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
        o[nt] = pack2(F16, fmaf(a.s, acc[nt][2 * h], half_lo_to_f32(F16, o[nt])),
                      fmaf(a.s, acc[nt][2 * h + 1], half_hi_to_f32(F16, o[nt])));
      // rows mt 16 + h 8 + 0..7 of the warp's tile; 16-byte chunk nt of a row
      // sits at chunk nt ^ (row & 7) (128-byte swizzle)
      const uint32_t lrow = uint32_t(mt * 16 + h * 8 + (lane & 7));
      const uint32_t rbase = st_u + lrow * 128u;
      const uint32_t ch = uint32_t(lane >> 3);
      stsm_x4(rbase + ((ch ^ (lrow & 7u)) << 4), o[0], o[1], o[2], o[3]);
      stsm_x4(rbase + (((ch + 4u) ^ (lrow & 7u)) << 4), o[4], o[5], o[6], o[7]);
    }
  }
  fence_proxy_async_smem();   // generic-proxy writes, read next by the TMA engine
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(&P.tm_out, stage + warp * 4096, int32_t(kb), int32_t(n0 + wn * 32));
    bulk_commit();
    bulk_wait_all();
  }
}

size_t merge_frag_smem_bytes(int rp) {
  return 1024 + size_t(kFragStage) + size_t(rp) * kFragBRow + size_t(kFragCols) * (rp * 2 + 16) +
         size_t(kFragRows) * kFragPkRow;
}

}  // namespace

size_t merge_smem_bytes(int r) {
  const int rp = (r + 15) / 16 * 16;
  const size_t operands = size_t(2) * kTile * (rp + 8) * 2;
  const size_t parked = size_t(kTile) * kPStride * 4;
  return operands > parked ? operands : parked;
}

cudaError_t launch_merge(const MergeArgs& a, const float code[16], cudaStream_t stream) {
  const int64_t ktiles = (a.K + kFragCols - 1) / kFragCols;
  const int64_t tiles = ktiles * ((a.N + kFragRows - 1) / kFragRows);
  if (a.K % 64 == 0 && a.N % 8 == 0 && a.r % 8 == 0 && a.K < (int64_t(1) << 31) && a.N < (int64_t(1) << 31) &&
      tiles < (int64_t(1) << 31)) {
    MergeFragParams P;
    P.a = a;
    for (int i = 0; i < 16; ++i) P.code.v[i] = code[i];
    P.km = make_shift_muls();
    P.rp = (a.r + 15) / 16 * 16;
    P.a_chunks = uint32_t(P.rp / 8);
    P.a_magic = uint32_t(((uint64_t(1) << 32) + P.a_chunks - 1) / P.a_chunks);
    P.ktiles = ktiles;
    if (!encode_tmap_2d(&P.tm_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.out, uint64_t(a.K), uint64_t(a.N),
                        uint64_t(a.K) * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    const size_t smem = merge_frag_smem_bytes(P.rp);
    void (*kern)(const MergeFragParams) = a.f16 ? nf4_merge_frag_kernel<true> : nf4_merge_frag_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    kern<<<unsigned(tiles), kFragThreads, smem, stream>>>(P);
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
