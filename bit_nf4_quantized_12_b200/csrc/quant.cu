// quant.cu -- NF4 blockwise quantization with double quantization of the
// block constants, and the standalone double dequantization to bf16.
//
// Quantize ("QLoRA 原理精讲" §2.1 示意代码, §2.2 核心机制):
//   scale1_b = max |w| over block b (64 consecutive weights),
//   code     = nearest NF4 value to w / scale1_b (ties to the lower code),
//   scale2_g = max scale1 over group g (256 blocks) / 448 (fp32),
//   c1q_b    = E4M3(scale1_b / scale2_g), round to nearest even, saturating.
// The normalization uses x = w * fp32(1/scale1) (IEEE reciprocal once per
// block, then one multiply per weight) compared with fp32 midpoints rounded
// down.  For every pair of bf16 values this yields the same code as the
// exact quotient (checked exhaustively on the host by the test suite); blocks
// whose absmax lies outside [2^-122, 2^125] are rescaled by a power of two
// first so that 16 / absmax (the cells below work on 16 x) stays a normal
// number.  A power-of-two rescaling leaves the computed x unchanged.
//
// Dequantize ("QLoRA 原理精讲" §2.2, reverse order): scale1' = fp32(E4M3 value
// of c1q * scale2), w' = bf16(fp32(code * scale1')).
//
// Both kernels also take the storage variants (a uniform INT4 table; FP32 or
// unsigned 8-bit first-level constants) and dequantize into fp16 as well as
// bf16: the table, the per-block constant and the final rounding change,
// nothing else.
//
// Both kernels are meant to be HBM-bandwidth bound, so both keep the
// instructions per weight low.  Quantize: 16-byte coalesced loads and
// stores, the per-block absmax by warp shuffles across the 8 lanes that own a
// block, and the code decision as one lookup in a 33-cell shared-memory table
// plus one compare.  Dequantize: one lane per block, the block's 16 values
// formed once and the codes looked up with byte permutes (about 2.3 integer
// operations per weight), the output leaving through TMA tile stores.
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include "common.cuh"
#include "kernels.h"
#include "nf4_lut.cuh"

namespace nf4 {
namespace {

// A CTA of four warps quantizes one group (16384 weights) at a time.  A pass
// is one 16-byte load per lane: 256 weights, four blocks of 8 lanes each.
// Warp w takes passes 16 w .. 16 w + 15 of the group as four batches of 4,
// and within a batch lane j < 4 of each 8-lane block group owns pass j (its
// block's reciprocal is taken once and shuffled to the other lanes).  Small
// batches keep a warp's registers low enough for 8 CTAs per SM, so that the
// 1024 groups of a 4096 x 4096 weight run in one round.
constexpr int kQuantWarps = 4;
constexpr int kQuantThreads = kQuantWarps * 32;
constexpr int kQuantBatch = 4;                                      // passes per batch
constexpr int kPassElems = 32 * 8;                                  // weights per pass
constexpr int kWarpBatches = kGroupElems / (kPassElems * kQuantBatch * kQuantWarps);   // 4
constexpr int kWarpBlocks = kWarpBatches * kQuantBatch * 4;         // blocks per warp and group: 64
constexpr int kQuantCtasPerSm = 8;
static_assert(kWarpBatches * kPassElems * kQuantBatch * kQuantWarps == kGroupElems, "whole batches per group");
constexpr int kCells = 33;           // cells of 16 x: floor(16 x) = -16 .. 16

// Code decision by cells of width 1/16 in x = w / absmax: cell c holds
// x in [(c-16)/16, (c-15)/16).  Consecutive NF4 thresholds are more than
// 0.08 apart (checked on the host), so a cell holds at most one threshold
// and code = #{thresholds below the cell} + (x > that threshold).  The
// comparison is made on 16 x against 16 T, both exact power-of-two scalings
// of the fp32 values, so the decision equals x > T.  Most weights fall in a
// few cells near 0, so the warp's table loads are mostly broadcasts.
__device__ __forceinline__ void build_cells(uint2* cells, const float* thr_smem) {
  for (int c = threadIdx.x; c < kCells; c += blockDim.x) {
    const float lo = float(c - 16) * 0.0625f, hi = float(c - 15) * 0.0625f;
    uint32_t base = 0;
    float t_in = INFINITY;
    for (int i = 0; i < 15; ++i) {
      if (thr_smem[i] < lo) ++base;
      else if (thr_smem[i] < hi) t_in = thr_smem[i] * 16.0f;
    }
    cells[c] = make_uint2(__float_as_uint(t_in), base);
  }
}

// Code decision for any x16, non-finite included: NaN or |x| > 1 (only with
// non-finite input) clamps into an end cell.
__device__ __forceinline__ uint32_t classify16(const uint2* cells, float x16) {
  const uint32_t idx = min(uint32_t(__float2int_rd(x16) + 16), uint32_t(kCells - 1));
  const uint2 e = cells[idx];
  return e.y + (x16 > __uint_as_float(e.x) ? 1u : 0u);
}

// Code decision for finite x16 in [-16, 16] (a block with a normal absmax:
// |w * fp32(1/absmax)| <= 1 holds after rounding).  r = RD(x16 + 2^23 + 16)
// is the integer 2^23 + 16 + floor(x16), so the low bits of its pattern are
// the cell index 0..32: one round-down add on the FMA pipe instead of a
// float-to-int conversion.  cells_biased is the cell table's shared address
// minus 8 * 0x4B000000 (mod 2^32), so the pattern times 8 (one integer
// multiply-add by the runtime constant k8 = 8, on the FMA pipe) addresses the
// cell directly.  The comparison x16 > 16 T is the sign bit of 16 T - x16,
// which is +0 for x16 == 16 T (ties go to the lower code) and +inf where the
// cell holds no threshold.
__device__ __forceinline__ uint32_t mad_lo(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t classify_fast(uint32_t cells_biased, float x16, uint32_t k8) {
  const float r = __fadd_rd(x16, 8388624.0f);
  const uint32_t addr = mad_lo(__float_as_uint(r), k8, cells_biased);
  uint32_t t, base;
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(t), "=r"(base) : "r"(addr));
  return base + (__float_as_uint(__uint_as_float(t) - x16) >> 31);
}

// Code decision with an exact comparison, for tables whose thresholds are
// dyadic (the uniform INT4 table: odd sixteenths).  There w / scale1 can hit a
// threshold exactly, and w * fp32(1/scale1) can then land on either side of
// it; the cell is still taken from the rounded x16 (a neighbouring cell gives
// the same code there), but the comparison w > T scale1 is made exactly: the
// fma forms 16 w - 16T scale1 with the exact product and one rounding, which
// keeps the sign.  c1 is the block absmax (after the same scaling as w).
__device__ __forceinline__ uint32_t classify_exact(const uint2* cells, float x16, float w, float c1) {
  const uint32_t idx = min(uint32_t(__float2int_rd(x16) + 16), uint32_t(kCells - 1));
  const uint2 e = cells[idx];
  return e.y + (fmaf(-__uint_as_float(e.x), c1, w * 16.0f) > 0.0f ? 1u : 0u);
}

// 8 consecutive bf16 (one uint4) -> 8 nibbles (element 0 in bits 0-3);
// inv16 = 16 / scale1 (of the weights first scaled by pre, a power of two,
// on the careful path for extreme or non-finite blocks); c1 = scale1 * pre.
// MODE 0: fast cells (NF4 blocks with a normal scale1); 1: clamped cells (any
// input); 2: exact comparison (dyadic thresholds).  k holds runtime copies of
// 8, 16, 256 and 2^16, so that those products stay integer multiply-adds on
// the FMA pipe (the integer pipe carries the rest of the classification).
struct PackMuls {
  uint32_t k8, k16, k256, k65536;
};
template <int MODE>
__device__ __forceinline__ uint32_t quantize8(const uint2* cells, uint32_t cells_biased, const uint4& v,
                                              float inv16, float pre, float c1,
                                              const PackMuls& k = PackMuls{8u, 16u, 256u, 65536u}) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out = 0;
  if constexpr (MODE == 0) {
    // byte j = lo + 16 hi; bytes 0-1 and 2-3 joined by x 256, the halves by
    // x 2^16: seven multiply-adds for the eight codes, no serial chain
    uint32_t b[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = classify_fast(cells_biased, __uint_as_float(mad_lo(w[j], k.k65536, 0u)) * inv16, k.k8);
      const uint32_t hi = classify_fast(cells_biased, bf16hi_to_f32(w[j]) * inv16, k.k8);
      b[j] = mad_lo(hi, k.k16, lo);
    }
    out = mad_lo(mad_lo(b[3], k.k256, b[2]), k.k65536, mad_lo(b[1], k.k256, b[0]));
  } else {
#pragma unroll
    for (int j = 3; j >= 0; --j) {
      float hi = bf16hi_to_f32(w[j]) * pre, lo = bf16lo_to_f32(w[j]) * pre;
      const float xh = hi * inv16, xl = lo * inv16;
      if (MODE == 1) {
        out = out * 16u + classify16(cells, xh);
        out = out * 16u + classify16(cells, xl);
      } else {
        out = out * 16u + classify_exact(cells, xh, hi, c1);
        out = out * 16u + classify_exact(cells, xl, lo, c1);
      }
    }
  }
  return out;
}

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t u) {
  return *reinterpret_cast<const __nv_bfloat162*>(&u);
}
// Largest |w| of each half of 8 bf16 as a bf16x2 pattern (NaN propagates, so
// Inf/NaN inputs give a pattern >= 0x7F80 in that half).
__device__ __forceinline__ uint32_t absmax_pair8(const uint4& v) {
  const __nv_bfloat162 m = __hmax2_nan(__hmax2_nan(__habs2(as_bf162(v.x)), __habs2(as_bf162(v.y))),
                                       __hmax2_nan(__habs2(as_bf162(v.z)), __habs2(as_bf162(v.w))));
  return *reinterpret_cast<const uint32_t*>(&m);
}
__device__ __forceinline__ uint32_t hmax2_bits(uint32_t a, uint32_t b) {
  const __nv_bfloat162 m = __hmax2_nan(as_bf162(a), as_bf162(b));
  return *reinterpret_cast<const uint32_t*>(&m);
}
// Block maxima of two passes at once: the per-lane maxima of passes i and
// i + 1 are folded into one bf16x2 word (max of pass i in the low half, of
// pass i + 1 in the high half) and reduced over the block's 8 lanes with one
// set of shuffles.  All values are |w| patterns (non-negative), so the bf16
// maximum orders them as their bit patterns do.
__device__ __forceinline__ uint32_t block_absmax2(const uint4& vi, const uint4& vj) {
  const uint32_t mi = absmax_pair8(vi), mj = absmax_pair8(vj);
  uint32_t m = hmax2_bits(prmt(mi, mj, 0x5410u), prmt(mi, mj, 0x7632u));
  m = hmax2_bits(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = hmax2_bits(m, __shfl_xor_sync(0xffffffffu, m, 2));
  m = hmax2_bits(m, __shfl_xor_sync(0xffffffffu, m, 4));
  return m;
}

struct QuantArgs {
  const uint16_t* W;
  int64_t numel;
  uint8_t* packed;
  uint8_t* c1q;        // first-level constants: bytes, or fp32 values for kDqNone
  float* c2;           // unused for kDqNone
  uint32_t* status;
  int64_t ngroups;
  int dq;              // DqFormat
  int exact;           // exact comparisons (tables with dyadic thresholds)
  uint32_t zero8;      // eight nibbles of the table's 0.0 code (all-zero blocks)
  PackMuls km;          // 8, 16, 256 and 2^16 as runtime values (see quantize8)
  float thr[15];
};

// Batch b (0 .. kWarpBatches - 1) of this warp in group g: passes
// P = (kWarpBatches w + b) 4 + i for i = 0..3; pass P covers weights
// P * 256 + lane * 8 .. + 7 of the group.  Elements past the end read as 0.
__device__ __forceinline__ int64_t batch_first(int64_t g, int b) {
  const int warp = threadIdx.x >> 5;
  return g * kGroupElems + int64_t((kWarpBatches * warp + b) * kQuantBatch) * kPassElems;
}
__device__ __forceinline__ void load_batch(const QuantArgs& p, int64_t e_first, uint4 (&v)[kQuantBatch]) {
  const int lane = threadIdx.x & 31;
  if (e_first + kQuantBatch * kPassElems <= p.numel) {   // one base pointer, constant offsets
    const uint4* src = reinterpret_cast<const uint4*>(p.W + e_first) + lane;
#pragma unroll
    for (int i = 0; i < kQuantBatch; ++i) v[i] = __ldcs(src + i * 32);
    return;
  }
#pragma unroll
  for (int i = 0; i < kQuantBatch; ++i) {
    const int64_t e0 = e_first + int64_t(i) * kPassElems + lane * 8;
    if (e0 + 8 <= p.numel) {
      v[i] = __ldcs(reinterpret_cast<const uint4*>(p.W + e0));
    } else {
      uint16_t t[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) t[k] = (e0 + k < p.numel) ? p.W[e0 + k] : uint16_t(0);
      v[i] = make_uint4(t[0] | (uint32_t(t[1]) << 16), t[2] | (uint32_t(t[3]) << 16),
                        t[4] | (uint32_t(t[5]) << 16), t[6] | (uint32_t(t[7]) << 16));
    }
  }
}

// Persistent CTAs walk the groups; each warp loads its next batch (of this
// group or of the CTA's next one) while it classifies the current one.  The
// 4-bit codes depend only on their own block's absmax, so they are written
// before the group's maximum is known; the four warps then meet once per
// group for scale2 and each writes the 8-bit codes of its own 64 blocks.
__global__ void __launch_bounds__(kQuantThreads, kQuantCtasPerSm) nf4_quantize_kernel(const __grid_constant__ QuantArgs p) {
  __shared__ uint2 cells[kCells];
  __shared__ float thr_s[16];
  __shared__ uint32_t warp_max[2][kQuantWarps];
  __shared__ uint32_t keep_s[kQuantWarps][kWarpBlocks];   // block maxima, block order within the warp
  if (threadIdx.x < 15) thr_s[threadIdx.x] = p.thr[threadIdx.x];
  __syncthreads();
  build_cells(cells, thr_s);
  __syncthreads();
  const uint32_t cells_biased = smem_u32(cells) - (0x4B000000u << 3);

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5, j = lane & 7;
  const int64_t nblk_total = nblocks_of(p.numel);
  uint32_t bad = 0;

  int64_t g = blockIdx.x;
  uint4 v[kQuantBatch];
  if (g < p.ngroups) load_batch(p, batch_first(g, 0), v);
  for (int parity = 0; g < p.ngroups; g += gridDim.x, parity ^= 1) {
    uint32_t gm2 = 0;   // group maximum so far, as a bf16x2 pattern
#pragma unroll 1
    for (int b = 0; b < kWarpBatches; ++b) {
      const int64_t e_first = batch_first(g, b);
      // prefetch: the next batch of this group, or the first of the next group
      uint4 vn[kQuantBatch];
      {
        const int64_t gn = (b + 1 < kWarpBatches) ? g : g + gridDim.x;
        if (gn < p.ngroups) load_batch(p, batch_first(gn, (b + 1) % kWarpBatches), vn);
      }
      // first level: absmax of each block (8 lanes x 8 weights)
      uint32_t bm[kQuantBatch];
#pragma unroll
      for (int i = 0; i < kQuantBatch; i += 2) {
        const uint32_t m = block_absmax2(v[i], v[i + 1]);
        bm[i] = m & 0xFFFFu;
        bm[i + 1] = m >> 16;
        gm2 = hmax2_bits(gm2, m);
      }
      uint32_t my_bm = bm[0];   // this lane's pass: i == j (lanes j >= 4: pass 0, unused)
#pragma unroll
      for (int i = 1; i < kQuantBatch; ++i) my_bm = (j == i) ? bm[i] : my_bm;
      if (j < kQuantBatch)   // block 4 j + lane / 8 of the batch
        keep_s[warp][b * (kQuantBatch * 4) + j * 4 + (lane >> 3)] = my_bm;
      const float my_c1 = __uint_as_float(my_bm << 16);
      // 16 / scale1 must stay a finite normal number: scale1 in [2^-122, 2^125]
      const bool normal = (my_c1 >= 0x1p-122f && my_c1 <= 0x1p125f) || my_c1 == 0.0f;
      const float my_inv = (my_c1 == 0.0f) ? 0.0f : (normal ? __frcp_rn(my_c1) : 0.0f);
      const bool fast = __all_sync(0xffffffffu, normal);
      const bool full = e_first + kQuantBatch * kPassElems <= p.numel;
      if (fast && full && !p.exact) {
        // the common case in straight-line code: every block of the batch
        // has a normal (or zero) scale1, no element is past the end and the
        // table's thresholds are not dyadic.  A zero block has inv16 = 0, so
        // x16 = 0 and its codes come out as the 0.0 code of the table.
        const float my_inv16 = my_inv * 16.0f;
        uint32_t* dst = reinterpret_cast<uint32_t*>(p.packed + (e_first >> 1)) + lane;
#pragma unroll
        for (int i = 0; i < kQuantBatch; ++i) {
          const float inv16 = __shfl_sync(0xffffffffu, my_inv16, (lane & ~7) | i);
          __stcs(dst + i * 32, quantize8<0>(cells, cells_biased, v[i], inv16, 1.0f, 0.0f, p.km));
        }
      } else {
#pragma unroll
        for (int i = 0; i < kQuantBatch; ++i) {
          const int64_t e0 = e_first + int64_t(i) * kPassElems + lane * 8;
          const float inv = __shfl_sync(0xffffffffu, my_inv, (lane & ~7) | i);
          if (e0 >= p.numel) continue;
          const float c1 = __uint_as_float(bm[i] << 16);
          uint32_t q8;
          if (c1 == 0.0f) {
            q8 = p.zero8;                            // all-zero block: the 0.0 code
          } else if (p.exact) {                      // dyadic thresholds: exact comparisons
            const bool nrm = c1 >= 0x1p-122f && c1 <= 0x1p125f;
            const float pre = nrm ? 1.0f : ((c1 < 1.0f) ? 0x1p64f : 0x1p-64f);
            q8 = quantize8<2>(cells, cells_biased, v[i], __frcp_rn(c1 * pre) * 16.0f, pre, c1 * pre);
          } else if (fast) {
            q8 = quantize8<0>(cells, cells_biased, v[i], inv * 16.0f, 1.0f, c1, p.km);
          } else if (c1 >= 0x1p-122f && c1 <= 0x1p125f) {
            q8 = quantize8<1>(cells, cells_biased, v[i], __frcp_rn(c1) * 16.0f, 1.0f, c1);
          } else {                                   // keep 16/c1 a normal number
            const float pre = (c1 < 1.0f) ? 0x1p64f : 0x1p-64f;
            q8 = quantize8<1>(cells, cells_biased, v[i], __frcp_rn(c1 * pre) * 16.0f, pre, c1);
          }
          uint8_t* dst = p.packed + (e0 >> 1);
          if (e0 + 8 <= p.numel) {
            __stcs(reinterpret_cast<unsigned int*>(dst), q8);
          } else {
            const int valid = int(p.numel - e0);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              if (2 * jj < valid) {
                uint32_t byte = (q8 >> (8 * jj)) & 0xFFu;
                if (2 * jj + 1 >= valid) byte &= 0x0Fu;   // pad nibble of an odd tail
                dst[jj] = uint8_t(byte);
              }
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kQuantBatch; ++i) v[i] = vn[i];
    }

    // second level: fp32 scale2 of the group (the four warps' maxima), then
    // the 8-bit codes of scale1 / scale2 of this warp's 64 blocks
    uint32_t gm = max(gm2 & 0xFFFFu, gm2 >> 16);
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) gm = max(gm, __shfl_xor_sync(0xffffffffu, gm, o));
    if (lane == 0) warp_max[parity][warp] = gm;
    __syncthreads();
    gm = max(max(warp_max[parity][0], warp_max[parity][1]), max(warp_max[parity][2], warp_max[parity][3]));
    if (gm >= 0x7F80u) bad = 1;
    const float gmax = __uint_as_float(gm << 16);
    const float s2 = __fdiv_rn(gmax, p.dq == kDqU8 ? 255.0f : 448.0f);
    if (tid == 0 && p.dq != kDqNone) p.c2[g] = s2;
#pragma unroll
    for (int k = 0; k < kWarpBlocks / 32; ++k) {
      const int64_t blk = g * kGroup + int64_t(warp) * kWarpBlocks + k * 32 + lane;
      const float c1 = __uint_as_float(keep_s[warp][k * 32 + lane] << 16);
      if (blk < nblk_total) {
        if (p.dq == kDqNone) {
          reinterpret_cast<float*>(p.c1q)[blk] = c1;
        } else if (c1 == 0.0f) {
          p.c1q[blk] = 0;
        } else {
          const float t = __fdiv_rn(c1, s2);
          p.c1q[blk] = uint8_t(p.dq == kDqU8 ? min(__float2uint_rn(t), 255u) : f32_to_e4m3_satfinite(t));
        }
      }
    }
    __syncwarp();   // keep_s is rewritten by other lanes in the next group
  }
  if (bad && p.status != nullptr && tid == 0) atomicOr(p.status, kStatusNonfinite);
}

// ---------------------------------------------------------------- dequantize
struct DequantArgs {
  CUtensorMap tm_out;   // out as [nfull rows x 64] 2-byte, box {64, 32}, 128-byte swizzle
  const uint8_t* packed;
  const uint8_t* c1q;   // first-level constants (bytes, or fp32 for kDqNone)
  const float* c2;
  uint16_t* out;
  int64_t numel;
  int64_t nfull;        // complete 64-weight blocks
  int dq;               // DqFormat
  int f16;              // output fp16 (else bf16)
  CodeTable code;
  ShiftMuls km;
};

// One lane per 64-weight block: the lane loads the block's 32 packed bytes and
// its constants, forms the block's 16 values once (code[q] * scale1 in fp32,
// rounded to bf16 or fp16) and looks the 64 codes up with byte permutes.  A
// warp's 32 blocks (4 KB of output, contiguous in memory) are written into
// shared memory as a 32 x 128-byte tile in the 128-byte swizzle (lane l's
// 16-byte chunk k at position k ^ (l mod 8): no bank conflicts) and leave by
// one TMA store, which also clips the last, partial tile.  The next blocks'
// bytes are loaded before the current ones are decoded.
constexpr int kDqWarps = 8;
__global__ void __launch_bounds__(kDqWarps * 32, 4) nf4_dequant_kernel(const __grid_constant__ DequantArgs p) {
  __shared__ __align__(1024) uint4 stage[kDqWarps][32 * 8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint4* st = stage[warp];
  const int64_t nchunks = (p.nfull + 31) / 32;
  const int64_t nw = int64_t(gridDim.x) * kDqWarps;
  const bool h = p.f16 != 0;
  auto load = [&](int64_t ch, uint4& a, uint4& b, uint32_t& q, float& s2) {
    const int64_t blk = ch * 32 + lane;
    if (ch < nchunks && blk < p.nfull) {
      const uint4* src = reinterpret_cast<const uint4*>(p.packed) + blk * 2;
      a = __ldcs(src);
      b = __ldcs(src + 1);
      load_scale_parts(p.dq, p.c1q, p.c2, blk, q, s2);
    } else {
      a = b = make_uint4(0u, 0u, 0u, 0u);
      q = 0u;
      s2 = 0.0f;
    }
  };
  int64_t ch = int64_t(blockIdx.x) * kDqWarps + warp;
  uint4 a, b;
  uint32_t q;
  float s2;
  load(ch, a, b, q, s2);
  for (; ch < nchunks; ch += nw) {
    uint4 na, nb;
    uint32_t nq;
    float ns2;
    load(ch + nw, na, nb, nq, ns2);
    const BlockTable t = make_table(p.code, scale_from_parts(p.dq, q, s2), h);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    // the previous tile's TMA store must have read the staging buffer
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 8; ++k) {   // 16-byte chunk k: weights 8k .. 8k + 7
      uint4 o;
      lookup8(t, w[k], p.km, o.x, o.y, o.z, o.w);
      st[lane * 8 + (k ^ (lane & 7))] = o;
    }
    fence_proxy_async_smem();   // generic-proxy writes, read next by the TMA engine
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&p.tm_out, st, 0, int32_t(ch * 32));
      bulk_commit();
    }
    a = na;
    b = nb;
    q = nq;
    s2 = ns2;
  }
  if (lane == 0) bulk_wait_all();
  // the last numel % 64 weights (a partial block), one thread
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (int64_t e = p.nfull * kBlock; e < p.numel; ++e) {
      const float sc = block_scale(p.dq, p.c1q, p.c2, e / kBlock);
      const uint32_t byte = p.packed[e >> 1];
      const uint32_t c = (e & 1) ? (byte >> 4) : (byte & 0xFu);
      p.out[e] = uint16_t(pack2(h, p.code.v[c] * sc, 0.0f) & 0xFFFFu);
    }
  }
}

}  // namespace

cudaError_t launch_quantize(const uint16_t* W, int64_t numel, int quant_type, int dq, uint8_t* packed, void* c1,
                            float* c2, uint32_t* status, int num_sms, cudaStream_t stream) {
  QuantArgs a{};
  a.W = W;
  a.numel = numel;
  a.packed = packed;
  a.c1q = static_cast<uint8_t*>(c1);
  a.c2 = c2;
  a.status = status;
  a.ngroups = ngroups_of(numel);
  a.dq = dq;
  a.zero8 = 0x11111111u * uint32_t(zero_code(quant_type));
  a.exact = quant_type == kQuantInt4 ? 1 : 0;
  a.km = PackMuls{8u, 16u, 256u, 65536u};
  const Codebook& cb = host_codebook(quant_type);
  for (int i = 0; i < 15; ++i) a.thr[i] = cb.thr[i];
  int64_t grid = a.ngroups;
  const int64_t cap = int64_t(num_sms) * kQuantCtasPerSm;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  nf4_quantize_kernel<<<dim3(unsigned(grid)), kQuantThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* packed, const uint8_t* c1, const float* c2, int64_t numel,
                           int quant_type, int dq, int f16, uint16_t* out, int num_sms, cudaStream_t stream) {
  DequantArgs a{};
  a.packed = packed;
  a.c1q = c1;
  a.c2 = c2;
  a.out = out;
  a.numel = numel;
  a.nfull = numel / kBlock;
  a.dq = dq;
  a.f16 = f16;
  const Codebook& cb = host_codebook(quant_type);
  for (int i = 0; i < 16; ++i) a.code.v[i] = cb.code[i];
  a.km = make_shift_muls();
  if (a.nfull >= (int64_t(1) << 31)) return cudaErrorInvalidValue;   // tile rows are int32 coordinates
  if (a.nfull > 0 && !encode_tmap_2d(&a.tm_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, 64, uint64_t(a.nfull), 128, 64,
                                     32, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int64_t grid = (a.nfull + 32 * kDqWarps - 1) / (32 * kDqWarps);
  // one wave: no more CTAs than fit on the SMs at once (the loop is
  // grid-stride, so any grid covers the weight), or a partial second wave
  // of short-lived CTAs would add a tail to every call
  static const int per_sm = [] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nf4_dequant_kernel, kDqWarps * 32, 0) != cudaSuccess ||
        n < 1)
      n = 1;
    return n;
  }();
  const int64_t cap = int64_t(num_sms) * per_sm;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  nf4_dequant_kernel<<<dim3(unsigned(grid)), kDqWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

// Host check that the quantize cell table is well formed: no cell of width
// 1/16 in x holds two thresholds.
bool quantize_table_ok(int quant_type) {
  const Codebook& cb = host_codebook(quant_type);
  for (int c = 0; c < kCells; ++c) {
    const float lo = float(c - 16) * 0.0625f, hi = float(c - 15) * 0.0625f;
    int n = 0;
    for (int i = 0; i < 15; ++i) n += (cb.thr[i] >= lo && cb.thr[i] < hi);
    if (n > 1) return false;
  }
  return true;
}

}  // namespace nf4
