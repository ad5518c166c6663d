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
// Both kernels are HBM-bandwidth bound: 16-byte coalesced loads and stores,
// the per-block absmax by warp shuffles across the 8 lanes that own a block,
// and the code decision as one lookup in a 33-cell shared-memory table plus
// one compare (about 8 instructions per weight, most on the FMA pipe).
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include "common.cuh"
#include "kernels.h"
#include "nf4_lut.cuh"

namespace nf4 {
namespace {

constexpr int kQuantThreads = 512;   // one group (16384 weights) per CTA iteration
constexpr int kQuantIters = kGroupElems / (kQuantThreads * 8);   // 16-byte loads per thread per group: 4
static_assert(kQuantIters * kQuantThreads * 8 == kGroupElems, "a group is an exact number of passes");
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
// minus 8 * 0x4B000000 (mod 2^32), so the pattern times 8 addresses the cell
// directly.  The comparison x16 > 16 T is the sign bit of 16 T - x16, which is
// +0 for x16 == 16 T (ties go to the lower code) and +inf where the cell holds
// no threshold.
__device__ __forceinline__ uint32_t classify_fast(uint32_t cells_biased, float x16) {
  const float r = __fadd_rd(x16, 8388624.0f);
  const uint32_t addr = cells_biased + (__float_as_uint(r) << 3);
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
// input); 2: exact comparison (dyadic thresholds).
template <int MODE>
__device__ __forceinline__ uint32_t quantize8(const uint2* cells, uint32_t cells_biased, const uint4& v,
                                              float inv16, float pre, float c1) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out = 0;
#pragma unroll
  for (int j = 3; j >= 0; --j) {
    float hi = bf16hi_to_f32(w[j]), lo = bf16lo_to_f32(w[j]);
    if (MODE != 0) {
      hi *= pre;
      lo *= pre;
    }
    const float xh = hi * inv16, xl = lo * inv16;
    if (MODE == 0) {
      out = out * 16u + classify_fast(cells_biased, xh);
      out = out * 16u + classify_fast(cells_biased, xl);
    } else if (MODE == 1) {
      out = out * 16u + classify16(cells, xh);
      out = out * 16u + classify16(cells, xl);
    } else {
      out = out * 16u + classify_exact(cells, xh, hi, c1);
      out = out * 16u + classify_exact(cells, xl, lo, c1);
    }
  }
  return out;
}

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t u) {
  return *reinterpret_cast<const __nv_bfloat162*>(&u);
}
// Largest |w| of 8 bf16 as a bf16 bit pattern (NaN propagates, so Inf/NaN
// inputs give a pattern >= 0x7F80).
__device__ __forceinline__ uint32_t absmax_bits8(const uint4& v) {
  const __nv_bfloat162 m = __hmax2_nan(__hmax2_nan(__habs2(as_bf162(v.x)), __habs2(as_bf162(v.y))),
                                       __hmax2_nan(__habs2(as_bf162(v.z)), __habs2(as_bf162(v.w))));
  const uint32_t u = *reinterpret_cast<const uint32_t*>(&m);
  return max(u & 0xFFFFu, u >> 16);
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
  float thr[15];
};

// Pass i of a group covers weights i * 4096 .. i * 4096 + 4095; thread tid
// loads 8 of them (tid * 8 ..), so the 8 lanes tid & ~7 .. tid | 7 hold one
// 64-weight block.
__device__ __forceinline__ void load_group(const QuantArgs& p, int64_t g, uint4 (&v)[kQuantIters]) {
  const int64_t gbase = g * kGroupElems;
  const bool full = gbase + kGroupElems <= p.numel;
#pragma unroll
  for (int i = 0; i < kQuantIters; ++i) {
    const int64_t e0 = gbase + int64_t(i) * (kQuantThreads * 8) + threadIdx.x * 8;
    if (full || e0 + 8 <= p.numel) {
      v[i] = __ldcs(reinterpret_cast<const uint4*>(p.W + e0));
    } else {
      uint16_t t[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) t[j] = (e0 + j < p.numel) ? p.W[e0 + j] : uint16_t(0);
      v[i] = make_uint4(t[0] | (uint32_t(t[1]) << 16), t[2] | (uint32_t(t[3]) << 16),
                        t[4] | (uint32_t(t[5]) << 16), t[6] | (uint32_t(t[7]) << 16));
    }
  }
}

// Persistent CTAs walk the groups; the next group's 32 KB are loaded while
// the current one is classified.
__global__ void __launch_bounds__(kQuantThreads, 2) nf4_quantize_kernel(const __grid_constant__ QuantArgs p) {
  __shared__ uint2 cells[kCells];
  __shared__ float thr_s[16];
  __shared__ __align__(16) uint32_t warp_max[2][kQuantThreads / 32];
  if (threadIdx.x < 15) thr_s[threadIdx.x] = p.thr[threadIdx.x];
  __syncthreads();
  build_cells(cells, thr_s);
  __syncthreads();
  const uint32_t cells_biased = smem_u32(cells) - (0x4B000000u << 3);

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int64_t nblk_total = nblocks_of(p.numel);
  uint32_t bad = 0;

  int64_t g = blockIdx.x;
  uint4 v[kQuantIters];
  if (g < p.ngroups) load_group(p, g, v);
  for (int parity = 0; g < p.ngroups; g += gridDim.x, parity ^= 1) {
    const int64_t gbase = g * kGroupElems;
    // first level: absmax of each block (8 lanes x 8 weights)
    uint32_t bm[kQuantIters];
    uint32_t gm = 0;
#pragma unroll
    for (int i = 0; i < kQuantIters; ++i) {
      uint32_t m = absmax_bits8(v[i]);
      m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = max(m, __shfl_xor_sync(0xffffffffu, m, 4));
      bm[i] = m;
      gm = max(gm, m);
    }
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) gm = max(gm, __shfl_xor_sync(0xffffffffu, gm, o));
    if (lane == 0) warp_max[parity][warp] = gm;

    // prefetch the next group while this one is finished
    const int64_t gn = g + gridDim.x;
    uint4 vn[kQuantIters];
    if (gn < p.ngroups) load_group(p, gn, vn);

    // 4-bit codes first: a code depends only on its own block's absmax, so
    // this work needs no other warp and comes before the group barrier.
    // Lane j < kQuantIters of each 8-lane block group owns pass j: it takes
    // that block's reciprocal once; the others receive it by shuffle.
    const int j = lane & 7;
    uint32_t my_bm = bm[0];
#pragma unroll
    for (int i = 1; i < kQuantIters; ++i) my_bm = (j == i) ? bm[i] : my_bm;
    const float my_c1 = __uint_as_float(my_bm << 16);
    // 16 / scale1 must stay a finite normal number: scale1 in [2^-122, 2^125]
    const bool normal = (my_c1 >= 0x1p-122f && my_c1 <= 0x1p125f) || my_c1 == 0.0f;
    const float my_inv = (my_c1 == 0.0f) ? 0.0f : (normal ? __frcp_rn(my_c1) : 0.0f);
    const bool fast = __all_sync(0xffffffffu, normal);
    const int64_t ebase = gbase + tid * 8;
    const bool full = gbase + kGroupElems <= p.numel;   // no element of this group is past the end
#pragma unroll
    for (int i = 0; i < kQuantIters; ++i) {
      const int64_t e0 = ebase + i * (kQuantThreads * 8);
      const float inv = __shfl_sync(0xffffffffu, my_inv, (lane & ~7) | i);
      if (!full && e0 >= p.numel) continue;
      const float c1 = __uint_as_float(bm[i] << 16);
      uint32_t q8;
      if (c1 == 0.0f) {
        q8 = p.zero8;                            // all-zero block: the 0.0 code
      } else if (p.exact) {                      // dyadic thresholds: exact comparisons
        const bool nrm = c1 >= 0x1p-122f && c1 <= 0x1p125f;
        const float pre = nrm ? 1.0f : ((c1 < 1.0f) ? 0x1p64f : 0x1p-64f);
        q8 = quantize8<2>(cells, cells_biased, v[i], __frcp_rn(c1 * pre) * 16.0f, pre, c1 * pre);
      } else if (fast) {
        q8 = quantize8<0>(cells, cells_biased, v[i], inv * 16.0f, 1.0f, c1);
      } else if (c1 >= 0x1p-122f && c1 <= 0x1p125f) {
        q8 = quantize8<1>(cells, cells_biased, v[i], __frcp_rn(c1) * 16.0f, 1.0f, c1);
      } else {                                   // keep 16/c1 a normal number
        const float pre = (c1 < 1.0f) ? 0x1p64f : 0x1p-64f;
        q8 = quantize8<1>(cells, cells_biased, v[i], __frcp_rn(c1 * pre) * 16.0f, pre, c1);
      }
      uint8_t* dst = p.packed + (e0 >> 1);
      if (full || e0 + 8 <= p.numel) {
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

    // second level: fp32 scale2 for the group (needs every warp's maximum),
    // then the 8-bit codes of scale1 / scale2 (lane j < kQuantIters of each
    // block group stores its block's)
    __syncthreads();
    {   // the group maximum over the warps' maxima, four per 16-byte load
      const uint4* wm = reinterpret_cast<const uint4*>(warp_max[parity]);
      gm = 0;
#pragma unroll
      for (int w = 0; w < kQuantThreads / 128; ++w) {
        const uint4 q = wm[w];
        gm = max(gm, max(max(q.x, q.y), max(q.z, q.w)));
      }
    }
    if (gm >= 0x7F80u) bad = 1;
    const float gmax = __uint_as_float(gm << 16);
    const float s2 = __fdiv_rn(gmax, p.dq == kDqU8 ? 255.0f : 448.0f);
    if (tid == 0 && p.dq != kDqNone) p.c2[g] = s2;
    if (j < kQuantIters) {
      const int64_t b = g * kGroup + int64_t(j) * (kQuantThreads / 8) + (tid >> 3);
      if (b < nblk_total) {
        if (p.dq == kDqNone) {
          reinterpret_cast<float*>(p.c1q)[b] = my_c1;
        } else if (my_c1 == 0.0f) {
          p.c1q[b] = 0;
        } else {
          const float t = __fdiv_rn(my_c1, s2);
          p.c1q[b] = uint8_t(p.dq == kDqU8 ? min(__float2uint_rn(t), 255u) : f32_to_e4m3_satfinite(t));
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kQuantIters; ++i) v[i] = vn[i];
  }
  if (bad && p.status != nullptr && tid == 0) atomicOr(p.status, kStatusNonfinite);
}

// ---------------------------------------------------------------- dequantize
struct DequantArgs {
  const uint8_t* packed;
  const uint8_t* c1q;   // first-level constants (bytes, or fp32 for kDqNone)
  const float* c2;
  uint16_t* out;
  int64_t numel;
  int dq;               // DqFormat
  int f16;              // output fp16 (else bf16)
  float code[16];
};

// Eight lanes per 64-weight block, eight weights (four packed bytes) per
// lane and unit, so that every warp load covers 128 contiguous packed bytes
// and every warp store 512 contiguous bytes of bf16; four units per lane per
// iteration keep enough bytes in flight.  code[q] comes from a 16-word shared
// table (one bank per entry), times the block scale in fp32, rounded to bf16.
constexpr int kDqUnits = 4;
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const __grid_constant__ DequantArgs p) {
  __shared__ float code_s[16];
  if (threadIdx.x < 16) code_s[threadIdx.x] = p.code[threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t nunits = p.numel / 8;                        // complete 8-weight units
  const int64_t warp_id = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t base = warp_id * (32 * kDqUnits); base < nunits; base += nwarps * (32 * kDqUnits)) {
    uint32_t w[kDqUnits];
    float s1[kDqUnits];
#pragma unroll
    for (int i = 0; i < kDqUnits; ++i) {
      const int64_t u = base + i * 32 + lane;
      if (u < nunits) {
        w[i] = __ldcs(reinterpret_cast<const unsigned int*>(p.packed) + u);
        s1[i] = block_scale(p.dq, p.c1q, p.c2, u >> 3);
      } else {
        w[i] = 0u;
        s1[i] = 0.0f;
      }
    }
#pragma unroll
    for (int i = 0; i < kDqUnits; ++i) {
      const int64_t u = base + i * 32 + lane;
      if (u >= nunits) break;
      const bool h = p.f16 != 0;
      uint4 o;
      o.x = pack2(h, code_s[w[i] & 0xFu] * s1[i], code_s[(w[i] >> 4) & 0xFu] * s1[i]);
      o.y = pack2(h, code_s[(w[i] >> 8) & 0xFu] * s1[i], code_s[(w[i] >> 12) & 0xFu] * s1[i]);
      o.z = pack2(h, code_s[(w[i] >> 16) & 0xFu] * s1[i], code_s[(w[i] >> 20) & 0xFu] * s1[i]);
      o.w = pack2(h, code_s[(w[i] >> 24) & 0xFu] * s1[i], code_s[w[i] >> 28] * s1[i]);
      __stcs(reinterpret_cast<uint4*>(p.out) + u, o);
    }
  }
  // ragged tail: the last numel % 8 weights, one thread
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (int64_t e = nunits * 8; e < p.numel; ++e) {
      const float s = block_scale(p.dq, p.c1q, p.c2, e / kBlock);
      const uint32_t byte = p.packed[e >> 1];
      const uint32_t q = (e & 1) ? (byte >> 4) : (byte & 0xFu);
      p.out[e] = uint16_t(pack2(p.f16 != 0, code_s[q] * s, 0.0f) & 0xFFFFu);
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
  const Codebook& cb = host_codebook(quant_type);
  for (int i = 0; i < 15; ++i) a.thr[i] = cb.thr[i];
  int64_t grid = a.ngroups;
  const int64_t cap = int64_t(num_sms) * 2;
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
  a.dq = dq;
  a.f16 = f16;
  const Codebook& cb = host_codebook(quant_type);
  for (int i = 0; i < 16; ++i) a.code[i] = cb.code[i];
  const int64_t nunits = numel / 8;
  int64_t grid = (nunits / (32 * kDqUnits) + 7) / 8;   // 8 warps per CTA
  // one wave: no more CTAs than fit on the SMs at once (the loop is
  // grid-stride, so any grid covers the weight), or a partial second wave
  // of short-lived CTAs would add a tail to every call
  static const int per_sm = [] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nf4_dequant_kernel, 256, 0) != cudaSuccess || n < 1) n = 1;
    return n;
  }();
  const int64_t cap = int64_t(num_sms) * per_sm;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  nf4_dequant_kernel<<<dim3(unsigned(grid)), 256, 0, stream>>>(a);
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
