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
// whose absmax lies outside [2^-126, 2^125] are rescaled by a power of two
// first so the reciprocal stays a normal number.
//
// Dequantize ("QLoRA 原理精讲" §2.2, reverse order): scale1' = fp32(E4M3 value
// of c1q * scale2), w' = bf16(fp32(code * scale1')).
//
// Both kernels are HBM-bandwidth bound: 16-byte coalesced loads and stores,
// the per-block absmax by warp shuffles across the 8 lanes that own a block,
// and the code decision as one shared-memory table lookup plus one compare.
#include <cstdint>
#include <cuda_runtime.h>
#include "common.cuh"
#include "kernels.h"

namespace nf4 {
namespace {

constexpr int kQuantThreads = 256;   // one group (16384 weights) per CTA iteration
constexpr int kLutBits = 11;         // sign(1) | exponent(8) | significand top 2
constexpr int kLutSize = 1 << kLutBits;

// Bucket table over the fp32 bit pattern of the normalized value x: every
// bucket holds at most one threshold (checked on the host), so
// code = base + (x > thr).  Built per CTA by binary search over the 15
// ascending thresholds.
__device__ __forceinline__ void build_lut(uint2* lut, const float* thr_smem) {
  for (int idx = threadIdx.x; idx < kLutSize; idx += blockDim.x) {
    const uint32_t lo_bits = uint32_t(idx) << (32 - kLutBits);
    const uint32_t hi_bits = lo_bits | ((1u << (32 - kLutBits)) - 1u);
    uint2 e;
    if (((lo_bits >> 23) & 0xFF) == 0xFF) {   // NaN / Inf: only with non-finite input
      e = make_uint2(__float_as_uint(INFINITY), kCodeZero);
    } else {
      const float a = __uint_as_float(lo_bits), b = __uint_as_float(hi_bits);
      const float xmin = fminf(a, b), xmax = fmaxf(a, b);
      int base = 0;                            // #{thr < xmin}: lower bound in 4 steps
#pragma unroll
      for (int step = 8; step >= 1; step >>= 1)
        if (base + step - 1 < 15 && thr_smem[base + step - 1] < xmin) base += step;
      const float t_in = (base < 15 && thr_smem[base] <= xmax) ? thr_smem[base] : INFINITY;
      e = make_uint2(__float_as_uint(t_in), uint32_t(base));
    }
    lut[idx] = e;
  }
}

__device__ __forceinline__ uint32_t classify(const uint2* lut, float x) {
  const uint2 e = lut[__float_as_uint(x) >> (32 - kLutBits)];
  return e.y + (x > __uint_as_float(e.x) ? 1u : 0u);
}

// 8 consecutive bf16 (one uint4) -> 8 nibbles (element 0 in bits 0-3).
__device__ __forceinline__ uint32_t quantize8(const uint2* lut, const uint4& v, float inv) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out = 0;
#pragma unroll
  for (int j = 3; j >= 0; --j) {
    out = (out << 4) | classify(lut, bf16hi_to_f32(w[j]) * inv);
    out = (out << 4) | classify(lut, bf16lo_to_f32(w[j]) * inv);
  }
  return out;
}
// Same with the weights first scaled by a power of two (extreme blocks).
__device__ __forceinline__ uint32_t quantize8_scaled(const uint2* lut, const uint4& v, float inv, float pre) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out = 0;
#pragma unroll
  for (int j = 3; j >= 0; --j) {
    out = (out << 4) | classify(lut, (bf16hi_to_f32(w[j]) * pre) * inv);
    out = (out << 4) | classify(lut, (bf16lo_to_f32(w[j]) * pre) * inv);
  }
  return out;
}

__device__ __forceinline__ uint32_t absmax_bits8(const uint4& v) {
  // |bf16| as 15-bit integers: their order is the order of magnitudes, and
  // Inf/NaN patterns (>= 0x7F80) come out on top.
  const uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                              __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}

struct QuantArgs {
  const uint16_t* W;
  int64_t numel;
  uint8_t* packed;
  uint8_t* c1q;
  float* c2;
  uint32_t* status;
  int64_t ngroups;
  float thr[15];
};

__device__ __forceinline__ void load_group(const QuantArgs& p, int64_t g, uint4 (&v)[8]) {
  const int64_t gbase = g * kGroupElems;
  const bool full = gbase + kGroupElems <= p.numel;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t e0 = gbase + i * 2048 + threadIdx.x * 8;
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
__global__ void __launch_bounds__(kQuantThreads) nf4_quantize_kernel(const __grid_constant__ QuantArgs p) {
  __shared__ uint2 lut[kLutSize];
  __shared__ float thr_s[16];
  __shared__ uint32_t warp_max[2][kQuantThreads / 32];
  if (threadIdx.x < 15) thr_s[threadIdx.x] = p.thr[threadIdx.x];
  __syncthreads();
  build_lut(lut, thr_s);
  __syncthreads();

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int64_t nblk_total = nblocks_of(p.numel);
  uint32_t bad = 0;

  int64_t g = blockIdx.x;
  uint4 v[8];
  if (g < p.ngroups) load_group(p, g, v);
  for (int parity = 0; g < p.ngroups; g += gridDim.x, parity ^= 1) {
    const int64_t gbase = g * kGroupElems;
    // first level: absmax of each block (8 lanes x 8 weights)
    uint32_t bm[8];
    uint32_t gm = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
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
    uint4 vn[8];
    if (gn < p.ngroups) load_group(p, gn, vn);

    __syncthreads();
    gm = warp_max[parity][0];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) gm = max(gm, warp_max[parity][w]);
    if (gm >= 0x7F80u) bad = 1;

    // second level: fp32 scale2 for the group, E4M3 codes of scale1/scale2
    const float gmax = __uint_as_float(gm << 16);
    const float s2 = __fdiv_rn(gmax, 448.0f);
    if (tid == 0) p.c2[g] = s2;
    if ((tid & 7) == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int64_t b = g * kGroup + i * 32 + (tid >> 3);
        if (b < nblk_total) {
          const float c1 = __uint_as_float(bm[i] << 16);
          p.c1q[b] = (c1 == 0.0f) ? uint8_t(0) : uint8_t(f32_to_e4m3_satfinite(__fdiv_rn(c1, s2)));
        }
      }
    }
    // 4-bit codes
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t e0 = gbase + i * 2048 + tid * 8;
      if (e0 >= p.numel) continue;
      const float c1 = __uint_as_float(bm[i] << 16);
      uint32_t q8;
      if (c1 >= 0x1p-126f && c1 <= 0x1p125f) {
        q8 = quantize8(lut, v[i], __frcp_rn(c1));
      } else if (c1 == 0.0f) {
        q8 = 0x77777777u;                        // all-zero block: the 0.0 code
      } else {                                   // keep 1/c1 a normal number
        const float pre = (c1 < 1.0f) ? 0x1p64f : 0x1p-64f;
        q8 = quantize8_scaled(lut, v[i], __frcp_rn(c1 * pre), pre);
      }
      uint8_t* dst = p.packed + (e0 >> 1);
      if (e0 + 8 <= p.numel) {
        __stcs(reinterpret_cast<unsigned int*>(dst), q8);
      } else {
        const int valid = int(p.numel - e0);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (2 * j < valid) {
            uint32_t byte = (q8 >> (8 * j)) & 0xFFu;
            if (2 * j + 1 >= valid) byte &= 0x0Fu;   // pad nibble of an odd tail
            dst[j] = uint8_t(byte);
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = vn[i];
  }
  if (bad && p.status != nullptr && tid == 0) atomicOr(p.status, kStatusNonfinite);
}

// ---------------------------------------------------------------- dequantize
struct DequantArgs {
  const uint8_t* packed;
  const uint8_t* c1q;
  const float* c2;
  uint16_t* out;
  int64_t numel;
  float code[16];
};

// Per-block table: the 16 values bf16(code[q] * scale1), split into low- and
// high-byte planes so that 4 lookups take a few byte permutes (prmt).
struct DqTable {
  uint32_t lo[4], hi[4];
};
__device__ __forceinline__ DqTable dq_table(const float (&code)[16], float s1) {
  uint32_t pr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pr[i] = pack_bf16x2(code[2 * i] * s1, code[2 * i + 1] * s1);
  DqTable t;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t.lo[k] = prmt(pr[2 * k], pr[2 * k + 1], 0x6420);
    t.hi[k] = prmt(pr[2 * k], pr[2 * k + 1], 0x7531);
  }
  return t;
}
// nibbles j = 0..3 of s -> bf16 pairs (elements 0,1) and (2,3)
__device__ __forceinline__ void dq_lookup4(const DqTable& t, uint32_t s, uint32_t& o01, uint32_t& o23) {
  const uint32_t sel2 = ((s >> 1) & 0x4444u) | 0x3210u;
  const uint32_t lo = prmt(prmt(t.lo[0], t.lo[1], s), prmt(t.lo[2], t.lo[3], s ^ 0x8888u), sel2);
  const uint32_t hi = prmt(prmt(t.hi[0], t.hi[1], s), prmt(t.hi[2], t.hi[3], s ^ 0x8888u), sel2);
  o01 = prmt(lo, hi, 0x5140);
  o23 = prmt(lo, hi, 0x7362);
}

// One thread expands whole 64-weight blocks: two 16-byte loads of codes, one
// table per block, eight 16-byte stores; two blocks per iteration.
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const __grid_constant__ DequantArgs p) {
  float code[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) code[i] = p.code[i];
  const int64_t nfull = p.numel / kBlock;                  // complete blocks
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t b0 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; b0 < nfull; b0 += 2 * stride) {
    const int64_t b1 = b0 + stride;
    const bool has1 = b1 < nfull;
    const uint4* src0 = reinterpret_cast<const uint4*>(p.packed + b0 * 32);
    const uint4 a0 = __ldcs(src0), a1 = __ldcs(src0 + 1);
    uint4 c0 = make_uint4(0, 0, 0, 0), c1 = c0;
    if (has1) {
      const uint4* src1 = reinterpret_cast<const uint4*>(p.packed + b1 * 32);
      c0 = __ldcs(src1);
      c1 = __ldcs(src1 + 1);
    }
    const float s0 = e4m3_to_f32(__ldg(p.c1q + b0)) * __ldg(p.c2 + (b0 >> 8));
    const float s1 = has1 ? e4m3_to_f32(__ldg(p.c1q + b1)) * __ldg(p.c2 + (b1 >> 8)) : 0.0f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (h == 1 && !has1) break;
      const DqTable t = dq_table(code, h ? s1 : s0);
      const uint4 q0 = h ? c0 : a0, q1 = h ? c1 : a1;
      const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
      uint4* dst = reinterpret_cast<uint4*>(p.out + (h ? b1 : b0) * kBlock);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint4 o;
        dq_lookup4(t, w[i] & 0xFFFFu, o.x, o.y);
        dq_lookup4(t, w[i] >> 16, o.z, o.w);
        __stcs(dst + i, o);
      }
    }
  }
  // ragged tail: the last, short block (numel % 64 weights), one thread
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.numel % kBlock != 0) {
    const int64_t b = nfull;
    const float s1 = e4m3_to_f32(p.c1q[b]) * p.c2[b >> 8];
    for (int64_t e = b * kBlock; e < p.numel; ++e) {
      const uint32_t byte = p.packed[e >> 1];
      const uint32_t q = (e & 1) ? (byte >> 4) : (byte & 0xFu);
      p.out[e] = uint16_t(pack_bf16x2(code[q] * s1, 0.0f) & 0xFFFFu);
    }
  }
}

}  // namespace

cudaError_t launch_quantize(const uint16_t* W, int64_t numel, uint8_t* packed, uint8_t* c1q, float* c2,
                            uint32_t* status, int num_sms, cudaStream_t stream) {
  QuantArgs a{};
  a.W = W;
  a.numel = numel;
  a.packed = packed;
  a.c1q = c1q;
  a.c2 = c2;
  a.status = status;
  a.ngroups = ngroups_of(numel);
  const Codebook& cb = host_codebook();
  for (int i = 0; i < 15; ++i) a.thr[i] = cb.thr[i];
  int64_t grid = a.ngroups;
  const int64_t cap = int64_t(num_sms) * 2;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  nf4_quantize_kernel<<<dim3(unsigned(grid)), kQuantThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* packed, const uint8_t* c1q, const float* c2, int64_t numel,
                           uint16_t* out, int num_sms, cudaStream_t stream) {
  DequantArgs a{};
  a.packed = packed;
  a.c1q = c1q;
  a.c2 = c2;
  a.out = out;
  a.numel = numel;
  const Codebook& cb = host_codebook();
  for (int i = 0; i < 16; ++i) a.code[i] = cb.code[i];
  const int64_t nfull = numel / kBlock;
  int64_t grid = (nfull / 2 + 255) / 256;
  const int64_t cap = int64_t(num_sms) * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  nf4_dequant_kernel<<<dim3(unsigned(grid)), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

// Host check that the quantize lookup table is well formed: no bucket of
// x values (fixed sign, exponent and top 3 significand bits) holds two
// thresholds.
bool quantize_table_ok() {
  const Codebook& cb = host_codebook();
  for (uint32_t idx = 0; idx < uint32_t(kLutSize); ++idx) {
    uint32_t lo_bits = idx << (32 - kLutBits), hi_bits = lo_bits | ((1u << (32 - kLutBits)) - 1u);
    if (((lo_bits >> 23) & 0xFF) == 0xFF) continue;
    float a, b;
    memcpy(&a, &lo_bits, 4);
    memcpy(&b, &hi_bits, 4);
    float xmin = a < b ? a : b, xmax = a < b ? b : a;
    int n = 0;
    for (int i = 0; i < 15; ++i) n += (cb.thr[i] >= xmin && cb.thr[i] <= xmax);
    if (n > 1) return false;
  }
  return true;
}

}  // namespace nf4
