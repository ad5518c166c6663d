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
constexpr int kLutBits = 12;         // sign(1) | exponent(8) | mantissa top 3
constexpr int kLutSize = 1 << kLutBits;

// Bucket table over the fp32 bit pattern of the normalized value x: every
// bucket holds at most one threshold (checked on the host), so
// code = base + (x > thr).
__device__ __forceinline__ void build_lut(uint2* lut, const float* thr) {
  for (int idx = threadIdx.x; idx < kLutSize; idx += blockDim.x) {
    uint32_t lo_bits = uint32_t(idx) << (32 - kLutBits);
    uint32_t hi_bits = lo_bits | ((1u << (32 - kLutBits)) - 1u);
    uint32_t expo = (lo_bits >> 23) & 0xFF;
    uint2 e;
    if (expo == 0xFF) {                       // NaN / Inf: only with non-finite input
      e = make_uint2(__float_as_uint(INFINITY), kCodeZero);
    } else {
      float a = __uint_as_float(lo_bits), b = __uint_as_float(hi_bits);
      float xmin = fminf(a, b), xmax = fmaxf(a, b);
      uint32_t base = 0;
      float t_in = INFINITY;
      for (int i = 0; i < 15; ++i) {
        if (thr[i] < xmin) ++base;
        else if (thr[i] <= xmax) t_in = thr[i];
      }
      e = make_uint2(__float_as_uint(t_in), base);
    }
    lut[idx] = e;
  }
}

__device__ __forceinline__ uint32_t classify(const uint2* lut, float x) {
  uint2 e = lut[__float_as_uint(x) >> (32 - kLutBits)];
  return e.y + (x > __uint_as_float(e.x) ? 1u : 0u);
}

// 8 consecutive bf16 (one uint4) -> 8 nibbles (element 0 in bits 0-3).
__device__ __forceinline__ uint32_t quantize8(const uint2* lut, const uint4& v, float inv, float pre) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out = 0;
#pragma unroll
  for (int j = 3; j >= 0; --j) {
    float hi = bf16hi_to_f32(w[j]) * pre;
    float lo = bf16lo_to_f32(w[j]) * pre;
    out = (out << 4) | classify(lut, hi * inv);
    out = (out << 4) | classify(lut, lo * inv);
  }
  return out;
}

__device__ __forceinline__ uint32_t absmax_bits8(const uint4& v) {
  // |bf16| as 15-bit integers: their order is the order of magnitudes, and
  // Inf/NaN patterns (>= 0x7F80) come out on top.
  uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
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

__global__ void __launch_bounds__(kQuantThreads) nf4_quantize_kernel(const __grid_constant__ QuantArgs p) {
  __shared__ uint2 lut[kLutSize];
  __shared__ uint32_t warp_max[kQuantThreads / 32];
  build_lut(lut, p.thr);
  __syncthreads();

  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int64_t nblk_total = nblocks_of(p.numel);
  uint32_t bad = 0;

  for (int64_t g = blockIdx.x; g < p.ngroups; g += gridDim.x) {
    const int64_t gbase = g * kGroupElems;
    const bool full = gbase + kGroupElems <= p.numel;
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t e0 = gbase + i * 2048 + tid * 8;
      if (full || e0 + 8 <= p.numel) {
        v[i] = __ldg(reinterpret_cast<const uint4*>(p.W + e0));
      } else {
        uint16_t t[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) t[j] = (e0 + j < p.numel) ? p.W[e0 + j] : uint16_t(0);
        v[i] = make_uint4(t[0] | (uint32_t(t[1]) << 16), t[2] | (uint32_t(t[3]) << 16),
                          t[4] | (uint32_t(t[5]) << 16), t[6] | (uint32_t(t[7]) << 16));
      }
    }
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
    if (lane == 0) warp_max[warp] = gm;
    __syncthreads();
    gm = warp_max[0];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) gm = max(gm, warp_max[w]);
    if (gm >= 0x7F80u) bad = 1;

    // second level: fp32 scale2 for the group, E4M3 codes of scale1/scale2
    const float gmax = __uint_as_float(gm << 16);
    const float s2 = __fdiv_rn(gmax, 448.0f);
    if (tid == 0) p.c2[g] = s2;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t b = g * kGroup + i * 32 + (tid >> 3);
      if ((tid & 7) == 0 && b < nblk_total) {
        const float c1 = __uint_as_float(bm[i] << 16);
        p.c1q[b] = (c1 == 0.0f) ? uint8_t(0) : uint8_t(f32_to_e4m3_satfinite(__fdiv_rn(c1, s2)));
      }
    }
    // 4-bit codes
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t e0 = gbase + i * 2048 + tid * 8;
      if (e0 >= p.numel) continue;
      float c1 = __uint_as_float(bm[i] << 16);
      float pre = 1.0f;
      if (c1 != 0.0f && !(c1 >= 0x1p-126f && c1 <= 0x1p125f)) {   // keep 1/c1 a normal number
        pre = (c1 < 1.0f) ? 0x1p64f : 0x1p-64f;
        c1 *= pre;
      }
      const float inv = (c1 == 0.0f) ? 0.0f : __frcp_rn(c1);
      const uint32_t q8 = quantize8(lut, v[i], inv, pre);
      uint8_t* dst = p.packed + (e0 >> 1);
      if (e0 + 8 <= p.numel) {
        *reinterpret_cast<uint32_t*>(dst) = q8;
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
    __syncthreads();   // warp_max is reused by the next group
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

// Each thread expands 16 packed bytes (32 weights, half a block) into 64
// bytes of bf16: one 16-byte load, four 16-byte stores.
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const __grid_constant__ DequantArgs p) {
  __shared__ float code[16];
  if (threadIdx.x < 16) code[threadIdx.x] = p.code[threadIdx.x];
  __syncthreads();
  const int64_t nchunks = (p.numel + 31) / 32;
  for (int64_t c = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; c < nchunks;
       c += int64_t(gridDim.x) * blockDim.x) {
    const int64_t e0 = c * 32;
    const int64_t b = e0 / kBlock;
    const float s1 = e4m3_to_f32(__ldg(p.c1q + b)) * __ldg(p.c2 + b / kGroup);
    uint4 pk;
    const bool whole = e0 + 32 <= p.numel;
    if (whole) {
      pk = __ldg(reinterpret_cast<const uint4*>(p.packed + (e0 >> 1)));
    } else {
      uint8_t t[16];
      const int64_t nbytes = (p.numel - e0 + 1) / 2;
#pragma unroll
      for (int j = 0; j < 16; ++j) t[j] = (j < nbytes) ? p.packed[(e0 >> 1) + j] : uint8_t(0);
      pk = make_uint4(t[0] | t[1] << 8 | t[2] << 16 | uint32_t(t[3]) << 24,
                      t[4] | t[5] << 8 | t[6] << 16 | uint32_t(t[7]) << 24,
                      t[8] | t[9] << 8 | t[10] << 16 | uint32_t(t[11]) << 24,
                      t[12] | t[13] << 8 | t[14] << 16 | uint32_t(t[15]) << 24);
    }
    const uint32_t words[4] = {pk.x, pk.y, pk.z, pk.w};
    uint32_t o[16];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t byte = (words[w] >> (8 * j)) & 0xFFu;
        o[w * 4 + j] = pack_bf16x2(code[byte & 0xF] * s1, code[byte >> 4] * s1);
      }
    }
    if (whole) {
      uint4* dst = reinterpret_cast<uint4*>(p.out + e0);
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[k] = make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
    } else {
      for (int j = 0; j < 32 && e0 + j < p.numel; ++j)
        p.out[e0 + j] = uint16_t((j & 1) ? (o[j >> 1] >> 16) : (o[j >> 1] & 0xFFFFu));
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
  const int64_t cap = int64_t(num_sms) * 4;
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
  const int64_t nchunks = (numel + 31) / 32;
  int64_t grid = (nchunks + 255) / 256;
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
