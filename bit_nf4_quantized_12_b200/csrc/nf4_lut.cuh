// nf4_lut.cuh -- per-block NF4 dequantization by byte permutes, shared by the
// fused GEMM (operand tiles) and the decode GEMV.
//
// A weight is w' = bf16(fp32(code[q] * scale1)) ("QLoRA 原理精讲" §2.2: the
// block constant is restored first, then each 4-bit code is mapped through the
// NF4 table and scaled); the 16 possible values of one block are formed once
// and looked up with prmt.
#pragma once
#include <cstdint>
#include "common.cuh"

namespace nf4 {

struct CodeTable {
  float v[16];
};

// 16-entry table of one block in the compute type (code[q] * scale1, each an
// fp32 multiply rounded to bf16, or to fp16) split into low-byte and
// high-byte planes so that four lookups are a handful of byte permutes.
struct BlockTable {
  uint32_t lo[4], hi[4];
};

__device__ __forceinline__ BlockTable make_table(const CodeTable& code, float s1, bool f16 = false) {
  uint32_t pr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pr[i] = pack2(f16, code.v[2 * i] * s1, code.v[2 * i + 1] * s1);
  BlockTable t;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t.lo[k] = prmt(pr[2 * k], pr[2 * k + 1], 0x6420);
    t.hi[k] = prmt(pr[2 * k], pr[2 * k + 1], 0x7531);
  }
  return t;
}

// Four nibbles (bits 0-15 of s, element j in nibble j) -> two bf16x2 words.
__device__ __forceinline__ void lookup4(const BlockTable& t, uint32_t s, uint32_t& o01, uint32_t& o23) {
  const uint32_t sel_a = s;                   // entries 0-7 (bit 3 clear)
  const uint32_t sel_b = s ^ 0x8888u;         // entries 8-15
  // pick a or b per byte by bit 3: ((s & 0x8888) >> 1) | 0x3210, the shift
  // and the OR (no bits in common) as one high multiply-add on the FMA pipe,
  // leaving the integer pipe to the byte permutes
  const uint32_t sel2 = __umulhi(s & 0x8888u, 0x80000000u) + 0x3210u;
  const uint32_t lo = prmt(prmt(t.lo[0], t.lo[1], sel_a), prmt(t.lo[2], t.lo[3], sel_b), sel2);
  const uint32_t hi = prmt(prmt(t.hi[0], t.hi[1], sel_a), prmt(t.hi[2], t.hi[3], sel_b), sel2);
  o01 = prmt(lo, hi, 0x5140);
  o23 = prmt(lo, hi, 0x7362);
}

// Multipliers of the high-multiply shifts below.  They reach the kernels as
// launch parameters, so the compiler cannot turn a multiply by a power of two
// back into a shift: the shifts then run on the FMA pipe as integer
// multiply-adds, next to the integer pipe that the byte permutes keep busy.
struct ShiftMuls {
  uint32_t k16;   // 2^16: x >> 16
  uint32_t k15;   // 2^15: x >> 17
  uint32_t k31;   // 2^31: x >> 1
};
inline ShiftMuls make_shift_muls() { return ShiftMuls{1u << 16, 1u << 15, 1u << 31}; }

__device__ __forceinline__ uint32_t mulhi_add(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Eight nibbles (one packed word, element j in nibble j) -> four bf16x2 words
// (elements 0-1, 2-3, 4-5, 6-7).  The flip of bit 3 and its mask are taken
// once for the eight nibbles; the upper four nibbles' selectors come from
// them by high multiplies.
__device__ __forceinline__ void lookup8(const BlockTable& t, uint32_t w, const ShiftMuls& k, uint32_t& o0,
                                        uint32_t& o1, uint32_t& o2, uint32_t& o3) {
  const uint32_t wb = w ^ 0x88888888u;     // selectors into entries 8-15
  const uint32_t m = w & 0x88888888u;      // bit 3 of every nibble
  const uint32_t sel2_lo = mulhi_add(m, k.k31, 0x3210u);   // ((m >> 1) & 0x4444) | 0x3210 (bits 16+ unused)
  const uint32_t sel2_hi = mulhi_add(m, k.k15, 0x3210u);   // the same for nibbles 4-7
  const uint32_t wa_hi = mulhi_add(w, k.k16, 0u), wb_hi = mulhi_add(wb, k.k16, 0u);   // >> 16
  {
    const uint32_t lo = prmt(prmt(t.lo[0], t.lo[1], w), prmt(t.lo[2], t.lo[3], wb), sel2_lo);
    const uint32_t hi = prmt(prmt(t.hi[0], t.hi[1], w), prmt(t.hi[2], t.hi[3], wb), sel2_lo);
    o0 = prmt(lo, hi, 0x5140);
    o1 = prmt(lo, hi, 0x7362);
  }
  {
    const uint32_t lo = prmt(prmt(t.lo[0], t.lo[1], wa_hi), prmt(t.lo[2], t.lo[3], wb_hi), sel2_hi);
    const uint32_t hi = prmt(prmt(t.hi[0], t.hi[1], wa_hi), prmt(t.hi[2], t.hi[3], wb_hi), sel2_hi);
    o2 = prmt(lo, hi, 0x5140);
    o3 = prmt(lo, hi, 0x7362);
  }
}

// 32 packed bytes (64 weights) -> 32 bf16x2 words in element order.
__device__ __forceinline__ void dequant64(const BlockTable& t, const uint4& p0, const uint4& p1, const ShiftMuls& km,
                                          uint32_t (&o)[32]) {
  const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) lookup8(t, w[i], km, o[4 * i + 0], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
}

}  // namespace nf4

namespace nf4 {

// First-level constant of block b in each storage format (include/qlora_nf4.h
// NF4_DQ_*): FP8 E4M3 code times the group's FP32 scale2 (the method,
// "QLoRA 原理精讲" §2.2), the FP32 scale1 itself, or an unsigned 8-bit code
// times scale2.  One fp32 multiply where there are two levels.
enum DqFormat : int { kDqE4M3 = 0, kDqNone = 1, kDqU8 = 2 };

__device__ __forceinline__ float block_scale(int dq, const uint8_t* c1, const float* c2, int64_t b) {
  if (dq == kDqNone) return __ldg(reinterpret_cast<const float*>(c1) + b);
  const uint32_t q = __ldg(c1 + b);
  const float s2 = __ldg(c2 + (b >> 8));
  return (dq == kDqU8 ? float(q) : e4m3_to_f32(q)) * s2;
}

// Raw first-level value of block b as loaded ahead of use: the 8-bit code or
// the FP32 bits, and the group's scale2 (0 for kDqNone).
__device__ __forceinline__ void load_scale_parts(int dq, const uint8_t* c1, const float* c2, int64_t b,
                                                 uint32_t& q, float& s2) {
  if (dq == kDqNone) {
    q = __float_as_uint(__ldg(reinterpret_cast<const float*>(c1) + b));
    s2 = 0.0f;
  } else {
    q = __ldg(c1 + b);
    s2 = __ldg(c2 + (b >> 8));
  }
}
__device__ __forceinline__ float scale_from_parts(int dq, uint32_t q, float s2) {
  if (dq == kDqNone) return __uint_as_float(q);
  return (dq == kDqU8 ? float(q) : e4m3_to_f32(q)) * s2;
}

}  // namespace nf4
