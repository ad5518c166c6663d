// format.h -- the NF4 + double-quantization storage format of libqlora_nf4.
//
// A frozen weight W [rows, cols] (bf16, row-major) is stored as three flat
// buffers over its row-major flattening (element e = row*cols + col):
//   packed[ceil(numel/2)]  4-bit code of element e in byte e/2, even e in the
//                          low nibble (pad nibble 0 when numel is odd);
//   c1q[nblocks]           FP8 E4M3 code of each first-level scale
//                          (block = 64 consecutive elements; the last one
//                          may be short);
//   c2[ngroups]            fp32 second-level scale of each group of 256
//                          consecutive blocks (the last group may be short).
// Block size 64 and group size 256 follow "QLoRA 原理精讲" §2.1/§2.2; FP8 for
// the quantized first-level scales and FP32 for the second level follow §2.2
// of the same page (its diagram: 4-bit weights + FP8 scale1 + FP32 scale2).
#pragma once
#include <cstdint>

#if defined(__CUDACC__)
#define NF4_HD __host__ __device__
#else
#define NF4_HD
#endif

namespace nf4 {
constexpr int kBlock = 64;    // weights per first-level block
constexpr int kGroup = 256;   // blocks per second-level group
constexpr int kGroupElems = kBlock * kGroup;  // 16384
constexpr int kCodeZero = 7;  // index of the exact 0.0 code (the table ascends)

NF4_HD inline int64_t nblocks_of(int64_t numel) { return (numel + kBlock - 1) / kBlock; }
NF4_HD inline int64_t ngroups_of(int64_t numel) { return (nblocks_of(numel) + kGroup - 1) / kGroup; }
NF4_HD inline int64_t packed_bytes_of(int64_t numel) { return (numel + 1) / 2; }

// The 16 NF4 values (ascending) and the 15 decision thresholds: T[i] is the
// midpoint of codes i and i+1 rounded down to fp32, so that for any fp32 x,
// #{i : x > T[i]} is the index of the nearest code with ties to the lower.
struct Codebook {
  float code[16];
  float thr[15];
};

// Table selectors (include/qlora_nf4.h NF4_QUANT_*).
constexpr int kQuantNf4 = 0;
constexpr int kQuantInt4 = 1;

// Built once on the host (codebook.cpp): the NF4 table, or the table of a
// quant_type.
const Codebook& host_codebook();
const Codebook& host_codebook(int quant_type);
// Index of the exact 0.0 code of a quant_type's table.
inline int zero_code(int quant_type) { return quant_type == kQuantInt4 ? 8 : kCodeZero; }
}  // namespace nf4
