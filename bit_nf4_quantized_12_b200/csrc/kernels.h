// kernels.h -- internal launchers of libqlora_nf4 (not part of the C ABI).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace nf4 {

// How a kernel orders itself against the previous kernel of its stream when
// it is launched as a programmatic dependent (see griddep_wait in common.cuh).
enum PdlMode : int {
  kPdlWaitFirst = 0,    // wait for the previous kernel, then let the next one start
  kPdlWaitLast = 1,     // let the next kernel start, work, wait before exiting
  kPdlWaitLowRank = 2,  // fused GEMM: main product first, wait before the low-rank operand; a CTA with
                        // low-rank steps releases the next kernel only after that wait
};

// Quantize W (numel bf16) into the storage format (quant_type: table;
// dq: DqFormat of the first-level constants, c1 holds bytes or fp32).
cudaError_t launch_quantize(const uint16_t* W, int64_t numel, int quant_type, int dq, uint8_t* packed, void* c1,
                            float* c2, uint32_t* status, int num_sms, cudaStream_t stream);
// Dequantize into the compute type (f16: fp16, else bf16).
cudaError_t launch_dequant(const uint8_t* packed, const uint8_t* c1, const float* c2, int64_t numel,
                           int quant_type, int dq, int f16, uint16_t* out, int num_sms, cudaStream_t stream);
bool quantize_table_ok(int quant_type);

// Copy src [rows, cols] (2-byte elements, pitch cols) into dst with row pitch
// ld >= cols (elements); the columns past cols are left as they are.
cudaError_t launch_repitch(const uint16_t* src, int64_t rows, int64_t cols, uint16_t* dst, int64_t ld, int num_sms,
                           cudaStream_t stream);

// ---------------------------------------------------------------- LoRA merge
// out[n, k] = round(Wd[n, k] + s sum_j A[k, j] B[j, n]) in the compute type.
struct MergeArgs {
  const uint8_t* packed;
  const uint8_t* c1;      // first-level constants (bytes, or fp32 for dq == kDqNone)
  const float* c2;
  int64_t N, K;
  int double_quant;       // DqFormat
  const uint16_t* A;      // [K, r]
  const uint16_t* B;      // [r, N]
  int r;
  float s;
  int f16;                // compute type fp16 (else bf16)
  uint16_t* out;          // [N, K]
};
cudaError_t launch_merge(const MergeArgs& a, const float code[16], cudaStream_t stream);
size_t merge_smem_bytes(int r);

// ---------------------------------------------------------------- fused NF4 GEMM
// Computes, for a tile grid over (W-dim x tokens):
//   forward : Y[m, n]  = sum_k X[m,k] Wd[n,k]  + sum_j (sT)[m,j] B[j,n]
//   backward: dX[m, k] = sum_n dY[m,n] Wd[n,k] + sum_j G[m,j]  A[k,j]
// with Wd dequantized on chip from (packed, c1q, c2); the low-rank operand
// (sT or G) arrives as a bf16 hi/lo pair [M, 2*rp] (columns [0,rp) hi,
// [rp,2rp) lo).  When the tile grid is small the reduction is split over a
// cluster of up to 8 CTAs that sum through distributed shared memory.
struct Nf4GemmPlan {
  int backward;      // 0 forward, 1 backward
  int bt;            // token tile (MMA N): 16..256, multiple of 16
  int splits;        // split of the main reduction
  int64_t tiles_w;   // tiles along the W dimension (128 each)
  int64_t tiles_t;   // tiles along tokens
  int64_t main_steps;  // 64-wide reduction steps of the main product
  int lora_steps;    // 64-wide steps of the low-rank product (hi and lo)
};
Nf4GemmPlan plan_nf4_gemm(int backward, int64_t M, int64_t N, int64_t K, int r, int num_sms);

struct Nf4GemmArgs {
  // problem
  int64_t M, N, K;      // tokens, W rows, W cols
  int r, rp;            // LoRA rank and its padding to 64
  const uint8_t* packed;
  const uint8_t* c1q;
  const float* c2;
  const uint16_t* act;       // X (forward) or dY (backward), [M, K] or [M, N]
  const uint16_t* lora_w;    // B [r, N] (forward; read by the dequant warps) or A [K, r] (backward)
  const uint16_t* lora_act;  // sT hi/lo (forward) or G hi/lo (backward), [M, 2*rp] bf16
  uint16_t* out;             // Y [M, N] or dX [M, K], bf16
  uint32_t* status;          // kStatusTimeout on a failed wait
  int pdl_mode;              // PdlMode
  int quant_type;            // table (kQuantNf4 / kQuantInt4)
  int dq;                    // DqFormat of the first-level constants (c1q holds fp32 for kDqNone)
  int f16;                   // compute type fp16 (else bf16)
  int64_t packed_bytes;      // size of the packed array (loads past it read zeros)
  int64_t ld_act;            // row pitch (elements) of act: K or N, or a re-pitched copy's
  int64_t ld_lw;             // row pitch of lora_w (forward: B's, N or its copy's; backward: r)
};
// pdl: launch as a programmatic dependent of the previous kernel of the stream
cudaError_t launch_nf4_gemm(const Nf4GemmPlan& plan, const Nf4GemmArgs& a, cudaStream_t stream, bool pdl);

// ---------------------------------------------------------------- skinny GEMM
// D[i, j] = sum_k Aop[i,k] Bop[j,k] for the low-rank products, j < rp <= 256.
enum SkinnyKind : int {
  kSkinnyT = 0,   // T = X A      -> T bf16 [M,r], sT hi/lo [M,2rp]
  kSkinnyG = 1,   // G = s dY B^T -> G hi/lo [M,2rp]
  kSkinnyDA = 2,  // dA = X^T G   -> fp32 [K,r]   (reduction over tokens, G hi then lo)
  kSkinnyDB = 3,  // dB = s T^T dY-> fp32 [r,N]   (computed transposed, reduction over tokens)
};
struct SkinnyPlan {
  int kind;
  int64_t rows;        // extent of i
  int64_t red;         // reduction length
  int64_t tiles;       // 128-row tiles of i
  int64_t steps;       // 64-wide reduction steps (total, all passes)
  int splits;
};
SkinnyPlan plan_skinny(int kind, int64_t M, int64_t N, int64_t K, int r, int num_sms);

struct SkinnyArgs {
  int64_t M, N, K;
  int r, rp;
  float s;
  const uint16_t* X;
  const uint16_t* dY;
  const uint16_t* A;
  const uint16_t* B;
  const uint16_t* T;        // bf16 [M, r] (input of kSkinnyDB)
  const uint16_t* hilo_in;  // G hi/lo (input of kSkinnyDA)
  uint16_t* T_out;          // kSkinnyT
  uint16_t* hilo_out;       // kSkinnyT (sT) / kSkinnyG (G)
  float* f32_out;           // kSkinnyDA / kSkinnyDB
  uint32_t* status;
  int pdl_mode;             // PdlMode (kPdlWaitFirst or kPdlWaitLast)
  int f16;                  // compute type fp16 (else bf16)
  int64_t ld_x, ld_dy, ld_b;  // row pitches of X, dY, B when they are re-pitched copies (0: K, N, N)
};
cudaError_t launch_skinny(const SkinnyPlan& plan, const SkinnyArgs& a, cudaStream_t stream, bool pdl);

// ---------------------------------------------------------------- decode (1-16 tokens)
// Forward of the linear layer for M <= 16 tokens: every weight decoded once
// in registers and multiplied with all tokens on mma.sync; persistent CTAs
// over (256-row tile, 256-column chunk) units, split tiles summed in a fixed
// order by the CTA that finishes last.
struct Nf4DecodeArgs {
  int64_t M, N, K;
  int r;
  float s;
  const uint16_t* X;         // [M, K]
  const uint8_t* packed;
  const uint8_t* c1q;        // first-level constants (bytes, or fp32 for kDqNone)
  const float* c2;
  const uint16_t* T;         // [M, r] from the previous kernel of the stream
  const uint16_t* B;         // [r, N]
  uint16_t* Y;               // [M, N]
  uint32_t* status;          // kStatusTimeout on a failed wait
  int dq;                    // DqFormat
  int f16;                   // compute type fp16 (else bf16)
  float* partial;            // workspace: plan.partial_floats fp32
  int* counters;             // workspace: plan.tiles int32, zero before the launch
};
struct DecodePlan {
  int64_t tiles, nk, units, ctas;
  int64_t partial_floats;
};
bool decode_supported(int64_t M, int64_t K);
DecodePlan plan_decode(int64_t M, int64_t N, int64_t K, int num_sms);
cudaError_t launch_nf4_decode(const DecodePlan& plan, const Nf4DecodeArgs& a, const float code[16],
                              cudaStream_t stream, bool pdl);

// ---------------------------------------------------------------- generic GEMM
// C[i, j] = sum over segments of scale * sum_p a(i, p) b(j, p), on CUDA cores,
// for the linear layer's shapes outside the fused kernels.  An operand
// element (i, p) sits at base[i * si + p * sp] (bf16, fp16 or fp32); C is
// [I, J] row-major, bf16 / fp16 (round to nearest even) or fp32.
enum OperandKind : int { kOpBF16 = 0, kOpF32 = 1, kOpF16 = 2 };
struct GenericOperand {
  const void* base;
  int64_t si, sp;
  int kind;        // OperandKind
};
struct GenericSegment {
  GenericOperand a, b;
  int64_t P;       // reduction length
  float scale;
};
struct GenericGemm {
  int64_t I, J;
  int nseg;        // 1 or 2
  GenericSegment seg[2];
  void* out;
  int out_kind;    // OperandKind
};
cudaError_t launch_generic_gemm(const GenericGemm& g, int num_sms, cudaStream_t stream);

// Tensor-map helper (driver entry point resolved through the runtime).
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                    uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swizzle);

}  // namespace nf4
