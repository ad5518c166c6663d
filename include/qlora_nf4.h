/*
 * qlora_nf4.h -- C ABI of libqlora_nf4.so: 4-bit NormalFloat (NF4) storage
 * of a frozen weight with double quantization of its block constants, and
 * the QLoRA linear layer that computes in BF16 from that storage, on NVIDIA
 * B200 (sm_100a).
 *
 * Sources (web pages about QLoRA; titles and sections):
 *   [P1] "从LoRA到QLoRA：量化技术如何改变预训练模型的微调方式" -- §2.3 NF4
 *        (quantiles of N(0,1), normalized to [-1,1]); §3.1 storage type NF4,
 *        compute type BF16, gradients only for the LoRA parameters.
 *   [P2] "QLoRA 原理精讲" -- §2.1 NF4 (block of 64, absmax, nearest code);
 *        §2.2 double quantization (FP8 scale1 per 64 weights, one FP32
 *        scale2 per 256 scale1, dequantize in reverse order); §三 误区1 (LoRA
 *        factors stay BF16); §三 误区3 (serve with the adapter kept separate,
 *        dequantizing on the fly).
 *   [P4] "LoRA、Q-LoRA 与 PortLLM" (developer.volcengine.com) -- §3.1-§3.4,
 *        the QLoRA linear layer for one layer of the quantized base model.
 *
 * Conventions (all calls):
 *   - bf16 tensors are passed as uint16_t bit patterns, row-major.
 *   - Every pointer argument named d_* or documented "device" is a device
 *     pointer owned by the caller; the library allocates no memory and keeps
 *     no state between calls besides the constant NF4 table.  The one
 *     exception is qlora_linear_fwd_noalloc (below): a fixed per-device
 *     scratch array in the library's device image, and the host-side table
 *     of its device addresses, persist across its calls.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it; the return value reports argument validation and
 *     launch errors only.  Device pointers must be 16-byte aligned
 *     (NF4_ERR_MISALIGNED otherwise).
 *   - Sizes are element counts.  No kernel traps, asserts or waits without a
 *     bound: a wait that gives up sets bit 1 of the status word (below).
 *   - Status words: a device int32 the caller zero-fills and reads after the
 *     stream synchronizes: bit 0 = a NaN/Inf weight was seen by the
 *     quantizer (outputs then unspecified), bit 1 = a bounded device wait
 *     timed out (outputs unspecified).
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NF4_OK = 0,
  NF4_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad rank */
  NF4_ERR_MISALIGNED = 2,  /* a device pointer is not 16-byte aligned */
  NF4_ERR_UNSUPPORTED = 3, /* a shape the library does not handle */
  NF4_ERR_WORKSPACE = 4,   /* workspace missing or smaller than qlora_workspace_bytes() */
  NF4_ERR_NONFINITE = 5,   /* reserved for callers mapping status bit 0 */
  NF4_ERR_CUDA = 6         /* a CUDA runtime call or kernel launch failed */
} nf4_status;

/* Storage formats.  The method is NF4 codes with double quantization
 * (quant_type NF4_QUANT_NF4, double_quant NF4_DQ_E4M3; both 0, so a
 * zero-initialised format field selects it).  The variants are the ones the
 * pages set it against, selected like the pages' bnb_4bit_quant_type /
 * bnb_4bit_use_double_quant flags ([P2] §三 误区5):
 *   NF4_QUANT_INT4  the 16 evenly spaced integers -8..7 ([P2] §2.1), divided
 *                   by 8 so the table lies in [-1, 1] like NF4's: code i is
 *                   (i - 8) / 8; all-zero blocks take code 8 (0.0);
 *   NF4_DQ_NONE     no double quantization: one FP32 scale1 per block
 *                   (32/64 = 0.5 bit per weight, [P2] §2.2);
 *   NF4_DQ_U8       scale1 as an unsigned 8-bit linear code, scale2 =
 *                   max scale1 of the group / 255 (FP32), code = scale1 /
 *                   scale2 rounded to the nearest integer (ties to even),
 *                   at most 255 (an integer reading of the 8-bit scale1 of
 *                   [P4] §3.2). */
#define NF4_QUANT_NF4 0
#define NF4_QUANT_INT4 1
#define NF4_DQ_E4M3 0
#define NF4_DQ_NONE 1
#define NF4_DQ_U8 2

/* Compute types of the dequantized weight, the activations, the LoRA factors
 * and the layer's outputs: BF16 (the method, [P1] §3.1) or IEEE FP16 (the
 * pages' choice for GPUs without BF16, [P2] §三 误区4; the
 * bnb_4bit_compute_dtype flag).  Both are passed as uint16_t bit patterns. */
#define QLORA_BF16 0
#define QLORA_F16 1

/* A quantized weight W [rows, cols] (device buffers, see nf4_quantize). */
typedef struct {
  const uint8_t* packed; /* ceil(rows*cols/2) bytes */
  const uint8_t* c1q;    /* first-level constants: nblocks bytes (NF4_DQ_E4M3,
                            NF4_DQ_U8) or nblocks fp32 values, 4*nblocks bytes,
                            4-byte aligned (NF4_DQ_NONE) */
  const float* c2;       /* ngroups floats (unused, may be NULL, for NF4_DQ_NONE) */
  int64_t rows;          /* N: output features */
  int64_t cols;          /* K: input features */
  int32_t quant_type;    /* NF4_QUANT_* (0: NF4) */
  int32_t double_quant;  /* NF4_DQ_* (0: E4M3 scale1 + FP32 scale2) */
} nf4_weight;

/* The 16 NF4 values, ascending (codes) and the 15 decision thresholds
 * (thresholds[i] = midpoint of codes i and i+1 rounded down to fp32), as
 * used by the kernels.  [P1] §2.3, [P2] §2.1.  Host only; never fails. */
nf4_status nf4_build_codebook(float codes[16], float thresholds[15]);

/* Storage sizes for numel weights: packed bytes = ceil(numel/2), nblocks =
 * ceil(numel/64), ngroups = ceil(nblocks/256).  Any output may be NULL.
 * [P2] §2.2.  NF4_ERR_INVALID_ARG for numel < 1. */
nf4_status nf4_sizes(int64_t numel, size_t* packed_bytes, int64_t* nblocks, int64_t* ngroups);

/* Quantize a bf16 weight W [rows, cols] (device, row-major) to NF4 with
 * double quantization ([P2] §2.1 steps 1-3, §2.2):
 *   blocks are 64 consecutive elements of the row-major flattening, groups
 *   256 consecutive blocks (the last block and group may be short);
 *   scale1 = max |w| per block; code = nearest NF4 value to w / scale1,
 *   ties to the lower code (all-zero block -> the 0.0 code);
 *   c2 = fp32(max scale1 of the group / 448);
 *   c1q = FP8 E4M3 of fp32(scale1 / c2), nearest even, saturating at 448
 *   (0 for scale1 = 0);
 *   packed: element e in byte e/2, even e in the low nibble, pad nibble 0.
 * Outputs: packed, c1q, c2 (device, sizes from nf4_sizes).  d_status
 * (device int32, may be NULL) gets bit 0 OR-ed in when W holds NaN/Inf. */
nf4_status nf4_quantize_dq(const uint16_t* W, int64_t rows, int64_t cols, uint8_t* packed, uint8_t* c1q,
                           float* c2, int32_t* d_status, void* stream);

/* nf4_quantize_dq with a chosen storage format (NF4_QUANT_*, NF4_DQ_*):
 * same blocks, groups, nearest-code rule (on the chosen table) and packing;
 * c1 receives nblocks bytes, or nblocks fp32 values for NF4_DQ_NONE (then
 * 4-byte aligned); c2 receives ngroups floats and may be NULL for
 * NF4_DQ_NONE.  NF4_ERR_INVALID_ARG for an unknown format. */
nf4_status nf4_quantize(const uint16_t* W, int64_t rows, int64_t cols, int32_t quant_type, int32_t double_quant,
                        uint8_t* packed, void* c1, float* c2, int32_t* d_status, void* stream);

/* Double dequantization to bf16, reverse order ([P2] §2.2):
 * scale1' = fp32(E4M3 value of c1q * c2), out = bf16(fp32(code * scale1'))
 * (one fp32 multiply each, one round-to-nearest-even to bf16).
 * out: device bf16 [rows, cols]. */
nf4_status nf4_dequant_bf16(nf4_weight w, uint16_t* out, void* stream);

/* Dequantization of any storage format into a compute type (QLORA_BF16 or
 * QLORA_F16): scale1' = the FP32 scale1, or fp32(decoded 8-bit code *
 * scale2); out = round(fp32(code * scale1')) to the compute type.
 * nf4_dequant_bf16(w, out) is nf4_dequant(w, QLORA_BF16, out).
 * NF4_ERR_UNSUPPORTED above 2^37 weights (beyond any one GPU's memory). */
nf4_status nf4_dequant(nf4_weight w, int32_t dtype, uint16_t* out, void* stream);

/* Merge the adapter into the frozen weight for serving ([P2] §2.5: merged
 * weights are BF16 again and inference runs at the original speed; §三 误区3,
 * deployment path ②):
 *   out = round(Wd + s (A B)^T),  Wd = nf4_dequant(w, dtype),
 * A [K, r], B [r, N], out [N, K] (device, compute type dtype).  Arithmetic:
 * Wd as in nf4_dequant; p = sum_j A[k,j] B[j,n] accumulated in fp32 (exact
 * products, order unspecified); out = round(fma(s, p, Wd)).  1 <= r <= 256.
 * For K % 64 == 0 with N and r multiples of 8 the product runs on the tensor
 * cores behind bounded waits; there is no status word, so a wait that gave
 * up (a lost arrival, not seen in practice) would leave out unspecified. */
nf4_status nf4_lora_merge(nf4_weight w, const uint16_t* A, const uint16_t* B, int32_t r, float s, int32_t dtype,
                          uint16_t* out, void* stream);

/* Device workspace bytes needed by qlora_linear_fwd / qlora_linear_bwd for
 * M tokens, W [N, K] and rank r on the current device (0 on bad sizes). */
size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r);

/* QLoRA linear forward ([P4] §3.4; [P1] §3.1):
 *   T = bf16(X A),  Y = bf16(X Wd^T + s T B),  Wd = dequant(w) in bf16,
 * with X [M, K], A [K, r], B [r, N], Y [M, N], T [M, r] (T_out may be NULL),
 * all device bf16; s = alpha / r computed by the caller.  ws: device
 * workspace of at least qlora_workspace_bytes(M, N, K, r) bytes; its first 4
 * bytes are the status word (zeroed by the call).  1 <= r <= 256;
 * M, N, K <= 2^31, and M <= 65535 * 256 on the fused path below
 * (NF4_ERR_UNSUPPORTED otherwise, before anything is launched).
 * When K % 64 == 0, N % 8 == 0 and r % 8 == 0, Wd is formed on chip inside
 * the tensor-core product and never written to memory (1-16 tokens: the
 * decode kernel; more: the fused tensor-core GEMM).  Other shapes (rows of
 * W that do not start on an NF4 block, a row count or rank off the 8-element
 * granule) take a CUDA-core path that first dequantizes W into the workspace
 * (which then holds N * K bf16 more; N * K <= 2^40) and accumulates in fp32:
 * same results within rounding, far lower throughput. */
nf4_status qlora_linear_fwd(const uint16_t* X, int64_t M, nf4_weight w, const uint16_t* A, const uint16_t* B,
                            int32_t r, float s, uint16_t* Y, uint16_t* T_out, void* ws, size_t ws_bytes,
                            void* stream);

/* QLoRA linear backward ([P1] §3.1: the frozen weight gets no gradient; it
 * is dequantized again on chip):
 *   G = s dY B^T,  dX = bf16(dY Wd + G A^T),  dA = X^T G,  dB = s T^T dY,
 * dY [M, N] bf16, X [M, K] bf16, T [M, r] bf16 from the forward (NULL: the
 * call recomputes it), dX [M, K] bf16, dA [K, r] fp32, dB [r, N] fp32 (all
 * device).  Same workspace and shape rules as qlora_linear_fwd. */
nf4_status qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t M, nf4_weight w, const uint16_t* A,
                            const uint16_t* B, int32_t r, float s, const uint16_t* T, uint16_t* dX, float* dA,
                            float* dB, void* ws, size_t ws_bytes, void* stream);

/* qlora_linear_fwd / qlora_linear_bwd in a chosen compute type: dtype
 * QLORA_BF16 is exactly those calls; QLORA_F16 takes and returns fp16 in
 * every place they take bf16 (X, A, B, Y, T, dY, dX; Wd is formed in fp16;
 * s T and G are carried as fp16 hi/lo pairs), dA and dB stay fp32.  Any
 * storage format of w.  Same workspace, shapes and errors. */
nf4_status qlora_linear_fwd_ex(int32_t dtype, const uint16_t* X, int64_t M, nf4_weight w, const uint16_t* A,
                               const uint16_t* B, int32_t r, float s, uint16_t* Y, uint16_t* T_out, void* ws,
                               size_t ws_bytes, void* stream);
nf4_status qlora_linear_bwd_ex(int32_t dtype, const uint16_t* dY, const uint16_t* X, int64_t M, nf4_weight w,
                               const uint16_t* A, const uint16_t* B, int32_t r, float s, const uint16_t* T,
                               uint16_t* dX, float* dA, float* dB, void* ws, size_t ws_bytes, void* stream);

/* Size of the fixed scratch array behind qlora_linear_fwd_noalloc (4 MiB per
 * device, part of the library's device image). */
#define QLORA_NOALLOC_SCRATCH_BYTES (4u << 20)

/* qlora_linear_fwd with no workspace argument and no allocation.  The pages
 * have no counterpart: this is an integration entry point, not part of the
 * method.  Results equal those of qlora_linear_fwd with the same arguments.
 * Who needs it: callers that cannot allocate device memory at the point of
 * the call.  Examples are a decode loop driven from C with a device-memory
 * budget fixed at start-up (cudaMalloc / cudaFree would synchronize the
 * device between tokens and can fail once the budget is committed), and
 * hosts that only hand out input and output buffers.  The scratch is a
 * fixed device array of QLORA_NOALLOC_SCRATCH_BYTES per device:
 *  - the first call on a device, with that device current, does a one-time
 *    set-up (looks up the array's device address); make it before any
 *    stream capture begins;
 *  - when qlora_workspace_bytes(M, N, K, r) exceeds
 *    QLORA_NOALLOC_SCRATCH_BYTES the call returns NF4_ERR_WORKSPACE and
 *    launches nothing.  On the tensor-core path at r = 64 that allows M up to
 *    10922 tokens; shapes that take the generic path (see qlora_linear_fwd)
 *    also need N * K * 2 bytes for the dequantized weight, so only small
 *    ragged weights fit;
 *  - the status word (first 4 bytes of the array) is cleared on the stream by
 *    each call; qlora_linear_fwd_noalloc_info gives its device address so the
 *    caller can read it after the stream synchronizes;
 *  - calls that overlap in time on one device (other streams, other host
 *    threads) share the array and race: the caller orders them;
 *  - the device address is cached per device for the life of the process:
 *    do not use this entry point across cudaDeviceReset, which may move the
 *    array.
 * Same arguments and shape rules as qlora_linear_fwd, without ws/ws_bytes. */
nf4_status qlora_linear_fwd_noalloc(const uint16_t* X, int64_t M, nf4_weight w, const uint16_t* A,
                                    const uint16_t* B, int32_t r, float s, uint16_t* Y, uint16_t* T_out,
                                    void* stream);

/* Companion of qlora_linear_fwd_noalloc (no counterpart in the pages):
 * *scratch_bytes (may be NULL) receives QLORA_NOALLOC_SCRATCH_BYTES, and
 * *d_status_word (may be NULL) the device address, on the current device, of
 * the int32 status word the no-allocation calls write (bit 1: a bounded wait
 * gave up; outputs then unspecified).  Performs the same one-time set-up as
 * the first qlora_linear_fwd_noalloc call on the device; allocates nothing. */
nf4_status qlora_linear_fwd_noalloc_info(int32_t** d_status_word, size_t* scratch_bytes);

/* Launch plan of a qlora_linear_fwd / qlora_linear_bwd call, as the library
 * would choose it for these sizes on a device with num_sms SMs (num_sms <= 0:
 * the current device, or 148 when none is visible).  Host only: launches
 * nothing and touches no device memory.  The pages have no counterpart; it
 * exists so that callers and tests can see which kernels a shape runs.
 *   path        QLORA_PATH_FUSED: tensor-core GEMM with W dequantized on chip;
 *               QLORA_PATH_DECODE: forward with 1-16 tokens, each weight
 *               decoded once in registers and multiplied with every token
 *               (mma.sync), persistent CTAs over (tile, column chunk) units;
 *               QLORA_PATH_GENERIC: W dequantized into the workspace, then
 *               CUDA-core products (shapes off the fused kernels' granules).
 *   token_tile  fused: tokens per output tile (32, 64, 128 or 256); decode: 16.
 *   splits      fused: CTAs that share one output tile's reduction (1, 2, 4
 *               or 8, one thread-block cluster); every split gets >= 1 step.
 *               decode: persistent CTAs (min(units, SMs)).
 *   tiles_w     fused: 128-row tiles of the W dimension (N forward, K backward);
 *               decode: 256-row tiles of W.
 *   tiles_t     fused: token tiles; decode: 1.
 *   main_steps  fused: 64-wide steps of the main reduction (K forward, N
 *               backward); decode: 256-column chunks of K (units = tiles_w
 *               * main_steps).
 *   lora_steps  fused: 64-wide steps of the low-rank term (hi and lo halves).
 *   lowrank_splits[4]  splits of the low-rank products T = X A, G = s dY B^T,
 *               dA = X^T G, dB = s T^T dY (fused and decode paths; 0 where the
 *               call does not run that product).
 * Returns NF4_ERR_INVALID_ARG / NF4_ERR_UNSUPPORTED for the sizes that
 * qlora_linear_fwd / qlora_linear_bwd reject with those codes. */
#define QLORA_PATH_FUSED 0
#define QLORA_PATH_DECODE 1
#define QLORA_PATH_GENERIC 2
typedef struct {
  int32_t path;
  int32_t token_tile;
  int32_t splits;
  int32_t lora_steps;
  int64_t tiles_w;
  int64_t tiles_t;
  int64_t main_steps;
  int32_t lowrank_splits[4];
} qlora_plan;
nf4_status qlora_linear_plan(int64_t M, int64_t N, int64_t K, int32_t r, int32_t backward, int32_t num_sms,
                             qlora_plan* out);

/* Self-test of the bounded device wait every kernel of this library uses
 * (no counterpart in the pages).  Launches one thread on `stream` that waits
 * on a shared-memory barrier nothing arrives at, giving up after about
 * limit_cycles SM cycles (1 .. 2^40; the kernels use ~4e9, about 2 s): it
 * then ORs bit 1 (timeout) into *d_status (a device int32 the caller zeroed)
 * and returns, and the stream continues normally.  A lost arrival in any
 * kernel ends the same way: a status bit, never a hang. */
nf4_status nf4_wait_selftest(int32_t* d_status, int64_t limit_cycles, void* stream);

/* Human-readable name of a status code (static string). */
const char* nf4_status_str(nf4_status status);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
