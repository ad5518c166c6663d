// api.cu -- the extern "C" entry points of libqlora_nf4 (include/qlora_nf4.h):
// argument validation, workspace layout, and the launch sequence of each call.
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "qlora_nf4.h"
#include "format.h"
#include "kernels.h"

namespace {

using namespace nf4;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 148;
  return sms;
}

int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// A rank off the 8-element granule (the low-rank operands' 16-byte rows)
// takes the generic CUDA-core path of generic.cu.  Every other shape runs on
// the tensor cores: K % 64 != 0 (W rows not starting on an NF4 block) in the
// fused GEMM's ragged mode, and K or N off the 8-element granule with X, dY
// and B re-pitched into the workspace (16-byte row pitches for TMA).
bool needs_generic(int64_t /*N*/, int64_t /*K*/, int r) { return r % 8 != 0; }
int64_t pitch8(int64_t n) { return (n + 7) / 8 * 8; }

// Workspace, fused path:   [status word (256 B) | low-rank hi/lo pair [M, 2rp] bf16 | T scratch [M, r] bf16]
//   plus, for 1-16 tokens (decode kernel): [fp32 partials of split tiles | tile counters]
// Workspace, generic path: [status word (256 B) | Wd [N, K] bf16 | T scratch [M, r] bf16 | G [M, r] fp32]
//   plus, when K % 8 != 0: X re-pitched [M, pitch8(K)]; when N % 8 != 0: dY
//   re-pitched [M, pitch8(N)] and B re-pitched [r, pitch8(N)]
struct WsLayout {
  size_t hilo = 0, wd = 0, t_scratch = 0, g = 0, partial = 0, counters = 0, counters_bytes = 0;
  size_t xp = 0, dyp = 0, bp = 0, total = 0;
};
constexpr size_t kHeaderBytes = 256;

WsLayout ws_layout(int64_t M, int64_t N, int64_t K, int r, int sms) {
  WsLayout L;
  size_t off = kHeaderBytes;
  if (needs_generic(N, K, r)) {
    L.wd = off;
    off += size_t(round_up(N * K * 2, 256));
    L.t_scratch = off;
    off += size_t(round_up(M * r * 2, 256));
    L.g = off;
    off += size_t(round_up(M * r * 4, 256));
    L.total = off;
    return L;
  }
  const int64_t rp = round_up(r, 64);
  L.hilo = off;
  off += size_t(round_up(M * 2 * rp * 2, 256));
  L.t_scratch = off;
  off += size_t(round_up(M * r * 2, 256));
  if (decode_supported(M, K)) {
    const DecodePlan d = plan_decode(M, N, K, sms);
    L.partial = off;
    off += size_t(round_up(d.partial_floats * 4, 256));
    L.counters = off;
    L.counters_bytes = size_t(d.tiles) * 4;
    off += size_t(round_up(d.tiles * 4, 256));
  }
  if (K % 8 != 0) {
    L.xp = off;
    off += size_t(round_up(M * pitch8(K) * 2, 256));
  }
  if (N % 8 != 0) {
    L.dyp = off;
    off += size_t(round_up(M * pitch8(N) * 2, 256));
    L.bp = off;
    off += size_t(round_up(int64_t(r) * pitch8(N) * 2, 256));
  }
  L.total = off;
  return L;
}

// 16-bit operand in the compute type (kind kOpBF16 / kOpF16) or an fp32 one
GenericOperand half_operand(int kind, const uint16_t* base, int64_t si, int64_t sp) {
  return GenericOperand{base, si, sp, kind};
}
GenericOperand f32_operand(const float* base, int64_t si, int64_t sp) { return GenericOperand{base, si, sp, kOpF32}; }

// out[I, J] = scale * sum_p a(i, p) b(j, p)
GenericGemm generic_product(int64_t I, int64_t J, GenericOperand a, GenericOperand b, int64_t P, float scale,
                            void* out, int out_kind) {
  GenericGemm g{};
  g.I = I; g.J = J; g.nseg = 1;
  g.seg[0] = GenericSegment{a, b, P, scale};
  g.out = out; g.out_kind = out_kind;
  return g;
}

// The fused GEMM puts token tiles on grid.y (at most 65535 of at most 256).
constexpr int64_t kMaxFusedTokens = int64_t(65535) * 256;

nf4_status check_sizes(int64_t M, int64_t N, int64_t K, int32_t r) {
  if (M < 1 || N < 1 || K < 1 || r < 1 || r > 256) return NF4_ERR_INVALID_ARG;
  if (N > (int64_t(1) << 31) || K > (int64_t(1) << 31) || M > (int64_t(1) << 31)) return NF4_ERR_UNSUPPORTED;
  if (needs_generic(N, K, r)) {
    if (N > (int64_t(1) << 40) / K) return NF4_ERR_UNSUPPORTED;
  } else if (M > kMaxFusedTokens && !decode_supported(M, K)) {
    return NF4_ERR_UNSUPPORTED;
  }
  return NF4_OK;
}

bool format_ok(int32_t quant_type, int32_t double_quant) {
  return (quant_type == NF4_QUANT_NF4 || quant_type == NF4_QUANT_INT4) &&
         (double_quant == NF4_DQ_E4M3 || double_quant == NF4_DQ_NONE || double_quant == NF4_DQ_U8);
}

// The storage buffers of a weight: present, in a known format, aligned.
nf4_status check_weight(const nf4_weight& w) {
  if (!format_ok(w.quant_type, w.double_quant)) return NF4_ERR_INVALID_ARG;
  if (!w.packed || !w.c1q || (w.double_quant != NF4_DQ_NONE && !w.c2)) return NF4_ERR_INVALID_ARG;
  if (!aligned16(w.packed)) return NF4_ERR_MISALIGNED;
  if (w.double_quant == NF4_DQ_NONE && (reinterpret_cast<uintptr_t>(w.c1q) & 3u) != 0) return NF4_ERR_MISALIGNED;
  return NF4_OK;
}

nf4_status check_linear_shapes(int64_t M, const nf4_weight& w, int32_t r) {
  const nf4_status st = check_sizes(M, w.rows, w.cols, r);
  if (st != NF4_OK) return st;
  return check_weight(w);
}

bool dtype_ok(int32_t dtype) { return dtype == QLORA_BF16 || dtype == QLORA_F16; }
int operand_kind(int32_t dtype) { return dtype == QLORA_F16 ? kOpF16 : kOpBF16; }

}  // namespace

extern "C" {

nf4_status nf4_build_codebook(float codes[16], float thresholds[15]) {
  const Codebook& cb = host_codebook();
  if (codes) memcpy(codes, cb.code, sizeof(cb.code));
  if (thresholds) memcpy(thresholds, cb.thr, sizeof(cb.thr));
  return NF4_OK;
}

nf4_status nf4_sizes(int64_t numel, size_t* packed_bytes, int64_t* nblocks, int64_t* ngroups) {
  if (numel < 1) return NF4_ERR_INVALID_ARG;
  if (packed_bytes) *packed_bytes = size_t(packed_bytes_of(numel));
  if (nblocks) *nblocks = nblocks_of(numel);
  if (ngroups) *ngroups = ngroups_of(numel);
  return NF4_OK;
}

nf4_status nf4_quantize(const uint16_t* W, int64_t rows, int64_t cols, int32_t quant_type, int32_t double_quant,
                        uint8_t* packed, void* c1, float* c2, int32_t* d_status, void* stream) {
  if (!format_ok(quant_type, double_quant)) return NF4_ERR_INVALID_ARG;
  if (!W || !packed || !c1 || (double_quant != NF4_DQ_NONE && !c2) || rows < 1 || cols < 1)
    return NF4_ERR_INVALID_ARG;
  if (rows > (int64_t(1) << 40) / cols) return NF4_ERR_UNSUPPORTED;
  if (!aligned16(W) || !aligned16(packed)) return NF4_ERR_MISALIGNED;
  if (double_quant == NF4_DQ_NONE && (reinterpret_cast<uintptr_t>(c1) & 3u) != 0) return NF4_ERR_MISALIGNED;
  if (!quantize_table_ok(quant_type)) return NF4_ERR_UNSUPPORTED;
  cudaError_t e = launch_quantize(W, rows * cols, quant_type, double_quant, packed, c1, c2,
                                  reinterpret_cast<uint32_t*>(d_status), device_sms(),
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NF4_OK : NF4_ERR_CUDA;
}

nf4_status nf4_quantize_dq(const uint16_t* W, int64_t rows, int64_t cols, uint8_t* packed, uint8_t* c1q, float* c2,
                           int32_t* d_status, void* stream) {
  return nf4_quantize(W, rows, cols, NF4_QUANT_NF4, NF4_DQ_E4M3, packed, c1q, c2, d_status, stream);
}

nf4_status nf4_dequant(nf4_weight w, int32_t dtype, uint16_t* out, void* stream) {
  if (!dtype_ok(dtype) || !out || w.rows < 1 || w.cols < 1) return NF4_ERR_INVALID_ARG;
  const nf4_status st = check_weight(w);
  if (st != NF4_OK) return st;
  if (w.rows > (int64_t(1) << 37) / w.cols) return NF4_ERR_UNSUPPORTED;   // the output's tile rows are int32
  if (!aligned16(out)) return NF4_ERR_MISALIGNED;
  cudaError_t e = launch_dequant(w.packed, w.c1q, w.c2, w.rows * w.cols, w.quant_type, w.double_quant,
                                 dtype == QLORA_F16, out, device_sms(), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NF4_OK : NF4_ERR_CUDA;
}

nf4_status nf4_dequant_bf16(nf4_weight w, uint16_t* out, void* stream) {
  return nf4_dequant(w, QLORA_BF16, out, stream);
}

nf4_status nf4_lora_merge(nf4_weight w, const uint16_t* A, const uint16_t* B, int32_t r, float s, int32_t dtype,
                          uint16_t* out, void* stream) {
  if (!dtype_ok(dtype) || !A || !B || !out || w.rows < 1 || w.cols < 1 || r < 1 || r > 256)
    return NF4_ERR_INVALID_ARG;
  const nf4_status st = check_weight(w);
  if (st != NF4_OK) return st;
  if (w.rows > (int64_t(1) << 40) / w.cols || w.rows > int64_t(65535) * 128) return NF4_ERR_UNSUPPORTED;
  if (!aligned16(A) || !aligned16(B) || !aligned16(out)) return NF4_ERR_MISALIGNED;
  MergeArgs a{};
  a.packed = w.packed; a.c1 = w.c1q; a.c2 = w.c2;
  a.N = w.rows; a.K = w.cols; a.double_quant = w.double_quant;
  a.A = A; a.B = B; a.r = r; a.s = s; a.f16 = dtype == QLORA_F16 ? 1 : 0; a.out = out;
  cudaError_t e = launch_merge(a, host_codebook(w.quant_type).code, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NF4_OK : NF4_ERR_CUDA;
}

size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r) {
  if (check_sizes(M, N, K, r) != NF4_OK) return 0;
  return ws_layout(M, N, K, r, device_sms()).total;
}

nf4_status qlora_linear_fwd_ex(int32_t dtype, const uint16_t* X, int64_t M, nf4_weight w, const uint16_t* A,
                               const uint16_t* B, int32_t r, float s, uint16_t* Y, uint16_t* T_out, void* ws,
                               size_t ws_bytes, void* stream) {
  if (!dtype_ok(dtype)) return NF4_ERR_INVALID_ARG;
  const int f16 = dtype == QLORA_F16 ? 1 : 0;
  const int hk = operand_kind(dtype);
  nf4_status st = check_linear_shapes(M, w, r);
  if (st != NF4_OK) return st;
  if (!X || !A || !B || !Y) return NF4_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y) || (T_out && !aligned16(T_out)))
    return NF4_ERR_MISALIGNED;
  const int sms = device_sms();
  const int64_t N = w.rows, K = w.cols;
  const WsLayout L = ws_layout(M, N, K, r, sms);
  if (!ws || ws_bytes < L.total) return NF4_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return NF4_ERR_MISALIGNED;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(wsb);
  uint16_t* hilo = reinterpret_cast<uint16_t*>(wsb + L.hilo);
  uint16_t* t_dst = T_out ? T_out : reinterpret_cast<uint16_t*>(wsb + L.t_scratch);
  const int rp = int(round_up(r, 64));

  if (cudaMemsetAsync(ws, 0, kHeaderBytes, strm) != cudaSuccess) return NF4_ERR_CUDA;

  if (needs_generic(N, K, r)) {
    // Wd = dequant(W) into the workspace, T = bf16(X A), Y = bf16(X Wd^T + s T B)
    uint16_t* wd = reinterpret_cast<uint16_t*>(wsb + L.wd);
    if (launch_dequant(w.packed, w.c1q, w.c2, N * K, w.quant_type, w.double_quant, f16, wd, sms, strm) !=
        cudaSuccess)
      return NF4_ERR_CUDA;
    const GenericGemm gt = generic_product(M, r, half_operand(hk, X, K, 1), half_operand(hk, A, 1, r), K, 1.0f,
                                           t_dst, hk);
    if (launch_generic_gemm(gt, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
    GenericGemm gy = generic_product(M, N, half_operand(hk, X, K, 1), half_operand(hk, wd, K, 1), K, 1.0f, Y, hk);
    gy.nseg = 2;
    gy.seg[1] = GenericSegment{half_operand(hk, t_dst, r, 1), half_operand(hk, B, 1, N), r, s};
    if (launch_generic_gemm(gy, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
    return NF4_OK;
  }

  // X and B with 16-byte row pitches for TMA (re-pitched copies for ragged K, N)
  const uint16_t* Xa = X;
  const uint16_t* Ba = B;
  int64_t ldk = K, ldb = N;
  if (K % 8 != 0) {
    ldk = pitch8(K);
    uint16_t* xp = reinterpret_cast<uint16_t*>(wsb + L.xp);
    if (launch_repitch(X, M, K, xp, ldk, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
    Xa = xp;
  }
  if (N % 8 != 0 && !decode_supported(M, K)) {   // the decode kernel reads B by elements
    ldb = pitch8(N);
    uint16_t* bp = reinterpret_cast<uint16_t*>(wsb + L.bp);
    if (launch_repitch(B, r, N, bp, ldb, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
    Ba = bp;
  }

  SkinnyArgs sa{};
  sa.M = M; sa.N = N; sa.K = K; sa.r = r; sa.rp = rp; sa.s = s;
  sa.X = Xa; sa.A = A; sa.B = Ba;
  sa.ld_x = ldk;
  sa.T_out = t_dst; sa.hilo_out = hilo;
  sa.status = status;
  sa.pdl_mode = kPdlWaitFirst;
  sa.f16 = f16;

  if (decode_supported(M, K)) {
    // 1-16 tokens: bound by reading the packed weight; each weight is
    // decoded once and multiplied with every token on mma.sync.  It overlaps
    // T and waits for it only before the low-rank term.
    const DecodePlan dp = plan_decode(M, N, K, sms);
    int* counters = reinterpret_cast<int*>(wsb + L.counters);
    if (cudaMemsetAsync(counters, 0, L.counters_bytes, strm) != cudaSuccess) return NF4_ERR_CUDA;
    Nf4DecodeArgs da{};
    da.M = M; da.N = N; da.K = K; da.r = r; da.s = s;
    da.X = X; da.packed = w.packed; da.c1q = w.c1q; da.c2 = w.c2;
    da.T = t_dst; da.B = B; da.Y = Y; da.status = status;
    da.dq = w.double_quant; da.f16 = f16;
    da.partial = reinterpret_cast<float*>(wsb + L.partial);
    da.counters = counters;
    if (launch_skinny(plan_skinny(kSkinnyT, M, N, K, r, sms), sa, strm, false) != cudaSuccess) return NF4_ERR_CUDA;
    if (launch_nf4_decode(dp, da, host_codebook(w.quant_type).code, strm, true) != cudaSuccess) return NF4_ERR_CUDA;
    return NF4_OK;
  }

  if (launch_skinny(plan_skinny(kSkinnyT, M, N, K, r, sms), sa, strm, false) != cudaSuccess) return NF4_ERR_CUDA;
  // The fused GEMM may start while T is still being computed: its main
  // product does not need T, and it waits for T before the low-rank steps.
  Nf4GemmArgs ga{};
  ga.M = M; ga.N = N; ga.K = K; ga.r = r; ga.rp = rp;
  ga.packed = w.packed; ga.c1q = w.c1q; ga.c2 = w.c2;
  ga.act = Xa; ga.lora_w = Ba; ga.lora_act = hilo; ga.out = Y;
  ga.ld_act = ldk; ga.ld_lw = ldb; ga.packed_bytes = packed_bytes_of(N * K);
  ga.status = status;
  ga.pdl_mode = kPdlWaitLowRank;
  ga.quant_type = w.quant_type; ga.dq = w.double_quant; ga.f16 = f16;
  if (launch_nf4_gemm(plan_nf4_gemm(0, M, N, K, r, sms), ga, strm, true) != cudaSuccess) return NF4_ERR_CUDA;
  return NF4_OK;
}

nf4_status qlora_linear_fwd(const uint16_t* X, int64_t M, nf4_weight w, const uint16_t* A, const uint16_t* B,
                            int32_t r, float s, uint16_t* Y, uint16_t* T_out, void* ws, size_t ws_bytes,
                            void* stream) {
  return qlora_linear_fwd_ex(QLORA_BF16, X, M, w, A, B, r, s, Y, T_out, ws, ws_bytes, stream);
}

nf4_status qlora_linear_bwd_ex(int32_t dtype, const uint16_t* dY, const uint16_t* X, int64_t M, nf4_weight w,
                               const uint16_t* A, const uint16_t* B, int32_t r, float s, const uint16_t* T,
                               uint16_t* dX, float* dA, float* dB, void* ws, size_t ws_bytes, void* stream) {
  if (!dtype_ok(dtype)) return NF4_ERR_INVALID_ARG;
  const int f16 = dtype == QLORA_F16 ? 1 : 0;
  const int hk = operand_kind(dtype);
  nf4_status st = check_linear_shapes(M, w, r);
  if (st != NF4_OK) return st;
  if (!dY || !X || !A || !B || !dX || !dA || !dB) return NF4_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(dX) || !aligned16(dA) ||
      !aligned16(dB) || (T && !aligned16(T)))
    return NF4_ERR_MISALIGNED;
  const int sms = device_sms();
  const int64_t N = w.rows, K = w.cols;
  const WsLayout L = ws_layout(M, N, K, r, sms);
  if (!ws || ws_bytes < L.total) return NF4_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return NF4_ERR_MISALIGNED;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(wsb);
  uint16_t* hilo = reinterpret_cast<uint16_t*>(wsb + L.hilo);
  const int rp = int(round_up(r, 64));

  if (cudaMemsetAsync(ws, 0, kHeaderBytes, strm) != cudaSuccess) return NF4_ERR_CUDA;

  if (needs_generic(N, K, r)) {
    // Wd = dequant(W); [T = bf16(X A)]; G = s dY B^T (fp32);
    // dX = bf16(dY Wd + G A^T); dA = X^T G; dB = s T^T dY
    uint16_t* wd = reinterpret_cast<uint16_t*>(wsb + L.wd);
    float* g = reinterpret_cast<float*>(wsb + L.g);
    if (launch_dequant(w.packed, w.c1q, w.c2, N * K, w.quant_type, w.double_quant, f16, wd, sms, strm) !=
        cudaSuccess)
      return NF4_ERR_CUDA;
    const uint16_t* Tin = T;
    if (!Tin) {
      uint16_t* tw = reinterpret_cast<uint16_t*>(wsb + L.t_scratch);
      const GenericGemm gt = generic_product(M, r, half_operand(hk, X, K, 1), half_operand(hk, A, 1, r), K, 1.0f,
                                             tw, hk);
      if (launch_generic_gemm(gt, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
      Tin = tw;
    }
    const GenericGemm gg = generic_product(M, r, half_operand(hk, dY, N, 1), half_operand(hk, B, N, 1), N, s, g,
                                           kOpF32);
    if (launch_generic_gemm(gg, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
    GenericGemm gx = generic_product(M, K, half_operand(hk, dY, N, 1), half_operand(hk, wd, 1, K), N, 1.0f, dX, hk);
    gx.nseg = 2;
    gx.seg[1] = GenericSegment{f32_operand(g, r, 1), half_operand(hk, A, r, 1), r, 1.0f};
    if (launch_generic_gemm(gx, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
    const GenericGemm ga = generic_product(K, r, half_operand(hk, X, 1, K), f32_operand(g, 1, r), M, 1.0f, dA,
                                           kOpF32);
    if (launch_generic_gemm(ga, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
    const GenericGemm gb = generic_product(r, N, half_operand(hk, Tin, 1, r), half_operand(hk, dY, 1, N), M, s, dB,
                                           kOpF32);
    if (launch_generic_gemm(gb, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
    return NF4_OK;
  }

  // X, dY and B with 16-byte row pitches for TMA (re-pitched copies for ragged K, N)
  const uint16_t* Xa = X;
  const uint16_t* dYa = dY;
  const uint16_t* Ba = B;
  int64_t ldk = K, ldn = N;
  if (K % 8 != 0) {
    ldk = pitch8(K);
    uint16_t* xp = reinterpret_cast<uint16_t*>(wsb + L.xp);
    if (launch_repitch(X, M, K, xp, ldk, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
    Xa = xp;
  }
  if (N % 8 != 0) {
    ldn = pitch8(N);
    uint16_t* dyp = reinterpret_cast<uint16_t*>(wsb + L.dyp);
    uint16_t* bp = reinterpret_cast<uint16_t*>(wsb + L.bp);
    if (launch_repitch(dY, M, N, dyp, ldn, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
    if (launch_repitch(B, r, N, bp, ldn, sms, strm) != cudaSuccess) return NF4_ERR_CUDA;
    dYa = dyp;
    Ba = bp;
  }

  SkinnyArgs sa{};
  sa.M = M; sa.N = N; sa.K = K; sa.r = r; sa.rp = rp; sa.s = s;
  sa.X = Xa; sa.dY = dYa; sa.A = A; sa.B = Ba;
  sa.ld_x = ldk; sa.ld_dy = ldn; sa.ld_b = ldn;
  sa.status = status;
  sa.f16 = f16;

  // Launch order and overlap: the first kernel waits for all earlier work of
  // the stream; each later one is a programmatic dependent of the one before.
  // G waits for the T recompute (both write the hi/lo buffer).  The fused
  // GEMM starts its main product (dY Wd) while G is still running and waits
  // for G before its low-rank steps; it lets dA and dB start once G is
  // complete: they read only G and the inputs, so they fill the SMs the
  // GEMM's last wave leaves idle, and wait for the GEMM only before they exit.
  const uint16_t* Tin = T;
  bool after_kernel = false;
  sa.pdl_mode = kPdlWaitFirst;
  if (!Tin) {  // recompute T = bf16(X A) into scratch (the hi/lo output is overwritten by G below)
    uint16_t* tw = reinterpret_cast<uint16_t*>(wsb + L.t_scratch);
    sa.T_out = tw;
    sa.hilo_out = hilo;
    if (launch_skinny(plan_skinny(kSkinnyT, M, N, K, r, sms), sa, strm, false) != cudaSuccess) return NF4_ERR_CUDA;
    Tin = tw;
    after_kernel = true;
  }
  // G = s dY B^T as a bf16 hi/lo pair
  sa.T_out = nullptr;
  sa.hilo_out = hilo;
  if (launch_skinny(plan_skinny(kSkinnyG, M, N, K, r, sms), sa, strm, after_kernel) != cudaSuccess)
    return NF4_ERR_CUDA;

  // dX = dY Wd + G A^T
  Nf4GemmArgs ga{};
  ga.M = M; ga.N = N; ga.K = K; ga.r = r; ga.rp = rp;
  ga.packed = w.packed; ga.c1q = w.c1q; ga.c2 = w.c2;
  ga.act = dYa; ga.lora_w = A; ga.lora_act = hilo; ga.out = dX;
  ga.ld_act = ldn; ga.ld_lw = r; ga.packed_bytes = packed_bytes_of(N * K);
  ga.status = status;
  ga.pdl_mode = kPdlWaitLowRank;
  ga.quant_type = w.quant_type; ga.dq = w.double_quant; ga.f16 = f16;
  if (launch_nf4_gemm(plan_nf4_gemm(1, M, N, K, r, sms), ga, strm, true) != cudaSuccess) return NF4_ERR_CUDA;

  // dA = X^T G  (G hi + G lo)
  sa.hilo_in = hilo;
  sa.f32_out = dA;
  sa.pdl_mode = kPdlWaitLast;
  if (launch_skinny(plan_skinny(kSkinnyDA, M, N, K, r, sms), sa, strm, true) != cudaSuccess) return NF4_ERR_CUDA;
  // dB = s T^T dY
  sa.T = Tin;
  sa.f32_out = dB;
  if (launch_skinny(plan_skinny(kSkinnyDB, M, N, K, r, sms), sa, strm, true) != cudaSuccess) return NF4_ERR_CUDA;
  return NF4_OK;
}

nf4_status qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t M, nf4_weight w, const uint16_t* A,
                            const uint16_t* B, int32_t r, float s, const uint16_t* T, uint16_t* dX, float* dA,
                            float* dB, void* ws, size_t ws_bytes, void* stream) {
  return qlora_linear_bwd_ex(QLORA_BF16, dY, X, M, w, A, B, r, s, T, dX, dA, dB, ws, ws_bytes, stream);
}

nf4_status qlora_linear_plan(int64_t M, int64_t N, int64_t K, int32_t r, int32_t backward, int32_t num_sms,
                             qlora_plan* out) {
  if (!out) return NF4_ERR_INVALID_ARG;
  const nf4_status st = check_sizes(M, N, K, r);
  if (st != NF4_OK) return st;
  const int sms = num_sms > 0 ? num_sms : device_sms();
  qlora_plan p;
  memset(&p, 0, sizeof(p));
  if (needs_generic(N, K, r)) {
    p.path = QLORA_PATH_GENERIC;
  } else if (!backward && decode_supported(M, K)) {
    const DecodePlan d = plan_decode(M, N, K, sms);
    p.path = QLORA_PATH_DECODE;
    p.token_tile = 16;
    p.splits = int32_t(d.ctas);
    p.tiles_w = d.tiles;
    p.tiles_t = 1;
    p.main_steps = d.nk;
    p.lowrank_splits[kSkinnyT] = plan_skinny(kSkinnyT, M, N, K, r, sms).splits;
  } else {
    const Nf4GemmPlan g = plan_nf4_gemm(backward ? 1 : 0, M, N, K, r, sms);
    p.path = QLORA_PATH_FUSED;
    p.token_tile = g.bt;
    p.splits = g.splits;
    p.lora_steps = g.lora_steps;
    p.tiles_w = g.tiles_w;
    p.tiles_t = g.tiles_t;
    p.main_steps = g.main_steps;
    // the forward computes T; the backward recomputes it when not given
    p.lowrank_splits[kSkinnyT] = plan_skinny(kSkinnyT, M, N, K, r, sms).splits;
    if (backward) {
      for (int kind : {kSkinnyG, kSkinnyDA, kSkinnyDB}) p.lowrank_splits[kind] = plan_skinny(kind, M, N, K, r, sms).splits;
    }
  }
  *out = p;
  return NF4_OK;
}

const char* nf4_status_str(nf4_status status) {
  switch (status) {
    case NF4_OK: return "NF4_OK";
    case NF4_ERR_INVALID_ARG: return "NF4_ERR_INVALID_ARG";
    case NF4_ERR_MISALIGNED: return "NF4_ERR_MISALIGNED";
    case NF4_ERR_UNSUPPORTED: return "NF4_ERR_UNSUPPORTED";
    case NF4_ERR_WORKSPACE: return "NF4_ERR_WORKSPACE";
    case NF4_ERR_NONFINITE: return "NF4_ERR_NONFINITE";
    case NF4_ERR_CUDA: return "NF4_ERR_CUDA";
  }
  return "NF4_ERR_UNKNOWN";
}

}  // extern "C"
