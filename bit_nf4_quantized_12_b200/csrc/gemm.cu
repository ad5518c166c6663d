// gemm.cu -- tensor-core kernels of the QLoRA linear layer on sm_100a.
//
// The layer ("LoRA、Q-LoRA 与 PortLLM" §3.4; "从LoRA到QLoRA" §3.1) is
//     Y = X Wd^T + s (X A) B,    s = alpha / r,
// with Wd the frozen NF4 weight dequantized to BF16 on the fly.  Backward
// passes gradients to X, A and B only:
//     G = s dY B^T,  dX = dY Wd + G A^T,  dA = X^T G,  dB = s T^T dY,  T = X A.
//
// nf4_gemm_kernel: the two products with the frozen weight (Y and dX).  Both
// are computed transposed, with the W dimension as the 128-row MMA "M" and
// tokens as the MMA "N" (bt <= 256), so that the dequantized weight tile is
// the A operand, written into shared memory by the dequant warps:
//   forward : A = Wd[n0:n0+128, k:k+64], K-major 128-byte-swizzled rows;
//   backward: A = Wd[n:n+64, k0:k0+128]^T, MN-major (the NF4 blocks run along
//             k, which is the MN dimension there).
// The activation operand (X or dY) is staged by TMA.  The low-rank term is
// appended as extra 64-wide reduction steps into the same fp32 accumulator,
// using a bf16 hi/lo split of s*T (forward) or G (backward) so the low-rank
// product carries ~16 significant bits.  Small grids (k/v, few tokens) split
// the reduction over a cluster of up to 8 CTAs that sum their partials
// through distributed shared memory in a fixed order.
//
// skinny_gemm_kernel: the rank-r products T, G, dA, dB (N = r padded to 64),
// both operands by TMA, split reduction over a cluster in the same way.
//
// Warp roles (nf4_gemm, 640 threads): warp 0 activation TMA producer, warp 1
// MMA issuer, warp 2 tensor-memory allocator, warp 3 packed-weight TMA
// producer, warps 4-19 four dequant warpgroups that take every fourth
// reduction step and then run the epilogue.  Every wait is bounded
// (common.cuh) and reports kStatusTimeout instead of hanging.
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include "common.cuh"
#include "kernels.h"
#include "nf4_lut.cuh"

namespace nf4 {
namespace {

constexpr int kDequantWGs = 4;                          // dequant / epilogue warpgroups
constexpr int kGemmThreads = 128 + 128 * kDequantWGs;   // + producer, MMA, allocator, spare warp
constexpr int kSkinnyThreads = 192;
constexpr int kSkinnyStages = 2;

struct Nf4GemmParams {
  CUtensorMap tm_act;   // X [M,K] / dY [M,N], bf16, box {64, bt}, 128B swizzle
  CUtensorMap tm_pk;    // packed [N, K/2] bytes; box {32,128} fwd (32-byte swizzle), {64,64} bwd (64-byte)
  CUtensorMap tm_lact;  // hi/lo [M, 2rp] bf16, box {64, bt}, 128B swizzle
  CUtensorMap tm_lw;    // forward: B [r, N], box {64, 64}; backward: A [K, r], box {64, 128}; 128B swizzle
  Nf4GemmArgs a;
  CodeTable code;
  ShiftMuls km;
  int bt;
  int splits;
  int64_t main_steps;   // total 64-wide steps of the main reduction
  int lora_steps;
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void sts16(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(uint16_t(v)) : "memory");
}
__device__ __forceinline__ void stg128(void* p, const uint4& v) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
// Barrier over the 128 threads of one warpgroup (ids 1..4; 0 is __syncthreads).
__device__ __forceinline__ void warpgroup_sync(int id) {
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}


// ---------------------------------------------------------------- kernel
__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
// Wait ignoring the abort flag (used only to drain in-flight copies/MMAs),
// bounded to ~100 ms of SM cycles.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > 200000000ll) break;
  }
}

// Ring depths.  X: the activation tile ring (TMA), P: packed NF4 tiles (TMA,
// 4 KB each, recycled as soon as a dequant warpgroup has read them), A: the
// dequantized weight operand in shared memory (16 KB per step).  The dequant
// warps compute a step before they wait for its A slot, so they run ahead of
// the tensor core by up to SA steps.
// Backward: SX = 4, SP = 8, SA = 4.  Forward: its weight operand lives in
// tensor memory (below), so the shared-memory operand ring shrinks to the one
// slot the low-rank steps use, and the activation ring takes the space: 6
// slots (5 in ragged mode, whose per-thread scratch needs the 8-slot packed
// ring), with 4 packed slots.  The activation tile (32 KB at 256 tokens) is
// the largest refill of a step; a deeper ring covers its TMA latency.
__host__ __device__ constexpr int ring_x(bool bwd, bool ragged) { return bwd ? 4 : (ragged ? 5 : 6); }
__host__ __device__ constexpr int ring_p(bool bwd, bool ragged) { return (bwd || ragged) ? 8 : 4; }
__host__ __device__ constexpr int ring_a(bool bwd) { return bwd ? 4 : 1; }
constexpr int SP = 8, SA = 4;   // the backward's packed and operand rings (the largest of each)
// Each packed and operand slot must belong to a single dequant warpgroup
// (slot = step mod ring size, warpgroup = step mod kDequantWGs).  Otherwise two
// warpgroups share a slot, one can run two barrier phases ahead, and a parity
// wait would pass on the wrong phase.
static_assert(SP % kDequantWGs == 0 && SA % kDequantWGs == 0, "ring slots must map to one dequant warpgroup");
static_assert(ring_p(false, false) % kDequantWGs == 0, "ring slots must map to one dequant warpgroup");

// Forward main steps keep the dequantized weight operand in tensor memory:
// the dequant warps store it with tcgen05.st (thread t = row t = lane t, the
// 64 weights of its row segment as 32 columns of bf16x2) and the MMA reads A
// from there.  That takes the operand's 16 KB store and 16 KB read per step
// off shared memory, whose bandwidth the activation tile, the TMA fills and
// the operand otherwise share.  The ring of SA slots sits after the
// accumulator's columns.
// The tensor-memory ring has its own SAT slots and barriers; the forward's
// low-rank steps (A = a tile of B^T, by TMA) keep the shared-memory ring.  An
// 8-deep tensor-memory ring (the dequant warpgroups up to 8 steps ahead of the
// tensor core) measured slower than 4 (809 against 852 TFLOP/s on the
// forward calls of the 7B step), so the ring stays at the shared ring's depth.
constexpr bool kTmemA = true;
constexpr int SAT = 4;
static_assert(SAT % kDequantWGs == 0, "tensor-memory ring slots must map to one dequant warpgroup");
__host__ __device__ constexpr uint32_t acc_cols_of(int bt) { return uint32_t(bt < 32 ? 32 : bt); }
__host__ __device__ constexpr uint32_t tmem_cols_of(bool bwd, int bt) {
  // accumulator [+ operand ring], rounded up to a power of two (>= 32)
  return (bwd || !kTmemA) ? acc_cols_of(bt) : (acc_cols_of(bt) + SAT * 32 <= 256 ? 256u : 512u);
}

// Ragged mode reuses the idle packed ring: 48 bytes of load slot per dequant
// thread, then the 64 x 16 lane-mask table of the two-table dequantization.
constexpr uint32_t kRaggedMaskOffset = 128 * kDequantWGs * 48;
static_assert(kRaggedMaskOffset + 64 * 16 * 8 <= SP * 4096, "ragged scratch must fit the packed ring");

// The 64 codes of flat elements e0 .. e0 + 63 (element e in nibble e - e0),
// from global memory at any nibble phase: the three 16-byte chunks that
// cover them are copied into this thread's 48-byte slot (cp.async, zero fill
// past the end of the packed array), then shifted into place.
__device__ __forceinline__ void load_codes64(const uint8_t* packed, int64_t packed_bytes, int64_t e0, uint32_t slot,
                                             uint32_t (&w)[8]) {
  const int64_t byte0 = e0 >> 1;
  const int64_t base = byte0 & ~int64_t(15);
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int64_t off = base + 16 * j;
    const int64_t left = packed_bytes - off;
    const uint32_t valid = left <= 0 ? 0u : (left >= 16 ? 16u : uint32_t(left));
    const uint8_t* src = valid ? packed + off : packed;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(slot + 16 * j), "l"(src), "r"(valid)
                 : "memory");
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  const uint32_t ob = uint32_t(byte0 - base);          // 0 .. 15
  const uint32_t wb = slot + (ob & ~3u);
  uint32_t v[9];
#pragma unroll
  for (int i = 0; i < 9; ++i) asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v[i]) : "r"(wb + 4 * i));
  const uint32_t sel = 0x3210u + 0x1111u * (ob & 3u);   // bytes ob .. ob + 3 of a word pair
  uint32_t y[9];
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = prmt(v[i], v[i + 1], sel);
  y[8] = prmt(v[8], 0u, sel);
  const uint32_t ns = (e0 & 1) ? 4u : 0u;              // odd e0: its code is the high nibble
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = __funnelshift_r(y[i], y[i + 1], ns);
}

// 64 codes -> 32 bf16x2 (or f16x2) words in element order, each element taking
// its value from t0 or, where its lane of masks[group] is set, from t1.
__device__ __forceinline__ void dequant64_two(const BlockTable& t0, const BlockTable& t1, const uint32_t (&w)[8],
                                              const uint2* masks, const ShiftMuls& km, uint32_t (&o)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    lookup8(t0, w[i], km, o[4 * i + 0], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
    uint32_t b[4];
    lookup8(t1, w[i], km, b[0], b[1], b[2], b[3]);
    const uint4 m = *reinterpret_cast<const uint4*>(masks + 2 * i);
    o[4 * i + 0] = (o[4 * i + 0] & ~m.x) | (b[0] & m.x);
    o[4 * i + 1] = (o[4 * i + 1] & ~m.y) | (b[1] & m.y);
    o[4 * i + 2] = (o[4 * i + 2] & ~m.z) | (b[2] & m.z);
    o[4 * i + 3] = (o[4 * i + 3] & ~m.w) | (b[3] & m.w);
  }
}

// RAGGED: W rows do not start on an NF4 block (K % 64 != 0).  The packed
// codes then cannot be cut into TMA boxes; each dequant thread loads its row
// segment of 64 codes straight from global memory (cp.async into a private
// slot of the idle packed ring, at any nibble phase), and a segment that
// straddles two NF4 blocks is dequantized with both blocks' tables, each
// element taking its own block's value.
template <bool BWD, bool RAGGED>
__global__ void __launch_bounds__(kGemmThreads, 1) nf4_gemm_kernel(const __grid_constant__ Nf4GemmParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const Nf4GemmArgs& a = P.a;
  const int bt = P.bt;
  const uint32_t act_bytes = uint32_t(bt) * 128u;
  constexpr int SX = ring_x(BWD, RAGGED), SP = ring_p(BWD, RAGGED), SA = ring_a(BWD);
  uint8_t* act_s = smem;                                   // SX x act_bytes
  uint8_t* pk_s = act_s + SX * act_bytes;                  // SP x 4096
  uint8_t* a_s = pk_s + SP * 4096;                         // SA x 16384
  uint64_t* bars = reinterpret_cast<uint64_t*>(a_s + SA * 16384);
  uint64_t* x_full = bars;
  uint64_t* x_empty = x_full + SX;
  uint64_t* p_full = x_empty + SX;
  uint64_t* p_empty = p_full + SP;
  uint64_t* a_full = p_empty + SP;
  uint64_t* a_empty = a_full + SA;
  uint64_t* accf = a_empty + SA;
  uint64_t* t_full = accf + 1;             // tensor-memory operand ring (forward main steps)
  uint64_t* t_empty = t_full + SAT;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(t_empty + SAT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tile_w = blockIdx.x, tile_t = blockIdx.y;
  const int split = blockIdx.z;
  const int64_t w0 = tile_w * 128;          // forward: first W row; backward: first W column
  const int64_t m0 = tile_t * bt;
  const int64_t per = (P.main_steps + P.splits - 1) / P.splits;
  const int64_t g_begin = split * per;
  const int64_t g_end = (g_begin + per < P.main_steps) ? g_begin + per : P.main_steps;
  const int64_t my_main = g_end > g_begin ? g_end - g_begin : 0;
  const int my_lora = (split == 0) ? P.lora_steps : 0;
  const int64_t nsteps = my_main + my_lora;
  const uint32_t tmem_cols = tmem_cols_of(BWD, bt);
  const uint32_t a_tmem_col = acc_cols_of(bt);   // forward: operand ring column base

  if (threadIdx.x == 32) {   // descriptor fetches overlap the setup below
    tma_prefetch_desc(&P.tm_act);
    tma_prefetch_desc(&P.tm_lact);
    tma_prefetch_desc(&P.tm_pk);
    tma_prefetch_desc(&P.tm_lw);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) { mbar_init(&x_full[s], 1); mbar_init(&x_empty[s], 1); }
    for (int s = 0; s < SP; ++s) { mbar_init(&p_full[s], 1); mbar_init(&p_empty[s], 4); }
    // backward: the 4 warps of a dequant warpgroup arrive; forward: the
    // activation producer's one arrival with the low-rank tile's bytes
    for (int s = 0; s < SA; ++s) { mbar_init(&a_full[s], BWD ? 4 : 1); mbar_init(&a_empty[s], 1); }
    for (int s = 0; s < SAT; ++s) { mbar_init(&t_full[s], 4); mbar_init(&t_empty[s], 1); }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  if (RAGGED && warp >= 4) {
    // lane masks of the two-table dequantization: for a segment whose first
    // element sits at offset o of its NF4 block, elements 64 - o .. 63 belong
    // to the next block; entry (o, group of 4) selects those 16-bit lanes
    uint2* masks = reinterpret_cast<uint2*>(pk_s + kRaggedMaskOffset);
    for (int i = threadIdx.x - 128; i < 64 * 16; i += 128 * kDequantWGs) {
      const int o = i >> 4, grp = i & 15;
      uint32_t m[2] = {0u, 0u};
      for (int e = 0; e < 4; ++e)
        if (o != 0 && 4 * grp + e >= 64 - o) m[e >> 1] |= 0xFFFFu << (16 * (e & 1));
      masks[i] = make_uint2(m[0], m[1]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (a.pdl_mode == kPdlWaitFirst) griddep_wait();
  if (a.pdl_mode != kPdlWaitLowRank || my_lora == 0) griddep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------ X producer
    if (elect_one()) {
      int64_t issued = 0;
      int lr_issued = 0;
      for (int64_t ks = 0; ks < nsteps; ++ks) {
        const int s = int(ks % SX);
        const uint32_t ph = uint32_t(ks / SX) & 1u;
        if (ks >= SX && !mbar_wait(&x_empty[s], ph ^ 1u, a.status, abort_flag)) break;
        uint8_t* dst = act_s + s * act_bytes;
        mbar_arrive_expect_tx(&x_full[s], act_bytes);
        if (ks < my_main) {
          tma_load_2d(dst, &P.tm_act, &x_full[s], int32_t((g_begin + ks) * 64), int32_t(m0));
        } else {
          if (ks == my_main && a.pdl_mode == kPdlWaitLowRank) griddep_wait();   // s*T / G come from the previous kernel
          const int l = int(ks - my_main);
          const int nchunk = a.rp / 64;
          tma_load_2d(dst, &P.tm_lact, &x_full[s], int32_t((l / nchunk) * a.rp + (l % nchunk) * 64),
                      int32_t(m0));
          if (!BWD) {
            // forward: the low-rank A operand, B^T [128 features x 64 ranks]
            // as two MN-major boxes, into the one shared operand slot once the
            // previous low-rank step's MMA has released it
            if (l >= 1 && !mbar_wait(&a_empty[0], (uint32_t(l) & 1u) ^ 1u, a.status, abort_flag)) break;
            const int c = l % nchunk;
            mbar_arrive_expect_tx(&a_full[0], 16384u);
            tma_load_2d(a_s, &P.tm_lw, &a_full[0], int32_t(w0), int32_t(c * 64));
            tma_load_2d(a_s + 8192, &P.tm_lw, &a_full[0], int32_t(w0 + 64), int32_t(c * 64));
            lr_issued = l + 1;
          }
        }
        issued = ks + 1;
      }
      if (*abort_flag) {   // let copies already in flight land before the CTA exits
        for (int64_t ks = (issued > SX ? issued - SX : 0); ks < issued; ++ks)
          mbar_drain(&x_full[ks % SX], uint32_t(ks / SX) & 1u);
        if (!BWD && lr_issued > 0) mbar_drain(&a_full[0], uint32_t(lr_issued - 1) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // A CTA with low-rank steps lets the next kernel start only once the
    // previous one is complete: in the backward that kernel (dA = X^T G)
    // reads G from the previous one.  This warp is idle while the others run
    // the main product, so the wait delays nothing.
    if (a.pdl_mode == kPdlWaitLowRank && my_lora > 0 && lane == 0) {
      griddep_wait();
      griddep_launch();
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ packed-W producer
    if (!RAGGED && elect_one()) {
      int64_t issued = 0;
      for (int64_t ks = 0; ks < my_main; ++ks) {
        const int s = int(ks % SP);
        const uint32_t ph = uint32_t(ks / SP) & 1u;
        if (ks >= SP && !mbar_wait(&p_empty[s], ph ^ 1u, a.status, abort_flag)) break;
        const int64_t g = g_begin + ks;
        mbar_arrive_expect_tx(&p_full[s], 4096u);
        if (!BWD) tma_load_2d(pk_s + s * 4096, &P.tm_pk, &p_full[s], int32_t(g * 32), int32_t(w0));
        else      tma_load_2d(pk_s + s * 4096, &P.tm_pk, &p_full[s], int32_t(w0 / 2), int32_t(g * 64));
        issued = ks + 1;
      }
      if (*abort_flag) {
        for (int64_t ks = (issued > SP ? issued - SP : 0); ks < issued; ++ks)
          mbar_drain(&p_full[ks % SP], uint32_t(ks / SP) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // A operand layouts: forward main steps K-major (rows of W), backward
    // main steps MN-major (columns of W), forward low-rank steps MN-major
    // (B^T by TMA), backward low-rank steps K-major (A by TMA).
    // One thread runs the whole loop, waits included: a warp that loops and
    // elects a lane per step to issue the MMAs (with a warp sync after them)
    // takes ~1000 cycles per step on this part, against ~550 for the four
    // 128 x 256 x 16 MMAs themselves.  Ring slots and phases advance by one
    // per step (the activation ring's size is not a power of two).
    if (elect_one()) {
      const uint32_t idesc_k = make_idesc(128, bt, 0, 0, a.f16 != 0);
      const uint32_t idesc_mn = make_idesc(128, bt, 1, 0, a.f16 != 0);
      // descriptors and tensor-memory addresses of slot 0; a slot adds its
      // byte offset / 16 to a descriptor's address field
      const uint64_t bdesc0 = make_sdesc_sw128(smem_u32(act_s), 16, 1024);
      const uint64_t adesc0_k = make_sdesc_sw128(smem_u32(a_s), 16, 1024);
      const uint64_t adesc0_mn = make_sdesc_sw128(smem_u32(a_s), 8192, 1024);
      const uint32_t ta0 = tmem_base + a_tmem_col;
      int sx = 0, st = 0, ss = 0;               // activation, tensor-memory and shared operand slots
      uint32_t xph = 0, tph = 0, sph = 0;
      for (int64_t ks = 0; ks < nsteps; ++ks) {
        // operand slot: forward main steps in the tensor-memory ring, every
        // other step in the shared-memory ring (the forward's low-rank steps
        // counted from the first of them)
        const bool a_in_tmem = !BWD && kTmemA && ks < my_main;
        const int sa = a_in_tmem ? st : ss;
        if (!mbar_wait(&x_full[sx], xph, a.status, abort_flag)) break;
        if (!mbar_wait(a_in_tmem ? &t_full[sa] : &a_full[sa], a_in_tmem ? tph : sph, a.status, abort_flag)) break;
        tc_fence_after();
        const uint64_t bdesc = bdesc0 + uint32_t(sx) * (act_bytes >> 4);
        const uint32_t acc = ks > 0 ? 1u : 0u;
        if (a_in_tmem) {
          mma_ts_k64(tmem_base, ta0 + uint32_t(sa) * 32u, bdesc, idesc_k, acc);
        } else {
          const bool a_mn = (ks < my_main) == BWD;   // backward main steps: MN-major operand
          mma_ss_k64(tmem_base, (a_mn ? adesc0_mn : adesc0_k) + uint32_t(sa) * 1024u, a_mn ? 128u : 2u, bdesc, 2u,
                     a_mn ? idesc_mn : idesc_k, acc);
        }
        mma_commit(&x_empty[sx]);
        mma_commit(a_in_tmem ? &t_empty[sa] : &a_empty[sa]);
        if (++sx == SX) { sx = 0; xph ^= 1u; }
        if (a_in_tmem) {
          if (++st == SAT) { st = 0; tph ^= 1u; }
        } else {
          if (++ss == SA) { ss = 0; sph ^= 1u; }
        }
      }
      mma_commit(accf);
      if (*abort_flag) mbar_drain(accf, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ dequant warpgroups
    // Warpgroup wg takes reduction steps wg, wg + kDequantWGs, ...; the block
    // scales (c1q, c2) of its next four steps are loaded one window ahead so
    // their global-memory latency is off the critical path.
    const int wg = (warp - 4) >> 2;
    const int t = threadIdx.x - 128 - 128 * wg;               // 0..127
    // first flat element of this thread's 64-weight row segment at step ks
    // (row n, columns k0 .. k0 + 63), or -1 when the row or the columns lie
    // outside W; with K % 64 == 0 it is the start of NF4 block e0 / 64
    auto seg_of = [&](int64_t ks) -> int64_t {
      if (ks >= my_main) return -1;
      const int64_t g = g_begin + ks;
      const int64_t n = BWD ? g * 64 + (t & 63) : w0 + t;
      const int64_t k0 = BWD ? w0 + (t >> 6) * 64 : g * 64;
      return (n < a.N && k0 < a.K) ? n * a.K + k0 : -1;
    };
    const int64_t nblk = nblocks_of(a.N * a.K);
    const bool f16 = a.f16 != 0;
    uint32_t cq[4], nq[4], cq2[4], nq2[4];
    float cc[4], nc[4], cc2[4], nc2[4];
    // the constants of the segment's block, and in ragged mode of the next
    // block when the segment reaches into it
    auto load_consts = [&](int64_t ks, uint32_t& q, float& c, uint32_t& q2, float& c2) {
      q = q2 = 0u;
      c = c2 = 0.0f;
      const int64_t e0 = seg_of(ks);
      if (e0 < 0) return;
      load_scale_parts(a.dq, a.c1q, a.c2, e0 >> 6, q, c);
      if (RAGGED && (e0 & 63) != 0 && (e0 >> 6) + 1 < nblk) load_scale_parts(a.dq, a.c1q, a.c2, (e0 >> 6) + 1, q2, c2);
    };
#pragma unroll
    for (int j = 0; j < 4; ++j) load_consts(wg + int64_t(j) * kDequantWGs, cq[j], cc[j], cq2[j], cc2[j]);
    bool ok = true;
    for (int64_t base = wg; base < nsteps && ok; base += 4 * kDequantWGs) {
#pragma unroll
      for (int j = 0; j < 4; ++j) load_consts(base + int64_t(4 + j) * kDequantWGs, nq[j], nc[j], nq2[j], nc2[j]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t ks = base + int64_t(j) * kDequantWGs;
        if (!ok || ks >= nsteps) break;
        const int64_t ls = (!BWD && kTmemA) ? ks - my_main : ks;   // shared-ring step index
        const int sa = int(ls % SA);
        const uint32_t a_ph = uint32_t(ls / SA) & 1u;
        if (ks < my_main) {
          uint32_t o[32];
          if (!RAGGED) {
            const int sp = int(ks % SP);
            if (!(ok = mbar_wait(&p_full[sp], uint32_t(ks / SP) & 1u, a.status, abort_flag))) break;
            // The packed box is swizzled (32-byte mode forward, 64-byte mode
            // backward): 16-byte chunk c of a row sits at c ^ (address bits 7
            // and up), so the 8 lanes of each load phase hit 8 different bank
            // groups.  Forward: row t, 32 bytes, chunks 0 and 1; backward: row
            // t % 64, 64 bytes, chunks 2 (t / 64) and 2 (t / 64) + 1.
            const uint32_t row = smem_u32(pk_s + sp * 4096) + (BWD ? uint32_t(t & 63) * 64u : uint32_t(t) * 32u);
            const uint32_t c0 = BWD ? uint32_t(2 * (t >> 6)) ^ ((uint32_t(t & 63) >> 1) & 3u) : (uint32_t(t) >> 2) & 1u;
            const uint4 p0 = lds128(row + (c0 << 4)), p1 = lds128(row + ((c0 ^ 1u) << 4));
            // The slot is refilled by TMA, an async-proxy write: order these
            // generic-proxy reads before it, or the refill can land first.
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_empty[sp]);
            dequant64(make_table(P.code, scale_from_parts(a.dq, cq[j], cc[j]), f16), p0, p1, P.km, o);
          } else {
            const int64_t e0 = seg_of(ks);
            uint32_t wv[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            if (e0 >= 0)
              load_codes64(a.packed, a.packed_bytes, e0, smem_u32(pk_s) + uint32_t(threadIdx.x - 128) * 48u, wv);
            const uint2* masks = reinterpret_cast<const uint2*>(pk_s + kRaggedMaskOffset) + (e0 >= 0 ? (e0 & 63) : 0) * 16;
            dequant64_two(make_table(P.code, scale_from_parts(a.dq, cq[j], cc[j]), f16),
                          make_table(P.code, scale_from_parts(a.dq, cq2[j], cc2[j]), f16), wv, masks, P.km, o);
          }
          if (!BWD && kTmemA) {
            // forward: row t of Wd into tensor memory, lane t (this warp's
            // quarter), the slot's 32 columns, once the MMA of step ks - SAT
            // has released the slot (the fence orders its reads first)
            const int ts = int(ks % SAT);
            if (ks >= SAT && !(ok = mbar_wait(&t_empty[ts], (uint32_t(ks / SAT) & 1u) ^ 1u, a.status, abort_flag)))
              break;
            tc_fence_after();
            tmem_st_32x32b_x32(tmem_base + (uint32_t((warp & 3) * 32) << 16) + a_tmem_col + uint32_t(ts) * 32u, o);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&t_full[ts]);
            continue;
          }
          // the A slot must have been released by the MMA of step ks - SA
          if (ks >= SA && !(ok = mbar_wait(&a_empty[sa], a_ph ^ 1u, a.status, abort_flag))) break;
          // forward: row t of Wd (K-major, 128-byte rows); backward: row
          // t%64 of the MN atom t/64 (64 weights along k)
          const int row_i = BWD ? (t & 63) : t;
          const uint32_t row = smem_u32(a_s + sa * 16384) + (BWD ? (t >> 6) * 8192 : 0) + (row_i >> 3) * 1024 +
                               (row_i & 7) * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            sts128(row + ((c ^ (row_i & 7)) << 4), o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[sa]);
        } else {
          // low-rank step: the A operand is a tile of a LoRA factor, by TMA
          // (forward: loaded by the activation producer; backward: A [128
          // inputs x 64 ranks], one K-major box, by this warpgroup)
          if (!BWD) continue;
          if (ls >= SA && !(ok = mbar_wait(&a_empty[sa], a_ph ^ 1u, a.status, abort_flag))) break;
          __syncwarp();
          if (lane == 0) {
            if ((warp & 3) == 0) {
              const int c = int(ks - my_main) % (a.rp / 64);
              uint8_t* dst = a_s + sa * 16384;
              mbar_arrive_expect_tx(&a_full[sa], 16384u);
              if (!BWD) {
                tma_load_2d(dst, &P.tm_lw, &a_full[sa], int32_t(w0), int32_t(c * 64));
                tma_load_2d(dst + 8192, &P.tm_lw, &a_full[sa], int32_t(w0 + 64), int32_t(c * 64));
              } else {
                tma_load_2d(dst, &P.tm_lw, &a_full[sa], int32_t(c * 64), int32_t(w0));
              }
            } else {
              mbar_arrive(&a_full[sa]);
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        cq[j] = nq[j];
        cc[j] = nc[j];
        cq2[j] = nq2[j];
        cc2[j] = nc2[j];
      }
    }

    // ------------------------------------------------------------ epilogue
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const int64_t wdim = BWD ? a.K : a.N;       // extent of the W dimension of the output
    const int nchunks = bt / 32;
    // a CTA whose share of a split reduction is empty issued no MMA: its
    // accumulator was never written and its partial is zero
    const bool got_acc = ok && nsteps > 0 && mbar_wait(accf, 0, a.status, abort_flag);
    if (got_acc) tc_fence_after();
    float* red = reinterpret_cast<float*>(act_s);   // split partial [bt][128] (the X ring is free now)
    for (int c = wg; c < nchunks; c += kDequantWGs) {
      uint32_t v[32];
      if (got_acc) {
        tmem_ld_32x32b_x32(tmem_base + lane_base + c * 32, v);   // waits for the data
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0u;
      }
      if (P.splits == 1) {
        // Stage the chunk as bf16 [32 tokens][128 rows of W] in the idle X
        // ring, then write whole 16-byte pieces of output rows.
        const uint32_t stg = smem_u32(act_s) + uint32_t(c) * (32 * 256);
#pragma unroll
        for (int j = 0; j < 32; ++j) sts16(stg + j * 256 + t * 2, pack2(a.f16 != 0, __uint_as_float(v[j]), 0.0f));
        warpgroup_sync(1 + wg);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int e = q * 128 + t;                 // 16-byte piece: token row e / 16, columns (e % 16) * 8 ...
          const int64_t m = m0 + c * 32 + (e >> 4);
          const int64_t col = w0 + (e & 15) * 8;
          if (m < a.M && col < wdim) {
            const uint4 piece = lds128(stg + uint32_t(e) * 16);
            if ((wdim & 7) == 0) {            // whole 16-byte pieces of 16-byte aligned rows
              stg128(a.out + m * wdim + col, piece);
            } else {                          // ragged rows: element stores
              const uint32_t h[4] = {piece.x, piece.y, piece.z, piece.w};
              for (int u = 0; u < 8 && col + u < wdim; ++u)
                a.out[m * wdim + col + u] = uint16_t(h[u >> 1] >> (16 * (u & 1)));
            }
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) red[(c * 32 + j) * 128 + t] = __uint_as_float(v[j]);
      }
    }
  }

  // ------------------------------------------------------------ split reduction
  // The CTAs of one output tile form a cluster along z; each sums a slice of
  // the tile's columns over every CTA's partial (distributed shared memory,
  // fixed order, so results do not depend on timing).
  if (P.splits > 1) {
    cluster_sync_all();
    if (warp >= 4) {
      const int wg = (warp - 4) >> 2;
      const int t = threadIdx.x - 128 - 128 * wg;
      const int64_t wdim = BWD ? a.K : a.N;
      const int64_t i = w0 + t;
      const float* red = reinterpret_cast<const float*>(act_s);
      const int cps = bt / P.splits;
      const int c0 = int(cluster_ctarank()) * cps;
      for (int col = c0 + wg; col < c0 + cps; col += 4 * kDequantWGs) {
        float part[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int cu = col + u * kDequantWGs;
            part[u][q] = (q < P.splits && cu < c0 + cps) ? ld_dsmem_f32(red + cu * 128 + t, uint32_t(q)) : 0.0f;
          }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float acc = 0.0f;
#pragma unroll
          for (int q = 0; q < 8; ++q) acc += part[u][q];
          const int cu = col + u * kDequantWGs;
          const int64_t m = m0 + cu;
          if (cu < c0 + cps && i < wdim && m < a.M)
            a.out[m * wdim + i] = uint16_t(pack2(a.f16 != 0, acc, 0.0f) & 0xFFFFu);
        }
      }
    }
    cluster_sync_all();
  }

  if (a.pdl_mode != kPdlWaitFirst) griddep_wait();   // complete only after the previous kernel
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// ============================================================================
// skinny GEMM for the rank-r products
// ============================================================================
struct SkinnyParams {
  CUtensorMap tm_a;
  CUtensorMap tm_b;
  SkinnyArgs a;
  int kind;
  int a_mn, b_mn;      // operand majors (1 = MN-major)
  int splits;
  int64_t steps;       // total 64-wide reduction steps
  int64_t pass_steps;  // steps per pass (dA: one pass over G hi, one over G lo)
  int64_t rows;
};


// Final values of eight consecutive columns j0..j0+7 of row i (j0 % 8 == 0):
// one 16-byte store per output row segment where the row holds all eight.
__device__ __forceinline__ void skinny_finish8(const SkinnyParams& P, int64_t i, int j0, const float (&acc)[8]) {
  const SkinnyArgs& a = P.a;
  const bool f16 = a.f16 != 0;
  switch (P.kind) {
    case kSkinnyT:
    case kSkinnyG: {
      if (i >= a.M) return;
      uint32_t hi[4], lo[4], tb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float v[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int j = j0 + 2 * u + h;
          if (P.kind == kSkinnyT) {
            const float tval = round_to(f16, acc[2 * u + h]);   // T in the compute type
            v[h] = (j < a.r) ? a.s * tval : 0.0f;
          } else {
            v[h] = (j < a.r) ? a.s * acc[2 * u + h] : 0.0f;
          }
        }
        tb[u] = pack2(f16, acc[2 * u], acc[2 * u + 1]);
        hi[u] = pack2(f16, v[0], v[1]);
        const float h0 = half_lo_to_f32(f16, hi[u]), h1 = half_hi_to_f32(f16, hi[u]);
        lo[u] = pack2(f16, v[0] - h0, v[1] - h1);
      }
      uint16_t* row = a.hilo_out + i * 2 * a.rp;
      *reinterpret_cast<uint4*>(row + j0) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(row + a.rp + j0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      if (P.kind == kSkinnyT && a.T_out != nullptr) {
        if (j0 + 8 <= a.r) {
          *reinterpret_cast<uint4*>(a.T_out + i * a.r + j0) = make_uint4(tb[0], tb[1], tb[2], tb[3]);
        } else {
          for (int u = 0; u < 8 && j0 + u < a.r; ++u)
            a.T_out[i * a.r + j0 + u] = uint16_t((u & 1) ? (tb[u >> 1] >> 16) : (tb[u >> 1] & 0xFFFFu));
        }
      }
      break;
    }
    case kSkinnyDA: {
      if (i >= a.K) return;
      float* row = a.f32_out + i * a.r;
      if (j0 + 8 <= a.r) {
        *reinterpret_cast<float4*>(row + j0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(row + j0 + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
      } else {
        for (int u = 0; u < 8 && j0 + u < a.r; ++u) row[j0 + u] = acc[u];
      }
      break;
    }
    default:  // kSkinnyDB, computed as dB^T: column j of dB^T is row j of dB
      if (i >= a.N) return;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (j0 + u < a.r) a.f32_out[int64_t(j0 + u) * a.N + i] = a.s * acc[u];
      break;
  }
}

__global__ void __launch_bounds__(kSkinnyThreads, 2) skinny_gemm_kernel(const __grid_constant__ SkinnyParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const SkinnyArgs& a = P.a;
  const int rp = a.rp;
  const uint32_t b_bytes = uint32_t(rp) * 128u;
  constexpr uint32_t a_bytes = 16384u;
  const uint32_t stage_bytes = a_bytes + b_bytes;   // multiple of 8 KB: stages stay 1024-aligned
  float* recv = reinterpret_cast<float*>(smem + kSkinnyStages * stage_bytes);   // [splits][128][rp/splits]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSkinnyStages * stage_bytes +
                                               (P.splits > 1 ? uint32_t(rp) * 512u : 0u));
  uint64_t* full = bars;
  uint64_t* empty = bars + kSkinnyStages;
  uint64_t* accf = bars + 2 * kSkinnyStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int64_t tile = blockIdx.x;
  const int split = blockIdx.y;
  const int64_t i0 = tile * 128;
  const int64_t per = (P.steps + P.splits - 1) / P.splits;
  const int64_t g_begin = split * per;
  const int64_t g_end = (g_begin + per < P.steps) ? g_begin + per : P.steps;
  const int64_t nsteps = g_end > g_begin ? g_end - g_begin : 0;
  const uint32_t tmem_cols = rp <= 32 ? 32u : (rp <= 64 ? 64u : (rp <= 128 ? 128u : 256u));

  if (threadIdx.x == 32) {
    tma_prefetch_desc(&P.tm_a);
    tma_prefetch_desc(&P.tm_b);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSkinnyStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (a.pdl_mode == kPdlWaitFirst) griddep_wait();
  griddep_launch();

  if (warp == 0) {
    if (elect_one()) {
      int64_t issued = 0;
      for (int64_t ks = 0; ks < nsteps; ++ks) {
        const int s = int(ks % kSkinnyStages);
        const uint32_t ph = uint32_t(ks / kSkinnyStages) & 1u;
        if (ks >= kSkinnyStages && !mbar_wait(&empty[s], ph ^ 1u, a.status, abort_flag)) break;
        const int64_t g = g_begin + ks;
        const int64_t pass = g / P.pass_steps, gi = g % P.pass_steps;
        uint8_t* as = smem + s * stage_bytes;
        uint8_t* bs = as + a_bytes;
        mbar_arrive_expect_tx(&full[s], a_bytes + b_bytes);
        const int32_t kc = int32_t(gi * 64);
        if (P.a_mn) {   // two 64x64 boxes along the MN dimension
          tma_load_2d(as, &P.tm_a, &full[s], int32_t(i0), kc);
          tma_load_2d(as + 8192, &P.tm_a, &full[s], int32_t(i0 + 64), kc);
        } else {
          tma_load_2d(as, &P.tm_a, &full[s], kc, int32_t(i0));
        }
        if (P.b_mn) {
          for (int q = 0; q < rp / 64; ++q)
            tma_load_2d(bs + q * 8192, &P.tm_b, &full[s], int32_t(pass * rp + q * 64), kc);
        } else {
          tma_load_2d(bs, &P.tm_b, &full[s], kc, 0);
        }
        issued = ks + 1;
      }
      if (*abort_flag) {
        for (int64_t ks = (issued > kSkinnyStages ? issued - kSkinnyStages : 0); ks < issued; ++ks)
          mbar_drain(&full[ks % kSkinnyStages], uint32_t(ks / kSkinnyStages) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // one thread runs the whole MMA loop (see the fused kernel's issuer)
    if (elect_one()) {
      const uint32_t idesc = make_idesc(128, rp, P.a_mn, P.b_mn, a.f16 != 0);
      int s = 0;
      uint32_t ph = 0;
      for (int64_t ks = 0; ks < nsteps; ++ks) {
        if (!mbar_wait(&full[s], ph, a.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t aa = smem_u32(smem + s * stage_bytes);
        const uint32_t ba = aa + a_bytes;
        mma_ss_k64(tmem_base, make_sdesc_sw128(aa, P.a_mn ? 8192 : 16, 1024), P.a_mn ? 128u : 2u,
                   make_sdesc_sw128(ba, P.b_mn ? 8192 : 16, 1024), P.b_mn ? 128u : 2u, idesc, ks > 0 ? 1u : 0u);
        mma_commit(&empty[s]);
        if (++s == kSkinnyStages) { s = 0; ph ^= 1u; }
      }
      mma_commit(accf);
      if (*abort_flag) mbar_drain(accf, 0);
    }
    __syncwarp();
  } else {
    // epilogue: warps 2..5, TMEM lane quarter = warp % 4
    const int q = warp & 3;
    const int t = q * 32 + (threadIdx.x & 31);
    const uint32_t lane_base = uint32_t(q * 32) << 16;
    const int64_t i = i0 + t;
    const bool got = nsteps > 0 && mbar_wait(accf, 0, a.status, abort_flag);
    if (got) tc_fence_after();
    // Split partials: each CTA of the cluster owns rp/splits columns; every
    // CTA pushes its partial of those columns into the owner's receive
    // buffer with 16-byte remote stores (no round trips), then one cluster
    // barrier, then the owner sums the slices in a fixed order.
    const int jps = rp / P.splits;
    const uint32_t me = P.splits > 1 ? cluster_ctarank() : 0u;
    for (int c = 0; c < rp / 32; ++c) {
      uint32_t v[32];
      if (got) {
        tmem_ld_32x32b_x32(tmem_base + lane_base + c * 32, v);   // waits for the data
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0u;
      }
      if (P.splits == 1) {
#pragma unroll
        for (int j8 = 0; j8 < 32; j8 += 8) {
          float acc[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) acc[u] = __uint_as_float(v[j8 + u]);
          skinny_finish8(P, i, c * 32 + j8, acc);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const int jj = c * 32 + j;
          const int owner = jj / jps;
          float* slot = recv + (int(me) * 128 + t) * jps + (jj - owner * jps);
          st_dsmem_f32x4(dsmem_addr(slot, uint32_t(owner)), __uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                         __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
        }
      }
    }
  }

  if (P.splits > 1) {
    cluster_sync_all();
    if (warp >= 2) {
      const int t = (warp & 3) * 32 + (threadIdx.x & 31);
      const int64_t i = i0 + t;
      const int jps = rp / P.splits;
      const int j0 = int(cluster_ctarank()) * jps;
      for (int jj = 0; jj < jps; jj += 8) {
        float acc[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = 0.0f;
        for (int q = 0; q < P.splits; ++q) {
          const float4* src = reinterpret_cast<const float4*>(recv + (q * 128 + t) * jps + jj);
          const float4 x0 = src[0], x1 = src[1];
          acc[0] += x0.x; acc[1] += x0.y; acc[2] += x0.z; acc[3] += x0.w;
          acc[4] += x1.x; acc[5] += x1.y; acc[6] += x1.z; acc[7] += x1.w;
        }
        skinny_finish8(P, i, j0 + jj, acc);
      }
    }
  }

  if (a.pdl_mode != kPdlWaitFirst) griddep_wait();   // complete only after the previous kernel
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// ---------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Split of the reduction: 1, 2, 4 or 8 CTAs per output tile, launched as one
// thread-block cluster (portable size <= 8) that reduces through distributed
// shared memory.  Used only when the tile grid alone leaves SMs idle.
static int choose_splits(int64_t base_ctas, int64_t steps, int num_sms, int min_steps, int64_t cap8) {
  if (base_ctas >= num_sms) return 1;
  for (int s : {8, 4, 2}) {
    const int64_t cap = (s == 8) ? cap8 : num_sms;
    const int64_t per = (steps + s - 1) / s;
    // every split gets at least one step (the last one gets steps - (s-1) per)
    if (base_ctas * s <= cap && steps / s >= min_steps && (s - 1) * per < steps) return s;
  }
  return 1;
}

Nf4GemmPlan plan_nf4_gemm(int backward, int64_t M, int64_t N, int64_t K, int r, int num_sms) {
  Nf4GemmPlan p{};
  p.backward = backward;
  p.bt = M <= 32 ? 32 : (M <= 64 ? 64 : (M <= 128 ? 128 : 256));
  const int64_t wdim = backward ? K : N;
  p.tiles_w = cdiv(wdim, 128);
  p.tiles_t = cdiv(M, p.bt);
  p.main_steps = backward ? cdiv(N, 64) : cdiv(K, 64);
  const int rp = int(cdiv(r, 64) * 64);
  p.lora_steps = 2 * (rp / 64);
  p.splits = choose_splits(p.tiles_w * p.tiles_t, p.main_steps, num_sms, 4, (num_sms * 7) / 8);
  return p;
}

SkinnyPlan plan_skinny(int kind, int64_t M, int64_t N, int64_t K, int /*r*/, int num_sms) {
  SkinnyPlan p{};
  p.kind = kind;
  switch (kind) {
    case kSkinnyT: p.rows = M; p.red = K; p.steps = cdiv(K, 64); break;
    case kSkinnyG: p.rows = M; p.red = N; p.steps = cdiv(N, 64); break;
    case kSkinnyDA: p.rows = K; p.red = M; p.steps = 2 * cdiv(M, 64); break;
    default: p.rows = N; p.red = M; p.steps = cdiv(M, 64); break;
  }
  p.tiles = cdiv(p.rows, 128);
  p.splits = choose_splits(p.tiles, p.steps, 2 * num_sms, 2, (2 * num_sms * 7) / 8);
  // Beside a fused GEMM whose tiles fill the SMs without a split (more than
  // 16 tokens), the rank-r kernels compete with it for SMs, and fewer,
  // longer CTAs serve it better than clusters of short ones.  T runs beside
  // the forward GEMM's first wave, which its CTAs would keep off the SMs: at
  // most 2 ways while each partial sum stays within 128 steps (8192 terms);
  // a longer reduction keeps its split, so that the fp32 sums that T's bf16
  // rounding sees stay accurate (4 ways measured slower than 2 or 8 on the
  // 4096 x 11008 forward).  dA and dB run beside the dX GEMM's last wave on
  // the few SMs it leaves idle: unsplit.  G keeps its split (dA starts only
  // once G is complete) unless the dX GEMM runs in less than one wave: then
  // G's CTAs must fit in the SMs the GEMM leaves idle, 2 ways at most (the
  // 70B gate backward at 512 tokens: 228 instead of 274 us).  At 2048
  // tokens this took the 4096 x 4096 forward from 82 to 70 us and the
  // backward from 106 to 84 us.  A GEMM that splits its own reduction is
  // short, T must then finish early, and every kernel keeps its split.
  // (1-16 tokens: T runs beside the decode kernel, unchanged.)
  if (M > 16) {
    const bool bwd = kind != kSkinnyT;
    const Nf4GemmPlan g = plan_nf4_gemm(bwd ? 1 : 0, M, N, K, 64, num_sms);
    if (g.splits == 1) {
      int cap = 1;
      if (kind == kSkinnyT) cap = cdiv(p.steps, 2) <= 128 ? 2 : 8;
      if (kind == kSkinnyG) cap = g.tiles_w * g.tiles_t < num_sms ? 2 : 8;
      if (p.splits > cap) p.splits = cap;
    }
  }
  return p;
}

template <class Params>
static cudaError_t launch_clustered(void (*kern)(const Params), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t stream, dim3 cluster, bool pdl, const Params& P) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (cluster.x * cluster.y * cluster.z > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster.x;
    attr[n].val.clusterDim.y = cluster.y;
    attr[n].val.clusterDim.z = cluster.z;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, P);
}

static size_t nf4_gemm_smem(int backward, bool ragged, int bt) {
  return 1024 + size_t(ring_x(backward != 0, ragged)) * bt * 128 + size_t(ring_p(backward != 0, ragged)) * 4096 +
         size_t(ring_a(backward != 0)) * 16384 + 512;
}
static size_t skinny_smem(int rp, int splits) {
  return 1024 + size_t(kSkinnyStages) * (16384 + size_t(rp) * 128) + (splits > 1 ? size_t(rp) * 512 : 0) + 256;
}

cudaError_t launch_nf4_gemm(const Nf4GemmPlan& plan, const Nf4GemmArgs& a, cudaStream_t stream, bool pdl) {
  Nf4GemmParams P;
  memset(&P, 0, sizeof(P));
  P.a = a;
  P.bt = plan.bt;
  P.splits = plan.splits;
  P.main_steps = plan.main_steps;
  P.lora_steps = plan.lora_steps;
  const Codebook& cb = host_codebook(a.quant_type);
  for (int i = 0; i < 16; ++i) P.code.v[i] = cb.code[i];
  P.km = make_shift_muls();
  // 2-byte elements; TMA only moves them, so bf16 and fp16 share the map type
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  bool ok = true;
  const uint64_t M = a.M, N = a.N, K = a.K;
  const uint64_t hw = 2 * uint64_t(a.rp);
  const uint32_t act_box = uint32_t(plan.bt);
  // activations and B may sit in re-pitched copies (row pitch ld_act / ld_lw
  // elements, a multiple of 8); their extents stay the logical K and N, so TMA
  // fills everything past them with zeros
  const bool ragged = K % 64 != 0;
  const uint64_t lda = uint64_t(a.ld_act), ldl = uint64_t(a.ld_lw);
  if (!plan.backward) {
    ok &= encode_tmap_2d(&P.tm_act, BF, a.act, K, M, lda * 2, 64, act_box, SW);
    if (!ragged) ok &= encode_tmap_2d(&P.tm_pk, U8, a.packed, K / 2, N, K / 2, 32, 128, CU_TENSOR_MAP_SWIZZLE_32B);
    ok &= encode_tmap_2d(&P.tm_lw, BF, a.lora_w, N, uint64_t(a.r), ldl * 2, 64, 64, SW);
  } else {
    ok &= encode_tmap_2d(&P.tm_act, BF, a.act, N, M, lda * 2, 64, act_box, SW);
    if (!ragged) ok &= encode_tmap_2d(&P.tm_pk, U8, a.packed, K / 2, N, K / 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_64B);
    ok &= encode_tmap_2d(&P.tm_lw, BF, a.lora_w, uint64_t(a.r), K, uint64_t(a.r) * 2, 64, 128, SW);
  }
  ok &= encode_tmap_2d(&P.tm_lact, BF, a.lora_act, hw, M, hw * 2, 64, act_box, SW);
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = nf4_gemm_smem(plan.backward, ragged, plan.bt);
  dim3 grid(unsigned(plan.tiles_w), unsigned(plan.tiles_t), unsigned(plan.splits));
  void (*kern)(const Nf4GemmParams);
  if (ragged) kern = plan.backward ? nf4_gemm_kernel<true, true> : nf4_gemm_kernel<false, true>;
  else kern = plan.backward ? nf4_gemm_kernel<true, false> : nf4_gemm_kernel<false, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  return launch_clustered(kern, grid, dim3(kGemmThreads), smem, stream, dim3(1, 1, unsigned(plan.splits)), pdl, P);
}

cudaError_t launch_skinny(const SkinnyPlan& plan, const SkinnyArgs& a, cudaStream_t stream, bool pdl) {
  SkinnyParams P;
  memset(&P, 0, sizeof(P));
  P.a = a;
  P.kind = plan.kind;
  P.splits = plan.splits;
  P.steps = plan.steps;
  P.rows = plan.rows;
  P.pass_steps = plan.steps;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;   // 2-byte elements (bf16 or fp16)
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  const uint64_t M = a.M, N = a.N, K = a.K, r = uint64_t(a.r), rp = uint64_t(a.rp);
  // row pitches (elements) of X, dY and B: their re-pitched copies for ragged shapes
  const uint64_t ldk = a.ld_x ? uint64_t(a.ld_x) : K;
  const uint64_t ldn = a.ld_dy ? uint64_t(a.ld_dy) : N;
  const uint64_t ldb = a.ld_b ? uint64_t(a.ld_b) : N;
  bool ok = true;
  switch (plan.kind) {
    case kSkinnyT:   // A-op X [M,K] K-major; B-op A [K,r] MN-major
      P.a_mn = 0; P.b_mn = 1;
      ok &= encode_tmap_2d(&P.tm_a, BF, a.X, K, M, ldk * 2, 64, 128, SW);
      ok &= encode_tmap_2d(&P.tm_b, BF, a.A, r, K, r * 2, 64, 64, SW);
      break;
    case kSkinnyG:   // A-op dY [M,N] K-major; B-op B [r,N] K-major
      P.a_mn = 0; P.b_mn = 0;
      ok &= encode_tmap_2d(&P.tm_a, BF, a.dY, N, M, ldn * 2, 64, 128, SW);
      ok &= encode_tmap_2d(&P.tm_b, BF, a.B, N, r, ldb * 2, 64, uint32_t(rp), SW);
      break;
    case kSkinnyDA:  // A-op X^T (MN-major view of X); B-op G hi/lo MN-major
      P.a_mn = 1; P.b_mn = 1;
      P.pass_steps = plan.steps / 2;
      ok &= encode_tmap_2d(&P.tm_a, BF, a.X, K, M, ldk * 2, 64, 64, SW);
      ok &= encode_tmap_2d(&P.tm_b, BF, a.hilo_in, 2 * rp, M, 2 * rp * 2, 64, 64, SW);
      break;
    default:         // dB^T: A-op dY^T (MN-major view of dY); B-op T MN-major
      P.a_mn = 1; P.b_mn = 1;
      ok &= encode_tmap_2d(&P.tm_a, BF, a.dY, N, M, ldn * 2, 64, 64, SW);
      ok &= encode_tmap_2d(&P.tm_b, BF, a.T, r, M, r * 2, 64, 64, SW);
      break;
  }
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = skinny_smem(a.rp, plan.splits);
  cudaError_t e = cudaFuncSetAttribute(skinny_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(unsigned(plan.tiles), unsigned(plan.splits));
  return launch_clustered(skinny_gemm_kernel, grid, dim3(kSkinnyThreads), smem, stream,
                          dim3(1, unsigned(plan.splits), 1), pdl, P);
}

}  // namespace nf4
