// common.cuh -- sm_100a building blocks shared by the kernels of libqlora_nf4:
// bf16 helpers, mbarrier waits with a time bound, TMA (cp.async.bulk.tensor)
// and bulk-copy loads, programmatic dependent launch, and the tcgen05
// (5th-generation tensor core + tensor memory) instructions used by the GEMM
// kernels.  Inline PTX only; no CUTLASS.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "format.h"

#define NF4_DEV __device__ __forceinline__

namespace nf4 {

// ----------------------------------------------------------------------------
// Error word bits written by kernels (device status / workspace status word).
// ----------------------------------------------------------------------------
constexpr uint32_t kStatusNonfinite = 1u;   // quantize saw NaN or Inf in W
constexpr uint32_t kStatusTimeout   = 2u;   // a bounded wait gave up


NF4_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

NF4_DEV uint32_t elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "elect.sync _|P, 0xffffffff;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred;
}

// ----------------------------------------------------------------------------
// programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel of the stream runs;
// griddep_wait blocks until that kernel has completed and its memory is
// visible, griddep_launch lets the next kernel of the stream start early.
// Both are no-ops for a kernel launched without the attribute.
// ----------------------------------------------------------------------------
NF4_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
NF4_DEV void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ----------------------------------------------------------------------------
// mbarrier
// ----------------------------------------------------------------------------
NF4_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
NF4_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
NF4_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
NF4_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
NF4_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Same, but the thread may sleep in hardware until the phase completes (or
// about `hint_ns` passes), so waiting warps leave the issue slots to others.
NF4_DEV bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
// Wait for the phase with the given parity to complete.  Gives up after
// about kWaitLimitCycles SM cycles (~2 s), sets kStatusTimeout in *err (if
// any) and returns false, so a lost arrival can never hang the GPU.  Once any
// wait has failed (*abort set in shared memory), later waits return false at
// once.  Each poll lets the thread sleep in hardware until the phase completes
// (at most ~20 us), and the cycle counter is read every 16 polls, so waiting
// costs almost no issue slots and the bound stays coarse but finite.
constexpr long long kWaitLimitCycles = 4000000000ll;
NF4_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err, volatile int* abort_flag,
                       long long limit_cycles = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = -1;
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (((++spins) & 15u) == 0u) {
      if (abort_flag != nullptr && *abort_flag) return false;
      const long long now = clock64();
      if (t0 < 0) {
        t0 = now;
      } else if (now - t0 > limit_cycles) {
        if (err) atomicOr(err, kStatusTimeout);
        if (abort_flag) *abort_flag = 1;
        return false;
      }
    }
  }
}

// ----------------------------------------------------------------------------
// TMA (tensor memory accelerator)
// ----------------------------------------------------------------------------
NF4_DEV void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
// 2-D tiled load global -> shared, completion counted on *bar (bytes).
NF4_DEV void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
// Shared -> global tile store by TMA (2-D tensor map; rows past the tensor's
// extent are not written), tracked as a bulk async-group of this thread.
NF4_DEV void tma_store_2d(const CUtensorMap* m, const void* src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
NF4_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// this thread's committed bulk stores have read their shared source
NF4_DEV void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// this thread's committed bulk stores are complete
NF4_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Contiguous global -> shared copy by the bulk-copy engine, completing on an
// mbarrier; both addresses and the size are multiples of 16 bytes.
NF4_DEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Orders this thread's generic-proxy shared-memory accesses with later
// async-proxy accesses (TMA, bulk copies, MMA): after writing an operand the
// MMA will read, and after reading a slot a copy will refill.
NF4_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ----------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA, loads.
// ----------------------------------------------------------------------------
NF4_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
NF4_DEV void tmem_relinquish() {  // whole warp
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
NF4_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
NF4_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
NF4_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D(tmem) (+)= A(smem desc) * B(smem desc)^T, kind::f16 (bf16 inputs, fp32 accumulate).
NF4_DEV void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem) (+)= A(tmem) * B(smem desc)^T: A is read from tensor memory
// (M rows on the lanes, K along the 32-bit columns, two 16-bit elements per
// column, the lower index in the low half).
NF4_DEV void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The four MMAs of one 64-wide K step (K = 16 each) in one statement: A from
// tensor memory at columns a, a + 8, a + 16, a + 24, or from shared memory
// with its descriptor's address field advanced by a_inc per MMA; B's
// descriptor address field advanced by 2 (32 bytes) per MMA.  The address
// field (bits 0-13, address / 16) never carries into the next field for
// shared addresses below 256 KB.  The first MMA accumulates when acc != 0,
// the other three always.  One statement keeps the issuing thread's
// instruction count per step low: its loop paces the tensor pipe.
NF4_DEV void mma_ts_k64(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, t;\n\t.reg .b32 bl, bh, b1l, b2l, b3l, a1, a2, a3;\n\t.reg .b64 b1, b2, b3;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %4, %4;\n\t"
      "mov.b64 {bl, bh}, %2;\n\t"
      "add.u32 b1l, bl, 2;\n\tadd.u32 b2l, bl, 4;\n\tadd.u32 b3l, bl, 6;\n\t"
      "mov.b64 b1, {b1l, bh};\n\tmov.b64 b2, {b2l, bh};\n\tmov.b64 b3, {b3l, bh};\n\t"
      "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, t;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b2, %3, t;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b3, %3, t;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc)
      : "memory");
}
NF4_DEV void mma_ss_k64(uint32_t d_tmem, uint64_t a_desc, uint32_t a_inc, uint64_t b_desc, uint32_t b_inc,
                        uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, t;\n\t.reg .b32 al, ah, bl, bh, x1, x2, x3, y1, y2, y3;\n\t"
      ".reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "setp.eq.b32 t, %6, %6;\n\t"
      "mov.b64 {al, ah}, %1;\n\tmov.b64 {bl, bh}, %3;\n\t"
      "add.u32 x1, al, %2;\n\tadd.u32 x2, x1, %2;\n\tadd.u32 x3, x2, %2;\n\t"
      "add.u32 y1, bl, %4;\n\tadd.u32 y2, y1, %4;\n\tadd.u32 y3, y2, %4;\n\t"
      "mov.b64 a1, {x1, ah};\n\tmov.b64 a2, {x2, ah};\n\tmov.b64 a3, {x3, ah};\n\t"
      "mov.b64 b1, {y1, bh};\n\tmov.b64 b2, {y2, bh};\n\tmov.b64 b3, {y3, bh};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %3, %5, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %5, t;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %5, t;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %5, t;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "r"(a_inc), "l"(b_desc), "r"(b_inc), "r"(idesc), "r"(acc)
      : "memory");
}

// 32 lanes x 32 columns of 32 bit from registers into tensor memory (thread i
// of the warp -> lane base + i), then wait until the stores are done.
NF4_DEV void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),
      "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]),
      "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
// Arrive on *bar once all previously issued MMAs of this thread complete.
NF4_DEV void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Instruction descriptor, kind::f16: bf16 (or fp16) A/B, fp32 D, dense.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16, 0 = f16), 10-12 B
//   format, 15 A major (0 = K, 1 = MN), 16 B major, 17-22 N>>3, 24-28 M>>4.
// A and B always share one type.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, int a_mn_major, int b_mn_major, bool f16) {
  return (1u << 4) | (f16 ? 0u : (1u << 7) | (1u << 10)) | (uint32_t(a_mn_major) << 15) |
         (uint32_t(b_mn_major) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
  return make_idesc(M, N, a_mn_major, b_mn_major, false);
}

// Shared-memory matrix descriptor (sm_100 layout): start>>4 in bits 0-13,
// leading byte offset>>4 in 16-29, stride byte offset>>4 in 32-45,
// version 1 in bits 46-47, swizzle mode in 61-63 (2 = 128-byte swizzle).
NF4_DEV uint64_t make_sdesc_sw128(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= uint64_t((smem_addr >> 4) & 0x3FFF);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// 32 lanes x 32 columns of 32 bit: thread i of the warp <-> lane (base + i).
// Load 32 columns of this warp's 32 lanes and wait for them in the same
// statement: the destination registers of tcgen05.ld are undefined until
// tcgen05.wait::ld, and a separate wait statement would not stop the compiler
// from scheduling (non-volatile) uses of those registers ahead of it.
NF4_DEV void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]),
        "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
        "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

// ----------------------------------------------------------------------------
// thread-block clusters: rank, hardware barrier, distributed shared memory
// ----------------------------------------------------------------------------
NF4_DEV uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA in the cluster must call this (hardware barrier,
// release/acquire ordering of shared::cluster accesses around it).
NF4_DEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Address of `local`'s counterpart in the shared memory of CTA `rank`.
NF4_DEV uint32_t dsmem_addr(const void* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  return remote;
}
NF4_DEV void st_dsmem_f32x4(uint32_t remote, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(remote), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
// fp32 load from the shared memory of CTA `rank` of this cluster, at the
// address that `local` has in this CTA.
NF4_DEV float ld_dsmem_f32(const void* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// ----------------------------------------------------------------------------
// small numeric helpers
// ----------------------------------------------------------------------------
NF4_DEV float bf16lo_to_f32(uint32_t two) { return __uint_as_float(two << 16); }
NF4_DEV float bf16hi_to_f32(uint32_t two) { return __uint_as_float(two & 0xFFFF0000u); }
// Two fp32 -> packed bf16x2 (lo in bits 0-15), each rounded to nearest even.
NF4_DEV uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Same for IEEE fp16 (the FP16 compute type).
NF4_DEV uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Compute-type helpers: f16 selects IEEE fp16, else bf16 (16-bit patterns).
NF4_DEV uint32_t pack2(bool f16, float lo, float hi) { return f16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi); }
NF4_DEV float half_lo_to_f32(bool f16, uint32_t two) {
  return f16 ? __half2float(__ushort_as_half(static_cast<unsigned short>(two & 0xFFFFu))) : __uint_as_float(two << 16);
}
NF4_DEV float half_hi_to_f32(bool f16, uint32_t two) {
  return f16 ? __half2float(__ushort_as_half(static_cast<unsigned short>(two >> 16))) : __uint_as_float(two & 0xFFFF0000u);
}
// x rounded to the compute type (nearest even), as fp32.
NF4_DEV float round_to(bool f16, float x) { return half_lo_to_f32(f16, pack2(f16, x, 0.0f)); }
NF4_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}
// FP8 E4M3 code -> fp32 (exact: every E4M3 value is an fp16 value).
NF4_DEV float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  uint16_t in = static_cast<uint16_t>(code & 0xFF);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFF)));
}
// fp32 -> FP8 E4M3 code, round to nearest even, saturating to +-448.
NF4_DEV uint32_t f32_to_e4m3_satfinite(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFF;
}

}  // namespace nf4
