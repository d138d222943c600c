// fp8q_ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers with
// bounded waits, TMA tiled loads, tcgen05 (TMEM alloc, MMA, commit, loads),
// E4M3 conversion and packed FP32 FMA.  Hand-written; every wrapper is one
// PTX instruction (or a short fixed sequence) whose semantics are those of
// the PTX ISA.
#pragma once

#include <cuda.h>
#include <cstdint>

namespace fp8q {

// Device status word written by bounded waits that run out.
constexpr uint32_t kDevErrTimeout = 0x80000000u;
// Also set when a kernel's final drain (its own copies or MMAs still in
// flight after an abort) ran out of its fixed bound.
constexpr uint32_t kDevErrDrain = 0x40000000u;
// Fixed bound of those drains, independent of the caller's wait limit: the
// copies and MMAs being drained complete in microseconds on a healthy GPU.
constexpr uint64_t kDrainNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// `count` arrivals at once (count >= 1).
__device__ __forceinline__ void mbar_arrive_cnt(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Suspend-time hint of the blocking probe: short, so a waiting thread notices
// a completed phase quickly (measured faster than the default on B200).
constexpr uint32_t kTryWaitSuspendNs = 20;

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity), "n"(kTryWaitSuspendNs)
      : "memory");
  return done != 0;
}

// Non-blocking probe: true when the phase with the given parity has completed.
// Its result arrives after the probe's latency, so it can be issued early and
// consumed later.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Per-launch wait control: the time limit, the global status word, and a
// shared-memory abort flag that lets the other roles of the CTA stop quickly
// once one of them has given up.
struct WaitCtl {
  uint64_t timeout_ns;
  uint32_t* status;        // global
  volatile int* abort;     // shared
};

__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, WaitCtl w, uint32_t site) {
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    for (int i = 0; i < 128; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort) return false;
    if (globaltimer_ns() - t0 > w.timeout_ns) {
      atomicCAS(w.status, 0u, kDevErrTimeout | site);
      *w.abort = 1;
      return false;
    }
  }
}

// Drain wait: polls the phase for at most kDrainNs, whatever the caller's
// limit; if it runs out, records a drain timeout.  Returns whether the phase
// completed.
__device__ __noinline__ bool mbar_drain(uint32_t bar, uint32_t parity, uint32_t* status) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainNs) {
      atomicOr(status, kDevErrTimeout | kDevErrDrain);
      return false;
    }
  }
  return true;
}

// mbar_wait with its slow loop inlined.  For code that runs with more
// registers than the kernel was launched with (after setmaxnreg.inc): ptxas
// cannot allocate such a region if it calls an out-of-line function.
__device__ __forceinline__ bool mbar_wait_inl(uint32_t bar, uint32_t parity, const WaitCtl& w, uint32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    for (int i = 0; i < 128; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort) return false;
    if (globaltimer_ns() - t0 > w.timeout_ns) {
      atomicCAS(w.status, 0u, kDevErrTimeout | site);
      *w.abort = 1;
      return false;
    }
  }
}

// Register split between warpgroups (every warp of a warpgroup executes the
// same one): dec hands registers back to the CTA's pool, inc waits until the
// pool has them.  The counts must add up to at most the launch's allocation.
template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}

// Waits until the phase with the given parity has completed.  Returns false
// (after recording a timeout) if it does not within the limit.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCtl& w, uint32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, w, site);
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// 16 bytes of shared memory as two packed FP32 pairs; addr 16-byte aligned.
__device__ __forceinline__ void lds_v2_b64(uint32_t addr, uint64_t& a, uint64_t& b) {
  asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(addr) : "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled bulk copy global -> shared, completing on `bar` (tx bytes).
// x is the innermost (contiguous) coordinate in elements, y the row.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Untiled bulk copy global -> shared of `bytes` (a multiple of 16; both
// addresses 16-byte aligned), completing on `bar` (tx bytes).  No multicast.
__device__ __forceinline__ void bulk_load_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major operand tile stored with the
// 128-byte swizzle (rows of 128 bytes, 8-row groups 1024 bytes apart), as
// written by a TMA load with CU_TENSOR_MAP_SWIZZLE_128B into a 1024-byte
// aligned buffer.  Fields: start address >> 4 (bits 0-13), leading byte
// offset >> 4 (16-29, unused for this layout), stride byte offset >> 4
// (32-45), descriptor version 1 (46-47), swizzle mode 2 = 128B (61-63).
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma.kind::f8f6f4 with E4M3 x E4M3 -> F32,
// both operands K-major: D format (bits 4-5) = 1 (F32), A/B formats (7-9,
// 10-12) = 0 (E4M3), N >> 3 (17-22), M >> 4 (24-28).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int m, int n) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T for one K = 32 step of FP8 operands.
__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor, K-major without swizzle: 8-row core
// matrices of 16-byte rows stored contiguously (128 bytes), consecutive core
// matrices along M/N `sbo` bytes apart.  Fields as smem_desc_k_sw128, layout
// type 0 (no swizzle); the leading byte offset is unused for one 16-byte
// column.
__device__ __forceinline__ uint64_t smem_desc_k_none(uint32_t saddr, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(sbo >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// Instruction descriptor of tcgen05.mma.kind::mxf8f6f4.block_scale, E4M3 x
// E4M3 -> F32, both operands K-major, UE8M0 scale factors: B scale-factor id
// (bits 4-5), A/B formats (7-9, 10-12) = 0 (E4M3), N >> 3 (17-22), scale
// format (23) = 1 (E8M0), M >> 4 (24-28), A scale-factor id (29-30).  The ids
// pick the byte of each 32-bit scale-factor column that this K = 32 step uses.
__host__ __device__ constexpr uint32_t idesc_mx_e4m3(int m, int n, uint32_t sfa_id, uint32_t sfb_id) {
  return (sfb_id << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(m >> 4) << 24) | (sfa_id << 29);
}

// D[tmem] (+)= (A * SFA)[smem] * (B * SFB)[smem]^T for one K = 32 step: each
// row's 32-element block of A and of B scaled by 2^(sf - 127) in the tensor
// core.  sfa/sfb: TMEM addresses of the scale-factor columns (the byte this
// step uses also in bits 30-31, as the instruction descriptor's ids).
__device__ __forceinline__ void mma_mx_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
      : "memory");
}

// Shared -> TMEM copy of 32 rows x 128 bits (rows 16 bytes apart, described
// by `sdesc`) into 32 lanes x 4 columns at `taddr`, replicated into all four
// 32-lane quarters.  Executes in order with this thread's tcgen05.mma.
__device__ __forceinline__ void tmem_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Arrives once on `bar` when every previously issued tcgen05.mma of this
// thread has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}


// 32 lanes x 64 consecutive 32-bit columns (two 32-column loads), waited for
// and returned as 32 packed pairs of FP32 values (column 2i in the low half of
// p[i]).  The pairing happens after the wait inside one asm block, so the
// register allocator can place each pair directly.
__device__ __forceinline__ void tmem_ld_32x32b_x64_pairs(uint32_t taddr, uint64_t (&p)[32]) {
  asm volatile(
      "{\n\t.reg .b32 r0,r1,r2,r3,r4,r5,r6,r7,r8,r9,r10,r11,r12,r13,r14,r15,r16,r17,r18,r19,r20,r21,r22,r23,r24,r25,r26,r27,r28,r29,r30,r31;\n\t"
      ".reg .b32 q0,q1,q2,q3,q4,q5,q6,q7,q8,q9,q10,q11,q12,q13,q14,q15,q16,q17,q18,q19,q20,q21,q22,q23,q24,q25,q26,q27,q28,q29,q30,q31;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {r0,r1,r2,r3,r4,r5,r6,r7,r8,r9,r10,r11,r12,r13,r14,r15,r16,r17,r18,r19,r20,r21,r22,r23,r24,r25,r26,r27,r28,r29,r30,r31}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {q0,q1,q2,q3,q4,q5,q6,q7,q8,q9,q10,q11,q12,q13,q14,q15,q16,q17,q18,q19,q20,q21,q22,q23,q24,q25,q26,q27,q28,q29,q30,q31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t"
      "mov.b64 %0, {r0, r1};\n\t"
      "mov.b64 %1, {r2, r3};\n\t"
      "mov.b64 %2, {r4, r5};\n\t"
      "mov.b64 %3, {r6, r7};\n\t"
      "mov.b64 %4, {r8, r9};\n\t"
      "mov.b64 %5, {r10, r11};\n\t"
      "mov.b64 %6, {r12, r13};\n\t"
      "mov.b64 %7, {r14, r15};\n\t"
      "mov.b64 %8, {r16, r17};\n\t"
      "mov.b64 %9, {r18, r19};\n\t"
      "mov.b64 %10, {r20, r21};\n\t"
      "mov.b64 %11, {r22, r23};\n\t"
      "mov.b64 %12, {r24, r25};\n\t"
      "mov.b64 %13, {r26, r27};\n\t"
      "mov.b64 %14, {r28, r29};\n\t"
      "mov.b64 %15, {r30, r31};\n\t"
      "mov.b64 %16, {q0, q1};\n\t"
      "mov.b64 %17, {q2, q3};\n\t"
      "mov.b64 %18, {q4, q5};\n\t"
      "mov.b64 %19, {q6, q7};\n\t"
      "mov.b64 %20, {q8, q9};\n\t"
      "mov.b64 %21, {q10, q11};\n\t"
      "mov.b64 %22, {q12, q13};\n\t"
      "mov.b64 %23, {q14, q15};\n\t"
      "mov.b64 %24, {q16, q17};\n\t"
      "mov.b64 %25, {q18, q19};\n\t"
      "mov.b64 %26, {q20, q21};\n\t"
      "mov.b64 %27, {q22, q23};\n\t"
      "mov.b64 %28, {q24, q25};\n\t"
      "mov.b64 %29, {q26, q27};\n\t"
      "mov.b64 %30, {q28, q29};\n\t"
      "mov.b64 %31, {q30, q31};\n\t"
      "}"
      : "=l"(p[0]), "=l"(p[1]), "=l"(p[2]), "=l"(p[3]), "=l"(p[4]), "=l"(p[5]), "=l"(p[6]), "=l"(p[7]), "=l"(p[8]), "=l"(p[9]), "=l"(p[10]), "=l"(p[11]), "=l"(p[12]), "=l"(p[13]), "=l"(p[14]), "=l"(p[15]), "=l"(p[16]), "=l"(p[17]), "=l"(p[18]), "=l"(p[19]), "=l"(p[20]), "=l"(p[21]), "=l"(p[22]), "=l"(p[23]), "=l"(p[24]), "=l"(p[25]), "=l"(p[26]), "=l"(p[27]), "=l"(p[28]), "=l"(p[29]), "=l"(p[30]), "=l"(p[31])
      : "r"(taddr), "r"(taddr + 32)
      : "memory");
}

// acc += pair * scale2: two FP32 fused multiply-adds in one instruction.
__device__ __forceinline__ void ffma2(uint64_t& acc, uint64_t pair, uint64_t scale2) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(pair), "l"(scale2));
}

// Packed FP32 pair -> packed bf16 pair (round to nearest even); low half first in memory.
__device__ __forceinline__ uint32_t bf16x2_from_pair(uint64_t p) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}


// ---------------------------------------------------------------- arithmetic
// {x, x} as a packed pair of FP32 values.
__device__ __forceinline__ uint64_t pack_f32x2(float x) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(x));
  return r;
}





// Two FP32 values -> two E4M3 codes (round to nearest even, saturating to
// +-448).  The first argument lands in the low byte (lower address).
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t p;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(p) : "f"(hi), "f"(lo));
  return p;
}


// 16 bytes global -> shared through the L2 only (cp.async.cg); both addresses
// 16-byte aligned.  With src_bytes = 0 nothing is read and the 16 bytes are
// zero-filled.  Completion is tracked per thread by commit groups.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most N of this thread's committed groups are still pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 16 bytes in one 128-bit load (read-only, not kept in L1); p 16-byte aligned.
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 32 bytes in one 256-bit load (read-only, not kept in L1); p 32-byte aligned.
__device__ __forceinline__ void ld_nc_v8(const void* p, uint32_t (&w)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
               : "l"(p));
}

// The two bf16 of a 32-bit word as a packed pair of FP32 values (the bf16 at
// the lower address in the low half).  bf16 is the top half of a binary32.
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xFFFF0000u));
  return r;
}

// Per-half maximum of two packed bf16 pairs.
__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Packed FP32 product, each half rounded to nearest even.
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Two packed FP32 pairs -> four E4M3 codes (saturating RNE), in pair order,
// low byte first.
__device__ __forceinline__ uint32_t e4m3x4_from_f32x2(uint64_t p0, uint64_t p1) {
  uint32_t r;
  asm("{\n\t.reg .b16 c0, c1;\n\t.reg .f32 a0, a1, a2, a3;\n\t"
      "mov.b64 {a0, a1}, %1;\n\t"
      "mov.b64 {a2, a3}, %2;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 c0, a1, a0;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 c1, a3, a2;\n\t"
      "mov.b32 %0, {c0, c1};\n\t}"
      : "=r"(r)
      : "l"(p0), "l"(p1));
  return r;
}

}  // namespace fp8q
