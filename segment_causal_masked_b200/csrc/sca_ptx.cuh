// Device-side building blocks shared by the kernels of libsca (sm_100a):
// mbarriers with bounded waits, TMA copies, tcgen05 MMAs, TMEM loads and
// stores, shared-memory matrix descriptors, packed fp32 arithmetic, bf16
// packing and the pair predicate on descriptor words. Internal, not ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sca_internal.h"

namespace sca {

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// try_wait that may suspend the thread until the phase completes, for at
// most `ns` nanoseconds, instead of returning at once.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Longest a waiting thread sleeps in one try (it wakes as soon as the phase
// completes). Sleeping instead of spinning leaves the issue slots of the
// sub-partition to the warps that compute.
constexpr uint32_t kSuspendNs = 2000;

// Shared control block of one CTA.
struct Ctl {
  int32_t abort;   // set by the first wait that times out
};

// Wait for the phase of `bar` with the given parity. Gives up after
// `timeout_ns` (or as soon as another thread of the CTA gave up): then sets
// ctl->abort, writes SCA_ERR_DEVICE_TIMEOUT to *status (if any) and returns
// false. Every pipeline wait of this file goes through here, so a broken
// handshake ends the kernel with an error status instead of a hang.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile Ctl* ctl,
                                          int32_t* status, unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  // a try never sleeps longer than the limit itself (at a limit of 0 the
  // first incomplete try gives up)
  const uint32_t nap = timeout_ns < kSuspendNs ? uint32_t(timeout_ns) : kSuspendNs;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait_suspend(bar, parity, nap)) return true;
    if ((i & 15u) == 0) {
      if (ctl->abort) return false;
      if (global_ns() - t0 > timeout_ns) {
        ctl->abort = 1;
        if (status) atomicExch(status, SCA_ERR_DEVICE_TIMEOUT);
        return false;
      }
    }
  }
}

// Time a CTA gives the loads and products it armed itself to land before it
// exits (see wait_drain); independent of the pipeline waits' limit.
constexpr unsigned long long kDrainTimeoutNs = 2000000000ull;

// Wait for a phase the CTA armed itself (its own TMA loads, or a commit after
// its own MMAs) before it may free its tensor memory and exit. Unlike
// wait_bounded this ignores the abort flag, so an aborted CTA still lets
// every copy and product in flight complete; it gives up only after
// kDrainTimeoutNs. Returns whether the phase completed.
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait_suspend(bar, parity, kSuspendNs))
    if (global_ns() - t0 > kDrainTimeoutNs) return false;
  return true;
}

// One try first; the bounded polling loop only when the phase is not complete
// yet. (Everything is inlined: a shared out-of-line callee would stop ptxas
// from giving the warpgroups different register budgets.)
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile Ctl* ctl,
                                         int32_t* status, unsigned long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_bounded(bar, parity, ctl, status, timeout_ns);
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

// `count` arrivals at once.
__device__ __forceinline__ void mbar_arrive_n(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make this thread's shared-memory stores visible to the tensor cores.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
// K-major (rows of 128 bytes along K, 8-row groups 1024 bytes apart).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr) {
  return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
// MN-major (rows of 128 bytes along N = 64 elements; the next 64 N-elements
// 16 KB further; 8-row groups along K 1024 bytes apart).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr) {
  return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t(16384 >> 4) << 16) |
         (uint64_t(1024 >> 4) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor: kind::f16, bf16 A and B, fp32 D, M = 128, N = 128.
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) |
                              ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescQK | (1u << 16);  // B (V) is MN-major

// The eight MMAs of one 128 x 128 x 128 product (K = 8 x 16) in one asm
// block, so the single issuing thread spends a few instructions per MMA. The
// descriptors advance through their start-address field (bits 0..13, in
// 16-byte units) with 32-bit adds on the low word; smem addresses stay below
// 256 KB, so the field never carries into the next one.
// S = Q K^T: A (Q) and B (K) K-major, 32 B per K-step inside a 64-column
// half, 16 KB (1024 units) to the second half; D is overwritten.
__device__ __forceinline__ void mma_qk8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred pf, pt;\n\t.reg .b32 al, bl;\n\t.reg .b64 ad, bd;\n\t"
      "setp.ne.b32 pf, 0, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "mov.b64 ad, {%1, %2};\n\tmov.b64 bd, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pf;\n\t"
      "add.u32 al, %1, 2;\n\tadd.u32 bl, %3, 2;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.u32 al, %1, 4;\n\tadd.u32 bl, %3, 4;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.u32 al, %1, 6;\n\tadd.u32 bl, %3, 6;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.u32 al, %1, 1024;\n\tadd.u32 bl, %3, 1024;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.u32 al, %1, 1026;\n\tadd.u32 bl, %3, 1026;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.u32 al, %1, 1028;\n\tadd.u32 bl, %3, 1028;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t"
      "add.u32 al, %1, 1030;\n\tadd.u32 bl, %3, 1030;\n\tmov.b64 ad, {al, %2};\n\tmov.b64 bd, {bl, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %5, pt;\n\t}"
      ::"r"(d_tmem), "r"(uint32_t(a_desc)), "r"(uint32_t(a_desc >> 32)), "r"(uint32_t(b_desc)),
      "r"(uint32_t(b_desc >> 32)), "r"(idesc)
      : "memory");
}

// O (+)= P V: A = P from TMEM (8 columns per K-step of 16 keys), B = V
// MN-major, 2048 B (128 units) per K-step. `acc` = 0 overwrites O on the
// first K-step.
__device__ __forceinline__ void mma_pv8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred pf, pt;\n\t.reg .b32 ta, bl;\n\t.reg .b64 bd;\n\t"
      "setp.ne.b32 pf, %5, 0;\n\tsetp.eq.b32 pt, 0, 0;\n\t"
      "mov.b64 bd, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %4, pf;\n\t"
      "add.u32 ta, %1, 8;\n\tadd.u32 bl, %2, 128;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 16;\n\tadd.u32 bl, %2, 256;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 24;\n\tadd.u32 bl, %2, 384;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 32;\n\tadd.u32 bl, %2, 512;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 40;\n\tadd.u32 bl, %2, 640;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 48;\n\tadd.u32 bl, %2, 768;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t"
      "add.u32 ta, %1, 56;\n\tadd.u32 bl, %2, 896;\n\tmov.b64 bd, {bl, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], bd, %4, pt;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "r"(uint32_t(b_desc)), "r"(uint32_t(b_desc >> 32)), "r"(idesc),
      "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* r) {
  uint32_t* u = reinterpret_cast<uint32_t*>(r);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
        "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]),
        "=r"(u[14]), "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]),
        "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]), "=r"(u[24]), "=r"(u[25]),
        "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* r) {
  const uint32_t* u = reinterpret_cast<const uint32_t*>(r);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]),
      "r"(u[8]), "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]),
      "r"(u[15]), "r"(u[16]), "r"(u[17]), "r"(u[18]), "r"(u[19]), "r"(u[20]), "r"(u[21]),
      "r"(u[22]), "r"(u[23]), "r"(u[24]), "r"(u[25]), "r"(u[26]), "r"(u[27]), "r"(u[28]),
      "r"(u[29]), "r"(u[30]), "r"(u[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* u) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]),
      "r"(u[8]), "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]),
      "r"(u[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two 2-input maxima. (The 3-input max.f32 of sm_100 returned a wrong
// finite value for three -inf inputs in one instantiation of the attention
// kernel, where a row of masked scores must keep its running max at -inf.)
__device__ __forceinline__ float max3(float a, float b, float c) { return fmaxf(fmaxf(a, b), c); }

// Packed fp32 pairs (one instruction for two lanes of work on sm_100).
__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void unf2(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void named_sync(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// The pair predicate on descriptor words (layout documented in sca.h);
// `window` = how many earlier segments a query may see (65535: all).
__device__ __forceinline__ bool visible(uint32_t q0, uint32_t q1, uint32_t k, uint32_t window) {
  const uint32_t qs = q0 & SCA_DESC_SEG_MASK, ks = k & SCA_DESC_SEG_MASK;
  const bool own = (ks == qs) && (!(k & SCA_DESC_TAIL) ||
                                  ((q1 >> ((k >> SCA_DESC_ACTION_SHIFT) & 31u)) & 1u));
  const bool past = (ks < qs) && (qs - ks <= window) && (q0 & SCA_QDESC_SEES_PAST) &&
                    (k & SCA_DESC_ALIVE);
  return (q0 & SCA_QDESC_VALID) && (own || past);
}

}  // namespace sca
