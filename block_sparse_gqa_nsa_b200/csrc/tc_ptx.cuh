// Inline-PTX building blocks for sm_100a: mbarriers (bounded waits only), TMA tile
// loads, tensor-memory allocation and access, and tcgen05 bf16 MMAs.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "lsrm_common.cuh"

namespace lsrm {
namespace tc {

// ---- mbarrier -------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// try_wait: a waiting thread may sleep in hardware until the phase completes (or a
// system-dependent time limit passes) instead of spinning through issue slots.  No suspend-time
// hint: with a long hint the waiters measured slower to resume.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;\n" : "=l"(t));
  return t;
}

// Wait for the phase with `parity` to complete, giving up after kWaitLimitNs or when another
// thread of the CTA has set *abort.  Returns false when it gave up (the caller then unwinds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far above any legitimate wait
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      raise_status(status, LSRM_ERR_TIMEOUT);
      return false;
    }
  }
}

// every lane of a converged warp waits; true only when the wait succeeded in all of them
__device__ __forceinline__ bool mbar_wait_w(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* status) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, status));
}

// ---- TMA --------------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];\n" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tensor memory ----------------------------------------------------------------------------------
// whole warp: allocate ncols (power of two >= 32) columns, base address written to *dst
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}

// 32 lanes x 32 columns of 32-bit: thread i of the warp gets lane (base lane + i), 32 columns
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n" : "=r"(r) : "r"(taddr));
  return __uint_as_float(r);
}
__device__ __forceinline__ void tmem_st1(uint32_t taddr, float v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};\n" ::"r"(taddr), "r"(__float_as_uint(v))
               : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// ---- UMMA descriptors -------------------------------------------------------------------------------
// Shared-memory matrix descriptor (sm_100): start address, leading / stride byte offsets (16-byte
// units), version 1, layout type in bits 61..63 (2 = 128-byte swizzle, 4 = 64-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // version
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}
constexpr uint32_t kLayoutSW128 = 2, kLayoutSW64 = 4;

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4)                          // D format f32
         | (1u << 7)                        // A format bf16
         | (1u << 10)                       // B format bf16
         | (0u << 15)                       // A K-major
         | ((b_mn_major ? 1u : 0u) << 16)   // B major
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// ---- whole-warp issue ----
// The MMA warp runs its issue loop converged and one elected lane issues each tcgen05
// instruction: the operands are then warp-uniform values the compiler keeps in uniform
// registers, and an issue costs about 22 cycles instead of about 63 from a lone diverged lane.
// That pays where the issuing thread is the bottleneck; where it mostly waits on the softmax
// warps, the lone lane (no warp-wide vote after each wait) measured faster.
__device__ __forceinline__ void mma_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, e;\n setp.ne.b32 p, %4, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts_w(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p, e;\n setp.ne.b32 p, %4, 0;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit_w(uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(smem_u32(bar))
      : "memory");
}

// arrive on `bar` once every tcgen05 operation this thread issued so far has completed
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   smem_u32(bar))
               : "memory");
}


// 2^x on the FMA pipe, for x <= 127.  Cody-Waite style: x = j + f with j = round(x) taken from
// the low mantissa bits of x + 1.5 * 2^23 and f in [-0.5, 0.5]; 2^f from a degree-3 polynomial
// whose coefficients are the minimax fit of the relative error on [-0.5, 0.5] (Remez exchange,
// block_sparse_gqa_nsa_b200/exp2_fit.py: max relative error 7.5e-5, far below the bf16 rounding
// the result goes through); 2^j is added into the exponent field with one integer multiply-add
// ((1.5 * 2^23 + j) * 2^23 == j * 2^23 mod 2^32).  Inputs below -125 (masked keys at -inf among
// them) are clamped there and return about 2^-125, not 0: callers use it only where every key is
// valid (a key that far below the reference then weighs under 2^-125 against a row sum of at
// least 2^-64), and keep masked keys on the hardware ex2, whose ex2(-inf) is exactly 0.
// Two elements at once: the float steps run as packed f32x2 operations (the clamp and the
// exponent add stay scalar), about 5 issue slots per element.
__device__ __forceinline__ void poly_exp2_pair(float& r0, float& r1, float x0, float x1) {
  x0 = fmaxf(x0, -125.0f);
  x1 = fmaxf(x1, -125.0f);
  uint64_t rx, rt, rm, rn, rr, rf, rp, ra, rb, rc;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(rx) : "f"(x0), "f"(x1));
  asm("mov.b64 %0, {%1, %1};\n" : "=l"(rm) : "f"(12582912.0f));
  asm("add.rn.f32x2 %0, %1, %2;\n" : "=l"(rt) : "l"(rx), "l"(rm));        // t = x + 1.5 * 2^23
  asm("sub.rn.f32x2 %0, %1, %2;\n" : "=l"(rn) : "l"(rt), "l"(rm));        // round(x)
  asm("sub.rn.f32x2 %0, %1, %2;\n" : "=l"(rf) : "l"(rx), "l"(rn));        // f = x - round(x)
  asm("mov.b64 %0, {%1, %1};\n" : "=l"(ra) : "f"(0.0551716685f));
  asm("mov.b64 %0, {%1, %1};\n" : "=l"(rb) : "f"(0.2426111251f));
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(rp) : "l"(rf), "l"(ra), "l"(rb));
  asm("mov.b64 %0, {%1, %1};\n" : "=l"(rc) : "f"(0.6932609677f));
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(rr) : "l"(rp), "l"(rf), "l"(rc));
  asm("mov.b64 %0, {%1, %1};\n" : "=l"(rc) : "f"(0.9999280572f));
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(rp) : "l"(rr), "l"(rf), "l"(rc));
  float t0, t1, p0, p1;
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(t0), "=f"(t1) : "l"(rt));
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(p0), "=f"(p1) : "l"(rp));
  r0 = __uint_as_float(__float_as_uint(t0) * (1u << 23) + __float_as_uint(p0));
  r1 = __uint_as_float(__float_as_uint(t1) * (1u << 23) + __float_as_uint(p1));
}

// max of three floats in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// (r0, r1) = (a0, a1) * (b0, b1) with one packed f32x2 multiply
__device__ __forceinline__ void fmul2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
  uint64_t ra, rb, rd;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(ra) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(rb) : "f"(b0), "f"(b1));
  asm("mul.rn.ftz.f32x2 %0, %1, %2;\n" : "=l"(rd) : "l"(ra), "l"(rb));
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(r0), "=f"(r1) : "l"(rd));
}
// (c0, c1) += (a0, a1) * (b0, b1) with one packed f32x2 FMA
__device__ __forceinline__ void ffma2_acc(float& c0, float& c1, float a0, float a1, float b0, float b1) {
  uint64_t ra, rb, rc, rd;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(ra) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(rb) : "f"(b0), "f"(b1));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(rc) : "f"(c0), "f"(c1));
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;\n" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(c0), "=f"(c1) : "l"(rd));
}
// (a0, a1) += (b0, b1) with one packed f32x2 add
__device__ __forceinline__ void fadd2_acc(float& a0, float& a1, float b0, float b1) {
  uint64_t ra, rb, rd;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(ra) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(rb) : "f"(b0), "f"(b1));
  asm("add.rn.ftz.f32x2 %0, %1, %2;\n" : "=l"(rd) : "l"(ra), "l"(rb));
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(a0), "=f"(a1) : "l"(rd));
}
// (a0, a1) * (b, b) + (c, c) with one packed f32x2 FMA
__device__ __forceinline__ void ffma2(float& r0, float& r1, float a0, float a1, float b, float c) {
  uint64_t ra, rb, rc, rd;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(ra) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %1};\n" : "=l"(rb) : "f"(b));
  asm("mov.b64 %0, {%1, %1};\n" : "=l"(rc) : "f"(c));
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;\n" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(r0), "=f"(r1) : "l"(rd));
}

}  // namespace tc
}  // namespace lsrm
