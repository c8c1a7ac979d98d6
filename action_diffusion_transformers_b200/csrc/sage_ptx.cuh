// sage_ptx.cuh - inline-PTX helpers for sm_100a: mbarriers with bounded
// waits, TMA tile loads, tcgen05 (TMEM alloc, MMA, commit, ld/st, fences),
// and the FP8 / BF16 conversions the quantized-attention kernels use.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace sage {

// Programmatic dependent launch: wait until the grids this one depends on have
// completed and their writes are visible (a no-op when the launch did not allow
// an early start), then allow the next grid in the stream to be scheduled.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Two binary32 values held in one 64-bit register (first value in the low
// word), the operand form of the sm_100 add/mul/fma.f32x2 instructions.  The
// pair never leaves its register between operations, so no moves are needed
// to build operand pairs.
typedef unsigned long long f32x2_t;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread is parked (not spinning, so it
// takes no issue slots from other warps) until the phase completes or about
// hint_ns pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Gives up when the
// CTA-wide abort flag is raised, or after timeout_ns (then raises it itself).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort_flag, int64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (*abort_flag) return false;
    if (static_cast<int64_t>(globaltimer_ns() - t0) > timeout_ns) {
      *abort_flag = 1;
      return false;
    }
  }
}


// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}
// 2-D tiled tensor load into CTA shared memory, completion counted in bytes
// on `bar`.  x is the innermost coordinate (bytes here: 8-bit elements).
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Arrive on `bar` once all tcgen05 operations issued so far by this thread complete.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Shared-memory matrix descriptor, K-major operand with a swizzled layout:
// start address, leading byte offset 16 (unused for swizzled K-major),
// stride byte offset = bytes between consecutive 8-row groups, version 1,
// base offset 0, swizzle code (2 = 128 B, 4 = 64 B).
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t sbo_bytes, uint32_t swizzle_code) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(16u >> 4) << 16;
  d |= static_cast<uint64_t>((sbo_bytes & 0x3FFFFu) >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(swizzle_code & 7u) << 61;
  return d;
}

// Instruction descriptor: dense, K-major A and B, M = 128.
//   c_fmt: 1 = F32, 2 = S32;  ab_fmt: kind::i8 1 = signed, kind::f8f6f4 0 = E4M3.
__host__ __device__ constexpr uint32_t make_idesc(uint32_t c_fmt, uint32_t ab_fmt, uint32_t M, uint32_t N) {
  return (c_fmt << 4) | (ab_fmt << 7) | (ab_fmt << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane (warp w reads
// lanes 32*(w%4) .. +31; lane offset is encoded in taddr bits 31..16).
#define SAGE_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), \
                   "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : SAGE_R8(0), SAGE_R8(8), SAGE_R8(16), SAGE_R8(24)
      : "r"(taddr));
}
#undef SAGE_R8
// 32 consecutive 32-bit columns, waited for and returned as 16 pairs.
__device__ __forceinline__ void tmem_ld32_pairs(uint32_t taddr, f32x2_t (&r)[16]) {
  asm volatile(
      "{.reg .b32 t0, t1, t2, t3, t4, t5, t6, t7, t8, t9, t10, t11, t12, t13, t14, t15, t16, t17, t18, t19, t20, t21, t22, t23, t24, t25, t26, t27, t28, t29, t30, t31;\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {t0, t1, t2, t3, t4, t5, t6, t7, t8, t9, t10, t11, t12, t13, t14, t15, t16, t17, t18, t19, t20, t21, t22, t23, t24, t25, t26, t27, t28, t29, t30, t31}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n\t"
      "mov.b64 %0, {t0, t1};\n\t"
      "mov.b64 %1, {t2, t3};\n\t"
      "mov.b64 %2, {t4, t5};\n\t"
      "mov.b64 %3, {t6, t7};\n\t"
      "mov.b64 %4, {t8, t9};\n\t"
      "mov.b64 %5, {t10, t11};\n\t"
      "mov.b64 %6, {t12, t13};\n\t"
      "mov.b64 %7, {t14, t15};\n\t"
      "mov.b64 %8, {t16, t17};\n\t"
      "mov.b64 %9, {t18, t19};\n\t"
      "mov.b64 %10, {t20, t21};\n\t"
      "mov.b64 %11, {t22, t23};\n\t"
      "mov.b64 %12, {t24, t25};\n\t"
      "mov.b64 %13, {t26, t27};\n\t"
      "mov.b64 %14, {t28, t29};\n\t"
      "mov.b64 %15, {t30, t31};\n\t"
      "}"
      : "=l"(r[0]), "=l"(r[1]), "=l"(r[2]), "=l"(r[3]), "=l"(r[4]), "=l"(r[5]), "=l"(r[6]), "=l"(r[7]), "=l"(r[8]), "=l"(r[9]), "=l"(r[10]), "=l"(r[11]), "=l"(r[12]), "=l"(r[13]), "=l"(r[14]), "=l"(r[15])
      : "r"(taddr)
      : "memory");
}
// Store 16 pairs into 32 consecutive 32-bit TMEM columns (low word first);
// completion is awaited with tmem_wait_st().
__device__ __forceinline__ void tmem_st32_pairs(uint32_t taddr, const f32x2_t (&r)[16]) {
  asm volatile(
      "{.reg .b32 t0, t1, t2, t3, t4, t5, t6, t7, t8, t9, t10, t11, t12, t13, t14, t15, t16, t17, t18, t19, t20, t21, t22, t23, t24, t25, t26, t27, t28, t29, t30, t31;\n\t"
      "mov.b64 {t0, t1}, %1;\n\t"
      "mov.b64 {t2, t3}, %2;\n\t"
      "mov.b64 {t4, t5}, %3;\n\t"
      "mov.b64 {t6, t7}, %4;\n\t"
      "mov.b64 {t8, t9}, %5;\n\t"
      "mov.b64 {t10, t11}, %6;\n\t"
      "mov.b64 {t12, t13}, %7;\n\t"
      "mov.b64 {t14, t15}, %8;\n\t"
      "mov.b64 {t16, t17}, %9;\n\t"
      "mov.b64 {t18, t19}, %10;\n\t"
      "mov.b64 {t20, t21}, %11;\n\t"
      "mov.b64 {t22, t23}, %12;\n\t"
      "mov.b64 {t24, t25}, %13;\n\t"
      "mov.b64 {t26, t27}, %14;\n\t"
      "mov.b64 {t28, t29}, %15;\n\t"
      "mov.b64 {t30, t31}, %16;\n\t"
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {t0, t1, t2, t3, t4, t5, t6, t7, t8, t9, t10, t11, t12, t13, t14, t15, t16, t17, t18, t19, t20, t21, t22, t23, t24, t25, t26, t27, t28, t29, t30, t31};\n\t"
      "}"
      :
      : "r"(taddr), "l"(r[0]), "l"(r[1]), "l"(r[2]), "l"(r[3]), "l"(r[4]), "l"(r[5]), "l"(r[6]), "l"(r[7]), "l"(r[8]), "l"(r[9]), "l"(r[10]), "l"(r[11]), "l"(r[12]), "l"(r[13]), "l"(r[14]), "l"(r[15])
      : "memory");
}
// 64 consecutive 32-bit columns of this warp's 32 lanes set to v: the value is
// placed in one 8-register block once and stored 8 columns at a time (a 32-wide
// store would need 32 registers holding it).  Await with tmem_wait_st().
__device__ __forceinline__ void tmem_fill64(uint32_t taddr, uint32_t v) {
  asm volatile(
      "{.reg .b32 t0, t1, t2, t3, t4, t5, t6, t7;\n\t"
      "mov.b32 t0, %1;\n\tmov.b32 t1, %1;\n\tmov.b32 t2, %1;\n\tmov.b32 t3, %1;\n\t"
      "mov.b32 t4, %1;\n\tmov.b32 t5, %1;\n\tmov.b32 t6, %1;\n\tmov.b32 t7, %1;\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {t0, t1, t2, t3, t4, t5, t6, t7};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+8], {t0, t1, t2, t3, t4, t5, t6, t7};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+16], {t0, t1, t2, t3, t4, t5, t6, t7};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+24], {t0, t1, t2, t3, t4, t5, t6, t7};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+32], {t0, t1, t2, t3, t4, t5, t6, t7};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+40], {t0, t1, t2, t3, t4, t5, t6, t7};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+48], {t0, t1, t2, t3, t4, t5, t6, t7};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0+56], {t0, t1, t2, t3, t4, t5, t6, t7};\n\t"
      "}" ::"r"(taddr), "r"(v)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void reg_fence16(uint32_t (&r)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) asm volatile("" : "+r"(r[i])::"memory");
}
// After tmem_wait_ld(): ties the loaded registers to this point, so that no use
// of them is scheduled between the asynchronous tcgen05.ld and its wait.
__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i])::"memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- numerics
// Two floats -> two E4M3 bytes (round to nearest even, saturate to +-448);
// `lo` lands in bits 0..7, `hi` in bits 8..15.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return static_cast<uint32_t>(r);
}
__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}
// float -> BF16 bits, round to nearest even (hardware cvt).
__device__ __forceinline__ uint32_t float_to_bf16_bits(float x) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
  return static_cast<uint32_t>(r);
}

// double -> BF16 bits with one rounding (nearest even), by integer arithmetic
// on the binary64 encoding: the 53-bit significand is shifted onto the BF16
// unit of the value's binade (2^(E-7), or 2^-133 below the normal range) and
// rounded on the dropped bits; a carry into the next binade and overflow to
// infinity fall out of the additive encoding.
__device__ __forceinline__ uint32_t double_to_bf16_bits(double x) {
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
  const uint32_t sign = static_cast<uint32_t>(u >> 63) << 15;
  const uint64_t a = u & 0x7FFFFFFFFFFFFFFFull;
  const int e = static_cast<int>(a >> 52);
  if (e == 0x7FF) return (a & 0xFFFFFFFFFFFFFull) ? 0x7FC0u : (sign | 0x7F80u);
  if (e == 0) return sign;                    // |x| < 2^-1022: rounds to zero
  if (e - 1023 > 127) return sign | 0x7F80u;  // |x| >= 2^128
  const uint64_t mant = (a & 0xFFFFFFFFFFFFFull) | (1ull << 52);
  const int E = (e - 1023 >= -126) ? (e - 1023) : -126;
  const int shift = (E - 7) - (e - 1075);     // >= 45
  uint64_t q;
  if (shift >= 64) {
    q = 0;
  } else {
    q = mant >> shift;
    const uint64_t rem = mant & ((1ull << shift) - 1);
    const uint64_t half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (q & 1))) ++q;
  }
  uint32_t bits;
  if (e - 1023 >= -126) {
    bits = static_cast<uint32_t>(((E + 127) << 7) + (q - 128));  // q in [128, 256]
    if (bits >= 0x7F80u) bits = 0x7F80u;
  } else {
    bits = static_cast<uint32_t>(q);                              // subnormal, q in [0, 128]
  }
  return sign | bits;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
// Three-input maximum (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ---------------------------------------------------------------- FP32 pairs
// (f32x2_t, declared at the top of this file.)

__device__ __forceinline__ f32x2_t x2_splat(float v) {
  f32x2_t d;
  asm("mov.b64 %0, {%1, %1};" : "=l"(d) : "f"(v));
  return d;
}
__device__ __forceinline__ f32x2_t x2_add(f32x2_t a, f32x2_t b) {
  f32x2_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2_t x2_sub(f32x2_t a, f32x2_t b) {
  f32x2_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2_t x2_mul(f32x2_t a, f32x2_t b) {
  f32x2_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2_t x2_fma(f32x2_t a, f32x2_t b, f32x2_t c) {
  f32x2_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2_t x2_pack(uint32_t lo, uint32_t hi) {
  f32x2_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
  return d;
}
__device__ __forceinline__ float x2_lo(f32x2_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float x2_hi(f32x2_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
// Per 32-bit word: bits(p) + (bits(xr) << 23), i.e. the integer in the low bits
// of xr added to the exponent field of p.  The shift is written as a funnel
// shift of (xr : 0): a plain shl followed by the add is fused by the compiler
// into an integer multiply-add, which issues on the FMA pipe that the
// exponential pass saturates; in this form the shift and add stay on the
// integer ALU pipe (one instruction per word, measured).
__device__ __forceinline__ f32x2_t x2_add_exponent(f32x2_t p, f32x2_t xr) {
  f32x2_t d;
  asm("{.reg .b32 pl, ph, xl, xh, z;\n\t"
      "mov.b64 {pl, ph}, %1;\n\tmov.b64 {xl, xh}, %2;\n\tmov.b32 z, 0;\n\t"
      "shf.l.clamp.b32 xl, z, xl, 23;\n\tshf.l.clamp.b32 xh, z, xh, 23;\n\t"
      "add.u32 pl, pl, xl;\n\tadd.u32 ph, ph, xh;\n\t"
      "mov.b64 %0, {pl, ph};}"
      : "=l"(d) : "l"(p), "l"(xr));
  return d;
}
// Four binary32 values (two pairs) -> four E4M3 bytes, round to nearest even,
// saturating to +-448; a.lo lands in bits 0..7, a.hi 8..15, b.lo 16..23, b.hi 24..31.
__device__ __forceinline__ uint32_t x2_e4m3x4(f32x2_t a, f32x2_t b) {
  uint32_t d;
  asm("{.reg .f32 al, ah, bl, bh;\n\t.reg .b16 ca, cb;\n\t"
      "mov.b64 {al, ah}, %1;\n\tmov.b64 {bl, bh}, %2;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 ca, ah, al;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 cb, bh, bl;\n\t"
      "mov.b32 %0, {ca, cb};}"
      : "=r"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x with every step a binary32 operation whose rounding is fixed, so that the
// result is reproducible bit for bit on any IEEE machine (the CPU oracle runs
// the same steps): Cody-Waite split x = n + f with n = round(x) by the
// 1.5 * 2^23 addition (which leaves n, two's complement, in the low bits of
// xr), f = x - n exactly, 2^f from a polynomial with c0 = 1 fitted for minimax
// relative error on [-1/2, 1/2] (linear programming), Horner with fused
// multiply-adds, and n added to the exponent field of the polynomial's value:
// exactly p * 2^n for n >= -125.  The per-key weights use a quadratic
// (1.96e-3 relative after binary32 evaluation, 32 times below the 6.25% step
// of the E4M3 codes they feed); the per-tile rescale factor a quintic (2.2e-7).
// Requires x >= -126 (callers clamp).
constexpr float kExp2Round = 12582912.0f;  // 1.5 * 2^23
constexpr float kExp2C1 = 0.7029417753219604f;   // quadratic
constexpr float kExp2C2 = 0.2398640364408493f;
constexpr float kExp2Q1 = 0.6931465864181519f;   // quintic
constexpr float kExp2Q2 = 0.24022166430950165f;
constexpr float kExp2Q3 = 0.055510472506284714f;
constexpr float kExp2Q4 = 0.009674952365458012f;
constexpr float kExp2Q5 = 0.0013202981790527701f;
constexpr float kExp2Min = -126.0f;

// The constant pairs of exp2_fixed_x2, built once per thread.
struct Exp2Consts {
  f32x2_t round, c0, c1, c2;
  __device__ __forceinline__ Exp2Consts()
      : round(x2_splat(kExp2Round)), c0(x2_splat(1.0f)), c1(x2_splat(kExp2C1)), c2(x2_splat(kExp2C2)) {}
};

// Quadratic form on a pair.
__device__ __forceinline__ f32x2_t exp2_fixed_x2(f32x2_t x, const Exp2Consts& k) {
  const f32x2_t xr = x2_add(x, k.round);
  const f32x2_t nf = x2_sub(xr, k.round);
  const f32x2_t f = x2_sub(x, nf);
  f32x2_t p = x2_fma(k.c2, f, k.c1);
  p = x2_fma(p, f, k.c0);
  return x2_add_exponent(p, xr);
}
// Quintic scalar form, clamping x at -126 itself.
__device__ __forceinline__ float exp2_fixed5(float x) {
  x = fmaxf(x, kExp2Min);
  const float xr = __fadd_rn(x, kExp2Round);
  const float nf = __fadd_rn(xr, -kExp2Round);
  const float f = __fsub_rn(x, nf);
  float p = __fmaf_rn(kExp2Q5, f, kExp2Q4);
  p = __fmaf_rn(p, f, kExp2Q3);
  p = __fmaf_rn(p, f, kExp2Q2);
  p = __fmaf_rn(p, f, kExp2Q1);
  p = __fmaf_rn(p, f, 1.0f);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(xr) << 23));
}

}  // namespace sage
