// Device helpers shared by the AB-Attention kernels (sm_100a only).
//
// Inline PTX wrappers for mbarriers, cp.async, tcgen05 (TMEM allocation, MMA,
// commit, loads/stores) and the shared-memory matrix descriptors, plus the
// device status word and exact fp64 -> bf16 rounding.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "abattn.h"

#define AB_DEV __device__ __forceinline__

// ------------------------------------------------------------------ status word

// First device-side error since the last ab_get_status (0 = none).
__device__ int g_ab_status;

AB_DEV void ab_flag(int code) { atomicCAS(&g_ab_status, 0, code); }

AB_DEV uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

AB_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ bf16 rounding

// Nearest bf16 (ties to even) of a double, by rounding to fp32 with round-to-odd
// (truncate, then set the sticky lsb when inexact) and then to bf16 with
// round-to-nearest-even.  fp32 keeps 16 more bits than bf16 (>= 2 needed), so the
// two steps equal a single rounding of the double.
AB_DEV uint16_t bf16_bits_from_double(double x) {
  float f = __double2float_rz(x);
  uint32_t u = __float_as_uint(f);
  if ((double)f != x && !isnan(x)) u |= 1u;
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);  // NaN
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

AB_DEV float bf16_bits_to_float(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

AB_DEV uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

AB_DEV float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------ packed fp32 pairs
//
// sm_100 executes fp32 add and fma on register pairs (.f32x2), one instruction per pair.

AB_DEV uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
AB_DEV float2 f2_unpack(uint64_t r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
AB_DEV uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
AB_DEV uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for a pair on the FMA pipe (so that part of the exponentials stays off the MUFU).
// Range reduction x = j + f with j = round(x) (the 1.5 * 2^23 rounding constant) and
// |f| <= 1/2; 2^f by a degree-5 polynomial; 2^j added into the exponent field.  The
// coefficients are this library's own fit: Lawson's iteratively reweighted least squares
// for minimax relative error of 2^f on [-1/2, 1/2], rounded to fp32; evaluated by Horner
// in fp32 the maximum relative error is 2.4e-7 (ex2.approx: about 2^-22).  x is clamped
// to [-126, 127]; below -126 the result is a value under 2^-125 instead of the flushed 0.
constexpr float EXP2P_C0 = 1.0000001192092896f;
constexpr float EXP2P_C1 = 0.6931469440460205f;
constexpr float EXP2P_C2 = 0.24022120237350464f;
constexpr float EXP2P_C3 = 0.05550713092088699f;
constexpr float EXP2P_C4 = 0.009675541892647743f;
constexpr float EXP2P_C5 = 0.001327647129073739f;
constexpr float EXP2P_ROUND = 12582912.0f;  // 1.5 * 2^23

AB_DEV uint64_t exp2_poly_x2(float x0, float x1) {
  x0 = fminf(fmaxf(x0, -126.f), 127.f);
  x1 = fminf(fmaxf(x1, -126.f), 127.f);
  const uint64_t X = f2_pack(x0, x1);
  const uint64_t T = f2_add(X, f2_pack(EXP2P_ROUND, EXP2P_ROUND));  // its low bits hold j
  const uint64_t J = f2_add(T, f2_pack(-EXP2P_ROUND, -EXP2P_ROUND));
  const uint64_t F = f2_fma(J, f2_pack(-1.f, -1.f), X);  // x - j, exact
  uint64_t P = f2_fma(f2_pack(EXP2P_C5, EXP2P_C5), F, f2_pack(EXP2P_C4, EXP2P_C4));
  P = f2_fma(P, F, f2_pack(EXP2P_C3, EXP2P_C3));
  P = f2_fma(P, F, f2_pack(EXP2P_C2, EXP2P_C2));
  P = f2_fma(P, F, f2_pack(EXP2P_C1, EXP2P_C1));
  P = f2_fma(P, F, f2_pack(EXP2P_C0, EXP2P_C0));
  const float2 t = f2_unpack(T), pv = f2_unpack(P);
  return f2_pack(__uint_as_float(__float_as_uint(pv.x) + (__float_as_uint(t.x) << 23)),
                 __uint_as_float(__float_as_uint(pv.y) + (__float_as_uint(t.y) << 23)));
}

// ------------------------------------------------------------------ mbarriers

AB_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

AB_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

AB_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Arrive once the calling thread's earlier cp.async copies have landed (the arrival is
// one of the barrier's expected arrivals).
AB_DEV void mbar_arrive_cpasync(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Non-blocking probe of the phase with the given parity (no suspend hint).
AB_DEV bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity.  Gives up when *abort is raised
// by another thread of the CTA, or after timeout_ns (then records
// AB_ERR_DEVICE_TIMEOUT and raises *abort).  Returns true when the phase completed.
// Spins on the non-suspending probe: a thread parked in try_wait was observed to resume
// only long after an arrival made by tcgen05.commit.
AB_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t timeout_ns) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int k = 0; k < 64; ++k)
      if (mbar_test(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      ab_flag(AB_ERR_DEVICE_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// Arrive on `bar` (one of its expected arrivals) and add `bytes` to the transaction
// count that the bulk copies signalling it must complete.
AB_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Bounded wait that ignores the CTA's abort flag (used on the way out, to let copies that
// are already in flight land before the CTA exits).  Returns whether the phase completed.
AB_DEV bool mbar_wait_quiet(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_test(bar, parity))
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  return true;
}

// ------------------------------------------------------------------ TMA (tiled, no multicast)

// 3-D tiled bulk copy global -> shared of the box at (x, y, z) of `tmap`, completing `bytes`
// of transactions on `bar`.  x * element size must be a multiple of 16 bytes.
AB_DEV void tma_load_3d(uint32_t dst, const void* tmap, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"((uint64_t)tmap), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------------ cp.async

// 16-byte global -> shared copy; src_bytes = 0 writes zeros and reads nothing.
AB_DEV void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
AB_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Make this thread's generic-proxy shared-memory writes visible to async-proxy readers
// (the tensor cores) and order its later async-proxy operations after them.
AB_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ------------------------------------------------------------------ tcgen05 / TMEM

AB_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
AB_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
AB_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
AB_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
AB_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]^T-ish per the instruction descriptor.
AB_DEV void umma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]: A (M x K, K-major) read from tensor memory, lane =
// row, each 32-bit column holding two consecutive K elements (16 K elements = 8 columns).
AB_DEV void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` when every tcgen05 operation this thread issued so far has completed.
AB_DEV void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 columns of 32-bit values: thread i of the warp gets lane (base lane + i),
// columns [col, col+32).  The warp may only touch its own 32-lane sub-partition.
AB_DEV void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
AB_DEV void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
AB_DEV void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
// tcgen05.wait::ld that also names the destination registers of the loads it waits for,
// so the compiler cannot move a use of them above the wait.
AB_DEV void tmem_wait_ld_regs(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}
AB_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
AB_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: version bits = 1).
// Operand tiles are stored as [64-element column chunk][row][128 B], each 8-row group
// a 1024-byte swizzle atom whose 16-byte units are permuted by (row & 7); tile bases
// are 1024-byte aligned, so the base-offset field is 0.
//   K-major operand (rows = M or N, 64 elements of K per 128-byte row):
//       lbo unused (16), sbo = 1024 (next 8-row group)
//   MN-major operand (128-byte rows hold 64 consecutive M/N elements, rows = K):
//       lbo = byte distance between 64-element M/N chunks, sbo = 1024 (next 8 K rows)
AB_DEV uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;  // descriptor version for sm_100
  d |= (uint64_t)2u << 61;  // SWIZZLE_128B
  return d;
}

// Shared-memory matrix descriptor without swizzle (layout type 0).  K-major canonical
// layout of 8-row x 16-byte core matrices, each stored as 128 contiguous bytes (row i at
// byte 16 i):  sbo = byte distance between core matrices adjacent in M/N (the next 8
// rows), lbo = byte distance between core matrices adjacent in K (the next 8 elements).
AB_DEV uint64_t sdesc_noswizzle(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;  // descriptor version for sm_100
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A and B, fp32 D, dense.
//   a_mn / b_mn: 0 = K-major, 1 = MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                          // D format F32
         | (1u << 7)                        // A format BF16
         | (1u << 10)                       // B format BF16
         | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(N >> 3) << 17)         // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Byte offset of 16-byte unit `u` (0..7 within a 128-byte row) of row `r` inside a
// 128B-swizzled region whose base is 1024-byte aligned.
AB_DEV uint32_t sw128_off(uint32_t r, uint32_t u) { return r * 128u + ((u ^ (r & 7u)) << 4); }
