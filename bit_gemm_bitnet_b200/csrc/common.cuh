// Device helpers shared by the kernels of libbitnet_b200 (sm_100a only).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libbitnet_b200 is written for sm_100a (B200) only"
#endif

namespace bitnet {

// Error bits of the device status word (read by bitnet_device_status).
constexpr unsigned kDevErrTimeout = 1u;
constexpr unsigned kDevErrValue = 2u;  // an input outside a kernel's exact range

// Bounded waits give up after this many nanoseconds of global time (2 s; the
// failure-path test library is built with a 1 ms limit).
#ifndef BITNET_WAIT_LIMIT_NS
#define BITNET_WAIT_LIMIT_NS 2000000000ull
#endif
constexpr unsigned long long kWaitLimitNs = BITNET_WAIT_LIMIT_NS;

// Set by any kernel whose bounded wait gave up; cleared by the host.
__device__ unsigned int g_device_error = 0;
// Set by the pack kernel when an input value is outside {-1, 0, +1}.
__device__ unsigned int g_pack_bad_value = 0;

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- numerics

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) {
  return __uint_as_float(h << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Quantiser parameters of one row, from its fp32 absmax.
struct RowQuant {
  float s;    // absmax / 127 (IEEE fp32 division), the divisor of x
  float r;    // 1 / s (IEEE), used for a guarded fast path only
};

__device__ __forceinline__ RowQuant row_quant(float absmax) {
  RowQuant q;
  const float a = fmaxf(absmax, 1e-5f);
  q.s = __fdiv_rn(a, 127.0f);
  q.r = __fdiv_rn(1.0f, q.s);
  return q;
}

// q = clamp(rint(fl(x / s)), -127, 127) with rint rounding halves to even.
// Fast path: y = fl(x * r) differs from fl(x / s) by at most
// |x/s| * 3 * 2^-24 <= 2.3e-5 (|x/s| <= ~127), so whenever y is at least
// 1e-4 away from a half-integer both round to the same integer. Only inputs
// within 1e-4 of a tie take the true IEEE division.
// rint is the magic-number method: for |y| < 2^22, y + 1.5 * 2^23 lies in
// [2^23, 2^24), where the spacing of floats is 1, so the IEEE addition itself
// rounds y to the nearest integer, halves to even; that integer is the sum's
// bit pattern minus the pattern of 1.5 * 2^23, and subtracting 1.5 * 2^23
// back is exact. (Two adds on the FMA pipe instead of the conversion pipe.)
__device__ __forceinline__ int rint_small(float y, float* r) {
  const float t = __fadd_rn(y, 12582912.0f);
  *r = __fsub_rn(t, 12582912.0f);
  return __float_as_int(t) - 0x4B400000;
}

// The exact quotient of a near-tie, out of line: ties are rare, and kept out
// of the callers' code the IEEE division is neither executed for every
// element nor repeated in every unrolled copy of a quantisation loop.
__device__ __noinline__ int quant_tie(float x, float s) {
  float r;
  return rint_small(__fdiv_rn(x, s), &r);
}

__device__ __forceinline__ int quant_one(float x, const RowQuant& q) {
  float y = __fmul_rn(x, q.r);
  float ry;
  int v = rint_small(y, &ry);
  if (fabsf(fabsf(__fsub_rn(y, ry)) - 0.5f) < 1e-4f) v = quant_tie(x, q.s);
  v = v < -127 ? -127 : v;
  v = v > 127 ? 127 : v;
  return v;
}

// The layer's bias (BitLinear.forward on the bitnet-cpu page adds it to the
// bf16 output): bf16(float(y) + float(bias[n])); no bias when bias is null.
__device__ __forceinline__ uint16_t add_bias_bf16_v(uint16_t y, uint16_t b) {
  return f32_to_bf16_bits(__fadd_rn(bf16_bits_to_f32(y), bf16_bits_to_f32(b)));
}
__device__ __forceinline__ uint16_t add_bias_bf16(uint16_t y, const uint16_t* bias, int64_t n) {
  if (bias == nullptr) return y;
  return add_bias_bf16_v(y, bias[n]);
}

// --------------------------------------------------------- PDL (griddep)

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ------------------------------------------------------------ global loads

__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ldg_stream_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ int dp4a_s32(uint32_t a, uint32_t b, int c) {
  return __dp4a(static_cast<int>(a), static_cast<int>(b), c);
}
// dp4a with unsigned bytes in `a` and signed bytes in `b`.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// ------------------------------------------------------- shared / mbarrier

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar,
                                                      uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
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

// Wait for the phase of parity `parity` of the mbarrier at `bar`.
// Gives up after kWaitLimitNs, or as soon as *abort is set by another role:
// sets the device error word and *abort, and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicOr(&g_device_error, kDevErrTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}

// mbar_wait for a whole warp: every lane gets the same answer (false if any
// lane gave up), so warp-collective instructions that follow stay converged.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity,
                                               volatile int* abort) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort));
}

// Drain wait used on the way out of a kernel: ignores the abort flag (the
// copies or MMAs it waits for complete on their own), bounded by 200 ms.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 63u && global_ns() - t0 > 200000000ull) {
      atomicOr(&g_device_error, kDevErrTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}

// 2-D tiled bulk tensor load global -> this CTA's shared memory, completing
// `bytes` of transaction count on the mbarrier. No multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m,
                                            uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(m), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// Bulk (non-tensor) async copy global -> this CTA's shared memory of `bytes`
// (multiple of 16; both addresses 16-byte aligned), completing on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 8-byte async copy global -> shared (L1-cached path), any 8-byte alignment.
__device__ __forceinline__ void cp_async_8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
// Arrive on `bar` once this thread's prior cp.async copies have landed
// (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// --------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile(
      "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
          dst_smem),
      "r"(ncols)
      : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(
                   taddr),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, int8 x int8 -> int32.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc,
                                       uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, int8 x int8 -> int32 (A from tensor
// memory: lane = row of A, 4 consecutive K bytes per 32-bit column).
__device__ __forceinline__ void mma_i8_tmem_a(uint32_t d_tmem, uint32_t a_tmem,
                                              uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread t of the warp writes lane
// (base lane + t), columns [col, col + 16).
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Arrive once on the mbarrier when all prior tcgen05.mma of this thread end.
// The four kind::i8 MMAs of one 128-wide K block (A from tensor memory,
// columns a + 8k; B descriptor b + 2k), with a non-blocking test of the
// mbarrier phase the next K block needs issued ahead of them: its answer is
// read only after the four MMAs are issued, so the barrier's round trip
// overlaps them instead of preceding the next block. Returns whether that
// phase has completed (false: the caller waits for it).
__device__ __forceinline__ bool mma4_i8_tmem_a_test(uint32_t d_tmem, uint32_t a_tmem,
                                                    uint64_t bdesc, uint32_t idesc,
                                                    uint32_t accumulate, uint32_t next_bar,
                                                    uint32_t next_parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p, t, q;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q, [%5], %6;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.u32 t, 0, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%1], [%2], %3, %7, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%1], [%8], %9, %7, t;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%1], [%10], %11, %7, t;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%1], [%12], %13, %7, t;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(ok)
      : "r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(accumulate), "r"(next_bar), "r"(next_parity),
        "r"(idesc), "r"(a_tmem + 8u), "l"(bdesc + 2u), "r"(a_tmem + 16u), "l"(bdesc + 4u),
        "r"(a_tmem + 24u), "l"(bdesc + 6u)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 "
      "[%0];" ::"r"(bar)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives
// lane (base lane + t), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr,
                                                   uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]),
        "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]),
        "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 format) for a K-major operand in
// the 128-byte swizzle layout: rows of 128 bytes, 8-row atoms of 1024 bytes
// (stride byte offset), atoms 1024-byte aligned, descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);         // start address
  d |= static_cast<uint64_t>(1u) << 16;                         // LBO (unused)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;                 // SBO
  d |= static_cast<uint64_t>(1u) << 46;                         // version
  d |= static_cast<uint64_t>(2u) << 61;                         // SWIZZLE_128B
  return d;
}

// ------------------------------------------------ thread-block clusters

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Every thread of every CTA of the cluster; shared-memory writes before it
// are visible to the whole cluster after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 16 bytes of CTA `rank`'s shared memory at the address that `saddr` has in
// this CTA's shared window.
__device__ __forceinline__ uint4 dsmem_ld_v4(uint32_t saddr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(saddr), "r"(rank));
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(remote)
               : "memory");
  return v;
}

// 4 bytes of CTA `rank`'s shared memory at the address that `saddr` has in
// this CTA's shared window.
__device__ __forceinline__ uint32_t dsmem_ld_u32(uint32_t saddr, uint32_t rank) {
  uint32_t remote, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(saddr), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

}  // namespace bitnet
