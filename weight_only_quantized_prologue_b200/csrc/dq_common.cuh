// dq_common.cuh -- sm_100a building blocks shared by the kernels: mbarriers
// with bounded waits, bulk / tensor copies, tcgen05 (TMEM, MMA, commit), the
// shared-memory matrix descriptor, and the in-register unpack of the packed
// weight codes into bf16x2 tensor-core operands.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dq_layout.h"

namespace dq {

// ---------------------------------------------------------------------------
// device status word values (mirrors dqgemm_status)
// ---------------------------------------------------------------------------
constexpr int DEV_OK = 0;
constexpr int DEV_TIMEOUT = 6;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
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
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Control of a bounded wait, passed by value (it lives in registers or is
// rematerialised from kernel parameters; nothing of it goes to the stack):
// every wait gives up after `timeout_ns`, or as soon as another thread of
// the CTA has set the shared `abort` flag (null: ignore the flag); the
// first thread to give up records DEV_TIMEOUT in the global status word.
struct WaitCtl {
  volatile int* abort;   // shared memory flag, or null
  int* status;           // global status word (may be null)
  uint64_t timeout_ns;
};

// try_wait with a suspend-time hint: the waiting thread sleeps in hardware
// until the phase completes (or ~hint ns pass) instead of spinning on issue
// slots the producer and MMA threads need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool wait_give_up(const WaitCtl ctl, uint64_t t0) {
  if (ctl.abort && *ctl.abort) return true;
  if (globaltimer_ns() - t0 > ctl.timeout_ns) {
    if (ctl.abort) *ctl.abort = 1;
    if (ctl.status) *reinterpret_cast<volatile int*>(ctl.status) = DEV_TIMEOUT;   // every writer writes the same value
    return true;
  }
  return false;
}

// (the limit is checked before each sleep, so a wait that does not complete
// at once gives up as soon as its limit has passed, however short)
__device__ __forceinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, const WaitCtl ctl) {
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (wait_give_up(ctl, t0)) return false;
    if (mbar_try_wait_sleep(bar, parity)) return true;
  }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtl ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, ctl);
}

// Whole-warp wait.  Common case, the phase already complete: every lane
// observes it itself (acquire) and the warp agrees by a vote (one try_wait
// and a vote; lane 0 first, a shuffle, then every lane, cost ~230 cycles).
// Otherwise lane 0 sleeps on the barrier, the other lanes wait at the
// shuffle, then every lane observes the completed phase itself.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, const WaitCtl ctl) {
  if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, ctl) ? 1 : 0;
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  if (ok) mbar_try_wait(bar, parity);
  return ok != 0;
}



// ---------------------------------------------------------------------------
// bulk and tensor copies global -> shared (no multicast anywhere)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// one box of a 3-D tensor map {inner 64 k, rows, k-blocks of 64}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// global loads issued exactly where written (read-only data fetched early,
// ahead of the grid-dependency wait, and consumed in the epilogue)
__device__ __forceinline__ float ld_nc_f32(const float* p) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ float ld_nc_bf16(const __nv_bfloat16* p) {
  unsigned short v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return __uint_as_float((uint32_t)v << 16);
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// programmatic dependent launch: let the next grid in the stream start its
// prologue now / wait until every grid this one depends on has completed
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// thread-block cluster: rank, full barrier, distributed shared memory loads
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// split cluster barrier: arrive early (relaxed, no wait), wait much later
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
// distributed shared memory: the address of the same shared-memory location
// in cluster CTA `rank`, and asynchronous stores into it that count their
// bytes on a (remote) mbarrier's transaction count
__device__ __forceinline__ uint32_t dsmem_addr(const void* local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_async_v4(uint32_t raddr, float a, float b, float c, float d, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   raddr),
               "f"(a), "f"(b), "f"(c), "f"(d), "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t raddr, float a, float b, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(raddr),
               "f"(a), "f"(b), "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async_u32(uint32_t raddr, uint32_t v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(raddr), "r"(v),
               "r"(rbar)
               : "memory");
}

// wait on an mbarrier whose phase is completed by other CTAs of the cluster
// (st.async transactions): cluster-scope acquire, bounded like mbar_wait.
// No suspend-time hint: a thread suspended on the barrier is not woken
// promptly by remote transactions (it slept out the hint), so it polls.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, const WaitCtl ctl) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (wait_give_up(ctl, t0)) return false;
    if (mbar_try_wait_cluster(bar, parity)) return true;
  }
}


// e4m3 code of v, saturating to +-448, round to nearest even; a zero result
// keeps the sign of v (static FP8 activation codes)
__device__ __forceinline__ uint8_t e4m3_code(float v) {
  uint8_t c = (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
  if ((c & 0x7F) == 0) c = signbit(v) ? 0x80 : 0x00;
  return c;
}

// f32(v / s), correctly rounded, for the e4m3 conversion that follows,
// without a division: Markstein's correction step (P. Markstein, "Computation
// of elementary functions on the IBM RISC System/6000 processor", 1990).
// With r = f32(1 / s) correctly rounded, q0 = f32(v * r) lies within one
// unit in the last place of v / s, the residual v - q0 * s is then exact in
// one fused multiply-add, and f32(q0 + residual * r) is the correctly
// rounded quotient, provided nothing overflows or underflows.  Outside
// [2^-12, 2^9) the e4m3 code is +-0 or +-448 whatever the quotient's last
// bits, so q0 is used as it is there (which also keeps the residual in
// range).  r must be a normal fp32 value (s within [2^-126, 2^126]).
__device__ __forceinline__ float e4m3_quotient(float v, float s, float r) {
  const float q0 = __fmul_rn(v, r);
  const float a = fabsf(q0);
  if (!(a >= 0x1p-12f && a < 0x1p9f)) return q0;
  return __fmaf_rn(__fmaf_rn(-q0, s, v), r, q0);
}

// whether e4m3_quotient may be used for the scale s (its reciprocal normal)
__device__ __forceinline__ bool e4m3_quotient_ok(float r) {
  const uint32_t e = __float_as_uint(r) & 0x7F800000u;
  return e != 0u && e != 0x7F800000u;
}

// static-FP8 activation code of a value v (the Q node): e4m3(f32(v / s)),
// the IEEE quotient (r = f32(1 / s); the division itself where r is not a
// normal number)
__device__ __forceinline__ uint8_t act_code_r(float v, float s, float r) {
  if (e4m3_quotient_ok(r)) return e4m3_code(e4m3_quotient(v, s, r));
  return e4m3_code(__fdiv_rn(v, s));
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and MMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T, bf16 inputs, fp32 accumulate
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, e4m3 inputs, fp32 accumulate
__device__ __forceinline__ void mma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// e4m3 x e4m3 with A (128 x 32 e4m3, four codes a 32-bit column, the lower
// k in the lower byte) in tensor memory and B in shared memory
__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptors (M = 128 rows of W, N = BN rows of x, K-major A and B).
__host__ __device__ constexpr uint32_t idesc_bf16(int bn) {
  return (1u << 4)            // D format f32
         | (1u << 7)          // A bf16
         | (1u << 10)         // B bf16
         | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(TILE_N >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_e4m3(int bn) {
  return (1u << 4)  // D f32; A, B format 0 = E4M3
         | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(TILE_N >> 4) << 24);
}

// Block-scaled FP4 x FP4 (kind::mxf4 for MXFP4, kind::mxf4nvf4 for NVFP4):
// A and B packed E2M1 (two codes a byte, the even k in the low nibble),
// K-major, D fp32, 64 k per MMA.  Bits: 7-9 / 10-12 A / B format (1 = E2M1),
// 17-22 N / 8, 23 scale format (1 = E8M0, 0 = E4M3), 24-28 M / 16; the scale
// factors' byte selectors (bits 4-5, 29-30) stay 0: each operand's scale
// words start at byte 0 of their tensor-memory columns.
__host__ __device__ constexpr uint32_t idesc_fp4(int bn, bool e8m0) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(bn >> 3) << 17) | ((e8m0 ? 1u : 0u) << 23) |
         ((uint32_t)(TILE_N >> 4) << 24);
}

// D (+)= A . B^T with per-block scale factors read from tensor memory: for
// row m of A the word at lane m % 32 (every lane quadrant holds a copy),
// column sfa + m / 32, byte j = the scale of the j-th block of this MMA's
// 64 k (2 blocks of 32 for MXFP4, 4 of 16 for NVFP4); likewise for the rows
// of B at sfb.
template <bool MX>
__device__ __forceinline__ void mma_fp4_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  if constexpr (MX) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
  }
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row groups 1024 bytes apart.  `saddr` must lie in a
// 1024-byte-aligned swizzle atom (plus the k offset within its row).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// n consecutive 32-bit columns of this warp's 32 lanes (n = 1, 2, 4, 8)
template <int NC>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t* v) {
  if constexpr (NC == 1) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v[0]) : "memory");
  } else if constexpr (NC == 2) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(v[0]), "r"(v[1])
                 : "memory");
  } else if constexpr (NC == 4) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(v[0]),
                 "r"(v[1]), "r"(v[2]), "r"(v[3])
                 : "memory");
  } else {
    static_assert(NC == 8, "1, 2, 4 or 8 columns");
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
  }
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr)
               : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------------------
// shared-memory vector access
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ void sts128(void* p, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(p)), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// ---------------------------------------------------------------------------
// unpack: packed codes -> bf16x2 tensor-core operands
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                             *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t bsub2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                             *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// INT4: a nibble n with bits 0x4300 | (n ^ 8) is the bf16 value 136 + c for
// the two's-complement code c; subtracting 136 is exact, and one rounding
// multiply gives bf16(c * s) -- the page's dequantize_affine with zero-point 0.
__device__ __forceinline__ void unpack_int4(uint32_t q, uint32_t s2, uint32_t* o) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t v = ((q >> (4 * j)) & 0x000F000Fu) ^ 0x43084308u;
    o[j] = bmul2(bsub2(v, 0x43084308u), s2);
  }
}

// Unsigned INT4 (asymmetric format): 0x4300 | u is the bf16 of 128 + u, and
// zs2 holds bf16(128 + z) twice, so one sub and one mul give (u - z) * s
// exactly.
__device__ __forceinline__ void unpack_int4u(uint32_t q, uint32_t zs2, uint32_t s2, uint32_t* o) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t v = ((q >> (4 * j)) & 0x000F000Fu) | 0x43004300u;
    o[j] = bmul2(bsub2(v, zs2), s2);
  }
}

// E2M1: magnitude bits (e1 e0 m) placed at bf16 bits 8..6 with the sign at
// bit 15 read as a bf16 are exactly e2m1 * 2^-126 (the subnormal code 0.5
// lands on a bf16 subnormal, code 0 on zero).  The block scale word s2
// carries 2^126 times the wanted factor, so the product is exact.
__device__ __forceinline__ void unpack_e2m1(uint32_t q, uint32_t s2, uint32_t* o) {
  const uint32_t w0 = ((q << 6) & 0x01C001C0u) | ((q << 1) & 0x80008000u);
  const uint32_t w1 = (q << 3) & 0x81C081C0u;
  const uint32_t w2 = q & 0x81C081C0u;
  const uint32_t w3 = ((q >> 3) & 0x01C001C0u) | ((q << 2) & 0x80008000u);
  o[0] = bmul2(w0, s2);
  o[1] = bmul2(w1, s2);
  o[2] = bmul2(w2, s2);
  o[3] = bmul2(w3, s2);
}

// E4M3: magnitude bits at bf16 bits 10..4 with the sign at bit 15 read as a
// bf16 are exactly e4m3 * 2^-120; multiplying by 2^120 is exact.
constexpr uint32_t BF16X2_2P120 = 0x7B807B80u;
__device__ __forceinline__ void unpack_e4m3(uint32_t q, uint32_t* o) {
  const uint32_t w0 = ((q << 4) & 0x07F007F0u) | (q & 0x80008000u);
  const uint32_t w1 = ((q >> 3) & 0x07F007F0u) | ((q << 1) & 0x80008000u);
  o[0] = bmul2(w0, BF16X2_2P120);
  o[1] = bmul2(w1, BF16X2_2P120);
}

// NVFP4 block scale: bf16 of dec(sb) * 2^119 for a non-negative E4M3 code,
// so that (e2m1 * 2^-126) * it = e2m1 * dec(sb) * 2^-7 exactly; the epilogue
// multiplies by g * 2^7.
__device__ __forceinline__ uint32_t nvfp4_scale_bf16(uint32_t code) {
  const uint32_t e = (code >> 3) & 15u, m = code & 7u;
  const uint32_t normal = ((code & 0x7Fu) << 4) + 0x7780u;             // exponent field + 239
  const uint32_t sub = __float_as_uint((float)m * 0x1p110f) >> 16;    // m * 2^-9 * 2^119
  return e ? normal : sub;
}

// MXFP4 block scale: bf16 2^(e - 127) * 2^(126 - J) with the handle's shift
// J folded into `bias` = 126 - J; fields outside the normal range clamp.
__device__ __forceinline__ uint32_t mxfp4_scale_bf16(uint32_t code, int bias) {
  int f = (int)code + bias;
  f = f < 0 ? 0 : (f > 254 ? 254 : f);
  return (uint32_t)f << 7;
}

}  // namespace dq
