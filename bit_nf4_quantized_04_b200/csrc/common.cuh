// Shared device helpers for libqnf4: error flag, bounded waits, mbarrier, TMA and
// tcgen05 (5th-generation tensor core) wrappers written as inline PTX for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define QNF4_DEV __device__ __forceinline__

// ----------------------------------------------------------------------------
// Device error flag. A kernel whose bounded wait gives up records a nonzero code
// here (the first one wins) and returns; qnf4_check() reads and clears it.
// ----------------------------------------------------------------------------
__device__ unsigned int g_qnf4_err = 0;

QNF4_DEV void set_err(unsigned int code) { atomicCAS(&g_qnf4_err, 0u, code); }

// Index checks of the checked build (compiled with -DQNF4_CHECKED, libqnf4_checked.so): an
// access whose index falls outside its buffer records kErrBoundsBase + site in the device
// flag and is skipped, so a planning or indexing mistake shows as QNF4_ERR_BOUNDS instead
// of a fault. The default build compiles no check (the condition is dead code).
constexpr unsigned int kErrBoundsBase = 1000;
#ifdef QNF4_CHECKED
QNF4_DEV bool in_bounds(bool ok, unsigned int site) {
  if (!ok) set_err(kErrBoundsBase + site);
  return ok;
}
#else
QNF4_DEV bool in_bounds(bool, unsigned int) { return true; }
#endif

// Deadline of a drain: once a kernel gives up, it still waits for its own copies and
// MMAs in flight before it frees shared and tensor memory, however short the caller's
// wait limit; those always finish unless the hardware itself has stopped.
constexpr unsigned long long kDrainFloorNs = 1000000000ull;
QNF4_DEV unsigned long long drain_ns(unsigned long long wait_ns) {
  return wait_ns > kDrainFloorNs ? wait_ns : kDrainFloorNs;
}

// Clock of the bounded waits: the SM's cycle counter, a cheap register read. (Reading
// %globaltimer is a slow special-register access; many warps polling it measured 97-98 %
// busy on the SM's special-function / conversion pipe, which then throttled everything
// else that pipe serves.) Limits given in nanoseconds count as 2 cycles per ns (clocks up
// to 2 GHz), so a wait never gives up before its limit.
QNF4_DEV long long wait_clock() { return clock64(); }
QNF4_DEV long long ns_cycles(unsigned long long ns) {
  return static_cast<long long>(ns < (1ull << 61) ? ns : (1ull << 61)) * 2;
}


// Programmatic dependent launch (PDL) controls.
QNF4_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
QNF4_DEV void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

QNF4_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ----------------------------------------------------------------------------
// mbarrier
// ----------------------------------------------------------------------------
QNF4_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
QNF4_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
QNF4_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

QNF4_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
QNF4_DEV void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// Test for the completion of the phase with the given parity (returns at once).
QNF4_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
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
// The same test for long waits (a producer waiting for a free slot, an epilogue waiting
// for a whole tile's MMAs, a drain): a thread whose phase has not completed is suspended
// by the hardware until it completes or kWaitHintNs pass, so these loops poll rarely
// instead of taking issue slots from the working warps. Latency-critical hand-offs (data
// landed, a stage converted) poll with mbar_try_wait, which measured faster there.
constexpr uint32_t kWaitHintNs = 10000;
QNF4_DEV bool mbar_try_wait_long(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kWaitHintNs)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete, at most wait_ns.
// Returns false (and records `code`) on timeout.
QNF4_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned long long wait_ns,
                        unsigned int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = wait_clock();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (wait_clock() - t0 > ns_cycles(wait_ns)) {
      set_err(code);
      return false;
    }
  }
}

// Spin on a phase with a bound, in every lane of a warp, then agree: the result is
// the same in all lanes (all observed the phase, or the warp gives up together).
QNF4_DEV bool warp_wait(uint64_t* bar, uint32_t parity, unsigned long long wait_ns,
                        volatile int* abort_flag, unsigned int site) {
  bool ok = mbar_try_wait(bar, parity);
  if (!ok) {
    const long long t0 = wait_clock();
    while (!(ok = mbar_try_wait(bar, parity))) {
      if (*abort_flag) break;
      if (wait_clock() - t0 > ns_cycles(wait_ns)) {
        set_err(site);
        *abort_flag = 1;
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}

// ----------------------------------------------------------------------------
// TMA (bulk tensor copies global -> shared, completion on an mbarrier)
// ----------------------------------------------------------------------------
QNF4_DEV void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                          int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
QNF4_DEV void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                          int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// Tile shared -> global (bulk async group of the issuing thread; out-of-range
// elements of the box are not written).
QNF4_DEV void tma_store_2d(const CUtensorMap* map, const void* src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
QNF4_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// this thread's bulk stores have finished reading shared memory / have completed
QNF4_DEV void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
QNF4_DEV void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
QNF4_DEV void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// Bulk prefetch of a global range into L2 (16-byte aligned address, size a multiple of 16).
QNF4_DEV void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// 1-D bulk copy global -> shared (16-byte aligned addresses, size multiple of 16).
QNF4_DEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA, commit, loads/stores, fences
// ----------------------------------------------------------------------------
QNF4_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
QNF4_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
QNF4_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
QNF4_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
QNF4_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, fp32 accumulate)
QNF4_DEV void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                     uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T
QNF4_DEV void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                     uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on an mbarrier once all previously issued MMAs of this thread complete.
QNF4_DEV void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
QNF4_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
QNF4_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 8 consecutive columns per thread.
QNF4_DEV void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
// 32 lanes x 32 bits, 16 consecutive columns per thread.
QNF4_DEV void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
QNF4_DEV void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// Shared-memory matrix descriptor (sm_100 UMMA format):
//   bits  0-13 start address >> 4, 16-29 leading byte offset >> 4,
//   32-45 stride byte offset >> 4, 46-47 version (1), 61-63 layout (2 = 128B swizzle).
QNF4_DEV uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                            uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(layout & 0x7) << 61;
  return d;
}
constexpr uint32_t kLayoutSW128 = 2;

// Instruction descriptor for kind::f16 with bf16 A/B, fp32 D.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format (1 = bf16),
//   15 A major (0 = K, 1 = MN), 16 B major, 17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t M, uint32_t N, uint32_t a_mn,
                                                  uint32_t b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn << 15) | (b_mn << 16) | ((N >> 3) << 17) |
         ((M >> 4) << 24);
}

// ----------------------------------------------------------------------------
// small numeric helpers
// ----------------------------------------------------------------------------
QNF4_DEV float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
QNF4_DEV float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
// pack two fp32 to bf16x2 (round to nearest even); `lo` lands in bits 0-15.
QNF4_DEV uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// E4M3 byte -> fp32 (exact) through the hardware fp8 -> half conversion.
QNF4_DEV float e4m3_to_f32(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
  return __half2float(__half(h));
}
