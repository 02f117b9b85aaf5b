// Device helpers shared by the SVDQuant kernels: inline PTX for mbarriers,
// TMA, tcgen05 (TMEM allocation, MMA, loads and stores) and the FP4/FP8 conversions.
// Written for sm_100a from the public PTX ISA.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#define SVDQ_DEV __device__ __forceinline__

namespace svdq {

// ------------------------------------------------------------ error word ----
// Set by a kernel whose bounded wait ran out; read and cleared by the host
// (svdq_get_device_error).  Bit 0: timeout.  g_err_site: which wait.
__device__ unsigned int g_err_flags;
__device__ unsigned int g_err_site;

enum : unsigned { ERR_TIMEOUT = 1u, ERR_CHECK = 2u };

SVDQ_DEV void report_timeout(unsigned site) {
  // a failed copy check (which makes later waits run out) keeps its own site
  if (!(atomicOr(&g_err_flags, ERR_TIMEOUT) & ERR_CHECK)) atomicExch(&g_err_site, site);
}

// Debug build (-DSVDQ_CHECK, libsvdq_check.so): every TMA and bulk copy is checked before it is issued
// (alignment of the innermost coordinate, coordinates and sources inside their tensors, destination
// inside the launch's shared memory); a failed check records ERR_CHECK and the copy is skipped, so
// the kernel's bounded waits end it with the error word set instead of issuing a faulting copy.
SVDQ_DEV void report_check(unsigned site) {
  atomicOr(&g_err_flags, ERR_CHECK);
  atomicExch(&g_err_site, site);
}
#ifdef SVDQ_CHECK
#define SVDQ_CHECK_OK(cond, site) ((cond) || (::svdq::report_check(site), false))
#else
#define SVDQ_CHECK_OK(cond, site) true
#endif

// --------------------------------------------------------------- basics -----
SVDQ_DEV uint32_t dyn_smem_bytes() {
  uint32_t v;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(v));
  return v;
}

SVDQ_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory loads by 32-bit shared address (ld.shared: no generic-address resolution).
SVDQ_DEV uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
SVDQ_DEV float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

SVDQ_DEV uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------- mbarrier -----
SVDQ_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

SVDQ_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

SVDQ_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

SVDQ_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

SVDQ_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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


// Wait for the phase with parity `parity` to complete.  Gives up after
// `timeout_ns` of wall time, or as soon as `*abort` is set by another role of
// the same CTA; on a time-out it records `site` in the error word and sets
// `*abort`.  Returns false when it gave up.
SVDQ_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns, volatile int* abort,
                        unsigned site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      *abort = 1;
      report_timeout(site);
      return false;
    }
  }
}

// Non-blocking test of the phase with parity `parity`.
SVDQ_DEV bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// mbar_wait for the single threads on a pipeline's critical path (copy producers, MMA issuers):
// polls with the non-blocking test, so the thread sees the phase complete without the wake-up
// delay a suspended try_wait can add.  Same time-out and abort behaviour as mbar_wait.
SVDQ_DEV bool mbar_wait_spin(uint64_t* bar, uint32_t parity, uint64_t timeout_ns, volatile int* abort,
                             unsigned site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t n = 0;; ++n) {
    if (mbar_test_wait(a, parity)) return true;
    if ((n & 15u) == 15u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > timeout_ns) {
        *abort = 1;
        report_timeout(site);
        return false;
      }
    }
  }
}


// ------------------------------------------------------------------ TMA -----
SVDQ_DEV void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}

// 2-D tiled load: box at (x = innermost coordinate, y) into shared memory,
// completion counted in bytes on `bar`.
SVDQ_DEV void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(m), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled load: box at (x, y, z) into shared memory, completion counted in bytes on `bar`.
SVDQ_DEV void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int32_t x, int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(smem_u32(dst)), "l"(m), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size % 16 == 0).
SVDQ_DEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// -------------------------------------------------------------- tcgen05 -----
SVDQ_DEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
SVDQ_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
SVDQ_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
SVDQ_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
SVDQ_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive once on `bar` when every tcgen05 operation this thread issued before it has completed.
SVDQ_DEV void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

// D(tmem) (+)= A(smem) x B(smem)^T, E2M1 x E2M1 with UE4M3 scales per 16 along K (K = 64).
SVDQ_DEV void tc_mma_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                          uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
      ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
      : "memory");
}

// D(tmem) (+)= A(smem) x B(smem)^T, bf16 x bf16 -> f32 (K = 16).
SVDQ_DEV void tc_mma_bf16(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}


// Each thread of the warp reads 32 consecutive 32-bit columns of its TMEM lane.
SVDQ_DEV void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
// Each thread of the warp reads 16 consecutive 32-bit columns of its TMEM lane.
SVDQ_DEV void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
SVDQ_DEV void reg_fence16(uint32_t (&v)[16]) {
  asm volatile(""
      : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
        "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]));
}

// Each thread of the warp writes 16 consecutive 32-bit columns of its TMEM lane.
SVDQ_DEV void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// One 32-byte global store (the address must be 32-byte aligned).
SVDQ_DEV void st_global_v8(void* p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t a4, uint32_t a5,
                           uint32_t a6, uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a0), "r"(a1), "r"(a2),
               "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}
SVDQ_DEV void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Register budget of the calling warpgroup (all four warps execute it).
template <int N>
SVDQ_DEV void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N>
SVDQ_DEV void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }


SVDQ_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Ties registers filled by tcgen05.ld to a point after tcgen05.wait::ld, so that
// no use of them is scheduled before the wait.
SVDQ_DEV void reg_fence(uint32_t (&v)[32]) {
  asm volatile(""
      : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
        "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]),
        "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]), "+r"(v[23]),
        "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]), "+r"(v[30]), "+r"(v[31]));
}

// Shared-memory matrix descriptor: K-major operand tile whose rows are 128 bytes,
// stored with the 128-byte swizzle, 8-row groups 1024 bytes apart (tile base 1024-aligned).
SVDQ_DEV uint64_t sdesc_kmajor_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;            // leading byte offset (unused for this layout)
  d |= (uint64_t)(1024u >> 4) << 32;  // stride byte offset: next 8-row group
  d |= (uint64_t)1u << 46;            // descriptor version for tcgen05
  d |= (uint64_t)2u << 61;            // 128-byte swizzle
  return d;
}

// Same for a K-major tile whose rows are 64 bytes, stored with the 64-byte swizzle (8-row groups
// 512 bytes apart, tile base 512-aligned).
SVDQ_DEV uint64_t sdesc_kmajor_sw64(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(512u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)4u << 61;            // 64-byte swizzle
  return d;
}

// ------------------------------------------------- programmatic dependent launch ---
// Wait until the kernels this grid depends on (launched before it on the stream) have finished and
// their writes are visible; a no-op when the grid was launched without the programmatic attribute.
SVDQ_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the next kernel on the stream start its prologue while this grid runs (it still waits for
// this grid's completion before reading anything).
SVDQ_DEV void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Instruction descriptor, kind::mxf4nvf4: A, B = E2M1 (K-major), scales UE4M3, M x N, dense K = 64.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Instruction descriptor, kind::mxf4 (scale_vec::2X): A, B = E2M1 (K-major), E8M0 scales (bit 23), M x N,
// dense K = 64; `sf_id` is the byte of the 32-bit TMEM scale column where this MMA's two scales start
// (bits 29-30 for A, 4-5 for B).
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N, uint32_t sf_id) {
  return (sf_id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((uint32_t)(M >> 4) << 24) |
         (sf_id << 29);
}
// D(tmem) (+)= A(smem) x B(smem)^T, E2M1 x E2M1 with E8M0 scales per 32 along K (K = 64).
SVDQ_DEV void tc_mma_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                          uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
      ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::f16: A, B = bf16 (K-major), D = f32, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ----------------------------------------------------------- conversions ----
// Eight float32 -> eight E2M1 codes (round to nearest even, saturating), element i in nibble i.
SVDQ_DEV uint32_t cvt_e2m1x8(const float (&v)[8]) {
  uint32_t r;
  asm(
      "{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// Non-negative float32 -> UE4M3 byte (round to nearest even, saturating at 448).
SVDQ_DEV uint32_t cvt_ue4m3(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// UE4M3 byte -> float32 (exact, via the f16 conversion).
SVDQ_DEV float dec_ue4m3(uint32_t b) {
  uint32_t h2;
  const uint16_t in = (uint16_t)(b & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// ---------------------------------------------------------------- MXFP4 -----
// MX block scale of a block whose largest magnitude is `amax` (>= 0): the exponent
// X = floor(log2(amax)) - 2 (2: the exponent of the largest E2M1 value, 6 = 1.5 * 2^2), clamped to
// [-127, 127], -127 for amax = 0; returns the E8M0 byte X + 127 and sets `mul` = 2^-X (exact).
SVDQ_DEV uint32_t mx_scale(float amax, float& mul) {
  const uint32_t bits = __float_as_uint(amax);
  const int e = (int)((bits >> 23) & 0xFFu);
  int fl;
  if (e) fl = e - 127;                                           // normal: the exponent field
  else fl = (bits & 0x7FFFFFu) ? (31 - __clz(bits & 0x7FFFFFu)) - 149 : -129;   // subnormal / zero
  int X = fl - 2;
  X = X < -127 ? -127 : (X > 127 ? 127 : X);
  const int ne = -X;                                             // 2^ne, ne in [-127, 127]
  mul = ne >= -126 ? __uint_as_float((uint32_t)(ne + 127) << 23) : __uint_as_float(1u << 22);
  return (uint32_t)(X + 127);
}

// Element-wise arithmetic on float32 pairs, one packed instruction each; every element is one
// correctly rounded operation (an explicit rounding mode: never contracted into a fused multiply-add).
SVDQ_DEV uint64_t f2_bits(float2 a) {
  return (uint64_t)__float_as_uint(a.x) | ((uint64_t)__float_as_uint(a.y) << 32);
}
SVDQ_DEV float2 bits_f2(uint64_t d) {
  return make_float2(__uint_as_float((uint32_t)d), __uint_as_float((uint32_t)(d >> 32)));
}
SVDQ_DEV float2 mul_f32x2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(d);
}
SVDQ_DEV float2 add_f32x2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(d);
}
SVDQ_DEV float2 fma_f32x2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
  return bits_f2(d);
}
SVDQ_DEV float2 sub_f32x2(float2 a, float2 b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(d);
}

SVDQ_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
SVDQ_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

SVDQ_DEV uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<const uint32_t*>(&p);
}

// Byte offset of the 32-bit word holding scales kk4*4 .. kk4*4+3 of row `row`,
// in MMA scale order (see include/svdq.h).
SVDQ_DEV uint32_t sf_word_offset(uint32_t row, uint32_t kk4, uint32_t KS4) {
  return ((row >> 7) * KS4 + kk4) * 512u + (row & 31u) * 16u + ((row >> 5) & 3u) * 4u;
}

}  // namespace svdq
