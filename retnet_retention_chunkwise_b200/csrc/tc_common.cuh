// tc_common.cuh -- sm_100a building blocks written as inline PTX: mbarriers
// with bounded waits, TMA tile loads, tcgen05 MMA / TMEM access and the
// shared-memory matrix descriptors the tensor core reads.
//
// Conventions used by every kernel in this library:
//  * bf16 tiles live in shared memory in the 128-byte-swizzled layout that a
//    TMA load with CU_TENSOR_MAP_SWIZZLE_128B produces: rows of 128 bytes
//    (64 bf16), 8-row atoms of 1024 bytes, 16-byte chunk c of row r stored at
//    chunk (c ^ (r & 7)).  Every tile base is 1024-byte aligned.
//  * One M = 128 accumulator tile occupies TMEM lanes 0..127; warp w of the
//    epilogue reads lanes 32*(w%4) .. 32*(w%4)+31 (its sub-partition).
//  * Every wait is bounded (wall clock via %globaltimer plus an iteration cap);
//    on expiry the waiter raises the CTA abort flag and the device status word,
//    and all roles fall through to an orderly teardown.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace ret {

// Device status word (read and cleared by retention_get_device_status).
// 0 = ok, 4 = a bounded wait expired.  The library is one translation unit, so
// this is the single definition.
__device__ int g_device_status = 0;

// Bounds-checked builds (-DRET_BOUNDS_CHECK): RET_BC(cond, site) evaluates an
// index check; when it fails, the first failing site number is kept in
// g_bc_site, the device status word reads 5 (RET_EBOUNDS on the host) and the
// caller skips the access the check guards.  In the normal build RET_BC is the
// constant true and costs nothing.  Site numbers: 1xx chunkwise (dk <= 128),
// 2xx chunkwise dk = 256, 3xx blocks of 129..256 rows, 4xx segment sums and
// scan, 5xx parallel form, 6xx decode, 7xx GroupNorm.
#ifdef RET_BOUNDS_CHECK
__device__ unsigned int g_bc_site = 0;
__device__ __forceinline__ bool bc_ok(bool ok, unsigned int site) {
  if (!ok) {
    atomicCAS(&g_bc_site, 0u, site);
    atomicExch(&g_device_status, 5);
  }
  return ok;
}
#define RET_BC(cond, site) (::ret::bc_ok((cond), (site)))
#else
#define RET_BC(cond, site) (true)
#endif

// Optional event trace (builds with -DRET_TRACE only): %clock64 stamps (SM
// cycles; compare stamps of one CTA only) per (CTA, block, event) written to a
// caller-provided buffer.  RET_TRACE_INIT reads
// the buffer description once into registers; the stamps are plain stores.
// Both compile to nothing in the normal build.
#ifdef RET_TRACE
__device__ unsigned long long* g_trace_buf = nullptr;
__device__ int g_trace_events = 0;   // events per (CTA, block)
__device__ int g_trace_blocks = 0;   // block slots per CTA
#define RET_TRACE_INIT()                                \
  unsigned long long* trace_buf_ = g_trace_buf;         \
  const int trace_ev_ = g_trace_events;                 \
  const int trace_bl_ = g_trace_blocks
#define RET_TRACE_STAMP(cta, it, ev)                                                       \
  do {                                                                                     \
    if (trace_buf_ && (it) < trace_bl_ && (ev) < trace_ev_) {                              \
      unsigned long long t_;                                                               \
      asm volatile("mov.u64 %0, %%clock64;" : "=l"(t_));                             \
      trace_buf_[((size_t)(cta) * trace_bl_ + (it)) * trace_ev_ + (ev)] = t_;              \
    }                                                                                      \
  } while (0)
#else
#define RET_TRACE_INIT() \
  do {                   \
  } while (0)
#define RET_TRACE_STAMP(cta, it, ev) \
  do {                               \
  } while (0)
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Programmatic dependent launch.  griddep_wait blocks the calling thread until
// the grids this launch depends on have completed with their writes visible;
// it returns at once for a launch made without programmatic serialization.
// griddep_launch_dependents lets the next launch on the stream, if it was made
// with programmatic serialization, start before this grid has finished.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// One poll of a phase.  The suspend-time hint lets the hardware park the
// waiting thread (up to kSuspendNs) until the phase completes, so waiting warps
// do not take issue slots from working warps on the same sub-partition.
constexpr uint32_t kSuspendNs = 100000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Non-blocking test of four phases at once (a barrier may be repeated): the
// four tests go out back to back, so when every phase is already complete the
// answer costs one shared-memory round trip instead of four in a row.
__device__ __forceinline__ bool mbar_test4(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1, uint64_t* b2,
                                           uint32_t p2, uint64_t* b3, uint32_t p3) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred q0, q1, q2, q3;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q0, [%1], %2;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q1, [%3], %4;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q2, [%5], %6;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q3, [%7], %8;\n\t"
      "and.pred q0, q0, q1;\n\t"
      "and.pred q2, q2, q3;\n\t"
      "and.pred q0, q0, q2;\n\t"
      "selp.u32 %0, 1, 0, q0;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(b0)), "r"(p0), "r"(smem_u32(b1)), "r"(p1), "r"(smem_u32(b2)), "r"(p2), "r"(smem_u32(b3)),
        "r"(p3)
      : "memory");
  return ok != 0;
}

struct WaitLimit {
  uint64_t ns;        // wall-clock budget of one wait
  uint32_t max_iter;  // hard cap on polls, whatever the clock says
};

// Bounded phase wait.  Returns false (and raises *abort and the device status)
// when the limit expires, or false at once when another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          WaitLimit lim) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1; it < lim.max_iter; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > lim.ns) break;
  }
  *abort = 1;
  atomicExch(&g_device_status, 4);
  return false;
}

// Bounded wait for four phases (a barrier may be repeated): one joint test,
// then, only if some phase is not yet complete, the waits one by one.
__device__ __forceinline__ bool mbar_wait4(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1, uint64_t* b2,
                                           uint32_t p2, uint64_t* b3, uint32_t p3, volatile int* abort,
                                           WaitLimit lim) {
  if (mbar_test4(b0, p0, b1, p1, b2, p2, b3, p3)) return true;
  return mbar_wait(b0, p0, abort, lim) && mbar_wait(b1, p1, abort, lim) && mbar_wait(b2, p2, abort, lim) &&
         mbar_wait(b3, p3, abort, lim);
}

// --------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// 3-D tiled load (no multicast) completing on an mbarrier with a byte count.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// Prefetch one tile of a 3-D tensor map into L2 (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* map, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
// 3-D tiled store shared -> global (bulk-group completion).  Rows/columns past
// the tensor's extent are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1,
                                             int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until the shared-memory sources of every committed bulk store were read.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until every committed bulk store has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Named barrier over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Generic-proxy shared-memory writes -> visible to the async proxy (tensor core, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D(tmem) = A(smem) x B(smem) (+ D when accumulate != 0), kind::f16, 1 CTA.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem) = A(tmem) x B(smem) (+ D), A K-major packed two bf16 per 32-bit column.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every MMA issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> f32, M x N, operand majors.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                              // D format f32
         | (1u << 7)                            // A format bf16
         | (1u << 10)                           // B format bf16
         | ((a_mn_major ? 1u : 0u) << 15)       // A major (0 = K)
         | ((b_mn_major ? 1u : 0u) << 16)       // B major (0 = K)
         | ((uint32_t)(N >> 3) << 17)           // N / 8
         | ((uint32_t)(M >> 4) << 24);          // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bits.
//  K-major operand:  rows of the M/N dimension are 128-byte lines; 8-row groups
//                    `sbo` bytes apart; `lbo` unused (16).  A K step of 16
//                    elements inside a 64-element line advances the start by 32 B.
//  MN-major operand: 64 contiguous M/N elements per 128-byte line; consecutive
//                    64-element blocks `lbo` bytes apart; 8-row (K) groups `sbo`
//                    bytes apart.  A K step of 16 rows advances by 2 * sbo.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// TMEM -> registers: 32 lanes x 32 consecutive 32-bit columns; thread t of the
// warp gets lane (taddr.lane + t), r[i] = column (taddr.col + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  if (!RET_BC((taddr & 0xFFFFu) + 32u <= 512u && (taddr >> 16) + 32u <= 128u, 901)) return;
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// registers -> TMEM, 32 lanes x 16 columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  if (!RET_BC((taddr & 0xFFFFu) + 16u <= 512u && (taddr >> 16) + 32u <= 128u, 902)) return;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
// registers -> TMEM, 32 lanes x 32 columns.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  if (!RET_BC((taddr & 0xFFFFu) + 32u <= 512u && (taddr >> 16) + 32u <= 128u, 903)) return;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Pack two floats into a bf16x2 word (round to nearest even), lo in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Byte offset of 16-byte chunk `c` (0..7) of row `r` inside a 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(uint32_t r, uint32_t c) {
  return r * 128u + ((c ^ (r & 7u)) << 4);
}

}  // namespace ret
