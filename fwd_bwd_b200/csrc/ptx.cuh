// ptx.cuh -- hand-written PTX wrappers for sm_100a: mbarriers with bounded waits, TMA tile
// loads, tcgen05 (TMEM allocation, MMA, loads/stores, commits, fences) and the shared-memory
// and instruction descriptors the 5th-generation tensor cores read.
//
// Every wait here is bounded in time: when a barrier does not complete within the limit the
// thread records SAGE_ERR_TIMEOUT in the device status word and returns, so a broken pipeline
// ends with an error instead of hanging the GPU.  Once the status word is set, later waits use
// a 1 ms limit so the whole grid drains quickly.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sage {

// Device status word (one per device): SAGE_OK or the first error a kernel recorded.
__device__ int g_status;
// Identifier of the wait site that timed out first (for diagnosis).
__device__ int g_status_site;

constexpr int kStatusTimeout = -6;  // SAGE_ERR_TIMEOUT

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool device_aborted() {
  return *reinterpret_cast<volatile int*>(&g_status) != 0;
}

__device__ __forceinline__ void record_timeout(int site) {
  if (atomicCAS(&g_status, 0, kStatusTimeout) == 0) g_status_site = site;
}

// ---------------------------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// Makes barrier initialisation visible to the async proxy (TMA, tensor cores).
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
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

// Waits until the phase with the given parity has completed, for at most limit_ns
// nanoseconds; on timeout records SAGE_ERR_TIMEOUT (with `site`) and returns false.  Fully
// inlined: kernels that move registers between warpgroups (setmaxnreg) must not make calls.
__device__ __forceinline__ bool mbar_wait_ns(uint64_t* bar, uint32_t parity, int site,
                                             uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) {
      record_timeout(site);
      return false;
    }
  }
}

// The kernels' wait: 2 s, or 1 ms once any wait on the device has failed (so the whole grid
// drains quickly).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int site) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_ns(bar, parity, site, device_aborted() ? 1000000ull : 2000000000ull);
}

// Named barrier among `nthreads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------------------------
// TMA (no multicast anywhere in this library)
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled load of the box at (x = innermost element index, y = row) into shared memory,
// completing `bar`'s transaction count.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Contiguous global -> shared copy of `bytes` (a multiple of 16; both addresses 16-byte
// aligned), completing `bar`'s transaction count.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Asynchronous element-wise add of a shared-memory box into global memory (the TMA unit
// performs the reduction; float32 add for a float32 tensor map).  Tracked by bulk groups.
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int x,
                                                  int y) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%1, %2}], [%3];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(smem_u32(src))
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// At most one committed bulk group may still be reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// No committed bulk group is still reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_read_0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Every committed bulk group has completed (including its global writes).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Generic-proxy shared-memory writes -> visible to the async proxy (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------------------------
// tcgen05: tensor memory
// ---------------------------------------------------------------------------------------------
// Warp-collective.  Writes the allocated TMEM base address to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
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

// D[tmem] (+)= A[smem] * B[smem]; INT8 x INT8 -> INT32.  Issued by one thread.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]; FP16/BF16 -> FP32.  Issued by one thread.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05.mma previously issued by this thread has completed.
// D[tmem] (+)= (A * SFA)[smem] * (B * SFB)[smem]: NVFP4 operands (packed E2M1, two per byte,
// K = 64 per instruction) with one unsigned E4M3 scale per 16 elements along K; FP32
// accumulator.  sfa / sfb are the TMEM addresses of the scale factors (see tmem_cp_sf).
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], "
      "[%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Copy 32 rows x 16 bytes of shared memory (described by a no-swizzle K-major descriptor) into
// TMEM columns [taddr, taddr + 4) of all four 32-lane sub-partitions.  Ordered with later
// tcgen05.mma of the same thread.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its own TMEM lane.
// The warp may only address its lane quarter: lanes 32*(warp_id % 4) .. +31.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// One 32-column load (32x32b.x32) into two 16-register arrays: columns [0, 16) -> a,
// [16, 32) -> b.  A tcgen05.ld costs its warp's sub-partition about the same time whatever its
// width (measured on B200: ~200 B/clk per SM with .x16, ~420 B/clk with .x32), so the kernels
// load the widest chunks their registers allow.
__device__ __forceinline__ void tmem_ld32x(uint32_t taddr, uint32_t (&a)[16], uint32_t (&b)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
        "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]),
        "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]),
        "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15])
      : "r"(taddr));
}

// One 64-column load (32x32b.x64) into four 16-register arrays, in column order.
__device__ __forceinline__ void tmem_ld64x(uint32_t taddr, uint32_t (&a)[16], uint32_t (&b)[16],
                                           uint32_t (&c)[16], uint32_t (&d)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
        "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]),
        "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]),
        "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15]),
        "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3]), "=r"(c[4]), "=r"(c[5]), "=r"(c[6]), "=r"(c[7]),
        "=r"(c[8]), "=r"(c[9]), "=r"(c[10]), "=r"(c[11]), "=r"(c[12]), "=r"(c[13]), "=r"(c[14]), "=r"(c[15]),
        "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]), "=r"(d[7]),
        "=r"(d[8]), "=r"(d[9]), "=r"(d[10]), "=r"(d[11]), "=r"(d[12]), "=r"(d[13]), "=r"(d[14]), "=r"(d[15])
      : "r"(taddr));
}

// tcgen05.wait::ld that also ties four 16-register arrays (see tmem_ld_wait_regs).
__device__ __forceinline__ void tmem_ld_wait_regs4(uint32_t (&a)[16], uint32_t (&b)[16],
                                                   uint32_t (&c)[16], uint32_t (&d)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]),
                 "+r"(a[6]), "+r"(a[7]), "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]),
                 "+r"(a[12]), "+r"(a[13]), "+r"(a[14]), "+r"(a[15])
               :
               : "memory");
  asm volatile(""
               : "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]),
                 "+r"(b[6]), "+r"(b[7]), "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]),
                 "+r"(b[12]), "+r"(b[13]), "+r"(b[14]), "+r"(b[15])
               :
               : "memory");
  asm volatile(""
               : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3]), "+r"(c[4]), "+r"(c[5]),
                 "+r"(c[6]), "+r"(c[7]), "+r"(c[8]), "+r"(c[9]), "+r"(c[10]), "+r"(c[11]),
                 "+r"(c[12]), "+r"(c[13]), "+r"(c[14]), "+r"(c[15])
               :
               : "memory");
  asm volatile(""
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3]), "+r"(d[4]), "+r"(d[5]),
                 "+r"(d[6]), "+r"(d[7]), "+r"(d[8]), "+r"(d[9]), "+r"(d[10]), "+r"(d[11]),
                 "+r"(d[12]), "+r"(d[13]), "+r"(d[14]), "+r"(d[15])
               :
               : "memory");
}

// 8-column variant of tmem_ld16.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// tcgen05.wait::ld tying two 8-register arrays (see tmem_ld_wait_regs).
__device__ __forceinline__ void tmem_ld_wait_regs8(uint32_t (&a)[8], uint32_t (&b)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]),
                 "+r"(a[6]), "+r"(a[7]), "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]),
                 "+r"(b[4]), "+r"(b[5]), "+r"(b[6]), "+r"(b[7])
               :
               : "memory");
}

// Fills 16 consecutive 32-bit columns of the thread's TMEM lane with the same word.
__device__ __forceinline__ void tmem_fill16(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, "
      "%1, %1, %1, %1, %1, %1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}

// tcgen05.wait::ld that also ties the loaded registers: uses of a[] and b[] cannot be moved
// above the wait by the compiler.
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t (&a)[16], uint32_t (&b)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]),
                 "+r"(a[6]), "+r"(a[7]), "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]),
                 "+r"(a[12]), "+r"(a[13]), "+r"(a[14]), "+r"(a[15])
               :
               : "memory");
  asm volatile(""
               : "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]),
                 "+r"(b[6]), "+r"(b[7]), "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]),
                 "+r"(b[12]), "+r"(b[13]), "+r"(b[14]), "+r"(b[15])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------------------------
// Descriptors
// ---------------------------------------------------------------------------------------------
// Shared-memory swizzle modes as encoded in the matrix descriptor.
enum : uint32_t { kSwizzleNone = 0, kSwizzle128B = 2, kSwizzle64B = 4, kSwizzle32B = 6 };

// Shared-memory matrix descriptor: start address, leading / stride byte offsets (16-byte
// units), descriptor version 1, base offset 0 (tiles are aligned to the swizzle repeat),
// swizzle mode in bits 61..63.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes, uint32_t swizzle) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(swizzle) << 61;
  return d;
}

// Instruction descriptor of a dense tcgen05.mma (kind::i8 or kind::f16).
//   c_fmt: 1 = F32, 2 = S32 accumulator; a_fmt/b_fmt: kind::f16 0 = F16, 1 = BF16;
//   kind::i8 0 = U8, 1 = S8.  a_mn / b_mn: operand stored MN-major (transposed).
__host__ __device__ constexpr uint32_t instr_desc(uint32_t c_fmt, uint32_t a_fmt,
                                                  uint32_t b_fmt, bool a_mn, bool b_mn,
                                                  int M, int N) {
  return (c_fmt << 4) | (a_fmt << 7) | (b_fmt << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor of a block-scaled tcgen05.mma of kind::mxf4nvf4 with E2M1 A and B
// (format code 1), both K-major, unsigned E4M3 scales (bit 23 = 0), scale-factor IDs 0 and a
// dense K of 64.
__host__ __device__ constexpr uint32_t instr_desc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Byte offset of the 16-byte chunk `chunk` of row `row` inside a swizzled tile whose rows are
// `row_bytes` (64 or 128) long: the hardware XORs the chunk index with the row's position in
// the swizzle repeat (8 rows of 128 B, or 8 rows of 64 B in pairs).
__device__ __forceinline__ uint32_t swz_offset(uint32_t row, uint32_t chunk,
                                               uint32_t row_bytes) {
  if (row_bytes == 128) return row * 128u + ((chunk ^ (row & 7u)) << 4);
  return row * 64u + ((chunk ^ ((row >> 1) & 3u)) << 4);
}

// ---------------------------------------------------------------------------------------------
// Small numeric helpers
// ---------------------------------------------------------------------------------------------
// INT32 accumulators are preloaded with kMagicBits (the float 1.5 * 2^23) before the MMAs add
// into them, so a result a (|a| < 2^22) reads back as the bit pattern of the float
// 1.5 * 2^23 + a, with no integer instruction.
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr float kMagic = 12582912.0f;

// ---------------------------------------------------------------------------------------------
// Preloading accumulators with the tensor core
// ---------------------------------------------------------------------------------------------
// A kind::f16 MMA with accumulate = 0 can write the preload value itself, so the compute warps
// never store it into TMEM: with A[i][k] = 1 and B[j][k] = 1.5 * 2^22 (both exact in bf16) at
// k = 0 and k = 8 and zero elsewhere, D[i][j] = 2 * 1.5 * 2^22 = 1.5 * 2^23 exactly, whose float32
// bits are kMagicBits.  Every 16-byte chunk of the operand tiles holds the same 8 elements
// (element 0 set, 7 zeros), so each tile row reads k = 0 and k = 8 as set whatever the layout's
// row and chunk order: only the tiles' extent matters.
constexpr uint32_t kFillA = 0x00003F80u;  // bf16 1.0 in the chunk's first element
constexpr uint32_t kFillB = 0x00004AC0u;  // bf16 6291456.0 = 1.5 * 2^22
constexpr int kFillRowsA = 128;           // M rows of A
constexpr int kFillRowsB = 256;           // up to N = 256 rows of B
constexpr int kFillBytes = (kFillRowsA + kFillRowsB) * 32;

// Writes the fill operands (A then B, rows of 32 bytes) into `dst` (256-byte aligned); every
// thread of the calling group takes its share; the caller fences to the async proxy.
__device__ __forceinline__ void write_fill_operands(uint8_t* dst, int tid, int nthreads) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  for (int i = tid; i < kFillBytes / 16; i += nthreads)
    d4[i] = make_uint4(i < kFillRowsA * 2 ? kFillA : kFillB, 0u, 0u, 0u);
}

// D[tmem, columns 0 .. n) = 1.5 * 2^23 (bits kMagicBits) for all 128 lanes; n in {16 .. 256}, a
// multiple of 16.  `fill` is the operand tile pair written by write_fill_operands.  Issued by the
// MMA thread, in order with its other MMAs.
__device__ __forceinline__ void mma_fill_magic(uint32_t d_tmem, const uint8_t* fill, int n) {
  const uint32_t a = smem_u32(fill), b = a + kFillRowsA * 32;
  const uint32_t id = instr_desc(1, 1, 1, false, false, 128, n);  // F32 <- BF16 x BF16
  mma_f16(d_tmem, smem_desc(a, 16, 256, kSwizzle32B), smem_desc(b, 16, 256, kSwizzle32B), id, 0u);
}

// s rounded toward zero to 22 significant bits: kMagic * scale22(s) is then exact in float32.
__device__ __forceinline__ float scale22(float s) {
  return __uint_as_float(__float_as_uint(s) & 0xFFFFFFFCu);
}

// Exact fl(a * s22) from the bits of the float kMagic + a, given s22 = scale22(s) and
// neg_ms = -kMagic * s22: the fused multiply-add forms (kMagic + a) * s22 - kMagic * s22 =
// a * s22 without intermediate rounding and rounds once.
__device__ __forceinline__ float deq(uint32_t magic_plus_a, float s22, float neg_ms) {
  return __fmaf_rn(__uint_as_float(magic_plus_a), s22, neg_ms);
}

// Four codes (each the low byte of a float x + 1.5*2^23) packed into one word, byte 0 first.
__device__ __forceinline__ uint32_t pack_magic4(float a, float b, float c, float d) {
  const uint32_t lo = __byte_perm(__float_as_uint(a), __float_as_uint(b), 0x0040);
  const uint32_t hi = __byte_perm(__float_as_uint(c), __float_as_uint(d), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^z for a pair, on the FMA pipe instead of the special-function unit (the kernels route a
// share of their exponentials here so that both units work).  z = j + f with j = rint(z) (the
// 1.5 * 2^23 rounding trick) and f in [-1/2, 1/2] exact; p(f) ~ 2^f is the degree-5 polynomial
// of minimax relative error (Remez exchange, coefficients from fwd_bwd_b200/exp2_fit.py),
// evaluated by packed FMAs; j is added to the exponent field.  Maximum relative error
// 2.2e-7 (float32 evaluation included).  z < -125 gives 0, as the flushing ex2.approx does
// below -126; z must stay below 128.
__device__ __forceinline__ float2 exp2_poly2(float2 z) {
  constexpr float kC0 = 1.0000001192092896f, kC1 = 0.6931469440460205f,
                  kC2 = 0.24022120237350464f, kC3 = 0.05550713092088699f,
                  kC4 = 0.009675540961325169f, kC5 = 0.0013276472454890609f;
  const float2 lo = make_float2(-125.0f, -125.0f);
  const float2 zc = make_float2(fmaxf(z.x, lo.x), fmaxf(z.y, lo.y));
  const float2 t = __fadd2_rn(zc, make_float2(kMagic, kMagic));       // rint(z) + 1.5 * 2^23
  const float2 j = __fadd2_rn(t, make_float2(-kMagic, -kMagic));      // rint(z), exact
  const float2 f = __ffma2_rn(j, make_float2(-1.0f, -1.0f), zc);      // z - rint(z), exact
  float2 q = __ffma2_rn(make_float2(kC5, kC5), f, make_float2(kC4, kC4));
  q = __ffma2_rn(q, f, make_float2(kC3, kC3));
  q = __ffma2_rn(q, f, make_float2(kC2, kC2));
  q = __ffma2_rn(q, f, make_float2(kC1, kC1));
  q = __ffma2_rn(q, f, make_float2(kC0, kC0));
  const int jx = static_cast<int>(__float_as_uint(t.x) - kMagicBits);
  const int jy = static_cast<int>(__float_as_uint(t.y) - kMagicBits);
  const float rx = __int_as_float(__float_as_int(q.x) + (jx << 23));
  const float ry = __int_as_float(__float_as_int(q.y) + (jy << 23));
  return make_float2(z.x < lo.x ? 0.0f : rx, z.y < lo.y ? 0.0f : ry);
}

}  // namespace sage
