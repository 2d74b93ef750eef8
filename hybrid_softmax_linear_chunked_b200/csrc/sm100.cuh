// sm_100a building blocks: mbarriers with bounded waits, TMA tile loads, tcgen05 MMA / TMEM
// access, and the shared-memory matrix descriptors used by the hybrid-attention kernels.
//
// Conventions used throughout the library:
//  * Every bf16 operand tile in shared memory is stored in the 128-byte-swizzled layout that a
//    TMA load with CU_TENSOR_MAP_SWIZZLE_128B produces for a box whose inner extent is 64 bf16
//    (128 B): row r of a [rows x 64] slab sits at byte r*128, and its 16-byte chunk j is stored at
//    chunk position j ^ (r % 8).  A 128-wide operand is two such slabs, 16 KiB apart (for 128
//    rows).  Slabs start on 1024-byte boundaries.
//  * K-major operand (contraction dim contiguous, e.g. Q and K rows over D): descriptor with
//    SBO = 1024 B (next group of 8 rows); the 16-element K step of one MMA moves the start
//    address by 32 B inside the 128-B row, and by a whole slab every 64 elements.
//  * MN-major operand (M or N dim contiguous, e.g. V rows over D as the B of P.V): LBO = slab
//    stride (next 64 elements of M/N), SBO = 1024 B (next 8 rows of K); one MMA K step of 16 rows
//    moves the start address by 16 * 128 B.
//  * Waits are bounded in time; on expiry a CTA-wide abort flag and the library's device error
//    word are set, and every later wait returns at once so the CTA can tear down.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace rehyat {
namespace sm100 {

// Device error word (one per library load; the library is built as one translation unit);
// non-zero after a wait gave up or a bounds check failed.  Values: 1 = an mbarrier wait timed
// out; 2 = a TMA coordinate or a global store index failed a bounds check of a debug-bounds
// build (compiled with REHYAT_DEBUG_BOUNDS), and the access was redirected or skipped.
// g_bounds_info holds the first failed check: {site, value, limit}.
__device__ int g_device_error = 0;
__device__ long long g_bounds_info[3];

// In debug-bounds builds: true when lo <= value < hi, else the failure is recorded (the first
// one's site, value and upper limit) and false is returned.  In other builds: true, no code.
__device__ __forceinline__ bool bounds_ok(int site, long long value, long long lo, long long hi) {
#ifdef REHYAT_DEBUG_BOUNDS
  if (value >= lo && value < hi) return true;
  if (atomicCAS(&g_device_error, 0, 2) == 0) {
    g_bounds_info[0] = site;
    g_bounds_info[1] = value;
    g_bounds_info[2] = hi;
  }
  return false;
#else
  (void)site, (void)value, (void)lo, (void)hi;
  return true;
#endif
}

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------------------------------
// mbarrier
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
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
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Returns false if the CTA is aborting
// (flag already set by another thread) or if this wait ran past the limit (then sets the flag
// and the device error word).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicExch(&g_device_error, 1);
      return false;
    }
  }
}

// Wait used on the teardown path after an abort: bounded, ignores the abort flag.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs / 4) return;
  }
}

// ------------------------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched after this one with programmatic stream
// serialization may start once every CTA of this grid has signalled (or exited); a kernel so
// launched waits for the full completion (and memory) of the grid before it with grid_dep_wait.
// Both are no-ops for ordinary launches.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void grid_dep_signal() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------------------------------
// TMA
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// tma_load_3d of a bf16 tensor map with extents (ext0 inner elements, ext1 rows, ext2 depth) and
// boxes of box1 rows; in debug-bounds builds its coordinates are checked first: the inner
// coordinate a multiple of 8 elements (16 bytes) inside the row, the first row no more than one
// box before the tensor and inside it (rows past either end read zeros, a start further out is
// a wrong index), the depth inside the tensor.  A failed check is recorded and the copy goes to
// (0, 0, 0) instead, so that its barrier still completes.
__device__ __forceinline__ void tma_load_3d_chk(int site, void* dst, const CUtensorMap* map,
                                                uint64_t* bar, int c0, int c1, int c2,
                                                long long ext0, long long ext1, long long ext2,
                                                int box1 = 128) {
#ifdef REHYAT_DEBUG_BOUNDS
  const bool ok = bounds_ok(site, c0 & 7, 0, 1) & bounds_ok(site, c0, 0, ext0) &
                  bounds_ok(site, c1, -box1, ext1) & bounds_ok(site, c2, 0, ext2);
  if (!ok) c0 = c1 = c2 = 0;
#else
  (void)site, (void)ext0, (void)ext1, (void)ext2, (void)box1;
#endif
  tma_load_3d(dst, map, bar, c0, c1, c2);
}

// TMA tile store of one 3-D box from shared memory (128B-swizzled like the loads) into the
// tensor; the parts of the box past the tensor's extents are not written.  Completion is tracked
// by this thread's bulk async-groups (bulk_commit_group, then bulk_wait_read_all /
// bulk_wait_all).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0,
                                             int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// tma_store_3d with, in debug-bounds builds, the inner coordinate a multiple of 8 elements inside
// the row and the row and depth coordinates inside the tensor (a store never starts before it);
// a failed check is recorded and the store skipped.
__device__ __forceinline__ void tma_store_3d_chk(int site, const CUtensorMap* map, const void* src,
                                                 int c0, int c1, int c2, long long ext0,
                                                 long long ext1, long long ext2) {
#ifdef REHYAT_DEBUG_BOUNDS
  const bool ok = bounds_ok(site, c0 & 7, 0, 1) & bounds_ok(site, c0, 0, ext0) &
                  bounds_ok(site, c1, 0, ext1) & bounds_ok(site, c2, 0, ext2);
  if (!ok) return;
#else
  (void)site, (void)ext0, (void)ext1, (void)ext2;
#endif
  tma_store_3d(map, src, c0, c1, c2);
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Every committed bulk group of this thread has finished reading its shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Every committed bulk group of this thread is complete.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Named barrier `id` (1..15; 0 is __syncthreads) for `count` threads, a multiple of 32.
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Make generic-proxy shared-memory writes visible to the async proxy (tensor core reads).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------------------------------
// tcgen05: TMEM allocation, MMA, commit, TMEM <-> registers
// ------------------------------------------------------------------------------------------
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

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T, A packed as bf16 pairs per 32-bit TMEM column.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05 op issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                  // D format: f32
         | (1u << 7)                                // A format: bf16
         | (1u << 10)                               // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15)           // A major
         | ((b_mn_major ? 1u : 0u) << 16)           // B major
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
  return d;
}

// Byte offset of element (row, col) of a 128B-swizzled bf16 tile built from 64-column slabs of
// `rows` rows each.
__host__ __device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t col,
                                                          uint32_t rows) {
  const uint32_t slab = col >> 6;
  const uint32_t c = col & 63u;
  const uint32_t chunk = (c >> 3) ^ (row & 7u);
  return slab * rows * 128u + row * 128u + chunk * 16u + (c & 7u) * 2u;
}

#define REHYAT_R32(r, b)                                                                   \
  "=r"(r[b + 0]), "=r"(r[b + 1]), "=r"(r[b + 2]), "=r"(r[b + 3]), "=r"(r[b + 4]),          \
      "=r"(r[b + 5]), "=r"(r[b + 6]), "=r"(r[b + 7]), "=r"(r[b + 8]), "=r"(r[b + 9]),      \
      "=r"(r[b + 10]), "=r"(r[b + 11]), "=r"(r[b + 12]), "=r"(r[b + 13]), "=r"(r[b + 14]), \
      "=r"(r[b + 15]), "=r"(r[b + 16]), "=r"(r[b + 17]), "=r"(r[b + 18]), "=r"(r[b + 19]), \
      "=r"(r[b + 20]), "=r"(r[b + 21]), "=r"(r[b + 22]), "=r"(r[b + 23]), "=r"(r[b + 24]), \
      "=r"(r[b + 25]), "=r"(r[b + 26]), "=r"(r[b + 27]), "=r"(r[b + 28]), "=r"(r[b + 29]), \
      "=r"(r[b + 30]), "=r"(r[b + 31])
#define REHYAT_W32(r, b)                                                                     \
  "r"(r[b + 0]), "r"(r[b + 1]), "r"(r[b + 2]), "r"(r[b + 3]), "r"(r[b + 4]), "r"(r[b + 5]), \
      "r"(r[b + 6]), "r"(r[b + 7]), "r"(r[b + 8]), "r"(r[b + 9]), "r"(r[b + 10]),           \
      "r"(r[b + 11]), "r"(r[b + 12]), "r"(r[b + 13]), "r"(r[b + 14]), "r"(r[b + 15]),       \
      "r"(r[b + 16]), "r"(r[b + 17]), "r"(r[b + 18]), "r"(r[b + 19]), "r"(r[b + 20]),       \
      "r"(r[b + 21]), "r"(r[b + 22]), "r"(r[b + 23]), "r"(r[b + 24]), "r"(r[b + 25]),       \
      "r"(r[b + 26]), "r"(r[b + 27]), "r"(r[b + 28]), "r"(r[b + 29]), "r"(r[b + 30]),       \
      "r"(r[b + 31])

// Load 32 consecutive 32-bit TMEM columns of this thread's lane (warp w reads lanes
// 32*(w%4) .. +31; `taddr` carries that lane base in bits 31..16) and wait for them.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : REHYAT_R32(r, 0)
      : "r"(taddr)
      : "memory");
}
// Load 128 consecutive 32-bit columns of this thread's lane with four loads and one wait.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%128];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, "
      "%41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, "
      "%58, %59, %60, %61, %62, %63}, [%129];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%64, %65, %66, %67, %68, %69, %70, %71, %72, "
      "%73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, "
      "%90, %91, %92, %93, %94, %95}, [%130];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%96, %97, %98, %99, %100, %101, %102, %103, "
      "%104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, "
      "%118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%131];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : REHYAT_R32(r, 0), REHYAT_R32(r, 32), REHYAT_R32(r, 64), REHYAT_R32(r, 96)
      : "r"(taddr), "r"(taddr + 32), "r"(taddr + 64), "r"(taddr + 96)
      : "memory");
}
// Load 64 consecutive 32-bit columns of this thread's lane with two loads and one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, "
      "%41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, "
      "%58, %59, %60, %61, %62, %63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : REHYAT_R32(r, 0), REHYAT_R32(r, 32)
      : "r"(taddr), "r"(taddr + 32)
      : "memory");
}
// Load 16 consecutive columns and wait.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
// Store 32 consecutive columns of this thread's lane (no wait).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      REHYAT_W32(r, 0)
      : "memory");
}
// Store 16 consecutive columns of this thread's lane (no wait).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// Store 8 consecutive columns of this thread's lane (no wait).
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 2^x on the MUFU (approximate, subnormal results flushed to zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Paired fp32 arithmetic: one instruction for the two floats of a 64-bit register pair.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low 16 bits), .y = hi
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace sm100
}  // namespace rehyat
