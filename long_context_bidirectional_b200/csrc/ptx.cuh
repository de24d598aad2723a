// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA tile loads and the
// tcgen05 family (TMEM allocation, MMA issue, commit, TMEM loads/stores).
// Every wait in this file is bounded: it gives up after a wall-clock limit,
// records an error in the library's device status word and reports failure
// so that the calling role can unwind without hanging the GPU.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

#include "debug_checks.h"

namespace b2a {

// Status bits OR-ed into the device status word by kernels.
enum : uint32_t {
  kDevErrTimeout = 1u,      // a bounded mbarrier wait ran out
  kDevErrBounds = 2u,       // a debug-build bounds check failed (the access was skipped)
};

// The library's device status word (one per device, static device memory):
// set by kernels, read and cleared by b2a_check_status().  Defined here
// because the whole library is one translation unit (b200attn.cu includes
// every kernel header), so device code anywhere in it can name the word.
__device__ unsigned int g_status_word;

#ifdef B2A_DEBUG
constexpr bool kDebugBuild = true;
#else
constexpr bool kDebugBuild = false;
#endif

// Debug builds: a failed check sets kDevErrBounds and returns false, and the
// caller skips the access.  Release builds: always true, the check compiles
// away.
__device__ __forceinline__ bool dbg_check(bool ok) {
  if constexpr (kDebugBuild) {
    if (!ok) {
      atomicOr(&g_status_word, kDevErrBounds);
      return false;
    }
  }
  return true;
}
#define B2A_DBG(cond) (!::b2a::kDebugBuild || ::b2a::dbg_check(cond))

__device__ __forceinline__ int warp_quarter() { return static_cast<int>((threadIdx.x >> 5) & 3u); }

__device__ __forceinline__ uint32_t dyn_smem_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
  return r;
}

// Wall-clock limit of one bounded wait.  A healthy wait in these kernels is
// microseconds; two seconds means a lost arrival.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t lane_id() {
  uint32_t l;
  asm volatile("mov.u32 %0, %%laneid;" : "=r"(l));
  return l;
}

// ------------------------------------------------------------- mbarrier ----

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but the thread may sleep up to ``hint_ns`` for the phase.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Slow path of mbar_wait: sleep in try_wait, give up after kWaitLimitNs, on
// this CTA's abort flag, or when another CTA has set the status word.
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            unsigned int* status, uint64_t limit_ns = kWaitLimitNs) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    // sleeps until the phase completes or ~0.1 ms pass
    if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
    if (*abort_flag) return false;
    // Another CTA that gave up releases this one too (the status word is
    // sticky until the host reads it).
    if (*reinterpret_cast<volatile unsigned int*>(status) != 0u) {
      *abort_flag = 1;
      return false;
    }
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(status, kDevErrTimeout);
      return false;
    }
  }
}

// Bounded wait for the phase of ``bar`` with parity ``parity`` to complete.
// ``abort_flag`` (shared memory) lets one role that gave up release the
// others quickly.  Returns false on timeout or abort.  The fast path is a
// single try_wait: an MMA issuer calls this between tensor-core groups, and
// the tensor pipe only has about one instruction of work queued to hide it.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, abort_flag, status);
}

// Wait ignoring the abort flag, used only to drain in-flight async work.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return;
  }
}

// Warp-uniform variant: lane 0 polls, the verdict is broadcast, so that the
// warp-collective tcgen05 instructions after it see one decision.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity,
                                               volatile int* abort_flag, unsigned int* status) {
  int ok = 0;
  if (lane_id() == 0) ok = mbar_wait(bar, parity, abort_flag, status) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Non-blocking phase test with cluster-scope acquire: the thread is never
// suspended, so an arrival from the other CTA of a pair is seen as soon as
// it lands.
__device__ __forceinline__ bool mbar_test_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __noinline__ bool mbar_spin_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            unsigned int* status) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_test_wait_cluster(bar, parity)) return true;
    if ((i & 127u) != 0u) continue;
    if (*abort_flag) return false;
    if (*reinterpret_cast<volatile unsigned int*>(status) != 0u) {
      *abort_flag = 1;
      return false;
    }
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(status, kDevErrTimeout);
      return false;
    }
  }
}

// Bounded busy-wait, for barriers that another CTA of the cluster arrives on
// (a suspended try_wait is woken late by such arrivals).
__device__ __forceinline__ bool mbar_spin(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned int* status) {
  if (mbar_test_wait_cluster(bar, parity)) return true;
  return mbar_spin_slow(bar, parity, abort_flag, status);
}

// ------------------------------------------------------------------ TMA ----

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// Prefetch one tensor tile into L2 (no shared-memory destination, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* map, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// -------------------------------------------------------------- tcgen05 ----

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
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

// Arrive once on ``bar`` when every tcgen05 op issued so far by this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]; kind::f16, fp32 accumulate.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  if (!B2A_DBG(tmem_operand_ok(d_tmem, idesc_n(idesc)))) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]; A is K-major fp16 packed two per column.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  if (!B2A_DBG(tmem_operand_ok(d_tmem, idesc_n(idesc)) && tmem_operand_ok(a_tmem, 8))) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
// K-major operands: lbo = 16 (unused), sbo = 1024 (8 rows of 128 B).
// MN-major operands: lbo = byte stride between 64-element MN atoms,
//                    sbo = byte stride between 8-row K groups.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes,
                                               uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;  // descriptor version for sm_100
  d |= static_cast<uint64_t>(2u) << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor for kind::f16 with fp16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn_major,
                                                     bool b_mn_major) {
  return (1u << 4)                                  // D format: f32
         | (0u << 7) | (0u << 10)                   // A, B format: f16
         | (static_cast<uint32_t>(a_mn_major) << 15)
         | (static_cast<uint32_t>(b_mn_major) << 16)
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---- TMEM <-> registers, 32 lanes x 32-bit shape: thread i of the warp
// ---- owns TMEM lane (32*(warp%4) + i); .xN moves N consecutive columns.

#define B2A_R8(b) "=r"(r[b + 0]), "=r"(r[b + 1]), "=r"(r[b + 2]), "=r"(r[b + 3]), \
                  "=r"(r[b + 4]), "=r"(r[b + 5]), "=r"(r[b + 6]), "=r"(r[b + 7])
#define B2A_W8(b) "r"(r[b + 0]), "r"(r[b + 1]), "r"(r[b + 2]), "r"(r[b + 3]), \
                  "r"(r[b + 4]), "r"(r[b + 5]), "r"(r[b + 6]), "r"(r[b + 7])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  if (!B2A_DBG(tmem_ldst_ok(taddr, 32, warp_quarter()))) {
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = 0u;
    return;
  }
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : B2A_R8(0), B2A_R8(8), B2A_R8(16), B2A_R8(24)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  if (!B2A_DBG(tmem_ldst_ok(taddr, 32, warp_quarter()))) return;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      B2A_W8(0), B2A_W8(8), B2A_W8(16), B2A_W8(24)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  if (!B2A_DBG(tmem_ldst_ok(taddr, 16, warp_quarter()))) return;
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      B2A_W8(0), B2A_W8(8)
      : "memory");
}

#undef B2A_R8
#undef B2A_W8

// Wait for this thread's outstanding tcgen05.ld, then pin the loaded
// registers after the wait so no use of them is scheduled above it.
template <int N>
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[N]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------ 2-CTA (cluster pair) ----
// A cluster of two CTAs on two SMs runs each tensor-core MMA as one
// M = 256 operation: CTA rank 0 (the leader) issues it; each CTA supplies
// its 128 rows of A and half of B from its own shared memory / TMEM and
// holds its 128 rows of D in its own TMEM.

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Shared::cluster address of the same variable in CTA ``rank`` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Store to a shared::cluster address (possibly in the other CTA).
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// Arrive on an mbarrier that may live in the other CTA of the cluster.
// Relaxed: a cluster-scope release costs about a microsecond per arrival on
// B200; callers order their own prior work (e.g. tcgen05.wait::st) first.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  if (!B2A_DBG(tmem_operand_ok(d_tmem, idesc_n(idesc)))) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  if (!B2A_DBG(tmem_operand_ok(d_tmem, idesc_n(idesc)) && tmem_operand_ok(a_tmem, 8))) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at offset ``bar`` in both CTAs of the pair when
// every tcgen05 op issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  const uint16_t both = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(both)
      : "memory");
}

// Tile load into this CTA's shared memory whose completed bytes are counted
// on an mbarrier of the pair's leader CTA (``leader_bar``: shared::cluster).
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t leader_bar,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(leader_bar)
      : "memory");
}

// 2-D form of tma_load_3d_pair.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t leader_bar,
                                                 int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(leader_bar)
      : "memory");
}

// ----------------------------------------------- checked TMA tile loads ----
// The loads above with the debug build's checks: the box start (x, y, z)
// against the map's innermost extent nx (fp16 elements), y against ny and z
// against the end nz of the rows the launch covers; the destination's
// ``bytes`` against the CTA's dynamic shared memory starting at
// ``smem_base``.  A failed check skips the copy (its barrier then never
// completes, and the waits give up at once on the set status word).

__device__ __forceinline__ bool tma_box_checked(uint32_t dst, uint32_t bytes, uint32_t smem_base, int x, int nx,
                                                int y, int ny, int z, int nz) {
  return B2A_DBG(tma_coords_ok(x, 2, nx, y, ny, z, nz) && smem_box_ok(dst, bytes, smem_base, dyn_smem_size()));
}

__device__ __forceinline__ void tma_load_3d_chk(uint32_t dst, uint32_t bytes, uint32_t smem_base,
                                                const CUtensorMap* map, uint32_t bar, int x, int y, int z, int nx,
                                                int ny, int nz) {
  if (tma_box_checked(dst, bytes, smem_base, x, nx, y, ny, z, nz)) tma_load_3d(dst, map, bar, x, y, z);
}

__device__ __forceinline__ void tma_load_3d_pair_chk(uint32_t dst, uint32_t bytes, uint32_t smem_base,
                                                     const CUtensorMap* map, uint32_t leader_bar, int x, int y,
                                                     int z, int nx, int ny, int nz) {
  if (tma_box_checked(dst, bytes, smem_base, x, nx, y, ny, z, nz)) tma_load_3d_pair(dst, map, leader_bar, x, y, z);
}

__device__ __forceinline__ void tma_load_2d_pair_chk(uint32_t dst, uint32_t bytes, uint32_t smem_base,
                                                     const CUtensorMap* map, uint32_t leader_bar, int x, int z,
                                                     int nx, int nz) {
  if (tma_box_checked(dst, bytes, smem_base, x, nx, 0, 1, z, nz)) tma_load_2d_pair(dst, map, leader_bar, x, z);
}

// ------------------------------------------------------------ arithmetic ----

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 -> one packed f16x2 word, ``lo`` in the low half (round to nearest).
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace b2a
