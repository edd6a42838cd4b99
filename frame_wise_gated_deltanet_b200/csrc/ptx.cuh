// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA tile loads, tcgen05 (TMEM
// allocation, MMA, commit, loads) and the shared-memory matrix descriptors the MMA reads.
//
// Every wait here is bounded: a wait that does not complete within g_wait_limit_ns of
// %globaltimer returns false, and the caller records GDN_ERR_TIMEOUT in the device status
// word and unwinds instead of spinning forever.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

namespace gdn {

// Limit of every bounded wait, in ns of %globaltimer (4 s unless the host lowers it).
__device__ unsigned long long g_wait_limit_ns = 4000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31; }

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
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

// Wait until the phase with the given parity has completed. Returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if (globaltimer_ns() - t0 > g_wait_limit_ns) return false;
  }
}

// ------------------------------------------------------------------ cross-CTA flags (global)
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// A plain (relaxed) store at GPU scope: visible to other CTAs, ordered with nothing.
__device__ __forceinline__ void st_relaxed(int* p, int v) {
  asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Shared-memory counter with release/acquire at CTA scope.
__device__ __forceinline__ void red_add_release_cta(uint32_t* p, uint32_t v) {
  asm volatile("red.release.cta.shared::cta.add.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v)
               : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_cta(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}

// Orders this thread's generic-proxy global accesses with its async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Wait until *p >= target (acquire). Gives up, returning false, after g_wait_limit_ns or as soon
// as *abort is non-zero (another CTA gave up first).
__device__ __forceinline__ bool wait_flag_ge(const int* p, int target, const int* abort) {
  if (ld_acquire(p) >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (ld_acquire(p) >= target) return true;
    if (ld_acquire(abort) != 0) return false;
    if (globaltimer_ns() - t0 > g_wait_limit_ns) return false;
    __nanosleep(64);
  }
}

// Last phase of each pipeline stage a producer thread filled, so that on any exit path it can
// wait (bounded) for its own in-flight copies to land before the CTA releases its resources.
template <int N>
struct StageFills {
  uint32_t last[N];
  __device__ __forceinline__ StageFills() {
#pragma unroll
    for (int i = 0; i < N; ++i) last[i] = 0xFFFFFFFFu;
  }
  __device__ __forceinline__ void filled(int s, uint32_t phase) { last[s] = phase; }
  __device__ __forceinline__ void drain(uint64_t* full) {
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (last[i] != 0xFFFFFFFFu) mbar_wait(&full[i], last[i]);
  }
};

// ------------------------------------------------------------------ debug checks
// The debug library (libgdn_debug.so, compiled with -DGDN_DEBUG) checks every TMA, bulk and
// cp.async copy and every MMA operand address before it is issued: shared-memory ranges inside
// the CTA's allocation, the 16-byte alignments and sizes the copies require, TMA coordinates
// (innermost coordinate a multiple of 16 bytes' worth of elements, no negative store
// coordinate). A violation records its site and the offending value in g_debug_site /
// g_debug_value (first one wins; read and cleared by gdn_debug_report) and the copy is skipped,
// so the call ends on a bounded wait and an error status rather than on a memory fault. Release
// builds compile the checks out.
__device__ int g_debug_site;
__device__ long long g_debug_value;

enum DebugSite : int {
  kSiteTmaLoadSmem = 1,   // TMA load destination outside shared memory or not 128-B aligned
  kSiteTmaLoadCoord = 2,  // TMA load innermost coordinate not a multiple of 16
  kSiteTmaStoreSmem = 3,  // TMA store source outside shared memory or not 128-B aligned
  kSiteTmaStoreCoord = 4, // TMA store coordinate negative or innermost not a multiple of 16
  kSiteBulkSmem = 5,      // bulk copy shared range outside the allocation or misaligned
  kSiteBulkGlobal = 6,    // bulk copy global address or size not a multiple of 16
  kSiteCpAsync = 7,       // cp.async addresses misaligned or shared address out of range
  kSiteDescriptor = 8,    // MMA operand start address outside shared memory
};

#ifdef GDN_DEBUG
// The dynamic shared memory of the running kernel (every kernel here keeps all of its shared
// data there: its extern array starts at the same address as this one).
extern __shared__ uint8_t gdn_dyn_smem[];

__device__ __forceinline__ bool smem_range_ok(uint32_t saddr, uint32_t bytes) {
  uint32_t dyn;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(gdn_dyn_smem));
  return saddr >= base && saddr + bytes <= base + dyn;
}

// false (and the violation recorded) unless `ok`
__device__ __forceinline__ bool debug_check(bool ok, int site, long long value) {
  if (ok) return true;
  if (atomicCAS(&g_debug_site, 0, site) == 0) atomicExch(reinterpret_cast<unsigned long long*>(
                                                             &g_debug_value),
                                                         static_cast<unsigned long long>(value));
  return false;
}
#define GDN_DEBUG_CHECK(cond, site, value) \
  if (!::gdn::debug_check((cond), (site), static_cast<long long>(value))) return
#else
#define GDN_DEBUG_CHECK(cond, site, value) \
  do {                                     \
  } while (0)
#endif

// ------------------------------------------------------------------ TMA (no multicast)
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int c0,
                                            int c1, int c2, uint64_t policy) {
  GDN_DEBUG_CHECK((smem_u32(dst) & 127) == 0 && smem_range_ok(smem_u32(dst), 1), kSiteTmaLoadSmem,
                  smem_u32(dst));
  GDN_DEBUG_CHECK((c0 & 15) == 0, kSiteTmaLoadCoord, c0);
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::"
      "cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)),
      "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const void* tmap, uint64_t* bar, int c0,
                                            int c1, int c2, int c3, uint64_t policy) {
  GDN_DEBUG_CHECK((smem_u32(dst) & 127) == 0 && smem_range_ok(smem_u32(dst), 1), kSiteTmaLoadSmem,
                  smem_u32(dst));
  GDN_DEBUG_CHECK((c0 & 15) == 0, kSiteTmaLoadCoord, c0);
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::"
      "cache_hint [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// TMA tile store smem -> global (bulk-group completion), with an L2 cache policy.
__device__ __forceinline__ void tma_store_4d(const void* tmap, const void* src, int c0, int c1,
                                             int c2, int c3, uint64_t policy) {
  GDN_DEBUG_CHECK((smem_u32(src) & 127) == 0 && smem_range_ok(smem_u32(src), 1),
                  kSiteTmaStoreSmem, smem_u32(src));
  GDN_DEBUG_CHECK((c0 & 15) == 0 && (c0 | c1 | c2 | c3) >= 0, kSiteTmaStoreCoord,
                  (static_cast<long long>(c2) << 32) | static_cast<uint32_t>(c0));
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group.L2::cache_hint"
      " [%0, {%2, %3, %4, %5}], [%1], %6;" ::"l"(reinterpret_cast<uint64_t>(tmap)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_store_3d(const void* tmap, const void* src, int c0, int c1,
                                             int c2, uint64_t policy) {
  GDN_DEBUG_CHECK((smem_u32(src) & 127) == 0 && smem_range_ok(smem_u32(src), 1),
                  kSiteTmaStoreSmem, smem_u32(src));
  GDN_DEBUG_CHECK((c0 & 15) == 0 && (c0 | c1 | c2) >= 0, kSiteTmaStoreCoord,
                  (static_cast<long long>(c2) << 32) | static_cast<uint32_t>(c0));
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group.L2::cache_hint"
      " [%0, {%2, %3, %4}], [%1], %5;" ::"l"(reinterpret_cast<uint64_t>(tmap)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}

// Bulk (non-tensor) copy of `bytes` contiguous bytes shared -> global, bulk-group completion.
__device__ __forceinline__ void bulk_store(void* gdst, const void* src, uint32_t bytes) {
  GDN_DEBUG_CHECK((smem_u32(src) & 15) == 0 && smem_range_ok(smem_u32(src), bytes), kSiteBulkSmem,
                  smem_u32(src));
  GDN_DEBUG_CHECK((reinterpret_cast<uintptr_t>(gdst) & 15) == 0 && (bytes & 15) == 0,
                  kSiteBulkGlobal, reinterpret_cast<uintptr_t>(gdst));
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(gdst)),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N committed bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Prefetch a tile of a 3-D tensor into L2 (no shared memory, no completion tracking).
__device__ __forceinline__ void tma_prefetch_3d(const void* tmap, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

// Named barrier that also ORs a predicate over the participating threads: every thread gets
// the same answer, so a decision to unwind (e.g. after a wait timed out) stays uniform.
__device__ __forceinline__ bool named_bar_any(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %2, 0;\n\t"
      "bar.red.or.pred q, %1, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(pred ? 1u : 0u), "r"(count)
      : "memory");
  return r != 0;
}

// 16-byte asynchronous copy global -> shared through L2 only (no L1 allocation), tracked per
// thread by commit/wait groups.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  GDN_DEBUG_CHECK((smem_u32(smem_dst) & 15) == 0 && smem_range_ok(smem_u32(smem_dst), 16) &&
                      (reinterpret_cast<uintptr_t>(gsrc) & 15) == 0,
                  kSiteCpAsync, reinterpret_cast<uintptr_t>(gsrc));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// Wait until at most N of this thread's committed cp.async groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Prefetch `bytes` (a multiple of 16) of contiguous global memory into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)),
               "r"(bytes)
               : "memory");
}

// Barrier over a subset of warps (named barrier `id`, `count` threads).
__device__ __forceinline__ void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Bulk (non-tensor) copy of `bytes` contiguous bytes global -> shared, completing on an mbarrier.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
  GDN_DEBUG_CHECK((smem_u32(dst) & 15) == 0 && smem_range_ok(smem_u32(dst), bytes), kSiteBulkSmem,
                  smem_u32(dst));
  GDN_DEBUG_CHECK((reinterpret_cast<uintptr_t>(src) & 15) == 0 && (bytes & 15) == 0,
                  kSiteBulkGlobal, reinterpret_cast<uintptr_t>(src));
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}


// Generic-proxy writes to shared memory -> visible to the async proxy (TMA, tcgen05.mma).
__device__ __forceinline__ void fence_async_smem() {
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

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 inputs, f32 accumulate), one CTA.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A * B with e4m3 A and B (kind::f8f6f4), f32 accumulate; K = 32 per instruction.
__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier when every previously issued tcgen05.mma of this thread is done.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (quarter*32+i).
// The wait is inside the same asm statement, so the outputs are complete when it returns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 64 consecutive 32-bit columns in one load (wait included).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 16 consecutive 32-bit columns (wait included).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 e4m3 values (byte i = element i) -> 16 bf16 (lo: elements 0..7, hi: 8..15). Every e4m3
// value is exactly representable in fp16 and in bf16, so the conversion is exact.
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4& in, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const __nv_fp8x2_storage_t pair =
        static_cast<__nv_fp8x2_storage_t>((w[i >> 1] >> ((i & 1) * 16)) & 0xFFFFu);
    const __half2 h2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3));
    const __nv_bfloat162 b2 = __float22bfloat162_rn(__half22float2(h2));
    o[i] = *reinterpret_cast<const uint32_t*>(&b2);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// An fp8 operand tile converted in place into the bf16 operand layout. The tile holds 128 token
// rows; the bf16 form is two 128B-swizzled TMA boxes of 64 dims (box0 at `tile`, box1 at
// tile + 16 KB, row r at r * 128 in each); the fp8 form was TMA-loaded 128B-swizzled into the
// box1 region (row r: 128 e4m3 values at tile + 16 KB + r * 128). kParts adjacent lanes of one
// warp convert row `row` together, lane `part` taking fp8 chunks [part, part + 1) * 8 / kParts
// (16 dims each): every lane of the warp reads its chunks before any lane writes, since box1 row
// r occupies the bytes of fp8 row r. Every lane of the warp must call it.
template <int kParts>
__device__ __forceinline__ void e4m3_row_to_bf16_tile(uint8_t* tile, int row, int part) {
  static_assert(kParts == 1 || kParts == 2 || kParts == 4, "parts of a row");
  constexpr int kC = 8 / kParts;
  uint8_t* b0 = tile + row * 128;
  uint8_t* b1 = tile + 16384 + row * 128;
  const uint32_t sw = row & 7;
  uint4 in[kC];
#pragma unroll
  for (int i = 0; i < kC; ++i)
    in[i] = *reinterpret_cast<const uint4*>(b1 + (((part * kC + i) ^ sw) << 4));
  if (kParts > 1) __syncwarp();
#pragma unroll
  for (int i = 0; i < kC; ++i) {
    // fp8 chunk c = dims 16c..16c+15 -> bf16 chunks 2c, 2c+1 of the 16 chunks of 8 dims
    const int c = part * kC + i;
    uint4 lo, hi;
    e4m3x16_to_bf16(in[i], lo, hi);
    const int k0 = 2 * c, k1 = 2 * c + 1;  // 8-dim chunk index over 128 dims
    uint8_t* d0 = (k0 < 8 ? b0 : b1) + (((k0 & 7) ^ sw) << 4);
    uint8_t* d1 = (k1 < 8 ? b0 : b1) + (((k1 & 7) ^ sw) << 4);
    *reinterpret_cast<uint4*>(d0) = lo;
    *reinterpret_cast<uint4*>(d1) = hi;
  }
}

// Store 32 lanes x 32 consecutive 32-bit columns (thread i of the warp writes lane
// quarter*32+i), then wait until the stores are done, so a following tcgen05 fence and thread
// synchronisation order them before later MMAs.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

// 2^x by the hardware's approximate base-2 exponential (the PTX ex2.approx.ftz.f32
// instruction: about 2 ulp, flushes subnormals; 2^-inf = +0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Store one 32-bit column of 32 lanes (thread i writes lane quarter*32+i), wait included.
__device__ __forceinline__ void tmem_st1(uint32_t taddr, float v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(__float_as_uint(v))
      : "memory");
}

// 32 lanes x one 32-bit column (wait included).
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r)
      : "r"(taddr)
      : "memory");
  return __uint_as_float(r);
}


// ------------------------------------------------------------------ descriptors
// Shared-memory matrix descriptor, SWIZZLE_128B, sm_100 format (version 1).
//  K-major operand : rows of 128 B (64 bf16 along K), 8-row groups SBO bytes apart.
//  MN-major operand: 128 B runs along M/N (64 bf16), 64-element MN blocks LBO bytes apart,
//                    8-row K groups SBO bytes apart.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes) {
#ifdef GDN_DEBUG
  if (!debug_check(smem_range_ok(saddr, 16), kSiteDescriptor, saddr)) saddr = 0;
#endif
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // version for tcgen05
  d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
  return d;
}

// Same without swizzling, for a K-major operand made of 8-row x 16-byte core matrices (each
// 128 contiguous bytes): LBO = bytes between the two K-adjacent core matrices of one MMA step,
// SBO = bytes between core matrices adjacent along M/N.
__device__ __forceinline__ uint64_t smem_desc_noswz(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
#ifdef GDN_DEBUG
  if (!debug_check(smem_range_ok(saddr, 16), kSiteDescriptor, saddr)) saddr = 0;
#endif
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // version for tcgen05; layout type 0 = no swizzle
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and f32 accumulate.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major,
                                                  bool b_mn_major) {
  return (1u << 4)                                    // D format f32
         | (1u << 7)                                  // A bf16
         | (1u << 10)                                 // B bf16
         | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor of kind::f8f6f4 with e4m3 A and B (format code 0 for both) and f32 D.
// MN-major operands are valid for e4m3 (not for the 6- and 4-bit formats).
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn_major,
                                                  bool b_mn_major) {
  return (1u << 4)                                    // D format f32
         | (0u << 7)                                  // A e4m3
         | (0u << 10)                                 // B e4m3
         | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Byte offset of element (row r, column c) inside a K-major SWIZZLE_128B tile whose rows are
// 128 B (64 bf16) and whose 64-column blocks are `block_bytes` apart.
__device__ __forceinline__ uint32_t swz128_offset_bf16(uint32_t r, uint32_t c,
                                                       uint32_t block_bytes) {
  const uint32_t blk = c >> 6;
  const uint32_t cc = c & 63;
  const uint32_t chunk = (cc >> 3) ^ (r & 7);
  return blk * block_bytes + r * 128u + chunk * 16u + (cc & 7) * 2u;
}


__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace gdn
