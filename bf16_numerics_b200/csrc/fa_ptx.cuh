// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA (cp.async.bulk),
// tcgen05 (TMEM allocation, MMA, loads/stores, fences) and the UMMA shared
// memory / instruction descriptors.
//
// Descriptor bit layouts follow the public PTX ISA description of tcgen05
// matrix descriptors (cross-checked against the CuTe UMMA::SmemDescriptor and
// UMMA::InstrDescriptor definitions):
//   shared-memory descriptor (64 bit):
//     [0,14)  start address >> 4      [16,30) leading byte offset >> 4
//     [32,46) stride byte offset >> 4 [46,48) version (1 on sm_100)
//     [49,52) base offset (0: tiles are 1024-byte aligned)
//     [61,64) layout: 2 = 128-byte swizzle
//   instruction descriptor, kind::f16 (32 bit):
//     [4,6) D format (1 = f32)  [7,10) A format (1 = bf16) [10,13) B format
//     [15] A major (0 = K, 1 = MN)  [16] B major  [17,23) N >> 3  [24,29) M >> 4
//
// Every wait on an mbarrier is bounded (see BoundedWait): after a time limit
// the waiting thread records an error code in a device word, raises the CTA's
// abort flag and returns false, so the kernel can drain and free TMEM instead
// of spinning forever.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

// Profiling hook: a build that defines FA_TRACE_POINT(event) before including
// this header can record per-CTA timelines; the library build compiles it out.
#ifndef FA_TRACE_POINT
#define FA_TRACE_POINT(event) ((void)0)
#endif

namespace fa {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
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

// Error word shared by every kernel of the library (first error wins).
// Code layout: kernel id << 24 | wait site << 16 | low 16 bits of blockIdx.x.
__device__ unsigned int g_fa_error = 0;

// Time limit of every bounded wait (2 s by default: far above any legitimate
// wait).  A test may lower it (fa_debug_set_wait_limit_ns) to exercise the
// exit path quickly.
__device__ unsigned long long g_fa_wait_limit_ns = 2000000000ull;

// Test hook (fa_debug_inject_stall): when it equals a kernel's id, CTA 0 of
// that kernel withholds the first arrive of its elementwise warps on the
// barrier that hands P_bar (forward) or P^T (backward) to the MMA warp.  The
// MMA warp's bounded wait then runs out with no bulk copy outstanding on that
// barrier, and the kernel takes its error exit.  0: no injection.
__device__ unsigned int g_fa_inject = 0;

__device__ __forceinline__ uint64_t wait_limit_ns() { return g_fa_wait_limit_ns; }
__device__ __forceinline__ bool inject_stall_here(uint32_t kernel_id) {
  return blockIdx.x == 0 && g_fa_inject == kernel_id;
}

struct BoundedWait {
  volatile int* abort_flag;  // in shared memory, one per CTA
  uint32_t kernel_id;
  uint64_t limit_ns;

  // Returns true when the phase with the given parity has completed; false if
  // the CTA is aborting (this wait timed out, or another one did).
  __device__ __forceinline__ bool operator()(uint32_t bar, uint32_t parity, uint32_t site) const {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
      if (mbar_try_wait(bar, parity)) return true;
      if ((it & 255u) == 0u) {
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > limit_ns) {
          atomicCAS(&g_fa_error, 0u, (kernel_id << 24) | ((site & 0xFFu) << 16) | (blockIdx.x & 0xFFFFu));
          *abort_flag = 1;
          __threadfence_block();
          return false;
        }
      }
    }
  }
  // Warp-uniform form: true only if the wait succeeded in every lane, so the
  // warp's .sync.aligned instructions after it see one decision.
  __device__ __forceinline__ bool warp(uint32_t bar, uint32_t parity, uint32_t site) const {
    return __all_sync(0xffffffffu, (*this)(bar, parity, site));
  }
};

// Named barrier 1 over the first four warps (128 threads).
__device__ __forceinline__ void named_barrier_sync_128() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// ----------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}
// L2 prefetch of `bytes` bytes at a 16-byte aligned global address (a hint:
// no data is returned and nothing is ordered by it); bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
               : "memory");
}
// generic-proxy shared-memory writes -> visible to the async proxy (tensor core, TMA)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive (once) on an mbarrier when every tcgen05 operation this thread has
// issued so far has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The same two products with each descriptor given as its two 32-bit halves
// (the high half is the same for every tile of a layout)
__device__ __forceinline__ void mma_ss2(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo, uint32_t b_hi,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
      "mov.b64 da, {%1, %2};\n\t"
      "mov.b64 db, {%3, %4};\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts2(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
      "mov.b64 db, {%2, %3};\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 columns of 32-bit TMEM cells -> 32 registers per thread
// (thread i of the warp gets lane base+i, register r holds column col+r).
// The wait is inside the same asm statement so no use of the registers can be
// scheduled before the data has arrived.  TMEM accesses carry no "memory"
// clobber (they touch no generic memory, so shared/global accesses may be
// scheduled around them); being volatile, they stay ordered with respect to
// the mbarrier waits and tcgen05 fences, which are volatile too.
#define FA_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24)
      : "r"(taddr));
}
// Two 32-column loads, one wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t taddr0, uint32_t taddr1, uint32_t (&r)[32], uint32_t (&s)[32]) {
#define FA_S8(i) "=r"(s[i]), "=r"(s[i + 1]), "=r"(s[i + 2]), "=r"(s[i + 3]), "=r"(s[i + 4]), "=r"(s[i + 5]), "=r"(s[i + 6]), "=r"(s[i + 7])
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24), FA_S8(0), FA_S8(8), FA_S8(16), FA_S8(24)
      : "r"(taddr0), "r"(taddr1));
#undef FA_S8
}
// 32 lanes x 128 columns: four 32-column loads and one wait.  The loads
// leave their registers undefined until the wait; the wait names all 128 as
// in/out operands, so no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24)
      : "r"(taddr));
}
#define FA_U8(i) "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])
// wait for every outstanding tcgen05.ld; r (32 registers a no-wait load
// targets) is passed through so that no use of it moves above the wait
__device__ __forceinline__ void tmem_wait_ld32(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : FA_U8(0), FA_U8(8), FA_U8(16), FA_U8(24));
}
__device__ __forceinline__ void tmem_ld32x4(uint32_t taddr, uint32_t (&r)[128]) {
  tmem_ld32_nowait(taddr, &r[0]);
  tmem_ld32_nowait(taddr + 32, &r[32]);
  tmem_ld32_nowait(taddr + 64, &r[64]);
  tmem_ld32_nowait(taddr + 96, &r[96]);
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : FA_U8(0), FA_U8(8), FA_U8(16), FA_U8(24), FA_U8(32), FA_U8(40), FA_U8(48), FA_U8(56), FA_U8(64),
                 FA_U8(72), FA_U8(80), FA_U8(88), FA_U8(96), FA_U8(104), FA_U8(112), FA_U8(120));
}
#undef FA_U8
#undef FA_R8

#define FA_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      FA_W8(0), FA_W8(8), FA_W8(16), FA_W8(24));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      FA_W8(0), FA_W8(8));
}
#undef FA_W8
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// --------------------------------------------------------------- descriptors
// 128-byte-swizzled operand tile in shared memory (see layout table above).
// K-major:  rows of 128 bytes, 8-row groups SBO bytes apart (LBO unused: 16).
// MN-major: 64-element MN blocks LBO bytes apart, 8-row K groups SBO apart.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(lbo >> 4) << 16) |
         (static_cast<uint64_t>(sbo >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
// bf16 x bf16 -> f32, dense, no negation.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn_major) << 15) |
         (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// --------------------------------------------------------------- arithmetic
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// two floats -> packed bf16x2 (RNE), lo in bits 0..15
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void red_add_v4(float* gaddr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(gaddr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

}  // namespace fa

namespace fa {
// ---------------------------------------------------------- bulk (non-tensor)
// Named barrier `id` over `count` threads (id 0 is __syncthreads).
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Named barrier that also ANDs a predicate over the participating threads:
// every thread gets true only if every thread passed true.  Used where a group
// of warps must take the same branch after a bounded wait (a wait that gave up
// in one warp must make all of them skip the work and the later barriers).
__device__ __forceinline__ bool named_barrier_and(uint32_t id, uint32_t count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
      : "memory");
  return r != 0u;
}
// global[dst] += shared[src] element-wise (fp32), `bytes` a multiple of 16,
// both addresses 16-byte aligned; tracked by the issuing thread's bulk group.
__device__ __forceinline__ void bulk_reduce_add_f32(float* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until every committed bulk group has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// wait until every committed bulk group has completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// wait until at most one committed bulk group is still in flight
__device__ __forceinline__ void bulk_wait_all_but_one() { asm volatile("cp.async.bulk.wait_group 1;" ::: "memory"); }
}  // namespace fa

namespace fa {
// ------------------------------------------------------------ packed fp32x2
// Two fp32 lanes per 64-bit register (sm_100 f32x2 arithmetic).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// 2^y for a pair of fp32 arguments on the FMA and integer pipes instead of
// the MUFU (which the exponentials of the softmax keep busy).  Cody-Waite
// range reduction (Cody & Waite, "Software Manual for the Elementary
// Functions", 1980): y = k + r with k = round(y) taken by adding and removing
// 1.5 * 2^23, r in [-1/2, 1/2] exact; 2^r by a degree-5 polynomial with
// constant term 1, fitted for this library by relative least squares with
// Lawson reweighting on [-1/2, 1/2] (20001 equispaced points, 300 solves;
// the fit is re-run by the CPU test of this function; max relative error
// 1.1e-7 with the fp32-rounded coefficients in exact arithmetic, 1.9e-7 in
// fp32 Horner form, the accuracy class of ex2.approx); 2^k by adding k to the
// exponent field.  y = 0 gives exactly 1.  Arguments below -126 (masked
// scores are -inf) give exactly 0, as ex2.approx.ftz does: the range
// reduction works on the argument clamped to -126 and the result is replaced
// by 0 afterwards, so a masked key never enters the row sum or P_bar V.
__device__ __forceinline__ uint64_t exp2_poly_f2(uint64_t y) {
  float y0, y1;
  f2_unpack(y, y0, y1);
  const uint64_t yc = f2_pack(fmaxf(y0, -126.f), fmaxf(y1, -126.f));
  const uint64_t kMagic = f2_pack(12582912.f, 12582912.f);  // 1.5 * 2^23
  const uint64_t t = f2_add(yc, kMagic);                     // 1.5 * 2^23 + k
  const uint64_t r = f2_sub(yc, f2_sub(t, kMagic));          // y - k
  uint64_t q = f2_fma(f2_pack(0.0013264708686619997f, 0.0013264708686619997f), r,
                      f2_pack(0.009671511128544807f, 0.009671511128544807f));
  q = f2_fma(q, r, f2_pack(0.05550733953714371f, 0.05550733953714371f));
  q = f2_fma(q, r, f2_pack(0.24022242426872253f, 0.24022242426872253f));
  q = f2_fma(q, r, f2_pack(0.6931470036506653f, 0.6931470036506653f));
  q = f2_fma(q, r, f2_pack(1.f, 1.f));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  // the low bits of t hold k (two's complement): shifting them to the
  // exponent field drops the 1.5 * 2^23 part
  const float e0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  const float e1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
  return f2_pack(y0 < -126.f ? 0.f : e0, y1 < -126.f ? 0.f : e1);
}
}  // namespace fa

namespace fa {
// 32 lanes x 16 columns, load + wait in one statement (see tmem_ld32)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]));
}
}  // namespace fa

namespace fa {
// shared (128B-swizzled tile) -> global, tracked by the issuing thread's bulk group
__device__ __forceinline__ void tma_store_3d(const void* tmap, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(src), "r"(x), "r"(y), "r"(z)
               : "memory");
}
// One row (64 bf16 = 128 bytes, given as 32 packed bf16x2 words) of a
// 128-row tile in the 128B-swizzled layout TMA uses: 16-byte chunk c of row r
// lives at chunk c ^ (r & 7).  Conflict-free when consecutive threads write
// consecutive rows.
__device__ __forceinline__ void st_row_sw128(uint8_t* tile, int row, const uint32_t (&w)[32]) {
  uint8_t* rp = tile + row * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(rp + ((c ^ (row & 7)) << 4)) = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
}
}  // namespace fa

namespace fa {
// Register re-balancing between warpgroups (all four warps of a warpgroup
// execute the same instruction).  The block is launched with a fixed per-thread
// count; the warpgroups' new counts must sum to no more than four times it.
template <uint32_t N>
__device__ __forceinline__ void warpgroup_reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void warpgroup_reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
}  // namespace fa

namespace fa {
// Explicit shared-memory accesses by 32-bit shared address (ld/st.shared), so
// no access through a generic pointer can fall back to the generic path.
// (not volatile: free to be scheduled among arithmetic and TMEM accesses; the
// "memory" clobber keeps it after the mbarrier waits that publish the data)
__device__ __forceinline__ float4 lds128(uint32_t addr) {
  float4 v;
  asm("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ float lds32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void sts32(uint32_t addr, float a) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(a) : "memory");
}
// st_row_sw128 with an explicit shared address
__device__ __forceinline__ void sts_row_sw128(uint32_t tile, int row, const uint32_t (&w)[32]) {
  const uint32_t rp = tile + row * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c) sts128(rp + ((c ^ (row & 7)) << 4), w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
}
}  // namespace fa

namespace fa {
// three-input maximum (sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// 1.0f if a == b, else 0.0f
__device__ __forceinline__ float feq(float a, float b) {
  float r;
  asm("set.eq.f32.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
}  // namespace fa

namespace fa {
// Programmatic dependent launch: wait until the grid this one depends on has
// completed and its memory is visible (no-op when launched without the
// attribute), and allow the next grid in the stream to be scheduled.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
}  // namespace fa
