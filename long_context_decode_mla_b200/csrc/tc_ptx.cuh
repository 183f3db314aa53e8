// Thin inline-PTX wrappers for the sm_100a features the tensor-core kernels
// use: mbarriers, cp.async and TMA tensor loads, tcgen05 (TMEM allocation,
// MMA, collector buffers, commit, loads and stores) and shared-memory matrix
// descriptors.  Every wait is bounded:
// it gives up after a clock budget and reports failure to the caller.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace dcpmla {
namespace ptx {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------- mbarrier ----

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n .reg .b64 st;\n mbarrier.arrive.release.cta.shared::cta.b64 st, [%0];\n}\n" ::"r"(
          smem_addr(bar))
      : "memory");
}

// Tests the phase; if it is not complete the thread may sleep until it
// completes or about a millisecond passes (the hint only bounds the sleep:
// a completing phase wakes the waiting threads at once).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}

// Arrive on `bar` and add `bytes` to the transaction count it waits for (TMA).
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// Makes barrier initialisations visible to the async proxy (TMA arrivals).
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Waits for completion of the phase with the given parity.  Gives up only
// on its own clock budget (about two seconds), then sets *abort and returns
// false.  It never gives up because another thread set *abort: a phase that
// completes is then seen by every waiter, so threads that later meet at a
// hardware barrier have all passed or all failed the same waits.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_test(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_test(bar, parity)) return true;
    if (clock64() - t0 > (4ll << 30)) {
      *abort = 1;
      return false;
    }
  }
}

// Tests three phases with one shared-memory round trip (the three tests are
// issued back to back; while the tensor core streams its operands a single
// round trip of the load/store unit costs a few hundred cycles).  Returns a
// bit mask of the completed ones (bit k for barrier k).
__device__ __forceinline__ uint32_t mbar_test3(uint64_t* b0, uint32_t p0, uint64_t* b1,
                                               uint32_t p1, uint64_t* b2, uint32_t p2) {
  uint32_t m;
  asm volatile(
      "{\n .reg .pred q0, q1, q2;\n .reg .b32 t0, t1, t2;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 q0, [%1], %2;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 q1, [%3], %4;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 q2, [%5], %6;\n"
      " selp.b32 t0, 1, 0, q0;\n selp.b32 t1, 2, 0, q1;\n selp.b32 t2, 4, 0, q2;\n"
      " or.b32 t0, t0, t1;\n or.b32 %0, t0, t2;\n}\n"
      : "=r"(m)
      : "r"(smem_addr(b0)), "r"(p0), "r"(smem_addr(b1)), "r"(p1), "r"(smem_addr(b2)), "r"(p2)
      : "memory");
  return m;
}

// mbar_wait for three phases at once (any of them may repeat a barrier).
__device__ __forceinline__ bool mbar_wait3(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1,
                                           uint64_t* b2, uint32_t p2, volatile int* abort) {
  const uint32_t m = mbar_test3(b0, p0, b1, p1, b2, p2);
  if (m == 7u) return true;
  if (!(m & 1u) && !mbar_wait(b0, p0, abort)) return false;
  if (!(m & 2u) && !mbar_wait(b1, p1, abort)) return false;
  if (!(m & 4u) && !mbar_wait(b2, p2, abort)) return false;
  return true;
}

// mbar_wait for four phases at once, one shared-memory round trip for the
// first test of all four (any of them may repeat a barrier).
__device__ __forceinline__ bool mbar_wait4(uint64_t* const (&b)[4], const uint32_t (&p)[4],
                                           volatile int* abort) {
  uint32_t m;
  asm volatile(
      "{\n .reg .pred q0, q1, q2, q3;\n .reg .b32 t0, t1, t2, t3;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 q0, [%1], %2;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 q1, [%3], %4;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 q2, [%5], %6;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 q3, [%7], %8;\n"
      " selp.b32 t0, 1, 0, q0;\n selp.b32 t1, 2, 0, q1;\n selp.b32 t2, 4, 0, q2;\n"
      " selp.b32 t3, 8, 0, q3;\n"
      " or.b32 t0, t0, t1;\n or.b32 t2, t2, t3;\n or.b32 %0, t0, t2;\n}\n"
      : "=r"(m)
      : "r"(smem_addr(b[0])), "r"(p[0]), "r"(smem_addr(b[1])), "r"(p[1]), "r"(smem_addr(b[2])),
        "r"(p[2]), "r"(smem_addr(b[3])), "r"(p[3])
      : "memory");
  if (m == 15u) return true;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (!(m & (1u << k)) && !mbar_wait(b[k], p[k], abort)) return false;
  return true;
}

// ------------------------------------------------------------- cp.async ----

// 16-byte global -> shared copy; src_bytes = 0 zero-fills the destination.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

// Bulk copy of `bytes` contiguous global bytes into this CTA's own shared
// memory at `dst` (both 16-byte aligned, bytes a multiple of 16); completes
// as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Bulk prefetch of [src, src + bytes) into L2 (16-byte aligned, multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Arrive on `bar` once all of this thread's earlier cp.async copies landed
// (without raising the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (the tensor core reads shared memory through it).
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ------------------------------------------------------------------ TMA ----

// 3-D tiled tensor load into this CTA's own shared memory; completion is
// signalled on `bar` as transaction bytes.  x is the innermost coordinate.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}

// Four rows of a 2-D tensor map whose box is one row high: rows r.x .. r.w
// (any order, repeats allowed), inner coordinate x (x times the element size
// a multiple of 16 bytes), landing as four consecutive box rows at dst (128-
// byte aligned; with a swizzled map the pattern follows dst's address bits).
__device__ __forceinline__ void tma_gather4(uint32_t dst, const void* tmap, int x, int4 r,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(tmap), "r"(x), "r"(r.x), "r"(r.y), "r"(r.z), "r"(r.w), "r"(smem_addr(bar))
      : "memory");
}

// Named barrier over `threads` threads that also ORs a predicate across them.
__device__ __forceinline__ bool named_bar_or(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

// -------------------------------------------------------------- tcgen05 ----

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(dst_smem)),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, weight-stationary form.
__device__ __forceinline__ void mma_ws_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.ws.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, cta_group::1, kind::f8f6f4
// (e4m3 x e4m3 with fp32 accumulation for the descriptors used here).
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Weight-stationary form of mma_f8.
__device__ __forceinline__ void mma_ws_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.ws.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Weight-stationary MMAs that keep the B operand in one of the tensor
// core's four collector buffers: kFill reads B from shared memory and keeps
// it, kUse / kLastUse read the kept copy (kLastUse releases it) instead of
// shared memory.  The B descriptor passed with kUse / kLastUse must describe
// the same operand that was filled.  Two consecutive MMAs that share B (the
// hi and lo terms of one product) then read it from shared memory once.
enum CollectorOp { kFill = 0, kUse = 1, kLastUse = 2 };

#define DCPMLA_MMA_WS_COLL(KIND, BUF, OP)                                                  \
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"                              \
               " tcgen05.mma.ws.cta_group::1.kind::" KIND ".collector::b" #BUF "::" OP  \
               " [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),                               \
               "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)                     \
               : "memory")

template <int kBuf, int kOp>
__device__ __forceinline__ void mma_ws_f8_coll(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  static_assert(kBuf >= 0 && kBuf < 4, "collector buffers b0..b3");
  if constexpr (kBuf == 0) {
    if constexpr (kOp == kFill) DCPMLA_MMA_WS_COLL("f8f6f4", 0, "fill");
    else if constexpr (kOp == kUse) DCPMLA_MMA_WS_COLL("f8f6f4", 0, "use");
    else DCPMLA_MMA_WS_COLL("f8f6f4", 0, "lastuse");
  } else if constexpr (kBuf == 1) {
    if constexpr (kOp == kFill) DCPMLA_MMA_WS_COLL("f8f6f4", 1, "fill");
    else if constexpr (kOp == kUse) DCPMLA_MMA_WS_COLL("f8f6f4", 1, "use");
    else DCPMLA_MMA_WS_COLL("f8f6f4", 1, "lastuse");
  } else if constexpr (kBuf == 2) {
    if constexpr (kOp == kFill) DCPMLA_MMA_WS_COLL("f8f6f4", 2, "fill");
    else if constexpr (kOp == kUse) DCPMLA_MMA_WS_COLL("f8f6f4", 2, "use");
    else DCPMLA_MMA_WS_COLL("f8f6f4", 2, "lastuse");
  } else {
    if constexpr (kOp == kFill) DCPMLA_MMA_WS_COLL("f8f6f4", 3, "fill");
    else if constexpr (kOp == kUse) DCPMLA_MMA_WS_COLL("f8f6f4", 3, "use");
    else DCPMLA_MMA_WS_COLL("f8f6f4", 3, "lastuse");
  }
}
#undef DCPMLA_MMA_WS_COLL

// cta_group::1 kind::f16 (non weight-stationary), used with bf16 operands.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane
// (warp % 4) * 32 + i of the given address, 32 values.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns (see tmem_ld32).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------- descriptors ----

// Shared-memory matrix descriptor, 128-byte swizzle.  K-major operands: rows
// of 128 bytes, 8-row groups `sbo` bytes apart (lbo unused).  MN-major
// operands: 64 contiguous 16-bit elements per 128-byte row along MN, 8 K-rows
// per group `sbo` apart, and the next 64 MN-elements `lbo` bytes away.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;      // descriptor version for tcgen05
  d |= (uint64_t)2 << 61;      // 128-byte swizzle
  return d;
}

// Shared-memory matrix descriptor with an explicit swizzle mode (tcgen05
// encoding: 0 none, 2 = 128-byte, 4 = 64-byte).  `lbo` / `sbo` are the
// leading / stride byte offsets of the canonical layout.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                          uint32_t swizzle) {
  uint64_t d = 0;
  d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(swizzle & 7u) << 61;
  return d;
}
constexpr uint32_t kSwizzle128B = 2, kSwizzle64B = 4;

// Instruction descriptor with fp32 accumulation: `fmt` is the A and B format
// (kind::f8f6f4: 0 = e4m3; kind::f16: 0 = f16, 1 = bf16); a_mn / b_mn select
// MN-major operands.
__host__ __device__ constexpr uint32_t idesc_make(int M, int N, uint32_t fmt, bool a_mn,
                                                  bool b_mn) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor, kind::f16 with fp16 inputs and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool b_mn_major) {
  return (1u << 4)                       // D format: f32 (A, B format 0: f16)
         | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace ptx
}  // namespace dcpmla
